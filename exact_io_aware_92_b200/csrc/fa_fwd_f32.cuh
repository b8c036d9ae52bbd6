// fp32 check mode: the same blockwise online-softmax recurrence as the
// tensor-core kernel (wiki note "FlashAttention", section "what it is"), run in
// fp32 on CUDA cores with accurate exp2f.  It exists to compare against the
// fp64 oracle at 1e-5; speed is not its purpose.
//
// Block = 64 (d = 64) or 32 (d = 128) query rows of one (batch, head); thread
// = one row.  K/V tiles of 32 or 16 keys are staged in shared memory; per tile
// each thread forms its scores, moves its running max once, rescales its
// accumulator and adds the tile's weighted V rows.
#pragma once

#include <cstdint>

namespace fa {

struct F32Params {
  const float *q, *k, *v;
  float *o, *lse;
  const int *seqlens;
  int B, Hq, Hkv, N, group;
  int causal;
  float scale_log2;
};

template <int D>
struct F32Cfg {
  static constexpr int ROWS = D == 64 ? 64 : 32;  // query rows (= threads) per block
  static constexpr int KT = D == 64 ? 32 : 16;    // keys per staged tile
};

template <int D>
__global__ void __launch_bounds__(F32Cfg<D>::ROWS) fa_fwd_f32_kernel(const F32Params p) {
  constexpr int ROWS = F32Cfg<D>::ROWS, KT = F32Cfg<D>::KT;
  __shared__ float sQ[ROWS][D + 1];
  __shared__ float sK[KT][D];
  __shared__ float sV[KT][D];
  const int bh = blockIdx.y;
  const int b = bh / p.Hq, h = bh % p.Hq, g = h / p.group;
  const int row0 = blockIdx.x * ROWS;
  const int i = row0 + threadIdx.x;
  int L = p.N;
  if (p.seqlens) L = min(max(p.seqlens[b], 0), p.N);
  const float *qb = p.q + static_cast<size_t>(bh) * p.N * D;
  const float *kb = p.k + (static_cast<size_t>(b) * p.Hkv + g) * p.N * D;
  const float *vb = p.v + (static_cast<size_t>(b) * p.Hkv + g) * p.N * D;
  for (int e = threadIdx.x; e < ROWS * D; e += ROWS) {
    const int rr = e / D, c = e % D;
    sQ[rr][c] = (row0 + rr < p.N) ? qb[static_cast<size_t>(row0 + rr) * D + c] : 0.f;
  }
  const int limit = p.causal ? min(L, i + 1) : L;
  const int kv_end = p.causal ? min(L, row0 + ROWS) : L;
  float acc[D];
#pragma unroll
  for (int c = 0; c < D; ++c) acc[c] = 0.f;
  float m = -INFINITY, l = 0.f;
  for (int kt = 0; kt < kv_end; kt += KT) {
    __syncthreads();
    for (int e = threadIdx.x; e < KT * D; e += ROWS) {
      const int jj = e / D, c = e % D;
      const bool in = kt + jj < p.N;
      sK[jj][c] = in ? kb[static_cast<size_t>(kt + jj) * D + c] : 0.f;
      sV[jj][c] = in ? vb[static_cast<size_t>(kt + jj) * D + c] : 0.f;
    }
    __syncthreads();
    float s[KT];
    float mx = -INFINITY;
#pragma unroll
    for (int jj = 0; jj < KT; ++jj) {
      float dot = 0.f;
#pragma unroll
      for (int c = 0; c < D; ++c) dot = fmaf(sQ[threadIdx.x][c], sK[jj][c], dot);
      s[jj] = (kt + jj < limit) ? dot * p.scale_log2 : -INFINITY;
      mx = fmaxf(mx, s[jj]);
    }
    const float m_new = fmaxf(m, mx);
    if (m_new == -INFINITY) continue;  // nothing visible to this row yet
    const float alpha = exp2f(m - m_new);
    l *= alpha;
#pragma unroll
    for (int c = 0; c < D; ++c) acc[c] *= alpha;
    m = m_new;
#pragma unroll
    for (int jj = 0; jj < KT; ++jj) {
      const float pj = exp2f(s[jj] - m);
      l += pj;
#pragma unroll
      for (int c = 0; c < D; ++c) acc[c] = fmaf(pj, sV[jj][c], acc[c]);
    }
  }
  if (i >= p.N) return;
  const float inv = l > 0.f ? 1.0f / l : 0.f;
  float *orow = p.o + (static_cast<size_t>(bh) * p.N + i) * D;
#pragma unroll
  for (int c = 0; c < D; ++c) orow[c] = acc[c] * inv;
  p.lse[static_cast<size_t>(bh) * p.N + i] =
      l > 0.f ? (m + log2f(l)) * 0.69314718055994530942f : -INFINITY;
}

}  // namespace fa
