// Split-KV decode forward on CUDA cores: query rows per (batch, kv head)
// against a long key/value cache.  The wiki note "FlashAttention" (section on
// common misconceptions) observes that generating one token is bound by
// reading the cached K/V, not by arithmetic.  Calls with up to 16 query rows
// per kv head run on the tensor cores (fa_decode_tc.cuh); this kernel serves
// the rest, 4 query rows per CTA, any number of them.
//
// Phase 1 (fa_decode_split_kernel): grid = (splits, B * Hkv, row groups).
//   Each CTA streams the K and V rows of one key range of one (batch, kv head)
//   through a 3-stage shared-memory ring with 1-D bulk copies (TMA), for up
//   to 4 query rows (the query heads sharing the kv head, times Nq).  Each
//   key is spread over d/8 lanes (16 bytes each); scores are reduced with
//   shuffles; the online-softmax recurrence (wiki note, section "what it is")
//   runs per block of 8 keys.  The CTA writes its unnormalised partial output
//   with its row max and row sum.
// Phase 2 (fa_decode_combine_kernel): per query row, the partials of all
//   splits are merged through their log-sum-exp: with M = max_s m_s,
//   w_s = 2^(m_s - M), O = sum_s w_s O_s / sum_s w_s l_s and
//   LSE = (M + log2 sum_s w_s l_s) ln 2.
#pragma once

#include <cstdint>

#include "sm100_ptx.cuh"

namespace fa {

struct DecodeParams {
  const uint16_t *q, *k, *v;  // bf16 q [B,Hq,Nq,d]; k, v [B,Hkv,Nk,d]
  uint16_t *o;                // bf16 [B,Hq,Nq,d]
  float *lse;                 // fp32 [B,Hq,Nq]
  const int *seqlens;         // int32 [B] key lengths or nullptr
  float *part_o;              // fp32 [splits][B*Hq*Nq][d]
  float *part_ml;             // fp32 [splits][B*Hq*Nq][2]: row max (log2 units), row sum
  int *status;
  int B, Hq, Hkv, Nq, Nk, group;
  int splits, keys_per_split;
  int ctas;                   // tensor-core path: CTAs sharing the key tiles
  int part_rows;              // tensor-core path: row slots per workspace slot
  int causal;
  float scale_log2;
  unsigned long long wait_limit_ns;
};

template <int D>
struct DecodeCfg {
  static constexpr int WARPS = 8;   // two CTAs per SM (shared memory): 16 warps hide
                                    // the latency of the shuffle reductions
  static constexpr int THREADS = 32 * WARPS;
  static constexpr int ROWS = 4;                      // query rows per CTA
  static constexpr int CHUNK_BYTES = 16384;           // one K (or V) chunk
  static constexpr int KEYS = CHUNK_BYTES / (D * 2);  // keys per chunk: 64 (d=128), 128 (d=64)
  static constexpr int LPK = D / 8;                   // lanes per key (16 bytes each)
  static constexpr int KPW = 32 / LPK;                // keys per warp step
  static constexpr int KPS = WARPS * KPW;             // keys per CTA step
  static constexpr int STEPS = KEYS / KPS;            // steps per chunk (4)
  static constexpr int STAGES = 3;
  static constexpr int SMEM = STAGES * 2 * CHUNK_BYTES + 64;
  static_assert(STEPS * KPS == KEYS, "whole steps per chunk");
  static_assert(WARPS * 4 * D * 4 + WARPS * 4 * 8 <= STAGES * 2 * CHUNK_BYTES,
                "the cross-warp merge fits in the ring");
};

__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// Packed fp32 multiply of two pairs.
__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// Eight bf16 values (16 bytes) to fp32.
__device__ __forceinline__ void bf16x8_to_f32(const uint4 &u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

template <int D>
__global__ void __launch_bounds__(DecodeCfg<D>::THREADS)
    fa_decode_split_kernel(const DecodeParams p) {
  using C = DecodeCfg<D>;
  constexpr int R = C::ROWS;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int bkv = blockIdx.y;  // b * Hkv + hkv
  const int b = bkv / p.Hkv, hkv = bkv % p.Hkv;
  const int rows_total = p.group * p.Nq;  // query rows that share this kv head
  int L = p.Nk;
  if (p.seqlens) L = min(max(p.seqlens[b], 0), p.Nk);
  const int k0 = split * p.keys_per_split;
  const int k1 = min(k0 + p.keys_per_split, L);
  const int nkeys = max(k1 - k0, 0);
  const int nchunks = (nkeys + C::KEYS - 1) / C::KEYS;

  // This lane's query rows (ROWS of them) and its 8 columns.
  const int key_in_warp = lane / C::LPK;
  const int col8 = lane % C::LPK;
  float q[R][8];
  int hq[R], iq[R], limit[R];
  bool row_ok[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int rr = blockIdx.z * R + r;
    row_ok[r] = rr < rows_total;
    hq[r] = hkv * p.group + (row_ok[r] ? rr / p.Nq : 0);
    iq[r] = row_ok[r] ? rr % p.Nq : 0;
    // visible keys [0, limit): causal queries sit at the end of the sequence
    limit[r] = p.causal ? min(L, L - p.Nq + iq[r] + 1) : L;
    if (row_ok[r]) {
      const uint4 u = *reinterpret_cast<const uint4 *>(
          p.q + ((static_cast<size_t>(b) * p.Hq + hq[r]) * p.Nq + iq[r]) * D + col8 * 8);
      bf16x8_to_f32(u, q[r]);
    } else {
#pragma unroll
      for (int c = 0; c < 8; ++c) q[r][c] = 0.f;
    }
  }

  const uint32_t base = smem_u32(smem);
  const uint32_t bars = base + C::STAGES * 2 * C::CHUNK_BYTES;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::STAGES * 2 * C::CHUNK_BYTES + 32);
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) mbar_init(bars + 8 * s, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  const size_t kv_row0 = (static_cast<size_t>(bkv) * p.Nk + k0) * D;
  auto issue = [&](int c) {
    const int s = c % C::STAGES;
    const int n = min(C::KEYS, nkeys - c * C::KEYS);
    const uint32_t bytes = static_cast<uint32_t>(n) * D * 2;
    const uint32_t bar = bars + 8 * s;
    mbar_arrive_expect_tx(bar, 2 * bytes);
    bulk_load(base + s * 2 * C::CHUNK_BYTES, p.k + kv_row0 + static_cast<size_t>(c) * C::KEYS * D,
              bytes, bar);
    bulk_load(base + s * 2 * C::CHUNK_BYTES + C::CHUNK_BYTES,
              p.v + kv_row0 + static_cast<size_t>(c) * C::KEYS * D, bytes, bar);
  };
  int issued = 0;  // chunks whose copies were started (thread 0's count)
  if (threadIdx.x == 0)
    for (; issued < C::STAGES - 1 && issued < nchunks; ++issued) issue(issued);

  // q as packed pairs (columns 2k, 2k + 1 of this lane's 8).
  uint64_t q2[R][4];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int k = 0; k < 4; ++k) q2[r][k] = f32x2(q[r][2 * k], q[r][2 * k + 1]);

  // Online-softmax state, the same on every lane of a key group: row max
  // (log2 units), row sum, and this lane's 8 output columns as 4 pairs.
  float m[R], l[R];
  uint64_t o2[R][4];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) o2[r][k] = f32x2(0.f, 0.f);
  }

  // A chunk gives each key group NV = STEPS * R partial dot products (index
  // i = step * R + row).  They are summed over the group's LPK lanes by a
  // reduce-scatter, after which lane c of the group holds the scores of
  // indices c * VPL .. c * VPL + VPL - 1: one step, VPL consecutive rows.
  constexpr int NV = C::STEPS * R;
  constexpr int VPL = NV / C::LPK;       // 1 (d = 128) or 2 (d = 64)
  constexpr int RPL = R / VPL;           // lanes per step in a group
  static_assert(NV % C::LPK == 0 && R % VPL == 0 && RPL * C::STEPS == C::LPK, "lane map");
  const int gbase = lane - col8;                       // first lane of this key group
  const int own_step = col8 / RPL;
  const int own_row0 = (col8 % RPL) * VPL;
  int own_limit[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const int rr = blockIdx.z * R + own_row0 + v;
    const int iqv = rr < rows_total ? rr % p.Nq : 0;
    own_limit[v] = p.causal ? min(L, L - p.Nq + iqv + 1) : L;
  }

  bool ok = true;
  int consumed = 0;
  for (int c = 0; c < nchunks; ++c, consumed = c) {
    const int s = c % C::STAGES;
    const bool got = mbar_wait_bounded(bars + 8 * s, static_cast<uint32_t>((c / C::STAGES) & 1),
                                       abort_flag, p.status, p.wait_limit_ns, kErrTimeout);
    if (!__syncthreads_and(got)) {
      ok = false;
      break;
    }
    const uint8_t *ks = smem + s * 2 * C::CHUNK_BYTES;
    const uint8_t *vs = ks + C::CHUNK_BYTES;
    const int n_here = min(C::KEYS, nkeys - c * C::KEYS);  // keys copied into this stage
    // Partial dot products over this lane's 8 columns (packed FMA pairs).
    float red[NV];
#pragma unroll
    for (int st = 0; st < C::STEPS; ++st) {
      const int kl = st * C::KPS + warp * C::KPW + key_in_warp;  // key within the chunk
      float kf[8];
      bf16x8_to_f32(*reinterpret_cast<const uint4 *>(ks + (kl * D + col8 * 8) * 2), kf);
      uint64_t k2[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) k2[k] = f32x2(kf[2 * k], kf[2 * k + 1]);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        uint64_t acc = fma_f32x2(q2[r][0], k2[0], f32x2(0.f, 0.f));
#pragma unroll
        for (int k = 1; k < 4; ++k) acc = fma_f32x2(q2[r][k], k2[k], acc);
        float a0, a1;
        f32x2_split(acc, a0, a1);
        red[st * R + r] = a0 + a1;
      }
    }
    // Reduce-scatter over the key group: each level halves the values a lane
    // keeps and adds its partner's matching half.
#pragma unroll
    for (int lev = 1; lev < C::LPK; lev <<= 1) {
      const int mask = C::LPK / (2 * lev);
      const int h = NV / (2 * lev);
      const bool up = (col8 & mask) != 0;
#pragma unroll
      for (int i = 0; i < h; ++i) {
        const float send = up ? red[i] : red[h + i];
        const float keep = up ? red[h + i] : red[i];
        red[i] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
      }
    }
    // This lane's scores (log2 units), masked to -inf past the range, the
    // sequence or the causal limit of their row.
    const int own_key = k0 + c * C::KEYS + own_step * C::KPS + warp * C::KPW + key_in_warp;
    float sc[VPL], bm[VPL];
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      sc[v] = (own_key < k1 && own_key < own_limit[v]) ? red[v] * p.scale_log2 : -INFINITY;
      bm[v] = sc[v];
    }
    // Block max of each row over the group's steps, then on every lane.
#pragma unroll
    for (int sm = RPL; sm < C::LPK; sm <<= 1)
#pragma unroll
      for (int v = 0; v < VPL; ++v) bm[v] = fmaxf(bm[v], __shfl_xor_sync(0xffffffffu, bm[v], sm));
    float m_use[R], alpha[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float bmax = __shfl_sync(0xffffffffu, bm[r % VPL], gbase + r / VPL);
      const float m_new = fmaxf(m[r], bmax);
      m_use[r] = (m_new == -INFINITY) ? 0.f : m_new;
      alpha[r] = ex2_approx(m[r] - m_use[r]);
      m[r] = m_new;
    }
    // Probabilities of this lane's scores; row sums over the steps.
    float pw[VPL], ps[VPL];
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      const int r = own_row0 + v;
      const float mu = r == 0 ? m_use[0] : r == 1 ? m_use[1] : r == 2 ? m_use[2] : m_use[3];
      pw[v] = ex2_approx(sc[v] - mu);
      ps[v] = pw[v];
    }
#pragma unroll
    for (int sm = RPL; sm < C::LPK; sm <<= 1)
#pragma unroll
      for (int v = 0; v < VPL; ++v) ps[v] += __shfl_xor_sync(0xffffffffu, ps[v], sm);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float psum = __shfl_sync(0xffffffffu, ps[r % VPL], gbase + r / VPL);
      l[r] = l[r] * alpha[r] + psum;
#pragma unroll
      for (int k = 0; k < 4; ++k) o2[r][k] = mul_f32x2(o2[r][k], f32x2(alpha[r], alpha[r]));
    }
    // Every lane needs every probability of its group for O += P V.
    float pa[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) pa[i] = __shfl_sync(0xffffffffu, pw[i % VPL], gbase + i / VPL);
#pragma unroll
    for (int st = 0; st < C::STEPS; ++st) {
      const int kl = st * C::KPS + warp * C::KPW + key_in_warp;
      float vf[8];
      bf16x8_to_f32(*reinterpret_cast<const uint4 *>(vs + (kl * D + col8 * 8) * 2), vf);
      if (kl >= n_here) {  // past the copied keys: stale bytes, weight 0
#pragma unroll
        for (int e = 0; e < 8; ++e) vf[e] = 0.f;
      }
      uint64_t v2[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) v2[k] = f32x2(vf[2 * k], vf[2 * k + 1]);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const uint64_t p2 = f32x2(pa[st * R + r], pa[st * R + r]);
#pragma unroll
        for (int k = 0; k < 4; ++k) o2[r][k] = fma_f32x2(p2, v2[k], o2[r][k]);
      }
    }
    __syncthreads();  // every thread is done with this stage before it is refilled
    if (threadIdx.x == 0 && issued < nchunks) issue(issued++);
  }
  // After a time-out, the copies already started must land before exit.
  if (!ok && threadIdx.x == 0) {
    volatile int never = 0;
    for (int cc = consumed; cc < issued; ++cc)
      mbar_wait_bounded(bars + 8 * (cc % C::STAGES), static_cast<uint32_t>((cc / C::STAGES) & 1),
                        &never, nullptr, p.wait_limit_ns, 0);
  }

  float o[R][8];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int k = 0; k < 4; ++k) f32x2_split(o2[r][k], o[r][2 * k], o[r][2 * k + 1]);
  // Merge the lane groups of each warp (same columns, different keys), then
  // the warps through shared memory, then write the CTA's partial.
#pragma unroll
  for (int r = 0; r < R; ++r) {
#pragma unroll
    for (int off = C::LPK; off < 32; off <<= 1) {
      const float m_o = __shfl_xor_sync(0xffffffffu, m[r], off);
      const float l_o = __shfl_xor_sync(0xffffffffu, l[r], off);
      const float m_n = fmaxf(m[r], m_o);
      const float m_u = (m_n == -INFINITY) ? 0.f : m_n;
      const float a = ex2_approx(m[r] - m_u), bw = ex2_approx(m_o - m_u);
      l[r] = l[r] * a + l_o * bw;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float oo = __shfl_xor_sync(0xffffffffu, o[r][e], off);
        o[r][e] = o[r][e] * a + oo * bw;
      }
      m[r] = m_n;
    }
  }
  __syncthreads();  // the ring is free; reuse it for the cross-warp merge
  float *red_o = reinterpret_cast<float *>(smem);          // [WARPS][R][D]
  float *red_ml = red_o + C::WARPS * R * D;                 // [WARPS][R][2]
  if (lane < C::LPK) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
      for (int e = 0; e < 8; ++e) red_o[(warp * R + r) * D + col8 * 8 + e] = o[r][e];
      if (lane == 0) {
        red_ml[(warp * R + r) * 2 + 0] = m[r];
        red_ml[(warp * R + r) * 2 + 1] = l[r];
      }
    }
  }
  __syncthreads();
  if (!ok) return;
  const int rows_all = p.B * p.Hq * p.Nq;
  for (int idx = threadIdx.x; idx < R * D; idx += C::THREADS) {
    const int r = idx / D, col = idx % D;
    const int rr = blockIdx.z * R + r;
    if (rr >= rows_total) continue;
    float mm = -INFINITY;
#pragma unroll
    for (int w = 0; w < C::WARPS; ++w) mm = fmaxf(mm, red_ml[(w * R + r) * 2]);
    const float mu = (mm == -INFINITY) ? 0.f : mm;
    float acc = 0.f, ll = 0.f;
#pragma unroll
    for (int w = 0; w < C::WARPS; ++w) {
      const float wgt = ex2_approx(red_ml[(w * R + r) * 2] - mu);
      acc += wgt * red_o[(w * R + r) * D + col];
      ll += wgt * red_ml[(w * R + r) * 2 + 1];
    }
    const int hqr = hkv * p.group + rr / p.Nq, iqr = rr % p.Nq;
    const size_t row = (static_cast<size_t>(b) * p.Hq + hqr) * p.Nq + iqr;
    p.part_o[(static_cast<size_t>(split) * rows_all + row) * D + col] = acc;
    if (col == 0) {
      p.part_ml[(static_cast<size_t>(split) * rows_all + row) * 2 + 0] = mm;
      p.part_ml[(static_cast<size_t>(split) * rows_all + row) * 2 + 1] = ll;
    }
  }
}

// One warp per query row: merge the splits' partials through their LSE.
template <int D>
__global__ void __launch_bounds__(128) fa_decode_combine_kernel(const DecodeParams p) {
  const int rows_all = p.B * p.Hq * p.Nq;
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows_all) return;
  float M = -INFINITY;
  for (int s = 0; s < p.splits; ++s)
    M = fmaxf(M, p.part_ml[(static_cast<size_t>(s) * rows_all + row) * 2]);
  const float mu = (M == -INFINITY) ? 0.f : M;
  constexpr int PER = D / 32;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float L = 0.f;
  for (int s = 0; s < p.splits; ++s) {
    const size_t base = static_cast<size_t>(s) * rows_all + row;
    const float w = ex2_approx(p.part_ml[base * 2] - mu);
    L += w * p.part_ml[base * 2 + 1];
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] += w * p.part_o[base * D + lane * PER + e];
  }
  const float inv = L > 0.f ? 1.0f / L : 0.f;
  uint16_t *orow = p.o + static_cast<size_t>(row) * D + lane * PER;
#pragma unroll
  for (int e = 0; e < PER; e += 2) {
    const uint32_t w2 = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
    *reinterpret_cast<uint32_t *>(orow + e) = w2;
  }
  if (lane == 0)
    p.lse[row] = L > 0.f ? (M + __log2f(L)) * 0.69314718055994530942f : -INFINITY;
}

}  // namespace fa
