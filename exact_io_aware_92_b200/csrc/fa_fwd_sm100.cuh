// Exact attention forward on B200 tensor cores (sm_100a): one fused kernel
// that streams K/V tiles past two resident Q tiles and keeps the running row
// max, row sum and unnormalised output on chip (wiki note "FlashAttention",
// section "what it is": fix a Q block on chip, stream K, V blocks, update
// m' = max(m, max S_b), l' = e^(m-m') l + sum e^(S_b - m'),
// O' = (e^(m-m') l O + e^(S_b - m') V_b) / l').  Only O and LSE reach HBM.
//
// CTA = one (batch, query head, pair of 128-row Q tiles) work unit.
//   warps 0-3  softmax warpgroup for Q tile 0 (thread r owns row r = TMEM lane r)
//   warps 4-7  softmax warpgroup for Q tile 1
//   warp  8    TMA producer: Q tiles once, then K_j, V_j into a ring of stages
//   warp  9    MMA issuer: S_t = Q_t K_j^T and O_t += P_t V_j with tcgen05.mma
// Tensor memory (512 columns, fp32): S0 [0,128) S1 [128,256) O0 [256,256+d)
// O1 [384,384+d).  P_t (bf16, packed two per column) overwrites the first 64
// columns of S_t and feeds the PV product straight from tensor memory.
//
// Differences from the pages' statement of the recurrence, all algebraically
// equivalent: O is kept unnormalised (O~ = l * O) and divided by l once at the
// end; exponentials are base 2 on log2(e)-scaled scores; the max used for the
// exponentials (m_ref) is only moved when the row max grows by more than
// 2^8, so most tiles skip the O rescale (values stay below 2^8, far from fp32
// overflow).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace fa {

struct FwdParams {
  uint16_t *o;           // bf16 [B, Hq, N, d]
  float *lse;            // fp32 [B, Hq, N]
  const int *seqlens;    // int32 [B] or nullptr
  int *status;           // device status word (time-outs)
  int B, Hq, Hkv, N, group;
  int num_qpairs;        // ceil(N / 256)
  int causal;
  float scale_log2;      // scale * log2(e)
  unsigned long long wait_limit_ns;
};

// Status codes written by the kernel (negative, matching fa_status).
constexpr int kErrTimeout = -8;

template <int D>
struct Sm100Cfg {
  static_assert(D == 64 || D == 128, "head dim 64 or 128");
  static constexpr int BM = 128;                  // query rows per Q tile
  static constexpr int BN = 128;                  // keys per K/V tile
  static constexpr int ROWS_PER_CTA = 2 * BM;
  static constexpr int HALF_BYTES = 128 * 64 * 2; // one TMA box: 128 rows x 64 bf16
  static constexpr int TILE_BYTES = 128 * D * 2;  // one Q, K or V tile
  static constexpr int STAGES = (D == 128) ? 4 : 8;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = OFF_Q + 2 * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_KV + STAGES * TILE_BYTES;
  // barrier indices
  static constexpr int BAR_Q = 0;                     // 2
  static constexpr int BAR_KV_FULL = 2;               // STAGES
  static constexpr int BAR_KV_EMPTY = 2 + STAGES;     // STAGES
  static constexpr int BAR_S_FULL = 2 + 2 * STAGES;   // 2
  static constexpr int BAR_P_FULL = BAR_S_FULL + 2;   // 2
  static constexpr int BAR_O_FULL = BAR_P_FULL + 2;   // 2
  static constexpr int BAR_MMA_DONE = BAR_O_FULL + 2; // 1
  static constexpr int NUM_BARS = BAR_MMA_DONE + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;  // tmem base, abort flag
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;     // room to align the base to 1 KB
  static constexpr int THREADS = 320;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S0 = 0, COL_O0 = 256;
  static constexpr float RESCALE_THRESHOLD = 8.0f;         // log2 units
};

template <int D>
struct Sm100Ctx {
  using C = Sm100Cfg<D>;
  uint32_t smem;      // 1 KB aligned shared base (shared-window address)
  uint32_t tmem;      // tensor-memory base address
  volatile int *abort_flag;
  int b, h, hkv, bh, row0, L, nkv;

  __device__ uint32_t bar(int i) const { return smem + C::OFF_BAR + 8 * i; }
  __device__ uint32_t q_tile(int t) const { return smem + C::OFF_Q + t * C::TILE_BYTES; }
  __device__ uint32_t kv_tile(int slot) const { return smem + C::OFF_KV + slot * C::TILE_BYTES; }
};

// --------------------------------------------------------------------------
// TMA producer (one thread)
// --------------------------------------------------------------------------
template <int D>
__device__ void role_producer(const Sm100Ctx<D> &x, const FwdParams &p, const CUtensorMap *tm_q,
                              const CUtensorMap *tm_k, const CUtensorMap *tm_v) {
  using C = Sm100Cfg<D>;
  for (int t = 0; t < 2; ++t) {
    mbar_arrive_expect_tx(x.bar(C::BAR_Q + t), C::TILE_BYTES);
    for (int half = 0; half < D / 64; ++half)
      tma_load_3d(x.q_tile(t) + half * C::HALF_BYTES, tm_q, x.bar(C::BAR_Q + t), half * 64,
                  x.row0 + t * C::BM, x.bh);
  }
  const int kv_plane = x.b * p.Hkv + x.hkv;
  int seq = 0;
  bool ok = true;
  for (int j = 0; j < x.nkv && ok; ++j) {
    for (int w = 0; w < 2; ++w, ++seq) {
      const int slot = seq % C::STAGES;
      const uint32_t phase = (seq / C::STAGES) & 1;
      if (!mbar_wait_bounded(x.bar(C::BAR_KV_EMPTY + slot), phase ^ 1, x.abort_flag, p.status,
                             p.wait_limit_ns, kErrTimeout)) {
        ok = false;
        break;
      }
      const uint32_t full = x.bar(C::BAR_KV_FULL + slot);
      mbar_arrive_expect_tx(full, C::TILE_BYTES);
      const CUtensorMap *m = w ? tm_v : tm_k;
      for (int half = 0; half < D / 64; ++half)
        tma_load_3d(x.kv_tile(slot) + half * C::HALF_BYTES, m, full, half * 64, j * C::BN,
                    kv_plane);
    }
  }
  // Drain: every copy this thread started must land before the CTA may exit.
  volatile int never = 0;
  for (int t = 0; t < 2; ++t)
    mbar_wait_bounded(x.bar(C::BAR_Q + t), 0, &never, p.status, p.wait_limit_ns, kErrTimeout);
  for (int s = 0; s < C::STAGES && s < seq; ++s) {
    const int last = s + C::STAGES * ((seq - 1 - s) / C::STAGES);
    mbar_wait_bounded(x.bar(C::BAR_KV_FULL + s), (last / C::STAGES) & 1, &never, p.status,
                      p.wait_limit_ns, kErrTimeout);
  }
}

// --------------------------------------------------------------------------
// MMA issuer (one thread)
// --------------------------------------------------------------------------
template <int D>
__device__ void role_mma(const Sm100Ctx<D> &x, const FwdParams &p) {
  using C = Sm100Cfg<D>;
  constexpr uint32_t IDESC_S = idesc_bf16_f32(128, C::BN, 0, 0);  // Q, K both K-major
  constexpr uint32_t IDESC_O = idesc_bf16_f32(128, D, 0, 1);      // P from TMEM, V MN-major
  const uint32_t tS[2] = {x.tmem + C::COL_S0, x.tmem + C::COL_S0 + 128};
  const uint32_t tO[2] = {x.tmem + C::COL_O0, x.tmem + C::COL_O0 + 128};

  auto wait = [&](int bar, uint32_t parity) {
    return mbar_wait_bounded(x.bar(bar), parity, x.abort_flag, p.status, p.wait_limit_ns,
                             kErrTimeout);
  };
  // S_t = Q_t K^T: K = d in steps of 16; a K step of 16 bf16 is 32 bytes inside
  // a 128-byte swizzled row, and every 4 steps move to the next 64-column box.
  auto issue_s = [&](int t, uint32_t k_tile) {
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t off = (kk / 4) * C::HALF_BYTES + (kk % 4) * 32;
      const uint64_t a = smem_desc_sw128(x.q_tile(t) + off, 16, 1024);
      const uint64_t b = smem_desc_sw128(k_tile + off, 16, 1024);
      tc_mma_ss(tS[t], a, b, IDESC_S, kk > 0 ? 1u : 0u);
    }
  };
  // O_t += P_t V: K = 128 keys in steps of 16; P_t steps 8 columns (16 bf16)
  // in TMEM; V steps 16 key rows = 2048 bytes; its two 64-column boxes are
  // HALF_BYTES apart (leading byte offset), 8-row groups 1024 bytes apart.
  auto issue_pv = [&](int t, uint32_t v_tile, bool accumulate) {
#pragma unroll
    for (int kk = 0; kk < C::BN / 16; ++kk) {
      const uint64_t b = smem_desc_sw128(v_tile + kk * 2048, C::HALF_BYTES, 1024);
      tc_mma_ts(tO[t], tS[t] + kk * 8, b, IDESC_O, (accumulate || kk > 0) ? 1u : 0u);
    }
  };
  auto k_slot = [&](int j) { return (2 * j) % C::STAGES; };
  auto v_slot = [&](int j) { return (2 * j + 1) % C::STAGES; };
  auto k_par = [&](int j) { return (uint32_t)(((2 * j) / C::STAGES) & 1); };
  auto v_par = [&](int j) { return (uint32_t)(((2 * j + 1) / C::STAGES) & 1); };

  do {
    if (!wait(C::BAR_Q + 0, 0) || !wait(C::BAR_Q + 1, 0)) break;
    if (!wait(C::BAR_KV_FULL + k_slot(0), k_par(0))) break;
    tc_fence_after();
    issue_s(0, x.kv_tile(k_slot(0)));
    tc_commit(x.bar(C::BAR_S_FULL + 0));
    issue_s(1, x.kv_tile(k_slot(0)));
    tc_commit(x.bar(C::BAR_S_FULL + 1));
    tc_commit(x.bar(C::BAR_KV_EMPTY + k_slot(0)));
    bool ok = true;
    for (int j = 1; j < x.nkv; ++j) {
      const uint32_t pp = (uint32_t)((j - 1) & 1);
      if (!wait(C::BAR_P_FULL + 0, pp) || !wait(C::BAR_KV_FULL + v_slot(j - 1), v_par(j - 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      issue_pv(0, x.kv_tile(v_slot(j - 1)), j - 1 > 0);
      if (!wait(C::BAR_KV_FULL + k_slot(j), k_par(j))) {
        ok = false;
        break;
      }
      tc_fence_after();
      issue_s(0, x.kv_tile(k_slot(j)));
      tc_commit(x.bar(C::BAR_S_FULL + 0));
      if (!wait(C::BAR_P_FULL + 1, pp)) {
        ok = false;
        break;
      }
      tc_fence_after();
      issue_pv(1, x.kv_tile(v_slot(j - 1)), j - 1 > 0);
      tc_commit(x.bar(C::BAR_KV_EMPTY + v_slot(j - 1)));
      issue_s(1, x.kv_tile(k_slot(j)));
      tc_commit(x.bar(C::BAR_S_FULL + 1));
      tc_commit(x.bar(C::BAR_KV_EMPTY + k_slot(j)));
    }
    if (!ok) break;
    const int jl = x.nkv - 1;
    const uint32_t pp = (uint32_t)(jl & 1);
    if (!wait(C::BAR_P_FULL + 0, pp) || !wait(C::BAR_KV_FULL + v_slot(jl), v_par(jl))) break;
    tc_fence_after();
    issue_pv(0, x.kv_tile(v_slot(jl)), jl > 0);
    tc_commit(x.bar(C::BAR_O_FULL + 0));
    if (!wait(C::BAR_P_FULL + 1, pp)) break;
    tc_fence_after();
    issue_pv(1, x.kv_tile(v_slot(jl)), jl > 0);
    tc_commit(x.bar(C::BAR_O_FULL + 1));
    tc_commit(x.bar(C::BAR_KV_EMPTY + v_slot(jl)));
  } while (false);
  // Every MMA issued above must finish before tensor memory is released.
  tc_commit(x.bar(C::BAR_MMA_DONE));
  volatile int never = 0;
  mbar_wait_bounded(x.bar(C::BAR_MMA_DONE), 0, &never, p.status, p.wait_limit_ns, kErrTimeout);
}

// --------------------------------------------------------------------------
// Softmax warpgroup t (128 threads, one query row each)
// --------------------------------------------------------------------------
template <int D>
__device__ void role_softmax(const Sm100Ctx<D> &x, const FwdParams &p, int t) {
  using C = Sm100Cfg<D>;
  const int r = threadIdx.x & 127;
  const uint32_t lane_base = static_cast<uint32_t>((threadIdx.x >> 5) & 3) * 32u << 16;
  const uint32_t tS = x.tmem + lane_base + C::COL_S0 + 128 * t;
  const uint32_t tO = x.tmem + lane_base + C::COL_O0 + 128 * t;
  const int tile_row0 = x.row0 + t * C::BM;
  const int i = tile_row0 + r;  // this thread's query row
  const int limit = p.causal ? min(x.L, i + 1) : x.L;  // visible keys are [0, limit)
  const float sl2 = p.scale_log2;

  float m_ref = -INFINITY;  // reference max (log2 units) the exponentials use
  float l = 0.f;            // running row sum relative to m_ref
  for (int j = 0; j < x.nkv; ++j) {
    if (!mbar_wait_bounded(x.bar(C::BAR_S_FULL + t), j & 1, x.abort_flag, p.status,
                           p.wait_limit_ns, kErrTimeout))
      return;
    tc_fence_after();
    uint32_t s[128];
    tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
    tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
    tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&s[64]));
    tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&s[96]));
    tmem_wait_ld();

    const int kbase = j * C::BN;
    // Masks only on the tile that crosses the key length or the diagonal.
    const bool need_mask = (kbase + C::BN > x.L) || (p.causal && kbase + C::BN - 1 > tile_row0);
    if (need_mask) {
#pragma unroll
      for (int c = 0; c < 128; ++c)
        if (kbase + c >= limit) s[c] = __float_as_uint(-INFINITY);
    }
    float mx = fmax3(__uint_as_float(s[0]), __uint_as_float(s[1]), __uint_as_float(s[2]));
#pragma unroll
    for (int c = 3; c < 127; c += 2)
      mx = fmax3(mx, __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
    mx = fmaxf(mx, __uint_as_float(s[127]));
    const float m_new = fmaxf(m_ref, mx * sl2);

    // Lazy correction: move m_ref (and rescale l and O) only on a big jump.
    const bool need = m_new > m_ref + C::RESCALE_THRESHOLD;
    const float alpha = need ? ex2_approx(m_ref - m_new) : 1.0f;
    if (need) {
      l *= alpha;
      m_ref = m_new;
    }
    const float m_use = (m_ref == -INFINITY) ? 0.0f : m_ref;
    // p = 2^(s * scale * log2(e) - m_ref), rounded to bf16 for the PV
    // product.  The row sum adds the same rounded values, so the weights
    // applied to V sum to exactly one after the final division.
    const uint64_t scale2 = f32x2(sl2, sl2);
    const uint64_t shift2 = f32x2(-m_use, -m_use);
    uint64_t sum2 = f32x2(0.f, 0.f);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      uint32_t pk[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int c = half * 64 + 2 * e;
        float x0, x1;
        f32x2_split(fma_f32x2(f32x2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), scale2,
                              shift2),
                    x0, x1);
        pk[e] = pack_bf16x2(ex2_approx(x0), ex2_approx(x1));
        sum2 = add_f32x2(sum2, f32x2(__uint_as_float(pk[e] << 16),
                                     __uint_as_float(pk[e] & 0xFFFF0000u)));
      }
      tmem_st32(tS + 32 * half, pk);
    }
    float sum_lo, sum_hi;
    f32x2_split(sum2, sum_lo, sum_hi);
    l += sum_lo + sum_hi;
    // O holds earlier tiles' sum only for j > 0; nothing writes it until this
    // warpgroup publishes P (the PV product of tile j-1 finished before S_j).
    if (j > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * c, o);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
        tmem_st32(tO + 32 * c, o);
      }
    }
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(x.bar(C::BAR_P_FULL + t));
  }

  // Epilogue: O = O~ / l in bf16, LSE = (m_ref + log2 l) * ln 2.
  if (!mbar_wait_bounded(x.bar(C::BAR_O_FULL + t), 0, x.abort_flag, p.status, p.wait_limit_ns,
                         kErrTimeout))
    return;
  tc_fence_after();
  const bool valid = i < p.N;
  const float inv_l = l > 0.f ? 1.0f / l : 0.0f;
  uint16_t *orow = p.o + (static_cast<size_t>(x.bh) * p.N + (valid ? i : 0)) * D;
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    uint32_t o[32];
    tmem_ld32(tO + 32 * c, o);
    tmem_wait_ld();
    uint32_t w[16];
#pragma unroll
    for (int e = 0; e < 16; ++e)
      w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
    if (valid) {
      uint4 *dst = reinterpret_cast<uint4 *>(orow + 32 * c);
#pragma unroll
      for (int v4 = 0; v4 < 4; ++v4)
        dst[v4] = make_uint4(w[4 * v4], w[4 * v4 + 1], w[4 * v4 + 2], w[4 * v4 + 3]);
    }
  }
  if (valid)
    p.lse[static_cast<size_t>(x.bh) * p.N + i] =
        l > 0.f ? (m_ref + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
}

// Rows of a work unit that sees no key at all (key length 0): O = 0, LSE = -inf.
template <int D>
__device__ void write_empty_rows(const Sm100Ctx<D> &x, const FwdParams &p) {
  const int i = x.row0 + threadIdx.x;  // threads 0..255 cover the 256 rows
  if (i >= p.N) return;
  uint4 *dst = reinterpret_cast<uint4 *>(p.o + (static_cast<size_t>(x.bh) * p.N + i) * D);
#pragma unroll
  for (int v4 = 0; v4 < D / 8; ++v4) dst[v4] = make_uint4(0, 0, 0, 0);
  p.lse[static_cast<size_t>(x.bh) * p.N + i] = -INFINITY;
}

template <int D>
__global__ void __launch_bounds__(Sm100Cfg<D>::THREADS, 1)
    fa_fwd_bf16_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                             const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = Sm100Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *smem = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  Sm100Ctx<D> x;
  x.smem = base;
  x.abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
  // Work unit: causal units run longest first (the last Q-tile pair has the
  // most keys); consecutive units are consecutive query heads, so the heads
  // that share one kv head read the same K/V tiles close together in time.
  const int BH = p.B * p.Hq;
  const int unit = blockIdx.x;
  const int qp = p.num_qpairs - 1 - unit / BH;
  x.bh = unit % BH;
  x.b = x.bh / p.Hq;
  x.h = x.bh % p.Hq;
  x.hkv = x.h / p.group;
  x.row0 = qp * C::ROWS_PER_CTA;
  int L = p.N;
  if (p.seqlens) L = min(max(p.seqlens[x.b], 0), p.N);
  x.L = L;
  const int kv_end = p.causal ? min(L, x.row0 + C::ROWS_PER_CTA) : L;
  x.nkv = (kv_end + C::BN - 1) / C::BN;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) mbar_init(x.bar(C::BAR_Q + i), 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(x.bar(C::BAR_KV_FULL + s), 1);
      mbar_init(x.bar(C::BAR_KV_EMPTY + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(x.bar(C::BAR_S_FULL + t), 1);
      mbar_init(x.bar(C::BAR_P_FULL + t), 128);
      mbar_init(x.bar(C::BAR_O_FULL + t), 1);
    }
    mbar_init(x.bar(C::BAR_MMA_DONE), 1);
    *x.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(base + C::OFF_MISC, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  x.tmem = *reinterpret_cast<volatile uint32_t *>(smem + C::OFF_MISC);

  if (x.nkv > 0) {
    if (warp == 8) {
      if (lane == 0) role_producer<D>(x, p, &tm_q, &tm_k, &tm_v);
    } else if (warp == 9) {
      if (lane == 0) role_mma<D>(x, p);
    } else {
      role_softmax<D>(x, p, warp >> 2);
    }
  } else if (warp < 8) {
    write_empty_rows<D>(x, p);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(x.tmem, C::TMEM_COLS);
  }
}

}  // namespace fa
