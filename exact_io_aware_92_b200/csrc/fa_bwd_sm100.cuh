// Attention backward on B200 tensor cores (sm_100a), by recomputation: the
// probabilities are rebuilt from Q, K and the saved per-row log-sum-exp
// instead of being stored (interview notes "Why is FlashAttention faster",
// section on memory: training can store less by recomputing; exam explainer,
// "recomputation": the backward pass recomputes what it needs).  With
// P = exp(scale Q K^T - LSE), dP = dO V^T, D_i = sum_c dO_ic O_ic and
// dS = P * (dP - D):  dV = P^T dO,  dK = scale dS^T Q,  dQ = scale dS K.
//
// fa_bwd_prep_kernel   D and -LSE*log2(e) per query row, in a workspace padded
//                      to whole 128-row tiles (padding: D = 0, -LSE*log2(e) = -inf).
// fa_bwd_dkdv_kernel   one CTA per 128-key tile of one (batch, kv head); it
//                      walks the query tiles of every query head of the
//                      group, each as two halves of 64 queries.  Per half:
//                      S^T = K Q_h^T, dP^T = V dO_h^T (tcgen05, TMEM); the
//                      elementwise warpgroups (thread = key row = TMEM lane)
//                      form P^T and dS^T in bf16 over those TMEM columns; then
//                      dV += P^T dO_h and dK += dS^T Q_h with the left operand
//                      read from TMEM.
// fa_bwd_dq_kernel     one CTA per 128-row query tile; per key tile, as two
//                      halves of 64 keys: S = Q K_h^T, dP = dO V_h^T, dS in
//                      bf16 over S, dQ += dS K_h.
// Halves alternate between two tensor-memory buffers (S or S^T at columns
// 128b, dP or dP^T at 128b + 64), each with its own pair of barriers, so the
// next half's products run while the elementwise warps work on this one.
// Both tcgen05 kernels use 320 threads: warps 0-7 elementwise work in two
// warpgroups (each takes 32 of a half's 64 columns: thread = TMEM lane,
// warp w reaches lanes 32*(w%4)), warp 8 TMA producer, warp 9 MMA issuer
// (one elected lane).  A warpgroup writes its bf16 P or dS over the first 16
// of its own 32 columns (columns 0-15 and 32-47 of the buffer), so neither
// overwrites scores the other has not read yet.  Every wait is bounded.
#pragma once

#include <cstdint>

#include "sm100_ptx.cuh"

namespace fa {

struct BwdParams {
  const uint16_t *o, *dout;   // bf16 [B,Hq,N,d]
  const float *lse;           // fp32 [B,Hq,N]
  uint16_t *dq, *dk, *dv;     // bf16 [B,Hq,N,d], [B,Hkv,N,d] x2
  float *ws_nlse2;            // [B*Hq][Npad]: -LSE * log2(e); -inf on padding rows
  float *ws_delta;            // [B*Hq][Npad]: D; 0 on padding rows
  const int *seqlens;
  int *status;
  int B, Hq, Hkv, N, Npad, group, causal;
  int q_tiles;                // Npad / 128
  float scale, scale_log2;
  unsigned long long wait_limit_ns;
};

template <int D>
struct BwdCfg {
  static constexpr int HALF_BYTES = 128 * 64 * 2;
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int THREADS = 320;
  static constexpr uint32_t COL_A = 0, COL_B = 128, COL_C = 256, COL_D = 384;
  // dK/dV kernel: K, V resident; ring of (Q, dO, LSE2, D) stages.
  static constexpr int KV_STAGES = 2;
  static constexpr int OFF_K = 0, OFF_V = TILE_BYTES, OFF_RING = 2 * TILE_BYTES;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES + 1024;  // Q, dO, 128 LSE2 + 128 D floats
  static constexpr int OFF_BAR_KV = OFF_RING + KV_STAGES * STAGE_BYTES;
  static constexpr int SMEM_KV = OFF_BAR_KV + 128 + 1024;
  // dQ kernel: Q, dO resident; ring of (K, V) stages.
  static constexpr int Q_STAGES = 2;
  static constexpr int OFF_Q = 0, OFF_DO = TILE_BYTES, OFF_KVRING = 2 * TILE_BYTES;
  static constexpr int KVSTAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int OFF_BAR_Q = OFF_KVRING + Q_STAGES * KVSTAGE_BYTES;
  static constexpr int SMEM_Q = OFF_BAR_Q + 128 + 1024;
};

// ---------------------------------------------------------------------------
// Preprocess: D_i = sum_c dO_ic O_ic, NLSE2_i = -LSE_i * log2(e) (stored
// negated, so the elementwise steps add it in one fused multiply-add)
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128) fa_bwd_prep_kernel(const BwdParams p) {
  const long long row = static_cast<long long>(blockIdx.x) * 128 + threadIdx.x;  // over B*Hq*Npad
  if (row >= static_cast<long long>(p.B) * p.Hq * p.Npad) return;
  const int bh = static_cast<int>(row / p.Npad), i = static_cast<int>(row % p.Npad);
  if (i >= p.N) {
    p.ws_nlse2[row] = -INFINITY;
    p.ws_delta[row] = 0.f;
    return;
  }
  const size_t base = (static_cast<size_t>(bh) * p.N + i) * D;
  const uint4 *po = reinterpret_cast<const uint4 *>(p.o + base);
  const uint4 *pd = reinterpret_cast<const uint4 *>(p.dout + base);
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < D / 8; ++c) {
    const uint4 a = po[c], b = pd[c];
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc = fmaf(__uint_as_float(wa[e] << 16), __uint_as_float(wb[e] << 16), acc);
      acc = fmaf(__uint_as_float(wa[e] & 0xFFFF0000u), __uint_as_float(wb[e] & 0xFFFF0000u), acc);
    }
  }
  p.ws_delta[row] = acc;
  const float l = p.lse[static_cast<size_t>(bh) * p.N + i];
  // A row that saw no key keeps no gradient: -inf makes its probabilities 0.
  p.ws_nlse2[row] = (l == -INFINITY) ? -INFINITY : -l * 1.4426950408889634f;
}

// Bulk copy of `bytes` (multiple of 16) global -> shared, completing on `bar`.
__device__ __forceinline__ void bwd_bulk(uint32_t dst, const void *src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// Packed fp32 pair arithmetic beyond fma/add (sm100_ptx.cuh).
__device__ __forceinline__ uint64_t sub_f32x2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t mul_f32x2_bwd(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// Load one 128-row x D bf16 tile (two 64-column boxes) with TMA.
template <int D>
__device__ __forceinline__ void load_tile(uint32_t dst, const CUtensorMap *m, uint32_t bar,
                                          int row, int plane) {
#pragma unroll
  for (int half = 0; half < D / 64; ++half)
    tma_load_3d(dst + half * BwdCfg<D>::HALF_BYTES, m, bar, half * 64, row, plane);
}

// ---------------------------------------------------------------------------
// dK, dV
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(BwdCfg<D>::THREADS, 1)
    fa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_do, const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *smem = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Unit: (batch, kv head, key tile), groups outermost so that the CTAs in
  // flight share one group's Q and dO stream in L2; within a group, causal
  // units with the most query tiles (the first key tiles) run first.
  const int kt = static_cast<int>(blockIdx.x) % p.q_tiles;
  const int bkv = static_cast<int>(blockIdx.x) / p.q_tiles;
  const int b = bkv / p.Hkv, hkv = bkv % p.Hkv;
  int L = p.N;
  if (p.seqlens) L = min(max(p.seqlens[b], 0), p.N);
  const int key0 = kt * 128;
  const int qt0 = p.causal ? kt : 0;  // first query tile that sees these keys
  const int nq_per_head = p.q_tiles - qt0;
  const int nsteps = (key0 < L) ? p.group * nq_per_head : 0;

  const uint32_t bar_kv = base + C::OFF_BAR_KV;         // K, V loaded
  const uint32_t bar_full = bar_kv + 8;                  // [KV_STAGES]
  const uint32_t bar_empty = bar_full + 8 * C::KV_STAGES;  // [KV_STAGES]
  // Each 128-query step runs as two halves of 64 queries; half gh uses
  // tensor-memory buffer gh & 1 (S^T at columns 128b, dP^T at 128b + 64) and
  // that buffer's own pair of barriers, so a barrier's next phase needs
  // products issued only after its previous one was consumed.
  const uint32_t bar_st = bar_empty + 8 * C::KV_STAGES;  // [2]: S^T and dP^T of a half in TMEM
  const uint32_t bar_pds = bar_st + 16;                  // [2]: P^T and dS^T of a half in TMEM
  const uint32_t bar_done = bar_pds + 16;                // all products finished
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_BAR_KV + 120);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_BAR_KV + 124);

  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    for (int s = 0; s < C::KV_STAGES; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int b2 = 0; b2 < 2; ++b2) {
      mbar_init(bar_st + 8 * b2, 1);
      mbar_init(bar_pds + 8 * b2, 256);
    }
    mbar_init(bar_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(tmem_slot);

  auto step_head = [&](int s) { return hkv * p.group + s / nq_per_head; };
  auto step_qt = [&](int s) { return qt0 + s % nq_per_head; };

  if (nsteps > 0 && warp == 8) {
    if (lane == 0) {
      // --- producer ---
      mbar_arrive_expect_tx(bar_kv, 2 * C::TILE_BYTES);
      load_tile<D>(base + C::OFF_K, &tm_k, bar_kv, key0, bkv);
      load_tile<D>(base + C::OFF_V, &tm_v, bar_kv, key0, bkv);
      int s = 0;
      for (; s < nsteps; ++s) {
        const int st = s % C::KV_STAGES;
        if (!mbar_wait_bounded(bar_empty + 8 * st, ((s / C::KV_STAGES) & 1) ^ 1, abort_flag,
                               p.status, p.wait_limit_ns, kErrTimeout))
          break;
        const int h = step_head(s), qt = step_qt(s);
        const int bh = b * p.Hq + h;
        const uint32_t dst = base + C::OFF_RING + st * C::STAGE_BYTES;
        mbar_arrive_expect_tx(bar_full + 8 * st, 2 * C::TILE_BYTES + 1024);
        load_tile<D>(dst, &tm_q, bar_full + 8 * st, qt * 128, bh);
        load_tile<D>(dst + C::TILE_BYTES, &tm_do, bar_full + 8 * st, qt * 128, bh);
        const size_t vrow = static_cast<size_t>(bh) * p.Npad + qt * 128;
        bwd_bulk(dst + 2 * C::TILE_BYTES, p.ws_nlse2 + vrow, 512, bar_full + 8 * st);
        bwd_bulk(dst + 2 * C::TILE_BYTES + 512, p.ws_delta + vrow, 512, bar_full + 8 * st);
      }
      volatile int never = 0;
      mbar_wait_bounded(bar_kv, 0, &never, p.status, p.wait_limit_ns, kErrTimeout);
      for (int st = 0; st < C::KV_STAGES && st < s; ++st) {
        const int last = st + C::KV_STAGES * ((s - 1 - st) / C::KV_STAGES);
        mbar_wait_bounded(bar_full + 8 * st, (last / C::KV_STAGES) & 1, &never, p.status,
                          p.wait_limit_ns, kErrTimeout);
      }
    }
  } else if (nsteps > 0 && warp == 9) {
    // --- MMA issuer ---
    const bool leader = elect_one();
    constexpr uint32_t IDESC_SS = idesc_bf16_f32(128, 64, 0, 0);   // K-major A and B, 64 queries
    constexpr uint32_t IDESC_TS = idesc_bf16_f32(128, D, 0, 1);    // A in TMEM, B MN-major
    const uint64_t dK = smem_desc_sw128(base + C::OFF_K, 16, 1024);
    const uint64_t dV = smem_desc_sw128(base + C::OFF_V, 16, 1024);
    auto wait = [&](uint32_t bar, uint32_t par) {
      const bool ok = mbar_wait_bounded(bar, par, abort_flag, p.status, p.wait_limit_ns,
                                        kErrTimeout);
      return __all_sync(0xffffffffu, ok);
    };
    auto commit = [&](uint32_t bar) {
      if (leader) tc_commit(bar);
      __syncwarp();
    };
    auto stage_addr = [&](int st_step) {
      return base + C::OFF_RING + (st_step % C::KV_STAGES) * C::STAGE_BYTES;
    };
    auto wait_full = [&](int st_step) {
      return wait(bar_full + 8 * (st_step % C::KV_STAGES), (st_step / C::KV_STAGES) & 1);
    };
    // S^T = K Q_h^T and dP^T = V dO_h^T for half gh (64 queries; query row 64
    // starts 8 swizzle atoms into each box), K = d in steps of 16.
    auto issue_sdp = [&](int gh) {
      const uint32_t stage = stage_addr(gh >> 1), rows = (gh & 1) * 8192u;
      const uint64_t dQk = smem_desc_sw128(stage + rows, 16, 1024);
      const uint64_t dOk = smem_desc_sw128(stage + C::TILE_BYTES + rows, 16, 1024);
      const uint32_t colS = (gh & 1) * 128u;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = ((kk / 4) * C::HALF_BYTES + (kk % 4) * 32) >> 4;
        if (leader) tc_mma_ss(tmem + colS, dK + off, dQk + off, IDESC_SS, kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = ((kk / 4) * C::HALF_BYTES + (kk % 4) * 32) >> 4;
        if (leader) tc_mma_ss(tmem + colS + 64, dV + off, dOk + off, IDESC_SS, kk > 0);
      }
      __syncwarp();
    };
    // dV += P^T dO_h, dK += dS^T Q_h: K = 64 queries in steps of 16; the right
    // operand is the tile read MN-major (queries as rows).  The warpgroups'
    // bf16 halves sit at columns 0-15 and 32-47 of S^T (and of dP^T).
    auto issue_ts = [&](int gh) {
      const uint32_t stage = stage_addr(gh >> 1), rows = (gh & 1) * 8192u;
      const uint64_t dOm = smem_desc_sw128(stage + C::TILE_BYTES + rows, C::HALF_BYTES, 1024);
      const uint64_t dQm = smem_desc_sw128(stage + rows, C::HALF_BYTES, 1024);
      const uint32_t colS = (gh & 1) * 128u;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t a = 8u * kk + (kk >= 2 ? 16u : 0u);
        if (leader) {
          tc_mma_ts(tmem + C::COL_D, tmem + colS + a, dOm + ((kk * 2048) >> 4), IDESC_TS,
                    (gh > 0 || kk > 0) ? 1u : 0u);
          tc_mma_ts(tmem + C::COL_C, tmem + colS + 64 + a, dQm + ((kk * 2048) >> 4), IDESC_TS,
                    (gh > 0 || kk > 0) ? 1u : 0u);
        }
      }
      __syncwarp();
    };
    const int nhalves = 2 * nsteps;
    bool ok = wait(bar_kv, 0) && wait_full(0);
    if (ok) {
      tc_fence_after();
      issue_sdp(0);
      commit(bar_st);
    }
    for (int gh = 0; ok && gh < nhalves; ++gh) {
      // The next half's products go into the other buffer while this half's
      // P^T and dS^T are formed (that buffer's last readers, half gh - 1's
      // products, were issued before).
      const int nx = gh + 1;
      if (nx < nhalves) {
        if ((nx & 1) == 0) {
          if (!wait_full(nx >> 1)) break;
          tc_fence_after();
        }
        issue_sdp(nx);
        commit(bar_st + 8 * (nx & 1));
      }
      if (!wait(bar_pds + 8 * (gh & 1), (gh >> 1) & 1)) break;
      tc_fence_after();
      issue_ts(gh);
      if (gh & 1) commit(bar_empty + 8 * ((gh >> 1) % C::KV_STAGES));
    }
    commit(bar_done);
    volatile int never = 0;
    mbar_wait_bounded(bar_done, 0, &never, p.status, p.wait_limit_ns, kErrTimeout);
  } else if (warp < 8) {
    // --- elementwise warpgroups: thread = key row; in each 64-query half,
    // warpgroup e takes queries [32e, 32e + 32) ---
    const int e = warp >> 2;
    const int j = key0 + (threadIdx.x & 127);
    const uint32_t lane_base = static_cast<uint32_t>(warp & 3) * 32u << 16;
    const bool key_ok = j < L;
    bool ok = true;
    for (int gh = 0; gh < 2 * nsteps && ok; ++gh) {
      const int s = gh >> 1, hq = gh & 1;
      const int st = s % C::KV_STAGES;
      const bool got = mbar_wait_bounded(bar_st + 8 * hq, (gh >> 1) & 1, abort_flag, p.status,
                                         p.wait_limit_ns, kErrTimeout);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      // The per-row vectors came with the stage's bulk copies: observe that
      // stage's fill directly (it is refilled only after this step's second
      // half is consumed, so the phase cannot have moved on).
      const bool filled = mbar_wait_bounded(bar_full + 8 * st, (s / C::KV_STAGES) & 1, abort_flag,
                                            p.status, p.wait_limit_ns, kErrTimeout);
      if (!__all_sync(0xffffffffu, filled)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int c0 = 64 * hq + 32 * e;  // first query column of this thread's block
      const int q0 = step_qt(s) * 128;
      const float *nlse2 =
          reinterpret_cast<const float *>(smem + C::OFF_RING + st * C::STAGE_BYTES + 2 * C::TILE_BYTES);
      const float *delta = nlse2 + 128;
      const uint32_t tS = tmem + lane_base + hq * 128 + 32 * e;
      {
        uint32_t sv[32], dp[32];
        tmem_ld32(tS, sv);
        tmem_ld32(tS + 64, dp);
        tmem_wait_ld();
        // Only a block on the diagonal tile has queries above some key
        // (query tile == key tile): elsewhere every (i, j) of the block is
        // visible and the per-element test is skipped (warp-uniform).
        const bool diag = p.causal && q0 + c0 < key0 + 127;
        const uint64_t scl2 = f32x2(p.scale_log2, p.scale_log2);
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int x4 = 0; x4 < 8; ++x4) {
          // this block's -LSE2 and D values, four columns per shared load;
          // the arithmetic runs on pairs (fma/sub/mul.rn.f32x2)
          const float4 l4 = *reinterpret_cast<const float4 *>(nlse2 + c0 + 4 * x4);
          const float4 d4 = *reinterpret_cast<const float4 *>(delta + c0 + 4 * x4);
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int u = 4 * x4 + 2 * h2;  // first of the pair's two columns
            const uint64_t t = fma_f32x2(
                f32x2(__uint_as_float(sv[u]), __uint_as_float(sv[u + 1])), scl2,
                h2 ? f32x2(l4.z, l4.w) : f32x2(l4.x, l4.y));
            float t0, t1;
            f32x2_split(t, t0, t1);
            float p0 = ex2_approx(t0), p1 = ex2_approx(t1);
            if (diag) {
              const int i0 = q0 + c0 + u;
              if (i0 < j) p0 = 0.f;
              if (i0 + 1 < j) p1 = 0.f;
            }
            const uint64_t pp = f32x2(p0, p1);
            const uint64_t dd = sub_f32x2(
                f32x2(__uint_as_float(dp[u]), __uint_as_float(dp[u + 1])),
                h2 ? f32x2(d4.z, d4.w) : f32x2(d4.x, d4.y));
            float s0, s1;
            f32x2_split(mul_f32x2_bwd(pp, dd), s0, s1);
            pk[u >> 1] = pack_bf16x2(p0, p1);
            dk[u >> 1] = pack_bf16x2(s0, s1);
          }
        }
        // keys past the length get no gradient
        if (!key_ok) {
#pragma unroll
          for (int x = 0; x < 16; ++x) pk[x] = dk[x] = 0u;
        }
        // P^T over the first 16 of this block's 32 S^T columns, dS^T over dP^T's.
        tmem_st16(tS, pk);
        tmem_st16(tS + 64, dk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_pds + 8 * hq);
    }
    // Epilogue: dK = scale * sum dS^T Q (warpgroup 0), dV = sum P^T dO
    // (warpgroup 1), in bf16.
    if (ok && nsteps > 0) {
      const bool got = mbar_wait_bounded(bar_done, 0, abort_flag, p.status, p.wait_limit_ns,
                                         kErrTimeout);
      ok = __all_sync(0xffffffffu, got);
    }
    // tcgen05.ld is warp-collective: every lane loads (ok is warp-uniform);
    // only the stores are limited to rows that exist.
    if (ok) {
      const bool row_ok = j < p.N;
      const size_t row = (static_cast<size_t>(bkv) * p.N + (row_ok ? j : 0)) * D;
      if (nsteps > 0) tc_fence_after();
      {
        const int which = e;
        uint16_t *dst = (which == 0 ? p.dk : p.dv) + row;
        const float mult = which == 0 ? p.scale : 1.0f;
        const uint32_t tcol = tmem + lane_base + (which == 0 ? C::COL_C : C::COL_D);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          if (nsteps > 0) {
            tmem_ld32(tcol + 32 * c, r);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int x = 0; x < 32; ++x) r[x] = 0u;  // keys past the length: no gradient
          }
          uint32_t w[16];
#pragma unroll
          for (int x = 0; x < 16; ++x)
            w[x] = pack_bf16x2(__uint_as_float(r[2 * x]) * mult, __uint_as_float(r[2 * x + 1]) * mult);
          uint4 *d4 = reinterpret_cast<uint4 *>(dst + 32 * c);
          if (row_ok) {
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              d4[v4] = make_uint4(w[4 * v4], w[4 * v4 + 1], w[4 * v4 + 2], w[4 * v4 + 3]);
          }
        }
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// dQ
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(BwdCfg<D>::THREADS, 1)
    fa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_do, const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *smem = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Unit: (batch, head, query tile), heads outermost so that the CTAs in
  // flight share one group's K and V in L2; within a head, causal units
  // with the most key tiles (the last query tiles) first.
  const int qt = p.q_tiles - 1 - static_cast<int>(blockIdx.x) % p.q_tiles;
  const int bh = static_cast<int>(blockIdx.x) / p.q_tiles;
  const int b = bh / p.Hq, h = bh % p.Hq, hkv = h / p.group;
  const int bkv = b * p.Hkv + hkv;
  int L = p.N;
  if (p.seqlens) L = min(max(p.seqlens[b], 0), p.N);
  const int row0 = qt * 128;
  const int kv_end = p.causal ? min(L, row0 + 128) : L;
  const int nkv = (kv_end + 127) / 128;

  const uint32_t bar_q = base + C::OFF_BAR_Q;
  const uint32_t bar_full = bar_q + 8;
  const uint32_t bar_empty = bar_full + 8 * C::Q_STAGES;
  // Each 128-key tile runs as two halves of 64 keys; half gh uses
  // tensor-memory buffer gh & 1 (S at columns 128b, dP at 128b + 64; dQ at
  // 256) and that buffer's own pair of barriers.
  const uint32_t bar_sd = bar_empty + 8 * C::Q_STAGES;  // [2]: S and dP of a half in TMEM
  const uint32_t bar_ds = bar_sd + 16;                   // [2]: dS of a half in TMEM
  const uint32_t bar_done = bar_ds + 16;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_BAR_Q + 120);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_BAR_Q + 124);

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < C::Q_STAGES; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int b2 = 0; b2 < 2; ++b2) {
      mbar_init(bar_sd + 8 * b2, 1);
      mbar_init(bar_ds + 8 * b2, 256);
    }
    mbar_init(bar_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(tmem_slot);

  if (nkv > 0 && warp == 8) {
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_q, 2 * C::TILE_BYTES);
      load_tile<D>(base + C::OFF_Q, &tm_q, bar_q, row0, bh);
      load_tile<D>(base + C::OFF_DO, &tm_do, bar_q, row0, bh);
      int j = 0;
      for (; j < nkv; ++j) {
        const int st = j % C::Q_STAGES;
        if (!mbar_wait_bounded(bar_empty + 8 * st, ((j / C::Q_STAGES) & 1) ^ 1, abort_flag,
                               p.status, p.wait_limit_ns, kErrTimeout))
          break;
        const uint32_t dst = base + C::OFF_KVRING + st * C::KVSTAGE_BYTES;
        mbar_arrive_expect_tx(bar_full + 8 * st, 2 * C::TILE_BYTES);
        load_tile<D>(dst, &tm_k, bar_full + 8 * st, j * 128, bkv);
        load_tile<D>(dst + C::TILE_BYTES, &tm_v, bar_full + 8 * st, j * 128, bkv);
      }
      volatile int never = 0;
      mbar_wait_bounded(bar_q, 0, &never, p.status, p.wait_limit_ns, kErrTimeout);
      for (int st = 0; st < C::Q_STAGES && st < j; ++st) {
        const int last = st + C::Q_STAGES * ((j - 1 - st) / C::Q_STAGES);
        mbar_wait_bounded(bar_full + 8 * st, (last / C::Q_STAGES) & 1, &never, p.status,
                          p.wait_limit_ns, kErrTimeout);
      }
    }
  } else if (nkv > 0 && warp == 9) {
    const bool leader = elect_one();
    constexpr uint32_t IDESC_SS = idesc_bf16_f32(128, 64, 0, 0);  // 64 keys per half
    constexpr uint32_t IDESC_TS = idesc_bf16_f32(128, D, 0, 1);
    const uint64_t dQk = smem_desc_sw128(base + C::OFF_Q, 16, 1024);
    const uint64_t dOk = smem_desc_sw128(base + C::OFF_DO, 16, 1024);
    auto wait = [&](uint32_t bar, uint32_t par) {
      const bool ok = mbar_wait_bounded(bar, par, abort_flag, p.status, p.wait_limit_ns,
                                        kErrTimeout);
      return __all_sync(0xffffffffu, ok);
    };
    auto commit = [&](uint32_t bar) {
      if (leader) tc_commit(bar);
      __syncwarp();
    };
    auto stage_of = [&](int jj) {
      return base + C::OFF_KVRING + (jj % C::Q_STAGES) * C::KVSTAGE_BYTES;
    };
    auto wait_full = [&](int jj) {
      return wait(bar_full + 8 * (jj % C::Q_STAGES), (jj / C::Q_STAGES) & 1);
    };
    // S = Q K_h^T and dP = dO V_h^T for half gh (64 keys; key row 64 starts
    // 8 swizzle atoms into each box), K = d in steps of 16.
    auto issue_sdp = [&](int gh) {
      const uint32_t stage = stage_of(gh >> 1), rows = (gh & 1) * 8192u;
      const uint64_t dKk = smem_desc_sw128(stage + rows, 16, 1024);
      const uint64_t dVk = smem_desc_sw128(stage + C::TILE_BYTES + rows, 16, 1024);
      const uint32_t colS = (gh & 1) * 128u;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = ((kk / 4) * C::HALF_BYTES + (kk % 4) * 32) >> 4;
        if (leader) tc_mma_ss(tmem + colS, dQk + off, dKk + off, IDESC_SS, kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = ((kk / 4) * C::HALF_BYTES + (kk % 4) * 32) >> 4;
        if (leader) tc_mma_ss(tmem + colS + 64, dOk + off, dVk + off, IDESC_SS, kk > 0);
      }
      __syncwarp();
    };
    // dQ += dS_h K_h: K = 64 keys in steps of 16, K read MN-major; the
    // warpgroups' bf16 halves sit at columns 0-15 and 32-47 of S.
    auto issue_ts = [&](int gh) {
      const uint32_t stage = stage_of(gh >> 1), rows = (gh & 1) * 8192u;
      const uint64_t dKm = smem_desc_sw128(stage + rows, C::HALF_BYTES, 1024);
      const uint32_t colS = (gh & 1) * 128u;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t a = 8u * kk + (kk >= 2 ? 16u : 0u);
        if (leader)
          tc_mma_ts(tmem + C::COL_C, tmem + colS + a, dKm + ((kk * 2048) >> 4), IDESC_TS,
                    (gh > 0 || kk > 0) ? 1u : 0u);
      }
      __syncwarp();
    };
    const int nhalves = 2 * nkv;
    bool ok = wait(bar_q, 0) && wait_full(0);
    if (ok) {
      tc_fence_after();
      issue_sdp(0);
      commit(bar_sd);
    }
    for (int gh = 0; ok && gh < nhalves; ++gh) {
      // The next half's products go into the other buffer while this half's
      // dS is formed (that buffer's last reader, half gh - 1's dQ product,
      // was issued before).
      const int nx = gh + 1;
      if (nx < nhalves) {
        if ((nx & 1) == 0) {
          if (!wait_full(nx >> 1)) break;
          tc_fence_after();
        }
        issue_sdp(nx);
        commit(bar_sd + 8 * (nx & 1));
      }
      if (!wait(bar_ds + 8 * (gh & 1), (gh >> 1) & 1)) break;
      tc_fence_after();
      issue_ts(gh);
      if (gh & 1) commit(bar_empty + 8 * ((gh >> 1) % C::Q_STAGES));
    }
    commit(bar_done);
    volatile int never = 0;
    mbar_wait_bounded(bar_done, 0, &never, p.status, p.wait_limit_ns, kErrTimeout);
  } else if (warp < 8) {
    // thread = query row; in each 64-key half, warpgroup e takes keys
    // [32e, 32e + 32)
    const int e = warp >> 2;
    const int i = row0 + (threadIdx.x & 127);
    const uint32_t lane_base = static_cast<uint32_t>(warp & 3) * 32u << 16;
    const size_t vrow = static_cast<size_t>(bh) * p.Npad + i;
    const float nlse2 = p.ws_nlse2[vrow];
    const float delta = p.ws_delta[vrow];
    const int limit = p.causal ? min(L, i + 1) : L;
    bool ok = true;
    for (int gh = 0; gh < 2 * nkv && ok; ++gh) {
      const int jt = gh >> 1, hk = gh & 1;  // key tile, key half
      const bool got = mbar_wait_bounded(bar_sd + 8 * hk, (gh >> 1) & 1, abort_flag, p.status,
                                         p.wait_limit_ns, kErrTimeout);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tS = tmem + lane_base + hk * 128 + 32 * e;
      {
        uint32_t sv[32], dp[32];
        tmem_ld32(tS, sv);
        tmem_ld32(tS + 64, dp);
        tmem_wait_ld();
        uint32_t dk[16];
        // When every row of the warp sees all 32 keys of the block (most
        // blocks), the per-element limit test is skipped (warp-uniform).
        const int key_first = jt * 128 + 64 * hk + 32 * e;
        const bool masked = !__all_sync(0xffffffffu, key_first + 31 < limit);
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          float dv[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            float pp = ex2_approx(fmaf(__uint_as_float(sv[2 * x + u]), p.scale_log2, nlse2));
            if (masked && key_first + 2 * x + u >= limit) pp = 0.f;
            dv[u] = pp * (__uint_as_float(dp[2 * x + u]) - delta);
          }
          dk[x] = pack_bf16x2(dv[0], dv[1]);
        }
        // dS over the first 16 of this block's 32 S columns
        tmem_st16(tS, dk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_ds + 8 * hk);
    }
    if (ok && nkv > 0) {
      const bool got = mbar_wait_bounded(bar_done, 0, abort_flag, p.status, p.wait_limit_ns,
                                         kErrTimeout);
      ok = __all_sync(0xffffffffu, got);
    }
    // Warp-collective TMEM loads on every lane; stores only for real rows.
    if (ok) {
      const bool row_ok = i < p.N;
      uint16_t *dst = p.dq + (static_cast<size_t>(bh) * p.N + (row_ok ? i : 0)) * D;
      if (nkv > 0) tc_fence_after();
      // warpgroup e writes columns [e D/2, (e + 1) D/2) of the row
#pragma unroll
      for (int c0 = 0; c0 < D / 64; ++c0) {
        const int c = e * (D / 64) + c0;
        uint32_t r[32];
        if (nkv > 0) {
          tmem_ld32(tmem + lane_base + C::COL_C + 32 * c, r);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int x = 0; x < 32; ++x) r[x] = 0u;
        }
        uint32_t w[16];
#pragma unroll
        for (int x = 0; x < 16; ++x)
          w[x] = pack_bf16x2(__uint_as_float(r[2 * x]) * p.scale,
                             __uint_as_float(r[2 * x + 1]) * p.scale);
        uint4 *d4 = reinterpret_cast<uint4 *>(dst + 32 * c);
        if (row_ok) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            d4[v4] = make_uint4(w[4 * v4], w[4 * v4 + 1], w[4 * v4 + 2], w[4 * v4 + 3]);
        }
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fa
