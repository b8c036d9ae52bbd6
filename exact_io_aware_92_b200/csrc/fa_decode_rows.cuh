// Decode forward on the tensor cores for 17 to 128 query rows per (batch, kv
// head): the same operation and results as fa_decode_tc.cuh (wiki note
// "FlashAttention", section "what it is": the blockwise running max / sum /
// output recurrence; section on common misconceptions: one generated token is
// bound by reading the cache), for row counts where keeping every query row's
// statistics per key thread no longer fits.
//
// Orientation.  The G * Nq query rows of a (batch b, kv head g) are the
// 128 row slots of one Q tile (heads g*G .. g*G+G-1 are contiguous in q, Nq
// rows each), so the products are the forward's: S = Q K^T with M = 128 row
// slots and N = 128 keys, then O += P V with P from tensor memory.  Thread r
// of the softmax warps owns row slot r (tensor-memory lane r): its row max and
// row sum need no cross-thread reduction.  Warps whose 32 slots hold no query
// row do no softmax work; the MMA still covers all 128 slots, and those rows
// of O are never read.
//
// Work split and merge are those of fa_decode_tc.cuh: the call's 128-key tiles
// form one sequence, persistent CTA c takes an equal share, the part of a
// share inside one (b, g) is a piece, which writes one partial (O, m, l) per
// query row to workspace slot c + (b Hkv + g); the merge kernel combines each
// row's partials through their log-sum-exp.
//
// Pipeline.  S alternates between two tensor-memory buffers over the key
// tiles: S(ts + 1) is computed while the softmax works on tile ts, and it is
// issued after PV(ts - 1), the last reader of that buffer's P.  K and V have
// rings of their own (a K slot frees when its S product is done, a V slot
// when its PV product is).  O has one buffer: the piece's first PV waits until
// the softmax has read the previous piece's O.
//
// Roles (224 threads, one CTA per SM):
//   warps 0-3  softmax, one row slot per thread;
//   warp 4     TMA producer of each piece's Q tile and of the K tiles;
//   warp 5     MMA issuer;
//   warp 6     TMA producer of the V tiles.
#pragma once

#include <cstdint>

#include "fa_decode_tc.cuh"
#include "sm100_ptx.cuh"

namespace fa {

template <int D>
struct DecodeRowsCfg {
  static_assert(D == 64 || D == 128, "head dim 64 or 128");
  static constexpr int BM = 128;                  // row slots
  static constexpr int BN = 128;                  // keys per tile
  static constexpr int TILE_BYTES = 128 * D * 2;  // one Q, K or V tile
  static constexpr int NBOX = D / 64;             // 64-column TMA boxes per row
  static constexpr int BOX_BYTES = 128 * 128;     // one box: 128 rows x 128 bytes
  static constexpr int KSTEPS = D / 16;           // K steps of the S product
  static constexpr int STAGES = D == 128 ? 3 : 6; // per ring
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + TILE_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_V + STAGES * TILE_BYTES;
  static constexpr int BAR_K_FULL = 0;                 // [STAGES]
  static constexpr int BAR_K_EMPTY = STAGES;           // [STAGES]
  static constexpr int BAR_V_FULL = 2 * STAGES;        // [STAGES]
  static constexpr int BAR_V_EMPTY = 3 * STAGES;       // [STAGES]
  static constexpr int BAR_Q_FULL = 4 * STAGES;
  static constexpr int BAR_Q_EMPTY = BAR_Q_FULL + 1;
  static constexpr int BAR_S_FULL = BAR_Q_EMPTY + 1;   // [2]
  static constexpr int BAR_P_FULL = BAR_S_FULL + 2;    // [2], one arrival per softmax thread at work
  static constexpr int BAR_PV_DONE = BAR_P_FULL + 2;   // a PV product landed
  static constexpr int BAR_O_FULL = BAR_PV_DONE + 1;   // a piece's last PV product landed
  static constexpr int BAR_O_EMPTY = BAR_O_FULL + 1;   // the softmax read O out
  static constexpr int BAR_MMA_DONE = BAR_O_EMPTY + 1;
  static constexpr int NUM_BARS = BAR_MMA_DONE + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;  // tmem base, abort, share, cursor
  static constexpr int SMEM_BYTES = OFF_MISC + 64;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
  static constexpr int THREADS = 224;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S = 0;    // S buffers at 0 and 128
  static constexpr uint32_t COL_O = 256;  // O: D columns
  static constexpr float RESCALE_THRESHOLD = 8.0f;
  static_assert(SMEM_ALLOC <= 232448, "shared memory per CTA");
};

template <int D>
struct DecRowsCtx {
  using C = DecodeRowsCfg<D>;
  uint32_t smem;
  uint32_t tmem;
  volatile int *abort_flag;
  __device__ uint32_t bar(int i) const { return smem + C::OFF_BAR + 8 * i; }
  __device__ uint32_t q_tile() const { return smem + C::OFF_Q; }
  __device__ uint32_t k_tile(int st) const { return smem + C::OFF_K + st * C::TILE_BYTES; }
  __device__ uint32_t v_tile(int st) const { return smem + C::OFF_V + st * C::TILE_BYTES; }
};

// --------------------------------------------------------------------------
// TMA producers (one thread each): IS_V = false loads each piece's Q tile and
// the K tiles, IS_V = true the V tiles.
// --------------------------------------------------------------------------
template <int D, bool IS_V>
__device__ void decr_role_producer(const DecRowsCtx<D> &x, const DecodeParams &p, DecCursor cur,
                                   const CUtensorMap *tm_q, const CUtensorMap *tm_kv) {
  using C = DecodeRowsCfg<D>;
  constexpr int FULL = IS_V ? C::BAR_V_FULL : C::BAR_K_FULL;
  constexpr int EMPTY = IS_V ? C::BAR_V_EMPTY : C::BAR_K_EMPTY;
  int ts = 0, pc = 0;
  bool ok = true;
  DecPiece w;
  while (ok && cur.next(p, w)) {
    if (!IS_V) {
      // The Q tile is replaced once the previous piece's last S product has
      // read it.
      if (!mbar_wait_bounded(x.bar(C::BAR_Q_EMPTY), (pc & 1) ^ 1, x.abort_flag, p.status,
                             p.wait_limit_ns, kErrTimeout))
        break;
      mbar_arrive_expect_tx(x.bar(C::BAR_Q_FULL), C::TILE_BYTES);
      // the piece's query rows: heads g*G .. g*G+G-1, Nq rows each, contiguous
      const int row0 = (w.b * p.Hq + w.g * p.group) * p.Nq;
      for (int bx = 0; bx < C::NBOX; ++bx)
        tma_load_3d(x.q_tile() + bx * C::BOX_BYTES, tm_q, x.bar(C::BAR_Q_FULL), bx * 64, row0,
                    0);
      ++pc;
    }
    const int plane = w.b * p.Hkv + w.g;
    for (int i = 0; i < w.nt; ++i, ++ts) {
      const int st = ts % C::STAGES;
      if (!mbar_wait_bounded(x.bar(EMPTY + st), ((ts / C::STAGES) & 1) ^ 1, x.abort_flag,
                             p.status, p.wait_limit_ns, kErrTimeout)) {
        ok = false;
        break;
      }
      const uint32_t full = x.bar(FULL + st);
      mbar_arrive_expect_tx(full, C::TILE_BYTES);
      const uint32_t dst = IS_V ? x.v_tile(st) : x.k_tile(st);
      const int key0 = (w.i0 + i) * C::BN;
      for (int bx = 0; bx < C::NBOX; ++bx)
        tma_load_3d(dst + bx * C::BOX_BYTES, tm_kv, full, bx * 64, key0, plane);
    }
  }
  // Drain: every copy this thread started must land before the CTA exits.
  volatile int never = 0;
  if (!IS_V && pc > 0)
    mbar_wait_bounded(x.bar(C::BAR_Q_FULL), (pc - 1) & 1, &never, p.status, p.wait_limit_ns,
                      kErrTimeout);
  for (int s = 0; s < C::STAGES && s < ts; ++s) {
    const int last = s + C::STAGES * ((ts - 1 - s) / C::STAGES);
    mbar_wait_bounded(x.bar(FULL + s), (last / C::STAGES) & 1, &never, p.status,
                      p.wait_limit_ns, kErrTimeout);
  }
}

// --------------------------------------------------------------------------
// MMA issuer (one warp; one elected lane issues).  Order: S(ts), then
// PV(ts - 1), so S(ts) overlaps the softmax of tile ts - 1 and its buffer's P
// (tile ts - 2) was read by a PV product issued before it.
// --------------------------------------------------------------------------
template <int D>
__device__ void decr_role_mma(const DecRowsCtx<D> &x, const DecodeParams &p, DecCursor cur) {
  using C = DecodeRowsCfg<D>;
  constexpr uint32_t IDESC_S = idesc_bf16_f32(128, C::BN, 0, 0);  // Q, K both K-major
  constexpr uint32_t IDESC_O = idesc_bf16_f32(128, D, 0, 1);      // P from TMEM, V MN-major
  const bool leader = elect_one();
  auto tS = [&](int i) { return x.tmem + C::COL_S + 128u * static_cast<uint32_t>(i); };
  const uint32_t tO = x.tmem + C::COL_O;
  const uint64_t desc_q = smem_desc_sw128(x.q_tile(), 16, 1024);
  const uint64_t desc_k = smem_desc_sw128(x.k_tile(0), 16, 1024);
  const uint64_t desc_v = smem_desc_sw128(x.v_tile(0), C::BOX_BYTES, 1024);
  constexpr uint32_t STAGE16 = C::TILE_BYTES >> 4;
  auto wait = [&](int bar, uint32_t parity) {
    const bool ok = mbar_wait_bounded(x.bar(bar), parity, x.abort_flag, p.status,
                                      p.wait_limit_ns, kErrTimeout);
    return __all_sync(0xffffffffu, ok);
  };
  auto commit = [&](int bar) {
    if (leader) tc_commit(x.bar(bar));
    __syncwarp();
  };
  struct Pend {
    int ts, st, pc;
    bool first, last;
  };
  auto issue_pv = [&](const Pend &q) {
    if (!wait(C::BAR_V_FULL + q.st, (q.ts / C::STAGES) & 1)) return false;
    if (!wait(C::BAR_P_FULL + (q.ts & 1), (q.ts >> 1) & 1)) return false;
    // A piece's first PV product overwrites O: the softmax must have read
    // the previous piece's O out of tensor memory.
    if (q.first && q.pc > 0 && !wait(C::BAR_O_EMPTY, (q.pc - 1) & 1)) return false;
    tc_fence_after();
    const uint64_t vd = desc_v + q.st * STAGE16;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)  // 16 keys each; P steps 8 columns in TMEM
      if (leader)
        tc_mma_ts(tO, tS(q.ts & 1) + kk * 8, vd + ((kk * 2048) >> 4), IDESC_O,
                  (!q.first || kk > 0) ? 1u : 0u);
    __syncwarp();
    commit(C::BAR_V_EMPTY + q.st);
    commit(C::BAR_PV_DONE);
    if (q.last) commit(C::BAR_O_FULL);
    return true;
  };

  int ts = 0, pc = 0;
  bool ok = true, have = false;
  Pend pend{};
  DecPiece w;
  while (ok && cur.next(p, w)) {
    if (!wait(C::BAR_Q_FULL, pc & 1)) break;
    for (int i = 0; i < w.nt; ++i, ++ts) {
      const int st = ts % C::STAGES;
      if (!wait(C::BAR_K_FULL + st, (ts / C::STAGES) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t kd = desc_k + st * STAGE16;
#pragma unroll
      for (int kk = 0; kk < C::KSTEPS; ++kk) {
        const uint32_t off = ((kk / 4) * C::BOX_BYTES + (kk % 4) * 32) >> 4;
        if (leader) tc_mma_ss(tS(ts & 1), desc_q + off, kd + off, IDESC_S, kk > 0 ? 1u : 0u);
      }
      __syncwarp();
      commit(C::BAR_S_FULL + (ts & 1));
      commit(C::BAR_K_EMPTY + st);
      if (i == w.nt - 1) commit(C::BAR_Q_EMPTY);
      if (have && !issue_pv(pend)) {
        ok = false;
        break;
      }
      pend = Pend{ts, st, pc, i == 0, i == w.nt - 1};
      have = true;
    }
    ++pc;
  }
  if (ok && have) issue_pv(pend);
  commit(C::BAR_MMA_DONE);
  volatile int never = 0;
  mbar_wait_bounded(x.bar(C::BAR_MMA_DONE), 0, &never, p.status, p.wait_limit_ns, kErrTimeout);
}

// --------------------------------------------------------------------------
// Softmax (warps 0-3; thread r = row slot r = TMEM lane r).  Only warps that
// hold query rows run it.
// --------------------------------------------------------------------------
template <int D>
__device__ void decr_role_softmax(const DecRowsCtx<D> &x, const DecodeParams &p, DecCursor cur) {
  using C = DecodeRowsCfg<D>;
  const int r = threadIdx.x;  // row slot
  const uint32_t lane_base = static_cast<uint32_t>((r >> 5) * 32) << 16;
  const int rows = p.group * p.Nq;
  const bool valid = r < rows;
  const int qi = r % p.Nq;  // the row's query index within its head
  const float sl2 = p.scale_log2;
  const uint32_t tO = x.tmem + lane_base + C::COL_O;
  auto wait = [&](int bar, uint32_t parity) {
    const bool ok = mbar_wait_bounded(x.bar(bar), parity, x.abort_flag, p.status,
                                      p.wait_limit_ns, kErrTimeout);
    return __all_sync(0xffffffffu, ok);
  };

  int ts = 0, pc = 0;
  DecPiece w;
  while (cur.next(p, w)) {
    // visible keys [0, limit): causal queries sit at the end of the sequence
    const int limit = p.causal ? min(w.L, w.L - p.Nq + qi + 1) : w.L;
    float m_ref = -INFINITY;  // reference max (log2 units)
    float l = 0.f;            // row sum of the fp32 probabilities relative to m_ref
    for (int i = 0; i < w.nt; ++i, ++ts) {
      const uint32_t tSb = x.tmem + lane_base + C::COL_S + 128u * static_cast<uint32_t>(ts & 1);
      if (!wait(C::BAR_S_FULL + (ts & 1), (ts >> 1) & 1)) return;
      tc_fence_after();
      uint32_t s[128];
      tmem_ld32(tSb + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_ld32(tSb + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
      tmem_ld32(tSb + 64, *reinterpret_cast<uint32_t(*)[32]>(&s[64]));
      tmem_ld32(tSb + 96, *reinterpret_cast<uint32_t(*)[32]>(&s[96]));
      tmem_wait_ld();
      const int kbase = (w.i0 + i) * C::BN;
      if (kbase + C::BN > limit) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (kbase + c >= limit) s[c] = __float_as_uint(-INFINITY);
      }
      float mq[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint32_t *sq = s + 16 * q;
        mq[q] = fmax3(__uint_as_float(sq[0]), __uint_as_float(sq[1]), __uint_as_float(sq[2]));
#pragma unroll
        for (int c = 3; c < 15; c += 2)
          mq[q] = fmax3(mq[q], __uint_as_float(sq[c]), __uint_as_float(sq[c + 1]));
        mq[q] = fmaxf(mq[q], __uint_as_float(sq[15]));
      }
      const float m_tile =
          fmaxf(fmax3(mq[0], mq[1], mq[2]), fmax3(fmax3(mq[3], mq[4], mq[5]), mq[6], mq[7])) * sl2;
      const float m_new = fmaxf(m_ref, m_tile);
      const bool need = m_new > m_ref + C::RESCALE_THRESHOLD;
      if (__any_sync(0xffffffffu, need)) {
        const float alpha = need ? (m_ref == -INFINITY ? 0.f : ex2_approx(m_ref - m_new)) : 1.f;
        if (need) {
          l *= alpha;
          m_ref = m_new;
        }
        if (i > 0) {
          // O holds this piece's earlier tiles once the PV product of the
          // previous tile has landed.
          if (!wait(C::BAR_PV_DONE, static_cast<uint32_t>((ts - 1) & 1))) return;
          tc_fence_after();
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
      }
      const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
      const uint64_t scale2 = f32x2(sl2, sl2), shift2 = f32x2(-m_use, -m_use);
      uint64_t sum2 = f32x2(0.f, 0.f);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int c = half * 64 + 2 * e;
          float x0, x1, p0, p1;
          f32x2_split(fma_f32x2(f32x2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), scale2,
                                shift2),
                      x0, x1);
          p0 = ex2_approx(x0);
          p1 = ex2_approx(x1);
          pk[e] = pack_bf16x2(p0, p1);
          sum2 = add_f32x2(sum2, f32x2(p0, p1));
        }
        tmem_st32(tSb + 32 * half, pk);
      }
      float a0, a1;
      f32x2_split(sum2, a0, a1);
      l += a0 + a1;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(x.bar(C::BAR_P_FULL + (ts & 1)));
    }
    // Piece end: O out of tensor memory, partial (O, m_ref, l) to the slot.
    if (!wait(C::BAR_O_FULL, pc & 1)) return;
    tc_fence_after();
    const long long slot = static_cast<long long>(blockIdx.x) + w.b * p.Hkv + w.g;
    float *po = p.part_o + (slot * p.part_rows + r) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      tmem_ld32(tO + 32 * c, o);
      tmem_wait_ld();
      if (valid) {
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4 *>(po + 32 * c + e) =
              make_float4(__uint_as_float(o[e]), __uint_as_float(o[e + 1]),
                          __uint_as_float(o[e + 2]), __uint_as_float(o[e + 3]));
      }
    }
    tc_fence_before();
    mbar_arrive(x.bar(C::BAR_O_EMPTY));
    if (valid) {
      float *pml = p.part_ml + (slot * p.part_rows + r) * 2;
      pml[0] = m_ref;
      pml[1] = l;
    }
    ++pc;
  }
}

template <int D>
__global__ void __launch_bounds__(DecodeRowsCfg<D>::THREADS, 1)
    fa_decode_rows_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
  using C = DecodeRowsCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *smem = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // softmax threads at work: the warps that hold query rows
  const int rows = p.group * p.Nq;
  const int busy = min(4, (rows + 31) / 32) * 32;

  DecRowsCtx<D> x;
  x.smem = base;
  x.abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
  long long *share = reinterpret_cast<long long *>(smem + C::OFF_MISC + 8);  // t0, t1
  int *start = reinterpret_cast<int *>(smem + C::OFF_MISC + 24);            // b, g, i

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(x.bar(C::BAR_K_FULL + s), 1);
      mbar_init(x.bar(C::BAR_K_EMPTY + s), 1);
      mbar_init(x.bar(C::BAR_V_FULL + s), 1);
      mbar_init(x.bar(C::BAR_V_EMPTY + s), 1);
    }
    mbar_init(x.bar(C::BAR_Q_FULL), 1);
    mbar_init(x.bar(C::BAR_Q_EMPTY), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(x.bar(C::BAR_S_FULL + i), 1);
      mbar_init(x.bar(C::BAR_P_FULL + i), busy);
    }
    mbar_init(x.bar(C::BAR_PV_DONE), 1);
    mbar_init(x.bar(C::BAR_O_FULL), 1);
    mbar_init(x.bar(C::BAR_O_EMPTY), busy);
    mbar_init(x.bar(C::BAR_MMA_DONE), 1);
    *x.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(base + C::OFF_MISC, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 5) {
    long long T, t0, t1;
    int sb, sg, si;
    dec_locate(p, lane, T, t0, t1, sb, sg, si);
    if (lane == 0) {
      share[0] = t0;
      share[1] = t1;
      start[0] = sb;
      start[1] = sg;
      start[2] = si;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  x.tmem = *reinterpret_cast<volatile uint32_t *>(smem + C::OFF_MISC);
  // The merge kernel may be scheduled now; it waits for this grid to finish
  // (griddepcontrol.wait) before it reads a partial.
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  DecCursor cur;
  cur.t = share[0];
  cur.t1 = share[1];
  cur.b = start[0];
  cur.g = start[1];
  cur.i = start[2];
  cur.L = cur.t < cur.t1 ? dec_len(p, cur.b) : 0;
  cur.n = dec_tiles(cur.L);

  if (warp < 4) {
    if (threadIdx.x < busy) decr_role_softmax<D>(x, p, cur);
  } else if (warp == 4) {
    if (lane == 0) decr_role_producer<D, false>(x, p, cur, &tm_q, &tm_k);
  } else if (warp == 6) {
    if (lane == 0) decr_role_producer<D, true>(x, p, cur, &tm_q, &tm_v);
  } else {
    decr_role_mma<D>(x, p, cur);
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
