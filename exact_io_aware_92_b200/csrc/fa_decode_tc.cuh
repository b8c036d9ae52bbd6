// Decode forward on the tensor cores: up to 16 query rows per (batch, kv
// head) against a long key/value cache, for the same operation and results
// as fa_decode.cuh (wiki note "FlashAttention", section "what it is": the
// blockwise running max / sum / output recurrence; section on common
// misconceptions: one generated token is bound by reading the cache).
//
// Why tensor cores for an HBM-bound path.  Both products are contractions:
// S^T = K Q^T over d, and O^T = V^T P^T over the keys.  With 4 query rows per
// kv head, doing them on CUDA cores costs 8 FMAs per cached bf16 pair (K and
// V), which at the B200's HBM rate is about 70 % of the SMs' FP32 FMA
// throughput before any unpacking or softmax work; the tensor cores do them
// with a handful of instructions per 128-key tile, so the kernel is left to
// stream K and V.
//
// Work split.  The call's key tiles (128 keys) form one sequence: for every
// (batch b, kv head g) with L_b valid keys, ceil(L_b / 128) tiles.  CTA c of
// the grid takes tiles [c T / grid, (c+1) T / grid): equal shares whatever
// the cache lengths.  The part of a CTA's share that lies in one (b, g) is a
// piece; it produces one partial (O, m, l) per query row in workspace slot
// c + (b Hkv + g), which is unique per piece.  A second kernel merges each
// row's pieces through their log-sum-exp; it is launched as a programmatic
// dependent of this one (this kernel triggers it after set-up, and it waits
// for this grid to finish before it reads a partial).
//
// Roles (224 threads, one CTA per SM):
//   warps 0-3  softmax: thread t owns key t of the tile (tensor-memory lane t)
//              and the NR query-row columns of S^T;
//   warp 4     TMA producer of the Q rows of each piece and of the K tiles;
//   warp 6     TMA producer of the V tiles.  K and V have rings of their own:
//              a K slot frees when its S^T product is done, a V slot when its
//              PV product is, so K runs further ahead than V;
//   warp 5     MMA issuer: S^T = K Q^T (M 128 keys, N 16 rows, K = d) and
//              O^T += V^T P^T (M = d, or at d = 64 two key halves stacked,
//              N 16 or 32, K = 128 keys), accumulators in tensor memory.
// The row max is shared by the CTA: the four warps post their per-row warp
// maxima each tile (one mbarrier exchange); the reference max m_ref moves
// only when a tile's max exceeds it by more than 8 (log2 units), and then O^T
// and the row sums are rescaled.  P (bf16) goes to shared memory in the
// 128-byte-swizzled K-major layout the MMA reads.
#pragma once

#include <cstdint>

#include "fa_decode.cuh"
#include "sm100_ptx.cuh"

namespace fa {

template <int D>
struct DecodeTcCfg {
  static_assert(D == 64 || D == 128, "head dim 64 or 128");
  static constexpr int BN = 128;                    // keys per tile (M of S^T)
  static constexpr int QROWS = 16;                  // query-row slots per piece (N of S^T)
  static constexpr int TILE_BYTES = BN * D * 2;     // one K or V tile
  static constexpr int NBOX = D / 64;               // 64-column TMA boxes per row
  static constexpr int BOX_BYTES = BN * 128;        // one box of a K/V tile
  static constexpr int STAGES = D == 128 ? 3 : 6;   // per ring: 192 KB of K and V
  static constexpr int Q_BOX_BYTES = QROWS * 128;   // one box of the Q rows
  static constexpr int Q_BYTES = NBOX * Q_BOX_BYTES;
  static constexpr int P_BYTES = QROWS * BN * 2;    // P^T of one tile, bf16
  // PV product: N = 16 rows at d = 128; at d = 64 the MMA's 128 rows are
  // (d, keys 0-63) and (d, keys 64-127), and the B operand stacks the two key
  // halves of P as 32 rows, so N = 32.
  static constexpr int N_O = D == 128 ? 16 : 32;
  static constexpr int OFF_KV = 0;
  static constexpr int OFF_V = OFF_KV + STAGES * TILE_BYTES;  // K ring, then V ring
  static constexpr int OFF_Q = OFF_V + STAGES * TILE_BYTES;
  static constexpr int OFF_P = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_XO = OFF_P + 2 * P_BYTES;
  // d = 64: warps 2-3 hand their half of O^T to warps 0-1 ([2][2 warps][32][16] fp32)
  static constexpr int XO_BYTES = D == 64 ? 2 * 2 * 32 * QROWS * 4 : 0;
  static constexpr int OFF_XCH = OFF_XO + XO_BYTES;  // [2][4 warps][16] fp32
  static constexpr int OFF_BAR = OFF_XCH + 2 * 4 * QROWS * 4;
  static constexpr int BAR_K_FULL = 0;                   // [STAGES]
  static constexpr int BAR_K_EMPTY = STAGES;             // [STAGES]
  static constexpr int BAR_V_FULL = 2 * STAGES;          // [STAGES]
  static constexpr int BAR_V_EMPTY = 3 * STAGES;         // [STAGES]
  static constexpr int BAR_Q_FULL = 4 * STAGES;          // [2]
  static constexpr int BAR_Q_EMPTY = BAR_Q_FULL + 2;     // [2]
  static constexpr int BAR_S_FULL = BAR_Q_EMPTY + 2;     // [2]
  static constexpr int BAR_P_FULL = BAR_S_FULL + 2;      // [2]
  static constexpr int BAR_P_EMPTY = BAR_P_FULL + 2;     // [2]: the PV product that read it is done
  static constexpr int BAR_O_FULL = BAR_P_EMPTY + 2;     // [2]
  static constexpr int BAR_O_EMPTY = BAR_O_FULL + 2;     // [2]
  static constexpr int BAR_XCH = BAR_O_EMPTY + 2;        // softmax warps' exchange
  static constexpr int BAR_MMA_DONE = BAR_XCH + 1;
  static constexpr int NUM_BARS = BAR_MMA_DONE + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;  // tmem base, abort, share, cursor
  static constexpr int SMEM_BYTES = OFF_MISC + 64;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;     // room to align the base to 1 KB
  static constexpr int THREADS = 224;
  static constexpr uint32_t TMEM_COLS = 128;
  static constexpr uint32_t COL_S = 0;    // S^T buffers at 0 and 32
  static constexpr uint32_t COL_O = 64;   // O^T buffers at 64 and 96
  static constexpr float RESCALE_THRESHOLD = 8.0f;
  static_assert(OFF_Q % 1024 == 0 && OFF_P % 1024 == 0 && Q_BYTES % 1024 == 0,
                "swizzled operands start on 1 KB boundaries");
  static_assert(SMEM_ALLOC <= 232448, "shared memory per CTA");
};

// Valid keys of sequence b, and its 128-key tiles.
__device__ __forceinline__ int dec_len(const DecodeParams &p, int b) {
  return p.seqlens ? min(max(p.seqlens[b], 0), p.Nk) : p.Nk;
}
__device__ __forceinline__ int dec_tiles(int L) { return (L + 127) >> 7; }

// A piece: tiles [i0, i0 + nt) of (batch b, kv head g), which has L keys.
struct DecPiece {
  int b, g, i0, nt, L;
};

// Walks a CTA's share [t, t1) of the tile sequence piece by piece.  Every
// role runs its own copy from the same start, so they see the same pieces.
struct DecCursor {
  int b, g, i, n, L;
  long long t, t1;

  __device__ bool next(const DecodeParams &p, DecPiece &pc) {
    if (t >= t1) return false;
    const int nt = static_cast<int>(min(static_cast<long long>(n - i), t1 - t));
    if (nt <= 0) return false;  // lengths changed under the kernel: stop
    pc.b = b;
    pc.g = g;
    pc.i0 = i;
    pc.nt = nt;
    pc.L = L;
    t += nt;
    i += nt;
    if (i == n && t < t1) {
      i = 0;
      if (++g == p.Hkv) {
        g = 0;
        n = 0;  // stays 0 past the last batch, which ends the walk
        while (n == 0 && b + 1 < p.B) {
          ++b;
          L = dec_len(p, b);
          n = dec_tiles(L);
        }
      }
    }
    return true;
  }
};

// One warp: T (tiles of the call), this CTA's share [t0, t1), and the
// (b, g, tile) where the share starts.
__device__ void dec_locate(const DecodeParams &p, int lane, long long &T, long long &t0,
                           long long &t1, int &sb, int &sg, int &si) {
  const unsigned full = 0xffffffffu;
  long long tiles = 0;  // per kv head
  for (int b0 = 0; b0 < p.B; b0 += 32) {
    const int b = b0 + lane;
    const int n = b < p.B ? dec_tiles(dec_len(p, b)) : 0;
    tiles += __reduce_add_sync(full, static_cast<unsigned>(n));
  }
  T = tiles * p.Hkv;
  const long long grid = gridDim.x, c = blockIdx.x;
  t0 = c * T / grid;
  t1 = (c + 1) * T / grid;
  sb = sg = si = 0;
  if (t0 >= t1) return;
  long long pre = 0;  // tiles per kv head of the batches before b0
  for (int b0 = 0; b0 < p.B; b0 += 32) {
    const int b = b0 + lane;
    const int n = b < p.B ? dec_tiles(dec_len(p, b)) : 0;
    int incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(full, incl, o);
      if (lane >= o) incl += y;
    }
    const unsigned hit = __ballot_sync(full, (pre + incl) * p.Hkv > t0);
    if (hit) {
      const int f = __ffs(hit) - 1;
      const int nf = __shfl_sync(full, n, f);
      const long long excl = pre + __shfl_sync(full, incl, f) - nf;
      const long long within = t0 - excl * p.Hkv;
      sb = b0 + f;
      sg = static_cast<int>(within / nf);
      si = static_cast<int>(within % nf);
      return;
    }
    pre += __shfl_sync(full, incl, 31);
  }
}

// tcgen05.ld / st of N consecutive 32-bit columns of this thread's lane.
template <int N>
__device__ __forceinline__ void tmem_ld_n(uint32_t taddr, uint32_t (&r)[N]) {
  static_assert(N == 4 || N == 8 || N == 16, "4, 8 or 16 columns");
  if constexpr (N == 4) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
  } else if constexpr (N == 8) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
  } else {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
  }
}
template <int N>
__device__ __forceinline__ void tmem_st_n(uint32_t taddr, const uint32_t (&r)[N]) {
  static_assert(N == 4 || N == 8 || N == 16, "4, 8 or 16 columns");
  if constexpr (N == 4) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3])
                 : "memory");
  } else if constexpr (N == 8) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(
                     taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
                 "r"(r[7])
                 : "memory");
  } else {
    tmem_st16(taddr, r);
  }
}

// Order this thread's shared-memory writes before later async-proxy reads
// (the tensor core reading P).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ float warp_max_f32(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// Round to bf16 (nearest even) and store the 16 bits.
__device__ __forceinline__ void st_shared_bf16(uint32_t addr, float v) {
  asm volatile(
      "{\n\t.reg .b16 h;\n\tcvt.rn.bf16.f32 h, %1;\n\tst.shared.b16 [%0], h;\n\t}" ::"r"(addr),
      "f"(v)
      : "memory");
}

template <int D>
struct DecTcCtx {
  using C = DecodeTcCfg<D>;
  uint32_t smem;  // 1 KB aligned shared base (shared-window address)
  uint8_t *smem_ptr;
  uint32_t tmem;
  volatile int *abort_flag;

  __device__ uint32_t bar(int i) const { return smem + C::OFF_BAR + 8 * i; }
  __device__ uint32_t k_tile(int stage) const { return smem + C::OFF_KV + stage * C::TILE_BYTES; }
  __device__ uint32_t v_tile(int stage) const { return smem + C::OFF_V + stage * C::TILE_BYTES; }
  __device__ uint32_t q_buf(int i) const { return smem + C::OFF_Q + i * C::Q_BYTES; }
  __device__ uint32_t p_buf(int i) const { return smem + C::OFF_P + i * C::P_BYTES; }
  __device__ float *xch(int i) const {
    return reinterpret_cast<float *>(smem_ptr + C::OFF_XCH) + i * 4 * C::QROWS;
  }
  __device__ float *xo(int i) const {
    return reinterpret_cast<float *>(smem_ptr + C::OFF_XO) + i * 2 * 32 * C::QROWS;
  }
};

// --------------------------------------------------------------------------
// TMA producers (one thread each): IS_V = false loads the Q rows and the K
// tiles, IS_V = true the V tiles.
// --------------------------------------------------------------------------
template <int D, bool IS_V>
__device__ void dec_role_producer(const DecTcCtx<D> &x, const DecodeParams &p, DecCursor cur,
                                  const CUtensorMap *tm_q, const CUtensorMap *tm_kv) {
  using C = DecodeTcCfg<D>;
  constexpr int FULL = IS_V ? C::BAR_V_FULL : C::BAR_K_FULL;
  constexpr int EMPTY = IS_V ? C::BAR_V_EMPTY : C::BAR_K_EMPTY;
  int ts = 0, pc = 0;
  bool ok = true;
  DecPiece w;
  while (ok && cur.next(p, w)) {
    if (!IS_V) {
      const int qb = pc & 1;
      if (!mbar_wait_bounded(x.bar(C::BAR_Q_EMPTY + qb), ((pc >> 1) & 1) ^ 1, x.abort_flag,
                             p.status, p.wait_limit_ns, kErrTimeout))
        break;
      mbar_arrive_expect_tx(x.bar(C::BAR_Q_FULL + qb), C::Q_BYTES);
      // the piece's query rows: heads g*G .. g*G+G-1, Nq rows each, contiguous
      const int row0 = (w.b * p.Hq + w.g * p.group) * p.Nq;
      for (int bx = 0; bx < C::NBOX; ++bx)
        tma_load_3d(x.q_buf(qb) + bx * C::Q_BOX_BYTES, tm_q, x.bar(C::BAR_Q_FULL + qb), bx * 64,
                    row0, 0);
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
  for (int q = 0; q < 2 && q < pc; ++q) {
    const int last = q + 2 * ((pc - 1 - q) / 2);
    mbar_wait_bounded(x.bar(C::BAR_Q_FULL + q), (last >> 1) & 1, &never, p.status,
                      p.wait_limit_ns, kErrTimeout);
  }
  for (int s = 0; s < C::STAGES && s < ts; ++s) {
    const int last = s + C::STAGES * ((ts - 1 - s) / C::STAGES);
    mbar_wait_bounded(x.bar(FULL + s), (last / C::STAGES) & 1, &never, p.status,
                      p.wait_limit_ns, kErrTimeout);
  }
}

// --------------------------------------------------------------------------
// MMA issuer (one warp; one elected lane issues)
// --------------------------------------------------------------------------
template <int D>
__device__ void dec_role_mma(const DecTcCtx<D> &x, const DecodeParams &p, DecCursor cur) {
  using C = DecodeTcCfg<D>;
  // S^T: A = K tile (keys x d, K-major), B = Q rows (K-major).
  // O^T: A = V tile read MN-major (d contiguous), B = P^T (K-major: a row of
  // keys per query row).
  constexpr uint32_t IDESC_S = idesc_bf16_f32(128, C::QROWS, 0, 0);
  constexpr uint32_t IDESC_O = idesc_bf16_f32(128, C::N_O, 1, 0);
  const bool leader = elect_one();
  // Buffer i of S^T / O^T is 32 columns after buffer 0; shared-memory
  // descriptors step in 16-byte units.  (Selects, not arrays, keep the
  // runtime buffer index out of local memory.)
  auto tS = [&](int i) { return x.tmem + C::COL_S + 32u * static_cast<uint32_t>(i); };
  auto tO = [&](int i) { return x.tmem + C::COL_O + 32u * static_cast<uint32_t>(i); };
  const uint64_t desc_k = smem_desc_sw128(x.k_tile(0), 16, 1024);
  // V: its 64-column boxes (d = 128), or its two 64-key halves (d = 64), are
  // the M chunks: leading byte offset between them, 8-key groups 1024 apart.
  const uint64_t desc_v = smem_desc_sw128(x.v_tile(0), D == 128 ? C::BOX_BYTES : 64 * 128, 1024);
  const uint64_t desc_q0 = smem_desc_sw128(x.q_buf(0), 16, 1024);
  const uint64_t desc_p0 = smem_desc_sw128(x.p_buf(0), 16, 1024);
  auto desc_q = [&](int i) { return desc_q0 + static_cast<uint64_t>(i * (C::Q_BYTES >> 4)); };
  auto desc_p = [&](int i) { return desc_p0 + static_cast<uint64_t>(i * (C::P_BYTES >> 4)); };
  constexpr uint32_t STAGE_STRIDE16 = C::TILE_BYTES >> 4;

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
  // O^T(piece) (+)= V^T P^T for one tile.
  auto issue_pv = [&](const Pend &q) {
    if (!wait(C::BAR_V_FULL + q.st, (q.ts / C::STAGES) & 1)) return false;
    if (!wait(C::BAR_P_FULL + (q.ts & 1), (q.ts >> 1) & 1)) return false;
    if (q.first && !wait(C::BAR_O_EMPTY + (q.pc & 1), ((q.pc >> 1) & 1) ^ 1)) return false;
    tc_fence_after();
    const uint64_t vd = desc_v + q.st * STAGE_STRIDE16;
    constexpr int KSTEPS = D == 128 ? 8 : 4;  // 16 keys each
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      const uint32_t poff = D == 128 ? (kk / 4) * 2048 + (kk % 4) * 32 : kk * 32;
      if (leader)
        tc_mma_ss(tO(q.pc & 1), vd + ((kk * 2048) >> 4), desc_p(q.ts & 1) + (poff >> 4), IDESC_O,
                  (!q.first || kk > 0) ? 1u : 0u);
    }
    __syncwarp();
    commit(C::BAR_P_EMPTY + (q.ts & 1));
    commit(C::BAR_V_EMPTY + q.st);
    if (q.last) commit(C::BAR_O_FULL + (q.pc & 1));
    return true;
  };

  int ts = 0, pc = 0;
  bool ok = true, have = false;
  Pend pend{};
  DecPiece w;
  while (ok && cur.next(p, w)) {
    const int qb = pc & 1;
    if (!wait(C::BAR_Q_FULL + qb, (pc >> 1) & 1)) break;
    for (int i = 0; i < w.nt; ++i, ++ts) {
      const int st = ts % C::STAGES;
      if (!wait(C::BAR_K_FULL + st, (ts / C::STAGES) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t kd = desc_k + st * STAGE_STRIDE16;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t koff = (kk / 4) * C::BOX_BYTES + (kk % 4) * 32;
        const uint32_t qoff = (kk / 4) * C::Q_BOX_BYTES + (kk % 4) * 32;
        if (leader)
          tc_mma_ss(tS(ts & 1), kd + (koff >> 4), desc_q(qb) + (qoff >> 4), IDESC_S,
                    kk > 0 ? 1u : 0u);
      }
      __syncwarp();
      commit(C::BAR_S_FULL + (ts & 1));
      commit(C::BAR_K_EMPTY + st);
      if (i == w.nt - 1) commit(C::BAR_Q_EMPTY + qb);
      // The previous tile's PV runs while the softmax works on this one.
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
  // Every MMA this warp issued must finish before tensor memory is freed.
  commit(C::BAR_MMA_DONE);
  volatile int never = 0;
  mbar_wait_bounded(x.bar(C::BAR_MMA_DONE), 0, &never, p.status, p.wait_limit_ns, kErrTimeout);
}

// --------------------------------------------------------------------------
// Softmax warps (128 threads; thread t = key t of a tile = TMEM lane t)
// --------------------------------------------------------------------------
template <int D, int NR>
__device__ void dec_role_softmax(const DecTcCtx<D> &x, const DecodeParams &p, DecCursor cur) {
  using C = DecodeTcCfg<D>;
  const int tid = threadIdx.x;
  const int wp = tid >> 5, lane = tid & 31;
  const uint32_t lane_off = static_cast<uint32_t>(wp * 32) << 16;
  // d = 64: warps 2-3 hold the keys 64-127 half of O^T in columns 16-31
  const uint32_t o_col = (D == 64 && wp >= 2) ? 16u : 0u;
  const int rows_total = p.group * p.Nq;
  // This key's byte offset inside a P^T buffer, without the row terms: the
  // 64-key box, the 16-byte chunk (swizzled by the row below) and the pair.
  const int kk = tid & 63;
  const uint32_t p_key = static_cast<uint32_t>((tid >> 6) * 2048 + (kk & 7) * 2);
  const uint32_t p_chunk = static_cast<uint32_t>(kk >> 3);

  auto wait = [&](int bar, uint32_t parity) {
    return mbar_wait_bounded(x.bar(bar), parity, x.abort_flag, p.status, p.wait_limit_ns,
                             kErrTimeout);
  };
  int ts = 0, pc = 0, xs = 0;  // tiles, pieces and exchanges so far
  // Post this warp's NR values (lane 0's) and collect all four warps'.
  auto exchange = [&](const float (&mine)[NR], float (&all)[4][NR]) {
    float *xb = x.xch(xs & 1);
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < NR; r += 4)
        *reinterpret_cast<float4 *>(xb + wp * C::QROWS + r) =
            make_float4(mine[r], mine[r + 1], mine[r + 2], mine[r + 3]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(x.bar(C::BAR_XCH));
    const bool ok = wait(C::BAR_XCH, xs & 1);
    ++xs;
    if (!ok) return false;
#pragma unroll
    for (int w4 = 0; w4 < 4; ++w4)
#pragma unroll
      for (int r = 0; r < NR; r += 4) {
        const float4 v = *reinterpret_cast<const float4 *>(xb + w4 * C::QROWS + r);
        all[w4][r] = v.x;
        all[w4][r + 1] = v.y;
        all[w4][r + 2] = v.z;
        all[w4][r + 3] = v.w;
      }
    return true;
  };

  DecPiece w;
  while (cur.next(p, w)) {
    // Visible keys [0, lim[r]) per row slot; slots past the rows get none.
    int lim[NR];
#pragma unroll
    for (int r = 0; r < NR; ++r)
      lim[r] = r < rows_total ? (p.causal ? min(w.L, w.L - p.Nq + (r % p.Nq) + 1) : w.L) : 0;
    float m_ref[NR], l[NR];
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      m_ref[r] = -INFINITY;
      l[r] = 0.f;
    }
    const uint32_t tO = x.tmem + C::COL_O + 32 * (pc & 1) + o_col + lane_off;
    for (int i = 0; i < w.nt; ++i, ++ts) {
      const int j = (w.i0 + i) * C::BN + tid;
      if (!wait(C::BAR_S_FULL + (ts & 1), (ts >> 1) & 1)) return;
      tc_fence_after();
      uint32_t sr[NR];
      tmem_ld_n<NR>(x.tmem + C::COL_S + 32 * (ts & 1) + lane_off, sr);
      tmem_wait_ld();
      float s[NR], tmax[NR];
#pragma unroll
      for (int r = 0; r < NR; ++r) {
        s[r] = j < lim[r] ? __uint_as_float(sr[r]) * p.scale_log2 : -INFINITY;
        tmax[r] = warp_max_f32(s[r]);
      }
      float all[4][NR];
      if (!exchange(tmax, all)) return;
      bool need = false;
#pragma unroll
      for (int r = 0; r < NR; ++r) {
        tmax[r] = fmaxf(fmaxf(all[0][r], all[1][r]), fmaxf(all[2][r], all[3][r]));
        need |= tmax[r] > m_ref[r] + C::RESCALE_THRESHOLD;
      }
      if (need) {  // the same decision in every thread: the inputs are shared
        float alpha[NR];
#pragma unroll
        for (int r = 0; r < NR; ++r) {
          const float m_new = fmaxf(m_ref[r], tmax[r]);
          alpha[r] = m_new == -INFINITY ? 1.f : ex2_approx(m_ref[r] - m_new);
          l[r] *= alpha[r];
          m_ref[r] = m_new;
        }
        if (i > 0) {
          // O^T holds this piece's earlier tiles once the last PV is done.
          const int tp = ts - 1;
          if (!wait(C::BAR_P_EMPTY + (tp & 1), (tp >> 1) & 1)) return;
          tc_fence_after();
          uint32_t o[NR];
          tmem_ld_n<NR>(tO, o);
          tmem_wait_ld();
#pragma unroll
          for (int r = 0; r < NR; ++r) o[r] = __float_as_uint(__uint_as_float(o[r]) * alpha[r]);
          tmem_st_n<NR>(tO, o);
          tmem_wait_st();
        }
      }
      // P buffer ts & 1 is free once the PV product of tile ts - 2 is done.
      if (!wait(C::BAR_P_EMPTY + (ts & 1), ((ts >> 1) & 1) ^ 1)) return;
      const uint32_t pb = x.p_buf(ts & 1) + p_key;
#pragma unroll
      for (int r = 0; r < NR; ++r) {
        const float mu = m_ref[r] == -INFINITY ? 0.f : m_ref[r];
        const float pr = ex2_approx(s[r] - mu);
        l[r] += pr;
        const uint32_t off = (r >> 3) * 1024 + (r & 7) * 128 + ((p_chunk ^ (r & 7)) << 4);
        st_shared_bf16(pb + off, pr);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(x.bar(C::BAR_P_FULL + (ts & 1)));
    }
    // Piece end: O^T from tensor memory, row sums over the CTA, partials out.
    if (!wait(C::BAR_O_FULL + (pc & 1), (pc >> 1) & 1)) return;
    tc_fence_after();
    uint32_t o[NR];
    tmem_ld_n<NR>(tO, o);
    tmem_wait_ld();
    tc_fence_before();
    mbar_arrive(x.bar(C::BAR_O_EMPTY + (pc & 1)));
    float lw[NR];
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      float v = l[r];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      lw[r] = v;
    }
    if constexpr (D == 64) {
      if (wp >= 2) {
        float *xo = x.xo(xs & 1) + ((wp - 2) * 32 + lane) * C::QROWS;
#pragma unroll
        for (int r = 0; r < NR; r += 4)
          *reinterpret_cast<float4 *>(xo + r) =
              make_float4(__uint_as_float(o[r]), __uint_as_float(o[r + 1]),
                          __uint_as_float(o[r + 2]), __uint_as_float(o[r + 3]));
      }
    }
    const int xo_buf = xs & 1;
    float all[4][NR];
    if (!exchange(lw, all)) return;
    const long long piece = static_cast<long long>(blockIdx.x) + w.b * p.Hkv + w.g;
    if (D == 128 || wp < 2) {
      float ov[NR];
#pragma unroll
      for (int r = 0; r < NR; ++r) ov[r] = __uint_as_float(o[r]);
      if constexpr (D == 64) {
        const float *xo = x.xo(xo_buf) + (wp * 32 + lane) * C::QROWS;
#pragma unroll
        for (int r = 0; r < NR; ++r) ov[r] += xo[r];
      }
      float *po = p.part_o + piece * C::QROWS * D + tid;
#pragma unroll
      for (int r = 0; r < NR; ++r)
        if (r < rows_total) po[r * D] = ov[r];
    }
    if (tid == 0) {
      float *pml = p.part_ml + piece * C::QROWS * 2;
#pragma unroll
      for (int r = 0; r < NR; ++r)
        if (r < rows_total) {
          pml[2 * r] = m_ref[r];
          pml[2 * r + 1] = all[0][r] + all[1][r] + all[2][r] + all[3][r];
        }
    }
    ++pc;
  }
}

template <int D, int NR>
__global__ void __launch_bounds__(DecodeTcCfg<D>::THREADS, 1)
    fa_decode_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
  using C = DecodeTcCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *smem = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  DecTcCtx<D> x;
  x.smem = base;
  x.smem_ptr = smem;
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
    for (int i = 0; i < 2; ++i) {
      mbar_init(x.bar(C::BAR_Q_FULL + i), 1);
      mbar_init(x.bar(C::BAR_Q_EMPTY + i), 1);
      mbar_init(x.bar(C::BAR_S_FULL + i), 1);
      mbar_init(x.bar(C::BAR_P_FULL + i), 128);
      mbar_init(x.bar(C::BAR_P_EMPTY + i), 1);
      mbar_init(x.bar(C::BAR_O_FULL + i), 1);
      mbar_init(x.bar(C::BAR_O_EMPTY + i), 128);
    }
    mbar_init(x.bar(C::BAR_XCH), 4);
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
  if (threadIdx.x < 128) {
    // P^T rows past the query rows stay zero (they only feed unused columns).
    uint4 *pz = reinterpret_cast<uint4 *>(smem + C::OFF_P);
    for (int i = threadIdx.x; i < 2 * C::P_BYTES / 16; i += 128) pz[i] = make_uint4(0, 0, 0, 0);
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
    dec_role_softmax<D, NR>(x, p, cur);
  } else if (warp == 4) {
    if (lane == 0) dec_role_producer<D, false>(x, p, cur, &tm_q, &tm_k);
  } else if (warp == 6) {
    if (lane == 0) dec_role_producer<D, true>(x, p, cur, &tm_q, &tm_v);
  } else {
    dec_role_mma<D>(x, p, cur);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(x.tmem, C::TMEM_COLS);
  }
}

// Merge of the pieces, one warp per query row: the pieces of (b, g) are
// those of the CTAs whose shares meet its tiles.  Serves both tensor-core
// split kernels (this file's and fa_decode_rows.cuh's): their workspace slots
// hold p.part_rows row slots each.
template <int D>
__global__ void __launch_bounds__(128) fa_decode_tc_combine_kernel(const DecodeParams p) {
  const int QROWS = p.part_rows;  // row slots per workspace slot
  constexpr int PER = D / 32;
  const int lane = threadIdx.x & 31;
  const int R = p.group * p.Nq;
  const long long idx = static_cast<long long>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  if (idx >= static_cast<long long>(p.B) * p.Hkv * R) return;
  const int b = static_cast<int>(idx / (static_cast<long long>(p.Hkv) * R));
  const int g = static_cast<int>((idx / R) % p.Hkv), r = static_cast<int>(idx % R);
  long long before = 0, all = 0;  // tiles per kv head: batches before b, every batch
  for (int i = lane; i < p.B; i += 32) {
    const int n = dec_tiles(dec_len(p, i));
    all += n;
    if (i < b) before += n;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    before += __shfl_xor_sync(0xffffffffu, before, off);
    all += __shfl_xor_sync(0xffffffffu, all, off);
  }
  const long long T = all * p.Hkv, grid = p.ctas;
  const int n = dec_tiles(dec_len(p, b));
  const size_t row = (static_cast<size_t>(b) * p.Hq + static_cast<size_t>(g) * p.group) * p.Nq + r;
  uint16_t *orow = p.o + row * D + lane * PER;
  if (n == 0) {
#pragma unroll
    for (int e = 0; e < PER; e += 2) *reinterpret_cast<uint32_t *>(orow + e) = 0u;
    if (lane == 0) p.lse[row] = -INFINITY;
    return;
  }
  auto start = [&](long long c) { return c * T / grid; };
  // the CTA whose share holds tile t: the largest c with start(c) <= t
  auto cta_of = [&](long long t) { return ((t + 1) * grid + T - 1) / T - 1; };
  const long long s = static_cast<long long>(b) * p.Hkv + g;
  const long long off = before * p.Hkv + static_cast<long long>(g) * n;
  const long long c0 = cta_of(off), c1 = cta_of(off + n - 1);
  const unsigned full = 0xffffffffu;
  // Launched as a programmatic dependent of the split kernel: everything
  // above overlapped its tail; the partials are read only after it is done.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // The row's pieces, 32 at a time, one per lane: (m, l) of each first and
  // the row max M, then each lane's weight 2^(m - M), and the weighted O
  // rows with 8 pieces' loads in flight at a time.  With at most 32 pieces
  // (the usual case) every (m, l) is read once.
  // share c holds tiles unless the call has fewer tiles than CTAs
  auto has = [&](long long c) { return T >= grid || start(c + 1) > start(c); };
  const float2 *ml_all = reinterpret_cast<const float2 *>(p.part_ml);
  auto load_ml = [&](long long cb) {
    const long long c = cb + lane;
    return c <= c1 && has(c) ? ml_all[(c + s) * QROWS + r] : make_float2(-INFINITY, 0.f);
  };
  const float2 ml0 = load_ml(c0);
  float M = warp_max_f32(ml0.x);
  for (long long cb = c0 + 32; cb <= c1; cb += 32) M = fmaxf(M, warp_max_f32(load_ml(cb).x));
  const float mu = M == -INFINITY ? 0.f : M;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float L = 0.f;
  for (long long cb = c0; cb <= c1; cb += 32) {
    const float2 ml = cb == c0 ? ml0 : load_ml(cb);
    const float wgt = ml.x == -INFINITY ? 0.f : ex2_approx(ml.x - mu);
    L += wgt * ml.y;
    const int cnt = static_cast<int>(min(32ll, c1 - cb + 1));
    for (int j0 = 0; j0 < cnt; j0 += 8) {
      float wj[8], v[8][PER];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        wj[u] = j0 + u < cnt ? __shfl_sync(full, wgt, (j0 + u) & 31) : 0.f;
        const float *po = p.part_o + ((cb + j0 + u + s) * QROWS + r) * D + lane * PER;
        if constexpr (PER == 4) {
          const float4 x = wj[u] != 0.f ? *reinterpret_cast<const float4 *>(po)
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
          v[u][0] = x.x;
          v[u][1] = x.y;
          v[u][2] = x.z;
          v[u][3] = x.w;
        } else {
          const float2 x = wj[u] != 0.f ? *reinterpret_cast<const float2 *>(po)
                                        : make_float2(0.f, 0.f);
          v[u][0] = x.x;
          v[u][1] = x.y;
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] += wj[u] * v[u][e];
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(full, L, o);
  const float inv = L > 0.f ? 1.0f / L : 0.f;
#pragma unroll
  for (int e = 0; e < PER; e += 2)
    *reinterpret_cast<uint32_t *>(orow + e) = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
  if (lane == 0) p.lse[row] = L > 0.f ? (M + __log2f(L)) * 0.69314718055994530942f : -INFINITY;
}

}  // namespace fa
