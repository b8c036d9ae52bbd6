// Exact attention forward on B200 tensor cores (sm_100a): one fused kernel
// that streams K/V tiles past two resident Q tiles and keeps the running row
// max, row sum and unnormalised output on chip (wiki note "FlashAttention",
// section "what it is": fix a Q block on chip, stream K, V blocks, update
// m' = max(m, max S_b), l' = e^(m-m') l + sum e^(S_b - m'),
// O' = (e^(m-m') l O + e^(S_b - m') V_b) / l').  Only O and LSE reach HBM.
//
// Work unit = (batch, query head, pair of 128-row Q tiles).  The kernel is
// persistent: one CTA per SM walks the units, heaviest first (for causal
// attention the last Q-tile pair sees the most keys), in "snake" order (every
// other round of gridDim.x units is taken in reverse), which balances the
// causal triangle across SMs.  Barrier phases run on across units, so the
// next unit's Q tiles load while the current unit's last products and
// epilogue run.
//   warps 0-3  softmax warpgroup for Q tile 0 (thread r owns row r = TMEM lane r)
//   warps 4-7  softmax warpgroup for Q tile 1
//   warp  8    TMA producer: Q tiles per unit, then K_j, V_j into a ring of stages
//   warp  9    MMA issuer: S_t = Q_t K_j^T and O_t += P_t V_j with tcgen05.mma
//              (role_mma_split at d = 128, role_mma_triple at d = 64)
//   warps 10-11 idle (they complete the third warpgroup, whose registers go
//              to the softmax warpgroups)
// Tensor memory (512 columns, fp32): S0 [0,128) S1 [128,256) O0 [256,256+d)
// O1 [384,384+d).  P_t (bf16, two per column; FP8: four E4M3 codes per
// column) is published in two halves of 64 keys so the PV product starts on
// the first half while the second is computed.  The first half overwrites the
// first columns of S_t and feeds the PV product straight from tensor memory.  At d = 128 the
// second half goes to a 16 KB shared-memory tile per Q tile (K-major,
// 128-byte swizzled), so S_t of the next key tile is issued right after the
// first half's PV product, while the softmax still computes the second half;
// at d = 64 (three S buffers) it overwrites columns 32-63.
// In a causal unit, Q tile 0 skips the last key tile when it lies wholly above
// its rows (Q tile 1 still needs it).
//
// The same body serves FP8 E4M3 inputs (F8 = true, head dim 128): 8-bit
// tiles, kind::f8f6f4 products, V given transposed so both products read
// K-major operands, and P stored as E4M3 (its second half in the first 64
// bytes of each shared-memory row) with a factor 2^2 and a rescale threshold
// of 6 (log2 units) so it never saturates.
//
// Differences from the pages' statement of the recurrence, all algebraically
// equivalent: O is kept unnormalised (O~ = l * O) and divided by l once at the
// end; exponentials are base 2 on log2(e)-scaled scores; the max used for the
// exponentials (m_ref) is only moved when the row max grows by more than
// 2^8 (bf16; 2^6 for FP8), so most tiles skip the O rescale (values stay
// below 2^8, far from fp32 overflow).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace fa {

// Division of non-negative 31-bit integers by a divisor fixed for the whole
// launch, without a division instruction sequence: with l = ceil(log2 d) and
// m = floor(2^32 (2^l - d) / d) + 1, n / d = (umulhi(n, m) + n) >> l
// (Granlund and Montgomery, "Division by invariant integers using
// multiplication", 1994).  The sum cannot overflow: n < 2^31 and
// umulhi(n, m) <= n.
struct FastDiv {
  uint32_t d, m, l;
  __device__ __forceinline__ int div(int n) const {
    const uint32_t un = static_cast<uint32_t>(n);
    return static_cast<int>((__umulhi(un, m) + un) >> l);
  }
};

inline FastDiv make_fast_div(uint32_t d) {
  FastDiv f;
  f.d = d;
  f.l = 0;
  while ((1ull << f.l) < d) ++f.l;
  f.m = static_cast<uint32_t>(((1ull << 32) * ((1ull << f.l) - d)) / d + 1);
  return f;
}

struct FwdParams {
  uint16_t *o;           // bf16 [B, Hq, N, d], or [total, Hq, d] when packed
  float *lse;            // fp32 [B, Hq, N], or [Hq, total] when packed
  const int *seqlens;    // int32 [B] key lengths or nullptr
  const int *cu_seqlens; // packed layout: int32 [B+1] token offsets, else nullptr
  int total;             // packed layout: tokens in all sequences
  int *status;           // device status word (time-outs)
  int B, Hq, Hkv, N, group;
  FastDiv div_bh, div_hq, div_group;  // by B * Hq, Hq and group
  int num_qpairs;        // ceil(N / 256)
  int num_units;         // B * Hq * num_qpairs
  int causal;
  float scale_log2;      // scale * log2(e) (times the Q and K descales for FP8 inputs)
  float out_scale;       // FP8 inputs: the V descale, applied with 1/l; 1 otherwise
  unsigned long long wait_limit_ns;
};

// F8: Q, K and V are FP8 E4M3 codes (head dim 128 only) and V arrives
// transposed ([d, keys], keys contiguous), so both products read K-major
// operands; otherwise bf16.
// V, the launch variant (bit flags):
//  kVarSkip0: causal launches at d = 64, where Q tile 0 skips a unit's last
//    key tile inside the three-buffer sequence;
//  kVarPacked: the packed layout (cu_seqlens), whose unit decode and tensor
//    map coordinates differ; dense launches compile without that branch.
constexpr int kVarSkip0 = 1;
constexpr int kVarPacked = 2;

template <int D, bool F8 = false, int V = 0>
struct Sm100Cfg {
  static_assert(D == 64 || D == 128, "head dim 64 or 128");
  static_assert(!F8 || D == 128, "FP8 inputs: head dim 128");
  static constexpr int EB = F8 ? 1 : 2;           // bytes per input element
  static constexpr int BM = 128;                  // query rows per Q tile
  static constexpr int BN = 128;                  // keys per K/V tile
  static constexpr int ROWS_PER_UNIT = 2 * BM;
  static constexpr int BOX_BYTES = 128 * 128;     // one TMA box: 128 rows x 128 bytes
  static constexpr int BOX_COLS = 128 / EB;       // elements in a box row
  static constexpr int TILE_BYTES = 128 * D * EB; // one Q, K or V tile
  static constexpr int NBOX = TILE_BYTES / BOX_BYTES;
  static constexpr int KSTEPS = D * EB / 32;      // 32-byte K steps of the S product
  static constexpr int STAGES = (TILE_BYTES == 32768) ? 4 : 8;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = OFF_Q + 2 * TILE_BYTES;
  // d = 128: the upper 64 keys of P go to shared memory (K-major, 128-byte
  // swizzled: 128 rows of 128 bytes, like a Q tile of 64 bf16 columns; E4M3
  // codes fill the first 64 bytes of each row) instead of tensor memory, so
  // the next S product may overwrite S_t as soon as the PV product has read
  // the lower half.  (At d = 64 the three S
  // buffers already decouple S from P, and the extra shared-memory stores
  // only lengthen the softmax, which bounds that head dimension.)
  static constexpr bool P_HI_SMEM = D == 128;
  static constexpr int P_HI_BYTES = 128 * 128;
  static constexpr int OFF_PHI = OFF_KV + STAGES * TILE_BYTES;  // [2 Q tiles]
  static constexpr int OFF_BAR = OFF_PHI + (P_HI_SMEM ? 2 * P_HI_BYTES : 0);
  // barrier indices
  static constexpr int BAR_Q_FULL = 0;                  // [2 tiles]
  static constexpr int BAR_Q_EMPTY = 2;                 // [2 tiles]
  static constexpr int BAR_KV_FULL = 4;                 // [STAGES]
  static constexpr int BAR_KV_EMPTY = 4 + STAGES;       // [STAGES]
  // D = 64 (bf16): tensor memory has room for a third S buffer.  Three
  // buffers rotate over the CTA's sequence of S products (both Q tiles
  // interleaved), so a Q tile's next S is computed while it still works on
  // the current one.
  static constexpr bool TRIPLE = (D == 64) && !F8;
  static constexpr bool SKIP0 = TRIPLE && (V & kVarSkip0) != 0;
  static constexpr bool PACKED = (V & kVarPacked) != 0;
  static constexpr int NSBUF = TRIPLE ? 3 : 2;
  static constexpr int BAR_S_FULL = 4 + 2 * STAGES;     // [NSBUF]
  static constexpr int BAR_P_HALF = BAR_S_FULL + NSBUF; // [NSBUF][2 halves of the keys]
  static constexpr int BAR_O_FULL = BAR_P_HALF + 2 * NSBUF;  // [2 tiles]
  static constexpr int BAR_MMA_DONE = BAR_O_FULL + 2;   // 1
  // [2 tiles] (TRIPLE or P_HI_SMEM): a Q tile's whole PV product landed
  static constexpr int BAR_PV_DONE = BAR_MMA_DONE + 1;
  static constexpr bool HAS_PV_DONE = TRIPLE || P_HI_SMEM;
  static constexpr int NUM_BARS = BAR_PV_DONE + (HAS_PV_DONE ? 2 : 0);
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;  // tmem base, abort flag
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;     // room to align the base to 1 KB
  static constexpr int THREADS = 384;
  // Registers per thread: 168 at launch (65536 / 384, rounded down to 8);
  // the producer/MMA warpgroup gives some up to the two softmax warpgroups.
  // 128 * REGS_CONTROL + 256 * REGS_SOFTMAX = 384 * 168.
  static constexpr uint32_t REGS_LAUNCH = 168;
  static constexpr uint32_t REGS_CONTROL = 56;
  static constexpr uint32_t REGS_SOFTMAX = 224;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S0 = 0;
  static constexpr uint32_t COL_O0 = TRIPLE ? 384 : 256;  // O0; O1 is O_STRIDE further
  static constexpr uint32_t O_STRIDE = TRIPLE ? 64 : 128;
  // The reference max moves when the row max grows by more than this (log2
  // units).  FP8: P is stored as E4M3 (largest finite 448) and carries a
  // factor 2^P_SHIFT that keeps small probabilities out of the subnormal
  // range, so P <= 2^(threshold + shift) = 256 must hold.  A shift of 2 with
  // a threshold of 6 sends about 3% of (warp, key tile) steps through the
  // rescale path on the GQA workload (4 and 4: about 19%) for a mean output
  // error within 4% of the 4-and-4 split.
  static constexpr float RESCALE_THRESHOLD = F8 ? 6.0f : 8.0f;
  static constexpr float P_SHIFT = F8 ? 2.0f : 0.0f;
  static constexpr int PK_WORDS = F8 ? 16 : 32;   // 32-bit words of P per 64 keys
  // Of every 8 consecutive pairs of probabilities, this many are computed on
  // the FMA pipe (exp2_poly_pair) instead of the MUFU pipe.  At d = 128 the
  // exponentials alone keep the MUFU pipe as busy as the MMAs keep the
  // tensor pipe; at d = 64 the MMAs take half as long, so more move over.
#ifndef FA_EXP2_EMU_PAIRS_D64
#define FA_EXP2_EMU_PAIRS_D64 2
#endif
#ifndef FA_EXP2_EMU_PAIRS_D128
#define FA_EXP2_EMU_PAIRS_D128 2
#endif
#ifndef FA_EXP2_EMU_PAIRS_F8
#define FA_EXP2_EMU_PAIRS_F8 2
#endif
  static constexpr int EXP2_EMU_PAIRS =
      F8 ? FA_EXP2_EMU_PAIRS_F8 : D == 64 ? FA_EXP2_EMU_PAIRS_D64 : FA_EXP2_EMU_PAIRS_D128;
};

// One work unit, as every role sees it.  Rows and keys are counted from the
// start of the unit's sequence; tok0 is where that sequence starts in the
// packed layout (0 otherwise).
struct Unit {
  int b, h, hkv, bh, row0, L, nkv;
  int nkv0;        // key tiles Q tile 0 needs: causal units skip a last tile
                   // that lies wholly above tile 0's rows
  int q_rows;      // query rows that exist (N, or the sequence length when packed)
  int tok0;        // first token of the sequence (packed layout)
  int q_plane;     // TMA plane of Q: b*Hq+h, or h when packed
  int kv_plane;    // TMA plane of K/V: b*Hkv+hkv, or hkv when packed
  size_t o_base;   // element offset of row 0 of this (sequence, head) in O
  size_t o_stride; // elements between consecutive rows of O
  size_t lse_base; // offset of row 0 in LSE
};

template <int D, bool F8, int V>
__device__ __forceinline__ Unit unit_at(const FwdParams &p, int u) {
  using C = Sm100Cfg<D, F8, V>;
  Unit x;
  const int BH = p.B * p.Hq;
  const int q_bh = p.div_bh.div(u);
  const int qp = p.num_qpairs - 1 - q_bh;
  x.bh = u - q_bh * BH;
  x.b = p.div_hq.div(x.bh);
  x.h = x.bh - x.b * p.Hq;
  x.hkv = p.div_group.div(x.h);
  x.row0 = qp * C::ROWS_PER_UNIT;
  int L = p.N;
  if constexpr (C::PACKED) {
    x.tok0 = p.cu_seqlens[x.b];
    L = max(p.cu_seqlens[x.b + 1] - x.tok0, 0);
    x.q_rows = L;
    x.q_plane = x.h;
    x.kv_plane = x.hkv;
    x.o_base = (static_cast<size_t>(x.tok0) * p.Hq + x.h) * D;
    x.o_stride = static_cast<size_t>(p.Hq) * D;
    x.lse_base = static_cast<size_t>(x.h) * p.total + x.tok0;
  } else {
    if (p.seqlens) L = min(max(p.seqlens[x.b], 0), p.N);
    x.tok0 = 0;
    x.q_rows = p.N;
    x.q_plane = x.bh;
    x.kv_plane = x.b * p.Hkv + x.hkv;
    x.o_base = static_cast<size_t>(x.bh) * p.N * D;
    x.o_stride = D;
    x.lse_base = static_cast<size_t>(x.bh) * p.N;
  }
  x.L = L;
  const int kv_end = p.causal ? min(L, x.row0 + C::ROWS_PER_UNIT) : L;
  // A unit past the end of its sequence (packed layout) has no rows at all.
  x.nkv = x.row0 < x.q_rows ? (kv_end + C::BN - 1) / C::BN : 0;
  x.nkv0 = ((!C::TRIPLE || C::SKIP0) && p.causal && x.nkv > 1 &&
             (x.nkv - 1) * C::BN >= x.row0 + C::BM)
               ? x.nkv - 1
               : x.nkv;
  return x;
}

// The k-th unit of this CTA in snake order, or -1 past the end / in a gap of
// the last, partial round.  Returns -2 when the rounds are exhausted.
__device__ __forceinline__ int snake_unit(int k, int num_units) {
  const int G = static_cast<int>(gridDim.x);
  const int base = k * G;
  if (base >= num_units) return -2;
  const int c = static_cast<int>(blockIdx.x);
  const int u = (k & 1) ? base + (G - 1 - c) : base + c;
  return u < num_units ? u : -1;
}

template <int D, bool F8, int V>
struct Sm100Ctx {
  using C = Sm100Cfg<D, F8, V>;
  uint32_t smem;      // 1 KB aligned shared base (shared-window address)
  uint32_t tmem;      // tensor-memory base address
  volatile int *abort_flag;

  __device__ uint32_t bar(int i) const { return smem + C::OFF_BAR + 8 * i; }
  __device__ uint32_t q_tile(int t) const { return smem + C::OFF_Q + t * C::TILE_BYTES; }
  __device__ uint32_t kv_tile(int slot) const { return smem + C::OFF_KV + slot * C::TILE_BYTES; }
  __device__ uint32_t p_hi(int t) const { return smem + C::OFF_PHI + t * C::P_HI_BYTES; }
};

// Ring position of K tile g (V tile g is the next one) in a CTA's stream.
template <int D, bool F8, int V>
__device__ __forceinline__ int ring_slot(int seq) { return seq % Sm100Cfg<D, F8, V>::STAGES; }
template <int D, bool F8, int V>
__device__ __forceinline__ uint32_t ring_parity(int seq) {
  return static_cast<uint32_t>((seq / Sm100Cfg<D, F8, V>::STAGES) & 1);
}

// --------------------------------------------------------------------------
// TMA producer (one thread)
// --------------------------------------------------------------------------
template <int D, bool F8, int V>
__device__ void role_producer(const Sm100Ctx<D, F8, V> &x, const FwdParams &p, const CUtensorMap *tm_q,
                              const CUtensorMap *tm_k, const CUtensorMap *tm_v) {
  using C = Sm100Cfg<D, F8, V>;
  int seq = 0;  // K/V tiles put into the ring so far (K and V counted apart)
  int qi = 0;   // units with keys loaded so far
  constexpr bool packed = C::PACKED;
  // K/V tiles are read by every query tile of their head, Q tiles once: keep
  // K/V in L2 ahead of Q (and of O, written with streaming stores).  On the
  // GQA layer this cut DRAM reads from 343 to 289 MB per launch.
  const uint64_t pol_kv = l2_policy_evict_last(), pol_q = l2_policy_evict_first();
  bool ok = true;
  for (int k = 0; ok; ++k) {
    const int u = snake_unit(k, p.num_units);
    if (u == -2) break;
    if (u < 0) continue;
    const Unit w = unit_at<D, F8, V>(p, u);
    if (w.nkv == 0) continue;
    // Q tile t of this unit replaces the previous unit's once its last
    // S product has read it.
    for (int t = 0; t < 2 && ok; ++t) {
      if (!mbar_wait_bounded(x.bar(C::BAR_Q_EMPTY + t), (qi & 1) ^ 1, x.abort_flag, p.status,
                             p.wait_limit_ns, kErrTimeout)) {
        ok = false;
        break;
      }
      mbar_arrive_expect_tx(x.bar(C::BAR_Q_FULL + t), C::TILE_BYTES);
      // The padded layout's maps are (d, rows, plane); the packed layout's
      // are (d, head, token), which keeps their strides increasing.
      const int qrow = w.tok0 + w.row0 + t * C::BM;
      for (int bx = 0; bx < C::NBOX; ++bx)
        tma_load_3d_hint(x.q_tile(t) + bx * C::BOX_BYTES, tm_q, x.bar(C::BAR_Q_FULL + t),
                         bx * C::BOX_COLS, packed ? w.q_plane : qrow, packed ? qrow : w.q_plane,
                         pol_q);
    }
    if (!ok) break;
    ++qi;
    const int kv_plane = w.kv_plane;
    for (int j = 0; j < w.nkv && ok; ++j) {
      for (int kv = 0; kv < 2; ++kv, ++seq) {
        const int slot = ring_slot<D, F8, V>(seq);
        if (!mbar_wait_bounded(x.bar(C::BAR_KV_EMPTY + slot), ring_parity<D, F8, V>(seq) ^ 1,
                               x.abort_flag, p.status, p.wait_limit_ns, kErrTimeout)) {
          ok = false;
          break;
        }
        const uint32_t full = x.bar(C::BAR_KV_FULL + slot);
        mbar_arrive_expect_tx(full, C::TILE_BYTES);
        const CUtensorMap *m = kv ? tm_v : tm_k;
        const int krow = w.tok0 + j * C::BN;
        if (F8 && kv) {
          // V^T tile: 128 keys (x, contiguous) by the d rows (y); one box.
          tma_load_3d_hint(x.kv_tile(slot), m, full, krow, 0, kv_plane, pol_kv);
        } else {
          for (int bx = 0; bx < C::NBOX; ++bx)
            tma_load_3d_hint(x.kv_tile(slot) + bx * C::BOX_BYTES, m, full, bx * C::BOX_COLS,
                             packed ? kv_plane : krow, packed ? krow : kv_plane, pol_kv);
        }
      }
    }
  }
  // Drain: every copy this thread started must land before the CTA may exit.
  volatile int never = 0;
  if (qi > 0)
    for (int t = 0; t < 2; ++t)
      mbar_wait_bounded(x.bar(C::BAR_Q_FULL + t), (qi - 1) & 1, &never, p.status,
                        p.wait_limit_ns, kErrTimeout);
  for (int s = 0; s < C::STAGES && s < seq; ++s) {
    const int last = s + C::STAGES * ((seq - 1 - s) / C::STAGES);
    mbar_wait_bounded(x.bar(C::BAR_KV_FULL + s), ring_parity<D, F8, V>(last), &never, p.status,
                      p.wait_limit_ns, kErrTimeout);
  }
}

// --------------------------------------------------------------------------
// MMA issuer for two S buffers with P's upper half in shared memory
// (D = 128, bf16 and FP8; every lane runs the loop and the waits, so the
// descriptor arithmetic stays warp-uniform, and one elected lane issues the
// tcgen05 instructions and their commits).  Per key tile j and Q tile t: PV_t(j-1) over the lower 64 keys
// (P from tensor memory), then S_t(j) into the same columns, then PV_t(j-1)
// over the upper 64 keys (P from shared memory).  S_t(j) thus waits only for
// the first half of the previous tile's probabilities.
// --------------------------------------------------------------------------
template <int D, bool F8, int V>
__device__ void role_mma_split(const Sm100Ctx<D, F8, V> &x, const FwdParams &p) {
  using C = Sm100Cfg<D, F8, V>;
  static_assert(C::P_HI_SMEM && !C::TRIPLE, "two S buffers, P's upper half in shared memory");
  // S: Q and K both K-major.  O: P K-major (tensor memory or shared memory);
  // V MN-major (bf16) or V^T K-major (FP8).
  constexpr uint32_t IDESC_S = F8 ? idesc_e4m3_f32(128, C::BN) : idesc_bf16_f32(128, C::BN, 0, 0);
  constexpr uint32_t IDESC_O = F8 ? idesc_e4m3_f32(128, D) : idesc_bf16_f32(128, D, 0, 1);
  const bool leader = elect_one();
  const uint32_t tS[2] = {x.tmem + C::COL_S0, x.tmem + C::COL_S0 + 128};
  const uint32_t tO[2] = {x.tmem + C::COL_O0, x.tmem + C::COL_O0 + C::O_STRIDE};
  const uint64_t desc_q[2] = {smem_desc_sw128(x.q_tile(0), 16, 1024),
                              smem_desc_sw128(x.q_tile(1), 16, 1024)};
  const uint64_t desc_p[2] = {smem_desc_sw128(x.p_hi(0), 16, 1024),
                              smem_desc_sw128(x.p_hi(1), 16, 1024)};
  const uint64_t desc_kv_k = smem_desc_sw128(x.kv_tile(0), 16, 1024);
  const uint64_t desc_kv_v = F8 ? smem_desc_sw128(x.kv_tile(0), 16, 1024)
                                : smem_desc_sw128(x.kv_tile(0), C::BOX_BYTES, 1024);
  auto wait = [&](int bar, uint32_t parity) {
    const bool ok = mbar_wait_bounded(x.bar(bar), parity, x.abort_flag, p.status,
                                      p.wait_limit_ns, kErrTimeout);
    return __all_sync(0xffffffffu, ok);
  };
  auto commit = [&](int bar) {
    if (leader) tc_commit(x.bar(bar));
    __syncwarp();
  };
  // S_t = Q_t K^T: K = d in steps of 32 bytes (16 bf16 or 32 FP8 values)
  // inside a 128-byte swizzled row; every 4 steps move to the next box.
  auto issue_s = [&](int t, int ks) {
    const uint64_t kd = desc_kv_k + ((ks * C::TILE_BYTES) >> 4);
#pragma unroll
    for (int kk = 0; kk < C::KSTEPS; ++kk) {
      const uint32_t off = ((kk / 4) * C::BOX_BYTES + (kk % 4) * 32) >> 4;
      if (leader) {
        if constexpr (F8)
          tc_mma_ss_f8(tS[t], desc_q[t] + off, kd + off, IDESC_S, kk > 0 ? 1u : 0u);
        else
          tc_mma_ss(tS[t], desc_q[t] + off, kd + off, IDESC_S, kk > 0 ? 1u : 0u);
      }
    }
    __syncwarp();
  };
  // O_t += P_t V over keys 0-63, P from tensor memory.  bf16: 16 keys per
  // step, 8 columns of P, V steps 16 key rows = 2048 bytes.  FP8: 32 keys per
  // step, 8 columns of P (four codes each), V^T steps 32 bytes of its rows.
  auto pv_lo = [&](int t, int vs, uint32_t parity, bool accumulate) {
    if (!wait(C::BAR_P_HALF + 2 * t, parity)) return false;
    tc_fence_after();
    const uint64_t vd = desc_kv_v + ((vs * C::TILE_BYTES) >> 4);
    if constexpr (F8) {
#pragma unroll
      for (int k2 = 0; k2 < 2; ++k2)
        if (leader)
          tc_mma_ts_f8(tO[t], tS[t] + k2 * 8, vd + ((k2 * 32) >> 4), IDESC_O,
                       (accumulate || k2 > 0) ? 1u : 0u);
    } else {
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4)
        if (leader)
          tc_mma_ts(tO[t], tS[t] + k4 * 8, vd + ((k4 * 2048) >> 4), IDESC_O,
                    (accumulate || k4 > 0) ? 1u : 0u);
    }
    __syncwarp();
    return true;
  };
  // O_t += P_t V over keys 64-127, P from shared memory (32 bytes per step
  // inside its 128-byte rows: 16 bf16 or 32 FP8 keys); then the whole
  // product is marked done.
  auto pv_hi = [&](int t, int vs, uint32_t parity) {
    if (!wait(C::BAR_P_HALF + 2 * t + 1, parity)) return false;
    tc_fence_after();
    const uint64_t vd = desc_kv_v + ((vs * C::TILE_BYTES) >> 4);
    if constexpr (F8) {
#pragma unroll
      for (int k2 = 0; k2 < 2; ++k2)
        if (leader)
          tc_mma_ss_f8(tO[t], desc_p[t] + ((k2 * 32) >> 4), vd + (((2 + k2) * 32) >> 4), IDESC_O,
                       1u);
    } else {
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4)
        if (leader)
          tc_mma_ss(tO[t], desc_p[t] + ((k4 * 32) >> 4), vd + (((4 + k4) * 2048) >> 4), IDESC_O,
                    1u);
    }
    __syncwarp();
    commit(C::BAR_PV_DONE + t);
    return true;
  };

  int g = 0;             // K/V tiles consumed by this CTA so far (ring position)
  int gs[2] = {0, 0};    // key tiles each Q tile has processed (its S/P phases)
  int qi = 0;            // units with keys processed so far
  bool ok = true;
  for (int k = 0; ok; ++k) {
    const int u = snake_unit(k, p.num_units);
    if (u == -2) break;
    if (u < 0) continue;
    const Unit w = unit_at<D, F8, V>(p, u);
    const int n1 = w.nkv, n0 = w.nkv0;  // n0 is n1 or n1 - 1
    if (n1 == 0) continue;
    const uint32_t qpar = static_cast<uint32_t>(qi & 1);
    if (!wait(C::BAR_Q_FULL + 0, qpar) || !wait(C::BAR_Q_FULL + 1, qpar) ||
        !wait(C::BAR_KV_FULL + ring_slot<D, F8, V>(2 * g), ring_parity<D, F8, V>(2 * g))) {
      ok = false;
      break;
    }
    tc_fence_after();
    issue_s(0, ring_slot<D, F8, V>(2 * g));
    commit(C::BAR_S_FULL + 0);
    if (n0 == 1) commit(C::BAR_Q_EMPTY + 0);
    issue_s(1, ring_slot<D, F8, V>(2 * g));
    commit(C::BAR_S_FULL + 1);
    commit(C::BAR_KV_EMPTY + ring_slot<D, F8, V>(2 * g));
    if (n1 == 1) commit(C::BAR_Q_EMPTY + 1);
    for (int j = 1; j < n1; ++j) {
      const int gp = g + j - 1, gc = g + j;
      const int vs = ring_slot<D, F8, V>(2 * gp + 1), ks = ring_slot<D, F8, V>(2 * gc);
      const uint32_t par0 = static_cast<uint32_t>((gs[0] + j - 1) & 1);
      const uint32_t par1 = static_cast<uint32_t>((gs[1] + j - 1) & 1);
      if (!wait(C::BAR_KV_FULL + vs, ring_parity<D, F8, V>(2 * gp + 1)) ||
          !pv_lo(0, vs, par0, j - 1 > 0) ||
          !wait(C::BAR_KV_FULL + ks, ring_parity<D, F8, V>(2 * gc))) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (j < n0) {
        issue_s(0, ks);
        commit(C::BAR_S_FULL + 0);
        if (j == n0 - 1) commit(C::BAR_Q_EMPTY + 0);
      }
      if (!pv_hi(0, vs, par0)) {
        ok = false;
        break;
      }
      if (j >= n0) commit(C::BAR_O_FULL + 0);  // Q tile 0's last PV was issued just above
      if (!pv_lo(1, vs, par1, j - 1 > 0)) {
        ok = false;
        break;
      }
      issue_s(1, ks);
      commit(C::BAR_S_FULL + 1);
      commit(C::BAR_KV_EMPTY + ks);
      if (j == n1 - 1) commit(C::BAR_Q_EMPTY + 1);
      if (!pv_hi(1, vs, par1)) {
        ok = false;
        break;
      }
      commit(C::BAR_KV_EMPTY + vs);
    }
    if (!ok) break;
    // Last tile's PV products, then the unit's output is complete.
    const int gl = g + n1 - 1;
    const int vs = ring_slot<D, F8, V>(2 * gl + 1);
    if (!wait(C::BAR_KV_FULL + vs, ring_parity<D, F8, V>(2 * gl + 1))) {
      ok = false;
      break;
    }
    if (n0 == n1) {
      const uint32_t par0 = static_cast<uint32_t>((gs[0] + n1 - 1) & 1);
      if (!pv_lo(0, vs, par0, n1 > 1) || !pv_hi(0, vs, par0)) {
        ok = false;
        break;
      }
      commit(C::BAR_O_FULL + 0);
    }
    const uint32_t par1 = static_cast<uint32_t>((gs[1] + n1 - 1) & 1);
    if (!pv_lo(1, vs, par1, n1 > 1) || !pv_hi(1, vs, par1)) {
      ok = false;
      break;
    }
    commit(C::BAR_O_FULL + 1);
    commit(C::BAR_KV_EMPTY + vs);
    g += n1;
    gs[0] += n0;
    gs[1] += n1;
    ++qi;
  }
  // Every MMA issued above must finish before tensor memory is released.
  commit(C::BAR_MMA_DONE);
  volatile int never = 0;
  mbar_wait_bounded(x.bar(C::BAR_MMA_DONE), 0, &never, p.status, p.wait_limit_ns, kErrTimeout);
}

// --------------------------------------------------------------------------
// MMA issuer with three S buffers (D = 64).  The CTA's S products form one
// sequence, index T = 2 * (key tiles so far) + Q tile, and S(T) goes to
// buffer T % 3.  S(T) is issued right after PV(T - 3), the last reader of
// that buffer's P, so a Q tile's next S is usually complete before its
// softmax finishes the current tile.  Barriers: S full and P halves per
// buffer (phase T / 3), PV done per Q tile (one phase per tile), O full per
// Q tile and unit.
// --------------------------------------------------------------------------
template <int D, bool F8, int V>
__device__ void role_mma_triple(const Sm100Ctx<D, F8, V> &x, const FwdParams &p) {
  using C = Sm100Cfg<D, F8, V>;
  static_assert(C::TRIPLE, "three S buffers: bf16, head dim 64");
  constexpr uint32_t IDESC_S = idesc_bf16_f32(128, C::BN, 0, 0);  // Q, K both K-major
  constexpr uint32_t IDESC_O = idesc_bf16_f32(128, D, 0, 1);      // P from TMEM, V MN-major
  const bool leader = elect_one();
  const uint64_t desc_q0 = smem_desc_sw128(x.q_tile(0), 16, 1024);
  const uint64_t desc_q1 = smem_desc_sw128(x.q_tile(1), 16, 1024);
  const uint64_t desc_kv_k = smem_desc_sw128(x.kv_tile(0), 16, 1024);
  const uint64_t desc_kv_v = smem_desc_sw128(x.kv_tile(0), C::BOX_BYTES, 1024);
  auto wait = [&](int bar, uint32_t parity) {
    const bool ok = mbar_wait_bounded(x.bar(bar), parity, x.abort_flag, p.status,
                                      p.wait_limit_ns, kErrTimeout);
    return __all_sync(0xffffffffu, ok);
  };
  auto commit = [&](int bar) {
    if (leader) tc_commit(x.bar(bar));
    __syncwarp();
  };
  auto sbuf = [&](int tt) { return x.tmem + C::COL_S0 + 128u * static_cast<uint32_t>(tt % 3); };

  int T = 0;   // S products issued by this CTA so far
  int g = 0;   // K/V tiles consumed (ring position)
  int qi = 0;  // units with keys processed so far
  bool ok = true;
  for (int k = 0; ok; ++k) {
    const int u = snake_unit(k, p.num_units);
    if (u == -2) break;
    if (u < 0) continue;
    const Unit w = unit_at<D, F8, V>(p, u);
    const int n = w.nkv;
    if (n == 0) continue;
    // In a causal unit Q tile 0 may skip the last key tile (it lies wholly
    // above tile 0's rows): that slot of the sequence issues no products, but
    // its barriers still complete, so every buffer keeps its phase count.
    const int n0 = w.nkv0;
    const uint32_t qpar = static_cast<uint32_t>(qi & 1);
    if (!wait(C::BAR_Q_FULL + 0, qpar) || !wait(C::BAR_Q_FULL + 1, qpar)) break;
    const int t0 = T, tend = T + 2 * n;
    const int t_skip = (C::SKIP0 && n0 < n) ? t0 + 2 * (n - 1) : -1;  // the skipped slot
    // S of sequence index tt (key tile j, Q tile q); K tile j is waited for
    // by Q tile 0's product and released after Q tile 1's.
    auto issue_s = [&](int tt) {
      const int j = (tt - t0) >> 1, q = (tt - t0) & 1;
      const int ks = ring_slot<D, F8, V>(2 * (g + j));
      if (q == 0) {
        if (!wait(C::BAR_KV_FULL + ks, ring_parity<D, F8, V>(2 * (g + j)))) return false;
        tc_fence_after();
      }
      const uint64_t kd = desc_kv_k + ((ks * C::TILE_BYTES) >> 4);
      if (!C::SKIP0 || tt != t_skip) {
#pragma unroll
        for (int kk = 0; kk < C::KSTEPS; ++kk) {
          const uint32_t off = ((kk / 4) * C::BOX_BYTES + (kk % 4) * 32) >> 4;
          if (leader)
            tc_mma_ss(sbuf(tt), (q ? desc_q1 : desc_q0) + off, kd + off, IDESC_S,
                      kk > 0 ? 1u : 0u);
        }
      }
      __syncwarp();
      commit(C::BAR_S_FULL + tt % 3);
      if (q == 1) commit(C::BAR_KV_EMPTY + ks);
      if (j == n - 1 - (C::SKIP0 && q == 0 && t_skip >= 0)) commit(C::BAR_Q_EMPTY + q);
      return true;
    };
    for (int tt = t0; ok && tt < t0 + 3 && tt < tend; ++tt) ok = issue_s(tt);
    for (int tp = t0; ok && tp < tend; ++tp) {
      const int j = (tp - t0) >> 1, q = (tp - t0) & 1;
      const int vs = ring_slot<D, F8, V>(2 * (g + j) + 1);
      if (q == 0 && !wait(C::BAR_KV_FULL + vs, ring_parity<D, F8, V>(2 * (g + j) + 1))) {
        ok = false;
        break;
      }
      const uint32_t par = static_cast<uint32_t>((tp / 3) & 1);
      const uint64_t vd = desc_kv_v + ((vs * C::TILE_BYTES) >> 4);
      const uint32_t tO = x.tmem + C::COL_O0 + C::O_STRIDE * q;
      // O_q += P V for each 64-key half as the softmax publishes it.
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        if (!wait(C::BAR_P_HALF + 2 * (tp % 3) + half, par)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (!C::SKIP0 || tp != t_skip) {
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const int kk = 4 * half + k4;
            if (leader)
              tc_mma_ts(tO, sbuf(tp) + kk * 8, vd + ((kk * 2048) >> 4), IDESC_O,
                        (j > 0 || kk > 0) ? 1u : 0u);
          }
        }
        __syncwarp();
      }
      if (!ok) break;
      commit(C::BAR_PV_DONE + q);
      if (q == 1) commit(C::BAR_KV_EMPTY + vs);
      if (j == n - 1) commit(C::BAR_O_FULL + q);
      // the buffer tp's P sat in is free once this PV has read it
      if (tp + 3 < tend && !issue_s(tp + 3)) {
        ok = false;
        break;
      }
    }
    if (!ok) break;
    T = tend;
    g += n;
    ++qi;
  }
  commit(C::BAR_MMA_DONE);
  volatile int never = 0;
  mbar_wait_bounded(x.bar(C::BAR_MMA_DONE), 0, &never, p.status, p.wait_limit_ns, kErrTimeout);
}

// --------------------------------------------------------------------------
// Softmax warpgroup t (128 threads, one query row each)
// --------------------------------------------------------------------------
template <int D, bool F8, int V>
__device__ void role_softmax(const Sm100Ctx<D, F8, V> &x, const FwdParams &p, int t) {
  using C = Sm100Cfg<D, F8, V>;
  const int r = threadIdx.x & 127;
  const uint32_t lane_base = static_cast<uint32_t>((threadIdx.x >> 5) & 3) * 32u << 16;
  const uint32_t tS = x.tmem + lane_base + C::COL_S0 + 128 * t;
  const uint32_t tO = x.tmem + lane_base + C::COL_O0 + C::O_STRIDE * t;
  const float sl2 = p.scale_log2;

  auto wait_all = [&](int bar, uint32_t parity) {
    const bool ok = mbar_wait_bounded(x.bar(bar), parity, x.abort_flag, p.status,
                                      p.wait_limit_ns, kErrTimeout);
    return __all_sync(0xffffffffu, ok);
  };

  int g = 0;   // K/V tiles processed by this CTA so far
  int qi = 0;  // units with keys processed so far
  for (int k = 0;; ++k) {
    const int u = snake_unit(k, p.num_units);
    if (u == -2) break;
    if (u < 0) continue;
    const Unit w = unit_at<D, F8, V>(p, u);
    const int tile_row0 = w.row0 + t * C::BM;
    const int i = tile_row0 + r;  // this thread's query row
    const bool valid = i < w.q_rows;
    if (w.nkv == 0) {
      // No visible key at all (key length 0): O = 0, LSE = -inf.
      if (valid) {
        uint4 *dst = reinterpret_cast<uint4 *>(p.o + w.o_base + i * w.o_stride);
#pragma unroll
        for (int v4 = 0; v4 < D / 8; ++v4) dst[v4] = make_uint4(0, 0, 0, 0);
        p.lse[w.lse_base + i] = -INFINITY;
      }
      continue;
    }
    const int limit = p.causal ? min(w.L, i + 1) : w.L;  // visible keys are [0, limit)
    const int nkv_t = t == 0 ? w.nkv0 : w.nkv;            // key tiles this Q tile needs

    float m_ref = -INFINITY;  // reference max (log2 units) the exponentials use
    float l = 0.f;            // row sum of the fp32 probabilities relative to m_ref
    for (int j = 0; j < nkv_t; ++j) {
      // This tile's S buffer and barriers: fixed per Q tile, or (three
      // buffers) sequence index tt = 2 (g + j) + t, buffer tt % 3.
      const int tt = 2 * (g + j) + t;
      const int sb = C::TRIPLE ? tt % 3 : t;
      const uint32_t spar =
          static_cast<uint32_t>(C::TRIPLE ? (tt / 3) & 1 : (g + j) & 1);
      const uint32_t tSj = C::TRIPLE ? x.tmem + lane_base + C::COL_S0 + 128u * sb : tS;
      if (!wait_all(C::BAR_S_FULL + sb, spar)) return;
      tc_fence_after();
      uint32_t s[128];
      tmem_ld32(tSj + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_ld32(tSj + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
      tmem_ld32(tSj + 64, *reinterpret_cast<uint32_t(*)[32]>(&s[64]));
      tmem_ld32(tSj + 96, *reinterpret_cast<uint32_t(*)[32]>(&s[96]));
      tmem_wait_ld();

      const int kbase = j * C::BN;
      // Masks only on the tile that crosses the key length or the diagonal.
      const bool need_mask = (kbase + C::BN > w.L) || (p.causal && kbase + C::BN - 1 > tile_row0);
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (kbase + c >= limit) s[c] = __float_as_uint(-INFINITY);
      }
      // p = 2^(s * scale * log2(e) - m_ref + P_SHIFT) for 64 keys: the row
      // sum takes p in fp32 and the PV product its bf16 (or E4M3) rounding.
      const uint64_t scale2 = f32x2(sl2, sl2);
      auto exp_half = [&](int half, float m_use, uint32_t(&pk)[C::PK_WORDS], uint64_t &sum2) {
        const float sh = F8 ? C::P_SHIFT - m_use : -m_use;
        const uint64_t shift2 = f32x2(sh, sh);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int c = half * 64 + 2 * e;
          float x0, x1, p0, p1;
          f32x2_split(fma_f32x2(f32x2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), scale2,
                                shift2),
                      x0, x1);
          if ((e & 7) >= 8 - C::EXP2_EMU_PAIRS) {
            exp2_poly_pair(x0, x1, p0, p1);
          } else {
            p0 = ex2_approx(x0);
            p1 = ex2_approx(x1);
          }
          if constexpr (F8) {
            const uint32_t h = pack_e4m3x2(p0, p1);
            if (e & 1)
              pk[e >> 1] |= h << 16;
            else
              pk[e >> 1] = h;
          } else {
            pk[e] = pack_bf16x2(p0, p1);
          }
          sum2 = add_f32x2(sum2, f32x2(p0, p1));
        }
      };
      // Row max in eight independent chains of 3-input maxima.
      auto row_max = [&]() {
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
        return fmaxf(fmax3(mq[0], mq[1], mq[2]), fmax3(fmax3(mq[3], mq[4], mq[5]), mq[6], mq[7]));
      };

      uint32_t pk[C::PK_WORDS];
      uint64_t sum2 = f32x2(0.f, 0.f);
      // P of one 64-key half over the first columns of S_t.
      auto store_p = [&](int half) {
        if constexpr (F8)
          tmem_st16(tSj + 16 * half, pk);
        else
          tmem_st32(tSj + 32 * half, pk);
      };
      bool need;
      float alpha = 1.0f;
      if (j > 0) {
        // The first half's exponentials start against the current reference
        // while the row max is found: the reference moves only when the max
        // rose by more than the threshold, which after the first tile is rare.
        exp_half(0, (m_ref == -INFINITY) ? 0.0f : m_ref, pk, sum2);
        const float m_new = fmaxf(m_ref, row_max() * sl2);
        need = m_new > m_ref + C::RESCALE_THRESHOLD;
        if (__any_sync(0xffffffffu, need)) {
          if (need) {
            alpha = ex2_approx(m_ref - m_new);
            l *= alpha;
            m_ref = m_new;
          }
          const float m_use = (m_ref == -INFINITY) ? 0.0f : m_ref;
          sum2 = f32x2(0.f, 0.f);
          exp_half(0, m_use, pk, sum2);
        }
      } else {
        // First tile of the unit: the reference is the tile's row max.
        const float m_new = row_max() * sl2;
        need = true;
        m_ref = m_new;
        l = 0.f;
        exp_half(0, (m_ref == -INFINITY) ? 0.0f : m_ref, pk, sum2);
      }
      const float m_use = (m_ref == -INFINITY) ? 0.0f : m_ref;
      store_p(0);
      // O holds earlier tiles' sum only for j > 0; nothing writes it until
      // this warpgroup publishes P.  When S_j is issued after the whole PV
      // product of tile j-1 (two S buffers in tensor memory, P entirely
      // there), that product finished before S_j did; otherwise (three S
      // buffers, or P's upper half in shared memory) it may still be
      // running, so its completion is awaited first.  O is rescaled before
      // the first half goes out.
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        if constexpr (C::HAS_PV_DONE) {
          if (!wait_all(C::BAR_PV_DONE + t, static_cast<uint32_t>((g + j - 1) & 1))) return;
          tc_fence_after();
        }
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * c, o);
          tmem_wait_ld();
#pragma unroll
          for (int e2 = 0; e2 < 32; ++e2) o[e2] = __float_as_uint(__uint_as_float(o[e2]) * alpha);
          tmem_st32(tO + 32 * c, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(x.bar(C::BAR_P_HALF + 2 * sb));
      // Second half of the keys.
      if constexpr (C::P_HI_SMEM) {
        // Row r of the K-major, 128-byte swizzled upper half of P: 16-byte
        // chunk c of the row's 128 bytes sits at chunk c ^ (r % 8).  The
        // buffer is free once this Q tile's previous PV product is done.
        const int gt = g + j;  // key tiles this Q tile processed before this one
        if (gt > 0 && !wait_all(C::BAR_PV_DONE + t, static_cast<uint32_t>((gt - 1) & 1))) return;
        exp_half(1, m_use, pk, sum2);
        // (Storing each chunk as soon as it is packed, interleaved with the
        // exponentials, measured 3 % slower on the GQA layer.)
        const uint32_t row = x.p_hi(t) + static_cast<uint32_t>(r) * 128u;
#pragma unroll
        for (int c = 0; c < C::PK_WORDS / 4; ++c)  // 8 chunks (bf16) or 4 (E4M3)
          st_shared_v4(row + (static_cast<uint32_t>(c ^ (r & 7)) << 4), pk[4 * c], pk[4 * c + 1],
                       pk[4 * c + 2], pk[4 * c + 3]);
        fence_proxy_async_shared();
      } else {
        exp_half(1, m_use, pk, sum2);
        store_p(1);
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(x.bar(C::BAR_P_HALF + 2 * sb + 1));
      float a0, a1;
      f32x2_split(sum2, a0, a1);
      l += a0 + a1;
    }

    if (C::SKIP0 && nkv_t < w.nkv) {
      // Q tile 0's skipped last key tile (three S buffers): the slot's S is
      // committed without products; once it has, both P halves are released
      // without any probabilities, which keeps the buffer's phases.
      const int tt = 2 * (g + w.nkv - 1) + t;
      if (!wait_all(C::BAR_S_FULL + tt % 3, static_cast<uint32_t>((tt / 3) & 1))) return;
      mbar_arrive(x.bar(C::BAR_P_HALF + 2 * (tt % 3)));
      mbar_arrive(x.bar(C::BAR_P_HALF + 2 * (tt % 3) + 1));
    }
    // Epilogue: O = O~ / l in bf16, LSE = (m_ref + log2 l) * ln 2.
    if (!wait_all(C::BAR_O_FULL + t, static_cast<uint32_t>(qi & 1))) return;
    tc_fence_after();
    float inv_l = l > 0.f ? 1.0f / l : 0.0f;
    if constexpr (F8) inv_l *= p.out_scale;
    uint16_t *orow = p.o + w.o_base + (valid ? i : 0) * w.o_stride;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      tmem_ld32(tO + 32 * c, o);
      tmem_wait_ld();
      uint32_t wv[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        wv[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l,
                            __uint_as_float(o[2 * e + 1]) * inv_l);
      if (valid) {
        uint4 *dst = reinterpret_cast<uint4 *>(orow + 32 * c);
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4)
          __stcs(dst + v4, make_uint4(wv[4 * v4], wv[4 * v4 + 1], wv[4 * v4 + 2], wv[4 * v4 + 3]));
      }
    }
    if (valid) {
      // l carries the factor 2^P_SHIFT of the stored probabilities.
      const float m_lse = F8 ? m_ref - C::P_SHIFT : m_ref;
      p.lse[w.lse_base + i] =
          l > 0.f ? (m_lse + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
    }
    // three S buffers: the sequence advances by the unit's tiles for both
    // Q tiles (a skipped slot included)
    g += C::SKIP0 ? w.nkv : nkv_t;
    ++qi;
  }
}

template <int D, bool F8, int V>
__device__ __forceinline__ void fwd_kernel_body(const CUtensorMap *tm_q, const CUtensorMap *tm_k,
                                                const CUtensorMap *tm_v, const FwdParams &p) {
  using C = Sm100Cfg<D, F8, V>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *smem = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  Sm100Ctx<D, F8, V> x;
  x.smem = base;
  x.abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(x.bar(C::BAR_Q_FULL + t), 1);
      mbar_init(x.bar(C::BAR_Q_EMPTY + t), 1);
      mbar_init(x.bar(C::BAR_O_FULL + t), 1);
      if (C::HAS_PV_DONE) mbar_init(x.bar(C::BAR_PV_DONE + t), 1);
    }
    for (int b = 0; b < C::NSBUF; ++b) {
      mbar_init(x.bar(C::BAR_S_FULL + b), 1);
      mbar_init(x.bar(C::BAR_P_HALF + 2 * b), 128);
      mbar_init(x.bar(C::BAR_P_HALF + 2 * b + 1), 128);
    }
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(x.bar(C::BAR_KV_FULL + s), 1);
      mbar_init(x.bar(C::BAR_KV_EMPTY + s), 1);
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
    tma_prefetch_desc(tm_q);
    tma_prefetch_desc(tm_k);
    tma_prefetch_desc(tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  x.tmem = *reinterpret_cast<volatile uint32_t *>(smem + C::OFF_MISC);

  static_assert(128 * C::REGS_CONTROL + 256 * C::REGS_SOFTMAX <= C::THREADS * 168,
                "register split exceeds the launch allocation");
  if (warp >= 8) {
    regs_decrease<C::REGS_CONTROL>();
    if (warp == 8) {
      if (lane == 0) role_producer<D, F8, V>(x, p, tm_q, tm_k, tm_v);
    } else if (warp == 9) {
      if constexpr (C::TRIPLE)
        role_mma_triple<D, F8, V>(x, p);
      else
        role_mma_split<D, F8, V>(x, p);
    }
  } else {
    regs_increase<C::REGS_SOFTMAX>();
    role_softmax<D, F8, V>(x, p, warp >> 2);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(x.tmem, C::TMEM_COLS);
  }
}

template <int D, int V>
__global__ void __launch_bounds__(Sm100Cfg<D>::THREADS, 1)
    fa_fwd_bf16_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                             const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  fwd_kernel_body<D, false, V>(&tm_q, &tm_k, &tm_v, p);
}

// FP8 E4M3 inputs (head dim 128); tm_v maps V^T.
__global__ void __launch_bounds__(Sm100Cfg<128, true>::THREADS, 1)
    fa_fwd_e4m3_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                             const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_vt, const FwdParams p) {
  fwd_kernel_body<128, true, 0>(&tm_q, &tm_k, &tm_vt, p);
}

}  // namespace fa
