// C ABI of the attention library (declared in include/fa.h).
//
// Host side only: argument checks, TMA tensor maps (cuTensorMapEncodeTiled,
// reached through the runtime's driver entry point so the library does not
// link libcuda), launch configuration, the status word, and the copy
// streams of the host-buffer call.  All attention arithmetic runs in the
// kernels: fa_fwd_sm100.cuh (bf16 and FP8 forward, packed layout),
// fa_fwd_f32.cuh (fp32 check mode), fa_bwd_sm100.cuh (backward) and
// fa_decode.cuh (split-KV decode).
#include <cmath>
#include <cstdint>
#include <algorithm>
#include <vector>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "fa.h"
#include "fa_bwd_sm100.cuh"
#include "fa_decode.cuh"
#include "fa_decode_tc.cuh"
#include "fa_decode_rows.cuh"
#include "fa_fwd_f32.cuh"
#include "fa_fwd_sm100.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s per wait
constexpr float kLog2e = 1.4426950408889634f;

// The library's own status word, used when the caller passes none.
__device__ int g_status_word;

struct DeviceState {
  bool checked = false;
  bool ok = false;
  int num_sms = 0;
  int *status_word = nullptr;  // device address of g_status_word
  bool fwd_attr[2][4] = {};  // [d = 64, 128][launch variant: fa::kVarSkip0 | fa::kVarPacked]
  bool dec_attr64 = false, dec_attr128 = false;
  bool dec_tc_attr[2][3] = {};  // [d = 64, 128][4, 8, 16 row slots]
  bool dec_rows_attr[2] = {};    // [d = 64, 128]: 17 to 128 rows per kv head
  bool bwd_attr64 = false, bwd_attr128 = false;
  bool fp8_attr = false;
  // fa_fwd_hostio's copy streams and per-slice events, created on first use
  // and kept for the process's lifetime.  io_mu is held for a whole call, so
  // host threads that call it on one device take turns.
  std::mutex io_mu;
  bool io_ready = false;
  cudaStream_t io_in = nullptr, io_out = nullptr;
  cudaEvent_t io_ev_in[16] = {}, io_ev_done[16] = {}, io_ev_end = nullptr;
  // The previous call's device buffers, shape and stream; a call with the
  // same ones (and no key lengths) is chained to it slice by slice.
  bool io_prev = false;
  const void *io_prev_ptr[5] = {};
  int io_prev_shape[5] = {};
  cudaStream_t io_prev_stream = nullptr;
  // fa_bwd's second stream: the dQ kernel runs beside the dK/dV kernel.
  // bwd_mu covers a call's fork and join, so concurrent callers do not
  // interleave them.
  std::mutex bwd_mu;
  bool bwd_ready = false;
  cudaStream_t bwd_side = nullptr;
  cudaEvent_t bwd_fork = nullptr, bwd_join = nullptr;
};
DeviceState g_dev[kMaxDevices];
std::mutex g_mu;

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

// Current device, checked once per device: must be sm_100 (B200).
int current_device(DeviceState **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return FA_ERR_ARCH;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState &s = g_dev[dev];
  if (!s.checked) {
    s.checked = true;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_ARCH;
    }
    if (prop.major != 10 || prop.minor != 0) return FA_ERR_ARCH;
    s.num_sms = prop.multiProcessorCount;
    void *addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_status_word) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
    s.status_word = static_cast<int *>(addr);
    s.ok = true;
  }
  if (!s.ok) return FA_ERR_ARCH;
  if (!g_encode) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  *out = &s;
  return FA_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_args(const void *q, const void *k, const void *v, const void *o, const float *lse,
               int B, int Hq, int Hkv, int N, int d, float scale) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_NULL;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || d <= 0) return FA_ERR_SHAPE;
  if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_SHAPE;
  if (Hq % Hkv != 0) return FA_ERR_HEADS;
  if (d != 64 && d != 128) return FA_ERR_HEADDIM;
  // element counts must fit the kernels' 64-bit offsets and the 32-bit grid
  const long long rows = static_cast<long long>(B) * Hq;
  if (rows > (1ll << 30) || static_cast<long long>(N) * d > (1ll << 40)) return FA_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return FA_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return FA_ERR_ALIGN;
  return FA_OK;
}

// 3-D map over a [planes, N, d] bf16 tensor: box = 64 columns x 128 rows x 1
// plane, 128-byte swizzle; rows past N read as zero.
int make_map(CUtensorMap *m, const void *ptr, int planes, int N, int d) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(planes)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(N) * static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// Packed layout: a [total, H, d] tensor seen as (d, head, token), box of 64
// columns x 1 head x 128 tokens, 128-byte swizzle; tokens past the end read
// as zero.
int make_map_packed(CUtensorMap *m, const void *ptr, int total, int H, int d) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(total)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(H) * static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// The query rows of a decode call, [rows, d] bf16: box = 64 columns x
// box_rows rows (16 or 128), 128-byte swizzle; rows past the end read as zero.
int make_map_qrows(CUtensorMap *m, const void *ptr, int rows, int d, int box_rows = 16) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows), 1};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(rows) * static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// 8-bit map over a [planes, rows, cols] tensor of E4M3 codes whose rows are
// `pitch` bytes apart: box = 128 columns x 128 rows x 1 plane, 128-byte
// swizzle; columns past `cols` and rows past `rows` read as zero.  Q and K:
// rows = N, cols = pitch = d.  V^T: rows = d, cols = N keys, pitch = ldvt.
int make_map_u8(CUtensorMap *m, const void *ptr, int planes, int rows, int cols, int pitch) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(planes)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(pitch),
                           static_cast<cuuint64_t>(rows) * static_cast<cuuint64_t>(pitch)};
  cuuint32_t box[3] = {128, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(ptr), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// The forward kernels split their registers between warpgroups with
// setmaxnreg: the softmax warpgroups' increase is served only by what the
// control warpgroup gives up from the launch allocation.  A build whose
// kernel was compiled with fewer registers per thread would leave that
// increase waiting for ever, so such a kernel is never launched.
template <typename Cfg, typename K>
int prepare_fwd_kernel(K kernel) {
  cudaFuncAttributes fa_attr{};
  if (cudaFuncGetAttributes(&fa_attr, kernel) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_LAUNCH;
  }
  if (static_cast<uint32_t>(fa_attr.numRegs) < Cfg::REGS_LAUNCH) return FA_ERR_LAUNCH;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           Cfg::SMEM_ALLOC) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_LAUNCH;
  }
  return FA_OK;
}

int launch_fp8(DeviceState *ds, const void *q, const void *k, const void *vt, void *o, float *lse,
               int B, int Hq, int Hkv, int N, int ldvt, float scale, float descale_q,
               float descale_k, float descale_v, int causal, const int *seqlens,
               cudaStream_t stream, int *status) {
  using C = fa::Sm100Cfg<128, true>;
  auto kernel = fa::fa_fwd_e4m3_sm100_kernel;
  if (!ds->fp8_attr) {
    const int rc = prepare_fwd_kernel<C>(kernel);
    if (rc != FA_OK) return rc;
    ds->fp8_attr = true;
  }
  CUtensorMap tq, tk, tvt;
  if (make_map_u8(&tq, q, B * Hq, N, 128, 128) != FA_OK ||
      make_map_u8(&tk, k, B * Hkv, N, 128, 128) != FA_OK ||
      make_map_u8(&tvt, vt, B * Hkv, 128, N, ldvt) != FA_OK)
    return FA_ERR_CUDA;
  fa::FwdParams p;
  p.o = static_cast<uint16_t *>(o);
  p.lse = lse;
  p.seqlens = seqlens;
  p.cu_seqlens = nullptr;
  p.total = 0;
  p.status = status;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.group = Hq / Hkv;
  p.div_bh = fa::make_fast_div(static_cast<uint32_t>(B * Hq));
  p.div_hq = fa::make_fast_div(static_cast<uint32_t>(Hq));
  p.div_group = fa::make_fast_div(static_cast<uint32_t>(Hq / Hkv));
  p.num_qpairs = (N + C::ROWS_PER_UNIT - 1) / C::ROWS_PER_UNIT;
  p.causal = causal ? 1 : 0;
  // scores of the codes times the two descales, in log2 units
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * descale_q * descale_k *
                                    1.4426950408889634);
  p.out_scale = descale_v;
  p.wait_limit_ns = kWaitLimitNs;
  const long long units = static_cast<long long>(B) * Hq * p.num_qpairs;
  if (units > 0x7fffffffll) return FA_ERR_SHAPE;
  p.num_units = static_cast<int>(units);
  const int grid = static_cast<int>(units < ds->num_sms ? units : ds->num_sms);
  kernel<<<grid, C::THREADS, C::SMEM_ALLOC, stream>>>(tq, tk, tvt, p);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_LAUNCH;
  return FA_OK;
}

template <int D>
int launch_bf16(DeviceState *ds, const void *q, const void *k, const void *v, void *o,
                float *lse, int B, int Hq, int Hkv, int N, float scale, int causal,
                const int *seqlens, cudaStream_t stream, int *status,
                const int *cu_seqlens = nullptr, int total = 0) {
  using C = fa::Sm100Cfg<D>;
  // Causal launches at d = 64 use the instance in which Q tile 0 skips a
  // unit's last key tile (wholly above its rows) inside the three-buffer
  // sequence; packed sequences their own instance, so that dense launches
  // decode units without the packed layout's branch.
  const int var = (D == 64 && causal ? fa::kVarSkip0 : 0) | (cu_seqlens ? fa::kVarPacked : 0);
  auto kernel = fa::fa_fwd_bf16_sm100_kernel<D, 0>;
  if (var == fa::kVarPacked) kernel = fa::fa_fwd_bf16_sm100_kernel<D, fa::kVarPacked>;
  if constexpr (D == 64) {
    if (var == fa::kVarSkip0) kernel = fa::fa_fwd_bf16_sm100_kernel<64, fa::kVarSkip0>;
    if (var == (fa::kVarSkip0 | fa::kVarPacked))
      kernel = fa::fa_fwd_bf16_sm100_kernel<64, fa::kVarSkip0 | fa::kVarPacked>;
  }
  bool &attr = ds->fwd_attr[D == 128][var];
  if (!attr) {
    const int rc = prepare_fwd_kernel<C>(kernel);
    if (rc != FA_OK) return rc;
    attr = true;
  }
  CUtensorMap tq, tk, tv;
  if (cu_seqlens) {
    if (make_map_packed(&tq, q, total, Hq, D) != FA_OK ||
        make_map_packed(&tk, k, total, Hkv, D) != FA_OK ||
        make_map_packed(&tv, v, total, Hkv, D) != FA_OK)
      return FA_ERR_CUDA;
  } else if (make_map(&tq, q, B * Hq, N, D) != FA_OK || make_map(&tk, k, B * Hkv, N, D) != FA_OK ||
             make_map(&tv, v, B * Hkv, N, D) != FA_OK) {
    return FA_ERR_CUDA;
  }
  fa::FwdParams p;
  p.o = static_cast<uint16_t *>(o);
  p.lse = lse;
  p.seqlens = seqlens;
  p.cu_seqlens = cu_seqlens;
  p.total = total;
  p.status = status;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.group = Hq / Hkv;
  p.div_bh = fa::make_fast_div(static_cast<uint32_t>(B * Hq));
  p.div_hq = fa::make_fast_div(static_cast<uint32_t>(Hq));
  p.div_group = fa::make_fast_div(static_cast<uint32_t>(Hq / Hkv));
  p.num_qpairs = (N + C::ROWS_PER_UNIT - 1) / C::ROWS_PER_UNIT;
  p.causal = causal ? 1 : 0;
  p.scale_log2 = scale * kLog2e;
  p.out_scale = 1.0f;
  p.wait_limit_ns = kWaitLimitNs;
  const long long units = static_cast<long long>(B) * Hq * p.num_qpairs;
  if (units > 0x7fffffffll) return FA_ERR_SHAPE;
  p.num_units = static_cast<int>(units);
  // Persistent: one CTA per SM (or per unit when there are fewer units).
  const int grid = static_cast<int>(units < ds->num_sms ? units : ds->num_sms);
  kernel<<<grid, C::THREADS, C::SMEM_ALLOC, stream>>>(tq, tk, tv, p);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_LAUNCH;
  return FA_OK;
}

template <int D>
int launch_f32(const float *q, const float *k, const float *v, float *o, float *lse, int B,
               int Hq, int Hkv, int N, float scale, int causal, const int *seqlens,
               cudaStream_t stream) {
  fa::F32Params p;
  p.q = q;
  p.k = k;
  p.v = v;
  p.o = o;
  p.lse = lse;
  p.seqlens = seqlens;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.group = Hq / Hkv;
  p.causal = causal ? 1 : 0;
  p.scale_log2 = scale * kLog2e;
  const long long bh = static_cast<long long>(B) * Hq;
  if (bh > 65535) return FA_ERR_SHAPE;
  constexpr int ROWS = fa::F32Cfg<D>::ROWS;
  dim3 grid((N + ROWS - 1) / ROWS, static_cast<unsigned>(bh));
  fa::fa_fwd_f32_kernel<D><<<grid, ROWS, 0, stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_LAUNCH;
  return FA_OK;
}

// Decode: how many key ranges, and how many keys each (a multiple of the
// kernel's chunk).  The automatic choice aims at about 16 CTAs per SM of a
// B200 (148 SMs, two resident at a time), so the last wave is a small part of
// the work, with at least 256 keys per range.
struct DecodeSplit {
  int splits, keys_per_split;
};
DecodeSplit decode_split(int B, int Hkv, int groups, int Nk, int d, int requested) {
  const int chunk = 16384 / (d * 2);
  const long long ctas_per_split = static_cast<long long>(B) * Hkv * groups;
  int s = requested > 0 ? requested
                        : static_cast<int>((16 * 148 + ctas_per_split - 1) / ctas_per_split);
  const int by_len = (Nk + 255) / 256;
  s = std::max(1, std::min(s, std::min(128, std::max(1, by_len))));
  int kps = (Nk + s - 1) / s;
  kps = (kps + chunk - 1) / chunk * chunk;
  DecodeSplit r;
  r.keys_per_split = kps;
  r.splits = (Nk + kps - 1) / kps;
  return r;
}

size_t decode_workspace_bytes(int B, int Hq, int Nq, int d, int splits) {
  const size_t rows = static_cast<size_t>(B) * Hq * Nq;
  const size_t o_bytes = static_cast<size_t>(splits) * rows * d * sizeof(float);
  const size_t ml_bytes = static_cast<size_t>(splits) * rows * 2 * sizeof(float);
  return ((o_bytes + 255) / 256) * 256 + ml_bytes;
}

int check_decode_args(const void *q, const void *k, const void *v, const void *o,
                      const float *lse, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                      float scale) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_NULL;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nk <= 0 || d <= 0) return FA_ERR_SHAPE;
  if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_SHAPE;
  if (Hq % Hkv != 0) return FA_ERR_HEADS;
  if (d != 64 && d != 128) return FA_ERR_HEADDIM;
  const long long groups = (static_cast<long long>(Hq / Hkv) * Nq + 3) / 4;
  if (static_cast<long long>(B) * Hkv > 65535 || groups > 65535) return FA_ERR_SHAPE;
  if (static_cast<long long>(B) * Hq * Nq > (1ll << 30)) return FA_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return FA_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return FA_ERR_ALIGN;
  return FA_OK;
}

template <int D>
int launch_decode(DeviceState *ds, const void *q, const void *k, const void *v, void *o,
                  float *lse, int B, int Hq, int Hkv, int Nq, int Nk, float scale, int causal,
                  const int *seqlens, const DecodeSplit &sp, void *workspace,
                  cudaStream_t stream, int *status) {
  using C = fa::DecodeCfg<D>;
  auto kernel = fa::fa_decode_split_kernel<D>;
  bool &attr = (D == 64) ? ds->dec_attr64 : ds->dec_attr128;
  if (!attr) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
        cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_LAUNCH;
    }
    attr = true;
  }
  const size_t rows = static_cast<size_t>(B) * Hq * Nq;
  fa::DecodeParams p;
  p.q = static_cast<const uint16_t *>(q);
  p.k = static_cast<const uint16_t *>(k);
  p.v = static_cast<const uint16_t *>(v);
  p.o = static_cast<uint16_t *>(o);
  p.lse = lse;
  p.seqlens = seqlens;
  p.part_o = static_cast<float *>(workspace);
  p.part_ml = reinterpret_cast<float *>(
      static_cast<char *>(workspace) +
      ((static_cast<size_t>(sp.splits) * rows * D * sizeof(float) + 255) / 256) * 256);
  p.status = status;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.group = Hq / Hkv;
  p.splits = sp.splits;
  p.part_rows = 0;
  p.keys_per_split = sp.keys_per_split;
  p.causal = causal ? 1 : 0;
  p.scale_log2 = scale * kLog2e;
  p.wait_limit_ns = kWaitLimitNs;
  const int groups = (p.group * Nq + C::ROWS - 1) / C::ROWS;
  dim3 grid(sp.splits, B * Hkv, groups);
  kernel<<<grid, C::THREADS, C::SMEM, stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_LAUNCH;
  const unsigned cblocks = static_cast<unsigned>((rows + 3) / 4);
  fa::fa_decode_combine_kernel<D><<<cblocks, 128, 0, stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_LAUNCH;
  return FA_OK;
}

// Decode on the tensor cores (up to 128 query rows per kv head): the call's
// key tiles are shared evenly by `ctas` persistent CTAs, one per SM by
// default, or num_splits per (batch, kv head) when given.  Each CTA leaves one
// partial per (batch, kv head) its share touches, so there are at most
// ctas + B * Hkv of them.  Up to 16 rows per kv head, fa_decode_tc.cuh (keys
// on the tensor-memory lanes, 16 row slots per partial); from 17 to 128,
// fa_decode_rows.cuh (rows on the lanes, the row count rounded up to 16 row
// slots per partial).
constexpr int kDecodeTcMaxRows = 16;
constexpr int kDecodeRowsMax = 128;
constexpr int kDecodeTcAutoCtasMax = 256;
constexpr long long kDecodeTcCtasMax = 1024;

bool decode_uses_tc(int Hq, int Hkv, int Nq) {
  return static_cast<long long>(Hq / Hkv) * Nq <= kDecodeRowsMax;
}

// Row slots per partial of the tensor-core decode.
int decode_tc_part_rows(int Hq, int Hkv, int Nq) {
  const int rows = (Hq / Hkv) * Nq;
  return rows <= kDecodeTcMaxRows ? kDecodeTcMaxRows : (rows + 15) / 16 * 16;
}

int decode_tc_ctas(int B, int Hkv, int num_splits, int num_sms) {
  if (num_splits > 0)
    return static_cast<int>(
        std::min(kDecodeTcCtasMax, static_cast<long long>(num_splits) * B * Hkv));
  return std::max(1, std::min(num_sms, kDecodeTcAutoCtasMax));
}

size_t decode_tc_workspace_bytes(int B, int Hkv, int d, int ctas, int part_rows) {
  const size_t pieces = static_cast<size_t>(ctas) + static_cast<size_t>(B) * Hkv;
  const size_t o_bytes = pieces * part_rows * d * sizeof(float);
  const size_t ml_bytes = pieces * part_rows * 2 * sizeof(float);
  return ((o_bytes + 255) / 256) * 256 + ml_bytes;
}

// The merge of a tensor-core decode call, as a programmatic dependent launch:
// it may start while the split kernel finishes and waits for it in the kernel
// before reading.
template <int D>
int launch_decode_tc_merge(const fa::DecodeParams &p, cudaStream_t stream);

template <int D, int NR>
int launch_decode_tc_rows(DeviceState *ds, const CUtensorMap &tq, const CUtensorMap &tk,
                          const CUtensorMap &tv, const fa::DecodeParams &p,
                          cudaStream_t stream) {
  using C = fa::DecodeTcCfg<D>;
  auto kernel = fa::fa_decode_tc_kernel<D, NR>;
  bool &attr = ds->dec_tc_attr[D == 128][NR == 4 ? 0 : NR == 8 ? 1 : 2];
  if (!attr) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM_ALLOC) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_LAUNCH;
    }
    attr = true;
  }
  kernel<<<p.ctas, C::THREADS, C::SMEM_ALLOC, stream>>>(tq, tk, tv, p);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_LAUNCH;
  return launch_decode_tc_merge<D>(p, stream);
}

// 17 to 128 query rows per kv head (fa_decode_rows.cuh).
template <int D>
int launch_decode_rows(DeviceState *ds, const CUtensorMap &tq, const CUtensorMap &tk,
                       const CUtensorMap &tv, const fa::DecodeParams &p, cudaStream_t stream) {
  using C = fa::DecodeRowsCfg<D>;
  auto kernel = fa::fa_decode_rows_kernel<D>;
  bool &attr = ds->dec_rows_attr[D == 128];
  if (!attr) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM_ALLOC) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_LAUNCH;
    }
    attr = true;
  }
  kernel<<<p.ctas, C::THREADS, C::SMEM_ALLOC, stream>>>(tq, tk, tv, p);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_LAUNCH;
  return launch_decode_tc_merge<D>(p, stream);
}

template <int D>
int launch_decode_tc_merge(const fa::DecodeParams &p, cudaStream_t stream) {
  // The merge is a programmatic dependent launch: it may start while the
  // split kernel finishes and waits for it in the kernel before reading.
  const long long rows = static_cast<long long>(p.B) * p.Hq * p.Nq;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((rows + 3) / 4));
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, fa::fa_decode_tc_combine_kernel<D>, p) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_LAUNCH;
  }
  return FA_OK;
}

template <int D>
int launch_decode_tc(DeviceState *ds, const void *q, const void *k, const void *v, void *o,
                     float *lse, int B, int Hq, int Hkv, int Nq, int Nk, float scale, int causal,
                     const int *seqlens, int ctas, void *workspace, cudaStream_t stream,
                     int *status) {
  const int part_rows = decode_tc_part_rows(Hq, Hkv, Nq);
  const bool wide = part_rows > kDecodeTcMaxRows;  // rows on the tensor-memory lanes
  CUtensorMap tq, tk, tv;
  if (make_map_qrows(&tq, q, B * Hq * Nq, D, wide ? 128 : 16) != FA_OK ||
      make_map(&tk, k, B * Hkv, Nk, D) != FA_OK || make_map(&tv, v, B * Hkv, Nk, D) != FA_OK)
    return FA_ERR_CUDA;
  const size_t pieces = static_cast<size_t>(ctas) + static_cast<size_t>(B) * Hkv;
  fa::DecodeParams p;
  p.q = static_cast<const uint16_t *>(q);
  p.k = static_cast<const uint16_t *>(k);
  p.v = static_cast<const uint16_t *>(v);
  p.o = static_cast<uint16_t *>(o);
  p.lse = lse;
  p.seqlens = seqlens;
  p.part_o = static_cast<float *>(workspace);
  p.part_ml = reinterpret_cast<float *>(
      static_cast<char *>(workspace) +
      ((pieces * part_rows * D * sizeof(float) + 255) / 256) * 256);
  p.part_rows = part_rows;
  p.status = status;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.group = Hq / Hkv;
  p.splits = 0;
  p.keys_per_split = 0;
  p.ctas = ctas;
  p.causal = causal ? 1 : 0;
  p.scale_log2 = scale * kLog2e;
  p.wait_limit_ns = kWaitLimitNs;
  const int rows = p.group * Nq;
  if (wide) return launch_decode_rows<D>(ds, tq, tk, tv, p, stream);
  if (rows <= 4) return launch_decode_tc_rows<D, 4>(ds, tq, tk, tv, p, stream);
  if (rows <= 8) return launch_decode_tc_rows<D, 8>(ds, tq, tk, tv, p, stream);
  return launch_decode_tc_rows<D, 16>(ds, tq, tk, tv, p, stream);
}

size_t bwd_workspace_bytes(int B, int Hq, int N) {
  const size_t npad = (static_cast<size_t>(N) + 127) / 128 * 128;
  return 2 * static_cast<size_t>(B) * Hq * npad * sizeof(float);
}

template <int D>
int launch_bwd(DeviceState *ds, const void *q, const void *k, const void *v, const void *o,
               const void *dout, const float *lse, void *dq, void *dk, void *dv, int B, int Hq,
               int Hkv, int N, float scale, int causal, const int *seqlens, void *workspace,
               cudaStream_t stream, int *status) {
  using C = fa::BwdCfg<D>;
  bool &attr = (D == 64) ? ds->bwd_attr64 : ds->bwd_attr128;
  if (!attr) {
    if (cudaFuncSetAttribute(fa::fa_bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM_KV) != cudaSuccess ||
        cudaFuncSetAttribute(fa::fa_bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM_Q) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_LAUNCH;
    }
    attr = true;
  }
  CUtensorMap tq, tk, tv, tdo;
  if (make_map(&tq, q, B * Hq, N, D) != FA_OK || make_map(&tk, k, B * Hkv, N, D) != FA_OK ||
      make_map(&tv, v, B * Hkv, N, D) != FA_OK || make_map(&tdo, dout, B * Hq, N, D) != FA_OK)
    return FA_ERR_CUDA;
  fa::BwdParams p;
  p.o = static_cast<const uint16_t *>(o);
  p.dout = static_cast<const uint16_t *>(dout);
  p.lse = lse;
  p.dq = static_cast<uint16_t *>(dq);
  p.dk = static_cast<uint16_t *>(dk);
  p.dv = static_cast<uint16_t *>(dv);
  p.Npad = (N + 127) / 128 * 128;
  const size_t vec = static_cast<size_t>(B) * Hq * p.Npad;
  p.ws_nlse2 = static_cast<float *>(workspace);
  p.ws_delta = p.ws_nlse2 + vec;
  p.seqlens = seqlens;
  p.status = status;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.group = Hq / Hkv;
  p.causal = causal ? 1 : 0;
  p.q_tiles = p.Npad / 128;
  p.scale = scale;
  p.scale_log2 = scale * kLog2e;
  p.wait_limit_ns = kWaitLimitNs;
  const long long prep_blocks = (static_cast<long long>(vec) + 127) / 128;
  const long long kv_units = static_cast<long long>(p.q_tiles) * B * Hkv;
  const long long q_units = static_cast<long long>(p.q_tiles) * B * Hq;
  if (prep_blocks > 0x7fffffffll || kv_units > 0x7fffffffll || q_units > 0x7fffffffll)
    return FA_ERR_SHAPE;
  // The dK/dV and dQ kernels read the same inputs and write disjoint outputs,
  // so they run side by side: dK/dV on `stream`, dQ on a second stream,
  // both after the prep kernel.  dK/dV is queued first; as its CTAs run out,
  // dQ CTAs take the SMs its causal tail leaves idle (about 12 % of its SM
  // time on the GQA layer when it runs alone).
  std::lock_guard<std::mutex> lock(ds->bwd_mu);
  if (!ds->bwd_ready) {
    if (cudaStreamCreateWithFlags(&ds->bwd_side, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&ds->bwd_fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ds->bwd_join, cudaEventDisableTiming) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
    ds->bwd_ready = true;
  }
  fa::fa_bwd_prep_kernel<D><<<static_cast<unsigned>(prep_blocks), 128, 0, stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_LAUNCH;
  if (cudaEventRecord(ds->bwd_fork, stream) != cudaSuccess ||
      cudaStreamWaitEvent(ds->bwd_side, ds->bwd_fork, 0) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  fa::fa_bwd_dkdv_kernel<D><<<static_cast<unsigned>(kv_units), C::THREADS, C::SMEM_KV, stream>>>(
      tq, tk, tv, tdo, p);
  const bool kv_ok = cudaGetLastError() == cudaSuccess;
  fa::fa_bwd_dq_kernel<D>
      <<<static_cast<unsigned>(q_units), C::THREADS, C::SMEM_Q, ds->bwd_side>>>(tq, tk, tv, tdo, p);
  const bool q_ok = cudaGetLastError() == cudaSuccess;
  // Join whatever was queued, so `stream` never runs ahead of the dQ kernel.
  if (cudaEventRecord(ds->bwd_join, ds->bwd_side) != cudaSuccess ||
      cudaStreamWaitEvent(stream, ds->bwd_join, 0) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  return kv_ok && q_ok ? FA_OK : FA_ERR_LAUNCH;
}

// Waits on a barrier that nothing arrives at; the bounded wait must give up.
__global__ void bounded_wait_selftest_kernel(int *status, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  fa::mbar_init(fa::smem_u32(&bar), 1);
  fa::fence_barrier_init();
  fa::mbar_wait_bounded(fa::smem_u32(&bar), 0, reinterpret_cast<volatile int *>(&abort_flag), status,
                        limit_ns, fa::kErrTimeout);
}

// Calibration of the exponential unit: every thread runs 8 independent
// chains x <- 2^(-|x|) of ex2.approx.ftz.f32 (the instruction the softmax
// uses; the values stay in (0, 1]) and each block records its cycle count and
// SM.  Sized so that one block per SM keeps the unit busy: 32 warps, 8 chains.
constexpr int kEx2Threads = 1024, kEx2Chains = 8, kEx2Iters = 2048, kEx2MaxBlocks = 1024;
__device__ long long g_ex2_cycles[kEx2MaxBlocks];
__device__ int g_ex2_smid[kEx2MaxBlocks];
__device__ float g_ex2_sink[kEx2MaxBlocks];

__global__ void __launch_bounds__(kEx2Threads) ex2_rate_kernel() {
  float x[kEx2Chains];
#pragma unroll
  for (int c = 0; c < kEx2Chains; ++c) x[c] = -0.001f * static_cast<float>(threadIdx.x + 37 * c);
  __syncthreads();
  const long long t0 = clock64();
  for (int it = 0; it < kEx2Iters; ++it) {
#pragma unroll
    for (int c = 0; c < kEx2Chains; ++c) x[c] = fa::ex2_approx(-fabsf(x[c]));
  }
  __syncthreads();
  const long long t1 = clock64();
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < kEx2Chains; ++c) acc += x[c];
  if (acc == 12345.f) g_ex2_sink[blockIdx.x] = acc;  // keeps the chains live
  if (threadIdx.x == 0) {
    uint32_t smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    g_ex2_cycles[blockIdx.x] = t1 - t0;
    g_ex2_smid[blockIdx.x] = static_cast<int>(smid);
  }
}

}  // namespace

extern "C" {

int fa_version(void) { return 100; }

const char *fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "ok";
    case FA_ERR_NULL: return "a required pointer is NULL";
    case FA_ERR_SHAPE: return "bad shape or scale";
    case FA_ERR_HEADS: return "Hq is not a multiple of Hkv";
    case FA_ERR_HEADDIM: return "head dimension not supported (64 or 128)";
    case FA_ERR_ALIGN: return "pointer not 16-byte aligned";
    case FA_ERR_ARCH: return "no sm_100 (B200) CUDA device";
    case FA_ERR_LAUNCH: return "kernel launch failed";
    case FA_ERR_TIMEOUT: return "a bounded in-kernel wait ran out";
    case FA_ERR_DTYPE: return "unknown dtype code";
    case FA_ERR_CUDA: return "CUDA runtime error";
    case FA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    default: return "unknown status";
  }
}

int fa_fwd_ex(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
              int Hkv, int N, int d, float scale, int causal, const int *seqlens, int dtype,
              void *stream, int *status_dev) {
  int rc = check_args(q, k, v, o, lse, B, Hq, Hkv, N, d, scale);
  if (rc != FA_OK) return rc;
  if (dtype != FA_DTYPE_BF16 && dtype != FA_DTYPE_F32) return FA_ERR_DTYPE;
  DeviceState *ds = nullptr;
  rc = current_device(&ds);
  if (rc != FA_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == FA_DTYPE_F32) {
    const float *qf = static_cast<const float *>(q), *kf = static_cast<const float *>(k),
                *vf = static_cast<const float *>(v);
    float *of = static_cast<float *>(o);
    return d == 64 ? launch_f32<64>(qf, kf, vf, of, lse, B, Hq, Hkv, N, scale, causal, seqlens, st)
                   : launch_f32<128>(qf, kf, vf, of, lse, B, Hq, Hkv, N, scale, causal, seqlens,
                                     st);
  }
  int *status = status_dev ? status_dev : ds->status_word;
  return d == 64 ? launch_bf16<64>(ds, q, k, v, o, lse, B, Hq, Hkv, N, scale, causal, seqlens, st,
                                   status)
                 : launch_bf16<128>(ds, q, k, v, o, lse, B, Hq, Hkv, N, scale, causal, seqlens,
                                    st, status);
}

int fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
           int Hkv, int N, int d, float scale, int causal, const int *seqlens) {
  return fa_fwd_ex(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal, seqlens, FA_DTYPE_BF16,
                   nullptr, nullptr);
}

int fa_fwd_f32(const float *q, const float *k, const float *v, float *o, float *lse, int B,
               int Hq, int Hkv, int N, int d, float scale, int causal, const int *seqlens) {
  return fa_fwd_ex(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal, seqlens, FA_DTYPE_F32,
                   nullptr, nullptr);
}

int fa_check_status(const int *status_dev, void *stream) {
  DeviceState *ds = nullptr;
  int rc = current_device(&ds);
  if (rc != FA_OK) return rc;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  int word = 0;
  if (status_dev) {
    if (cudaMemcpy(&word, status_dev, sizeof word, cudaMemcpyDeviceToHost) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
  } else {
    if (cudaMemcpyFromSymbol(&word, g_status_word, sizeof word) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
    const int zero = 0;
    if (word != 0 && cudaMemcpyToSymbol(g_status_word, &zero, sizeof zero) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
  }
  return word == 0 ? FA_OK : word;
}

}  // extern "C"

namespace {
// fa_fwd_hostio and fa_fwd_hostio_async; `wait` makes the call synchronous.
int hostio_impl(const void *q_h, const void *k_h, const void *v_h, void *o_h, float *lse_h,
                const int *seqlens_h, void *q_d, void *k_d, void *v_d, void *o_d, float *lse_d,
                int *seqlens_d, int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                void *stream, bool wait) {
  if (!q_h || !k_h || !v_h || !o_h || !lse_h) return FA_ERR_NULL;
  if (seqlens_h && !seqlens_d) return FA_ERR_NULL;
  int rc = check_args(q_d, k_d, v_d, o_d, lse_d, B, Hq, Hkv, N, d, scale);
  if (rc != FA_OK) return rc;
  DeviceState *ds = nullptr;
  rc = current_device(&ds);
  if (rc != FA_OK) return rc;
  std::lock_guard<std::mutex> io_lock(ds->io_mu);
  if (!ds->io_ready) {
    bool ok = cudaStreamCreateWithFlags(&ds->io_in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&ds->io_out, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&ds->io_ev_end, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; ok && i < 16; ++i)
      ok = cudaEventCreateWithFlags(&ds->io_ev_in[i], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&ds->io_ev_done[i], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
    ds->io_ready = true;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // Slices run as problems of their own, so slice s's copies in and s-1's
  // copies out overlap the forward of slice s.  Without key lengths a slice
  // is a run of consecutive (batch, kv head) pairs -- contiguous in q, k, v,
  // o and lse, and an attention problem of its own with batch = its kv heads
  // and Hkv = 1; with key lengths it is a run of whole batches.
  // Eight slices: on the GQA layer (16 pieces, 201 MB in, 136 MB out) a call
  // took 5.55 ms with 16 slices, 4.81 with 8, 4.87 with 6, 4.98 with 4 and
  // 5.11 with 12.  Each slice costs a fixed amount beyond its copies, and
  // large slices lengthen the forward and copy-out after the last input
  // copy; both directions of the link together bound the call at 4.05 ms.
  const int G = Hq / Hkv;
  const int units = seqlens_h ? B : B * Hkv;            // indivisible pieces
  const int nslices = units < 8 ? units : 8;
  const size_t q_unit = static_cast<size_t>(seqlens_h ? Hq : G) * N * d;   // elements
  const size_t k_unit = static_cast<size_t>(seqlens_h ? Hkv : 1) * N * d;
  const size_t l_unit = static_cast<size_t>(seqlens_h ? Hq : G) * N;
  auto bytes16 = [](const void *p, size_t off) {
    return static_cast<const uint8_t *>(p) + off * 2;
  };
  auto fail = [&]() {
    ds->io_prev = false;
    cudaGetLastError();
    cudaStreamSynchronize(ds->io_in);
    cudaStreamSynchronize(ds->io_out);
    cudaStreamSynchronize(st);
    cudaGetLastError();
    return FA_ERR_CUDA;
  };
  // The slices' inputs must not be overwritten before earlier work has
  // finished with the device buffers.  An asynchronous call chained to the
  // previous asynchronous one (same device buffers, shape and stream, no key
  // lengths) waits per slice for the previous call's forward of that slice,
  // so its copies in start while the previous call's last slices are
  // computed and copied out; any other call waits for all earlier work on
  // `stream`.  The forward of a slice runs on `stream`, after the previous
  // call's copies out (joined to `stream` at the end of every call).
  const void *ptrs[5] = {q_d, k_d, v_d, o_d, lse_d};
  const int shape[5] = {B, Hq, Hkv, N, d};
  const bool chained = !wait && !seqlens_h && ds->io_prev && ds->io_prev_stream == st &&
                       std::equal(ptrs, ptrs + 5, ds->io_prev_ptr) &&
                       std::equal(shape, shape + 5, ds->io_prev_shape);
  ds->io_prev = false;
  if (!chained && (cudaEventRecord(ds->io_ev_end, st) != cudaSuccess ||
                   cudaStreamWaitEvent(ds->io_in, ds->io_ev_end, 0) != cudaSuccess))
    return fail();
  if (seqlens_h && cudaMemcpyAsync(seqlens_d, seqlens_h, sizeof(int) * B, cudaMemcpyHostToDevice,
                                   ds->io_in) != cudaSuccess)
    return fail();
  for (int s = 0; s < nslices; ++s) {
    const int u0 = static_cast<int>(static_cast<long long>(units) * s / nslices);
    const int u1 = static_cast<int>(static_cast<long long>(units) * (s + 1) / nslices);
    const int nu = u1 - u0;
    const size_t qo = q_unit * u0, ko = k_unit * u0, lo = l_unit * u0;
    if (chained && cudaStreamWaitEvent(ds->io_in, ds->io_ev_done[s], 0) != cudaSuccess)
      return fail();
    if (cudaMemcpyAsync(const_cast<uint8_t *>(bytes16(q_d, qo)), bytes16(q_h, qo),
                        q_unit * nu * 2, cudaMemcpyHostToDevice, ds->io_in) != cudaSuccess ||
        cudaMemcpyAsync(const_cast<uint8_t *>(bytes16(k_d, ko)), bytes16(k_h, ko),
                        k_unit * nu * 2, cudaMemcpyHostToDevice, ds->io_in) != cudaSuccess ||
        cudaMemcpyAsync(const_cast<uint8_t *>(bytes16(v_d, ko)), bytes16(v_h, ko),
                        k_unit * nu * 2, cudaMemcpyHostToDevice, ds->io_in) != cudaSuccess ||
        cudaEventRecord(ds->io_ev_in[s], ds->io_in) != cudaSuccess ||
        cudaStreamWaitEvent(st, ds->io_ev_in[s], 0) != cudaSuccess)
      return fail();
    rc = seqlens_h
             ? fa_fwd_ex(bytes16(q_d, qo), bytes16(k_d, ko), bytes16(v_d, ko),
                         const_cast<uint8_t *>(bytes16(o_d, qo)), lse_d + lo, nu, Hq, Hkv, N, d,
                         scale, causal, seqlens_d + u0, FA_DTYPE_BF16, stream, nullptr)
             : fa_fwd_ex(bytes16(q_d, qo), bytes16(k_d, ko), bytes16(v_d, ko),
                         const_cast<uint8_t *>(bytes16(o_d, qo)), lse_d + lo, nu, G, 1, N, d,
                         scale, causal, nullptr, FA_DTYPE_BF16, stream, nullptr);
    if (rc != FA_OK) {
      fail();
      return rc;
    }
    if (cudaEventRecord(ds->io_ev_done[s], st) != cudaSuccess ||
        cudaStreamWaitEvent(ds->io_out, ds->io_ev_done[s], 0) != cudaSuccess ||
        cudaMemcpyAsync(const_cast<uint8_t *>(bytes16(o_h, qo)), bytes16(o_d, qo),
                        q_unit * nu * 2, cudaMemcpyDeviceToHost, ds->io_out) != cudaSuccess ||
        cudaMemcpyAsync(lse_h + lo, lse_d + lo, l_unit * nu * sizeof(float),
                        cudaMemcpyDeviceToHost, ds->io_out) != cudaSuccess)
      return fail();
  }
  if (cudaEventRecord(ds->io_ev_end, ds->io_out) != cudaSuccess ||
      cudaStreamWaitEvent(st, ds->io_ev_end, 0) != cudaSuccess)
    return fail();
  if (!wait && !seqlens_h) {
    std::copy(ptrs, ptrs + 5, ds->io_prev_ptr);
    std::copy(shape, shape + 5, ds->io_prev_shape);
    ds->io_prev_stream = st;
    ds->io_prev = true;
  }
  return wait ? fa_check_status(nullptr, stream) : FA_OK;
}
}  // namespace

extern "C" {

int fa_fwd_hostio(const void *q_h, const void *k_h, const void *v_h, void *o_h, float *lse_h,
                  const int *seqlens_h, void *q_d, void *k_d, void *v_d, void *o_d, float *lse_d,
                  int *seqlens_d, int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                  void *stream) {
  return hostio_impl(q_h, k_h, v_h, o_h, lse_h, seqlens_h, q_d, k_d, v_d, o_d, lse_d, seqlens_d,
                     B, Hq, Hkv, N, d, scale, causal, stream, true);
}

int fa_fwd_hostio_async(const void *q_h, const void *k_h, const void *v_h, void *o_h,
                        float *lse_h, const int *seqlens_h, void *q_d, void *k_d, void *v_d,
                        void *o_d, float *lse_d, int *seqlens_d, int B, int Hq, int Hkv, int N,
                        int d, float scale, int causal, void *stream) {
  return hostio_impl(q_h, k_h, v_h, o_h, lse_h, seqlens_h, q_d, k_d, v_d, o_d, lse_d, seqlens_d,
                     B, Hq, Hkv, N, d, scale, causal, stream, false);
}

int fa_fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse,
                  const int *cu_seqlens, int B, int Hq, int Hkv, int total, int max_seqlen, int d,
                  float scale, int causal, void *stream, int *status_dev) {
  if (!cu_seqlens) return FA_ERR_NULL;
  int rc = check_args(q, k, v, o, lse, B, Hq, Hkv, max_seqlen, d, scale);
  if (rc != FA_OK) return rc;
  if (total <= 0 || static_cast<long long>(total) * Hq * d > (1ll << 40)) return FA_ERR_SHAPE;
  DeviceState *ds = nullptr;
  rc = current_device(&ds);
  if (rc != FA_OK) return rc;
  int *status = status_dev ? status_dev : ds->status_word;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return d == 64 ? launch_bf16<64>(ds, q, k, v, o, lse, B, Hq, Hkv, max_seqlen, scale, causal,
                                   nullptr, st, status, cu_seqlens, total)
                 : launch_bf16<128>(ds, q, k, v, o, lse, B, Hq, Hkv, max_seqlen, scale, causal,
                                    nullptr, st, status, cu_seqlens, total);
}

int fa_fwd_fp8(const void *q, const void *k, const void *vt, void *o, float *lse, int B, int Hq,
               int Hkv, int N, int ldvt, int d, float scale, float descale_q, float descale_k,
               float descale_v, int causal, const int *seqlens, void *stream, int *status_dev) {
  int rc = check_args(q, k, vt, o, lse, B, Hq, Hkv, N, d, scale);
  if (rc != FA_OK) return rc;
  if (d != 128) return FA_ERR_HEADDIM;
  for (float f : {descale_q, descale_k, descale_v})
    if (!(std::isfinite(f) && f > 0.f)) return FA_ERR_SHAPE;
  if (ldvt < N) return FA_ERR_SHAPE;
  if (ldvt % 16 != 0) return FA_ERR_ALIGN;
  DeviceState *ds = nullptr;
  rc = current_device(&ds);
  if (rc != FA_OK) return rc;
  int *status = status_dev ? status_dev : ds->status_word;
  return launch_fp8(ds, q, k, vt, o, lse, B, Hq, Hkv, N, ldvt, scale, descale_q, descale_k,
                    descale_v, causal, seqlens, static_cast<cudaStream_t>(stream), status);
}

size_t fa_bwd_workspace_size(int B, int Hq, int N) {
  if (B <= 0 || Hq <= 0 || N <= 0) return 0;
  return bwd_workspace_bytes(B, Hq, N);
}

int fa_bwd(const void *q, const void *k, const void *v, const void *o, const void *dout,
           const float *lse, void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int N, int d,
           float scale, int causal, const int *seqlens, void *workspace, size_t workspace_bytes,
           void *stream, int *status_dev) {
  int rc = check_args(q, k, v, o, lse, B, Hq, Hkv, N, d, scale);
  if (rc != FA_OK) return rc;
  if (!dout || !dq || !dk || !dv) return FA_ERR_NULL;
  if (!aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv)) return FA_ERR_ALIGN;
  if (!workspace || !aligned16(workspace) || workspace_bytes < bwd_workspace_bytes(B, Hq, N))
    return FA_ERR_WORKSPACE;
  DeviceState *ds = nullptr;
  rc = current_device(&ds);
  if (rc != FA_OK) return rc;
  int *status = status_dev ? status_dev : ds->status_word;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return d == 64 ? launch_bwd<64>(ds, q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, N, scale,
                                  causal, seqlens, workspace, st, status)
                 : launch_bwd<128>(ds, q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, N, scale,
                                   causal, seqlens, workspace, st, status);
}

size_t fa_decode_workspace_size(int B, int Hq, int Hkv, int Nq, int Nk, int d, int num_splits) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nk <= 0 || (d != 64 && d != 128) ||
      Hq % Hkv != 0 || num_splits < 0)
    return 0;
  if (decode_uses_tc(Hq, Hkv, Nq))
    return decode_tc_workspace_bytes(B, Hkv, d,
                                     decode_tc_ctas(B, Hkv, num_splits, kDecodeTcAutoCtasMax),
                                     decode_tc_part_rows(Hq, Hkv, Nq));
  const int groups = ((Hq / Hkv) * Nq + 3) / 4;
  const DecodeSplit sp = decode_split(B, Hkv, groups, Nk, d, num_splits);
  return decode_workspace_bytes(B, Hq, Nq, d, sp.splits);
}

int fa_fwd_decode(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                  int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                  const int *seqlens_k, int num_splits, void *workspace, size_t workspace_bytes,
                  void *stream, int *status_dev) {
  int rc = check_decode_args(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale);
  if (rc != FA_OK) return rc;
  if (num_splits < 0 || num_splits > 128) return FA_ERR_SHAPE;
  // The workspace must hold what fa_decode_workspace_size reports, which does
  // not depend on the device.
  if (!workspace || !aligned16(workspace) ||
      workspace_bytes < fa_decode_workspace_size(B, Hq, Hkv, Nq, Nk, d, num_splits))
    return FA_ERR_WORKSPACE;
  DeviceState *ds = nullptr;
  rc = current_device(&ds);
  if (rc != FA_OK) return rc;
  int *status = status_dev ? status_dev : ds->status_word;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (decode_uses_tc(Hq, Hkv, Nq)) {
    const int ctas = decode_tc_ctas(B, Hkv, num_splits, ds->num_sms);
    return d == 64 ? launch_decode_tc<64>(ds, q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, causal,
                                          seqlens_k, ctas, workspace, st, status)
                   : launch_decode_tc<128>(ds, q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale,
                                           causal, seqlens_k, ctas, workspace, st, status);
  }
  const int groups = ((Hq / Hkv) * Nq + 3) / 4;
  const DecodeSplit sp = decode_split(B, Hkv, groups, Nk, d, num_splits);
  return d == 64 ? launch_decode<64>(ds, q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, causal,
                                     seqlens_k, sp, workspace, st, status)
                 : launch_decode<128>(ds, q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, causal,
                                      seqlens_k, sp, workspace, st, status);
}

int fa_measure_ex2_rate(float *ex2_per_clk, void *stream) {
  if (!ex2_per_clk) return FA_ERR_NULL;
  DeviceState *ds = nullptr;
  int rc = current_device(&ds);
  if (rc != FA_OK) return rc;
  const int blocks = std::min(ds->num_sms, kEx2MaxBlocks);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ex2_rate_kernel<<<blocks, kEx2Threads, 0, st>>>();
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_LAUNCH;
  if (cudaStreamSynchronize(st) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  std::vector<long long> cyc(blocks);
  std::vector<int> sm(blocks);
  if (cudaMemcpyFromSymbol(cyc.data(), g_ex2_cycles, sizeof(long long) * blocks) != cudaSuccess ||
      cudaMemcpyFromSymbol(sm.data(), g_ex2_smid, sizeof(int) * blocks) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  // Per SM: the exponentials of its blocks over the longest of their times
  // (blocks that shared an SM ran side by side); the median over SMs.
  std::vector<std::pair<int, long long>> per;  // (smid, cycles), sorted by smid
  for (int i = 0; i < blocks; ++i) per.emplace_back(sm[i], cyc[i]);
  std::sort(per.begin(), per.end());
  std::vector<double> rates;
  const double ops_per_block = static_cast<double>(kEx2Threads) * kEx2Chains * kEx2Iters;
  for (size_t i = 0; i < per.size();) {
    size_t j = i;
    long long longest = 0;
    while (j < per.size() && per[j].first == per[i].first) longest = std::max(longest, per[j++].second);
    if (longest > 0) rates.push_back(ops_per_block * static_cast<double>(j - i) / longest);
    i = j;
  }
  if (rates.empty()) return FA_ERR_CUDA;
  std::sort(rates.begin(), rates.end());
  *ex2_per_clk = static_cast<float>(rates[rates.size() / 2]);
  return FA_OK;
}

int fa_selftest_bounded_wait(int *status_dev, unsigned long long limit_ns, void *stream) {
  if (!status_dev) return FA_ERR_NULL;
  DeviceState *ds = nullptr;
  int rc = current_device(&ds);
  if (rc != FA_OK) return rc;
  bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(status_dev,
                                                                              limit_ns);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_LAUNCH;
  return FA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode for callers that cannot allocate device memory (fa_fwd_decode_noalloc)
// ---------------------------------------------------------------------------
// The per-range partials live in one fixed array owned by this library
// instead of a caller-provided workspace.  Every GPU that loads the library
// keeps these 8 MiB until the process exits.  In host code the symbol is a
// host-side stand-in, so its device address is looked up once per device.
static __device__ __align__(256) float g_decode_noalloc_scratch[(8u << 20) / sizeof(float)];

namespace {
constexpr size_t kNoAllocScratchBytes = 8u << 20;
void *g_noalloc_scratch_addr[kMaxDevices];
std::mutex g_noalloc_mu;

// With `dev` current: the device address of the scratch array, looked up on
// the first call for that device and remembered.
int noalloc_scratch(int dev, void **out) {
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_scratch_addr[dev]) {
    void *ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_decode_noalloc_scratch);
    if (e != cudaSuccess || !ptr) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
    g_noalloc_scratch_addr[dev] = ptr;
  }
  *out = g_noalloc_scratch_addr[dev];
  return FA_OK;
}
}  // namespace

extern "C" int fa_fwd_decode_noalloc(const void *q, const void *k, const void *v, void *o,
                                     float *lse, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                                     float scale, int causal, const int *seqlens_k,
                                     int num_splits, void *stream, int *status_dev) {
  int rc = check_decode_args(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale);
  if (rc != FA_OK) return rc;
  if (num_splits < 0 || num_splits > 128) return FA_ERR_SHAPE;
  const bool tc = decode_uses_tc(Hq, Hkv, Nq);
  const int groups = ((Hq / Hkv) * Nq + 3) / 4;
  const DecodeSplit sp = decode_split(B, Hkv, groups, Nk, d, num_splits);
  // the size fa_decode_workspace_size reports, so a shape is accepted or
  // rejected whatever the device
  const size_t need = tc ? decode_tc_workspace_bytes(
                               B, Hkv, d, decode_tc_ctas(B, Hkv, num_splits, kDecodeTcAutoCtasMax),
                               decode_tc_part_rows(Hq, Hkv, Nq))
                         : decode_workspace_bytes(B, Hq, Nq, d, sp.splits);
  if (need > kNoAllocScratchBytes) return FA_ERR_WORKSPACE;
  DeviceState *ds = nullptr;
  rc = current_device(&ds);
  if (rc != FA_OK) return rc;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  void *scratch = nullptr;
  rc = noalloc_scratch(dev, &scratch);
  if (rc != FA_OK) return rc;
  int *status = status_dev ? status_dev : ds->status_word;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tc) {
    const int ctas = decode_tc_ctas(B, Hkv, num_splits, ds->num_sms);
    return d == 64 ? launch_decode_tc<64>(ds, q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, causal,
                                          seqlens_k, ctas, scratch, st, status)
                   : launch_decode_tc<128>(ds, q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale,
                                           causal, seqlens_k, ctas, scratch, st, status);
  }
  return d == 64 ? launch_decode<64>(ds, q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, causal,
                                     seqlens_k, sp, scratch, st, status)
                 : launch_decode<128>(ds, q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, causal,
                                      seqlens_k, sp, scratch, st, status);
}
