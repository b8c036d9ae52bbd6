/*
 * fa.h - exact, IO-aware attention for NVIDIA B200 (sm_100a).
 *
 * The forward operation, which every fa_fwd* call computes (fa_bwd
 * differentiates it, fa_fwd_decode evaluates it for a few query rows
 * against a long key range): for every batch b, query head h and query
 * row i,
 *
 *     O[b,h,i,:] = softmax_j( scale * Q[b,h,i,:] . K[b,g,j,:] + mask(i,j) ) V[b,g,j,:]
 *     LSE[b,h,i] = log sum_j exp( scale * Q[b,h,i,:] . K[b,g,j,:] + mask(i,j) )
 *
 * with g = h / (Hq / Hkv) (query heads [g*G, (g+1)*G) share kv head g) and
 * mask(i,j) = -inf when j >= len_b or (causal and j > i), else 0.
 *
 * Sources, by page title and section:
 *  - wiki note "FlashAttention", section "what it is": the formula
 *    O = softmax(QK^T / sqrt(d)) V; the blockwise recurrence for the running
 *    row max m, row sum l and output O when a new block S_b = Q_b K_b^T/sqrt(d)
 *    arrives; causal mask, padding mask and multiple heads handled inside the
 *    tile; the SDPA call with is_causal and enable_gqa that states the problem.
 *  - explainer "FlashAttention" (liu-gong-zi): only the final result is stored.
 * The result is exact up to floating-point rounding (same page; interview
 * notes "Why is FlashAttention faster", section on exactness): no N x N
 * score or probability matrix is ever written to device memory.
 *
 * LSE is not on the pages: it is the per-row statistic a backward pass
 * recomputes from (interview notes, section on recomputation), exported in
 * natural-log units.
 *
 * Common conventions for every fa_fwd* call
 *  - Layout: all tensors contiguous, row-major, head dimension innermost.
 *      q, o : [B, Hq, N, d]      k, v : [B, Hkv, N, d]      lse : [B, Hq, N] fp32
 *  - Key padding: seqlens is NULL (every key of the N is visible) or a
 *    DEVICE pointer to int32[B] with 0 <= seqlens[b] <= N; keys
 *    j >= seqlens[b] are masked; every query row is still computed.  A row
 *    with no visible key (seqlens[b] == 0) gets O = 0 and LSE = -inf.
 *  - Causal: key j is visible to query i iff j <= i (queries and keys share
 *    the index range [0, N)).
 *  - Ownership: the caller allocates and owns every buffer; the library
 *    allocates no device memory per call and keeps no pointer after the call
 *    returns.  Device pointers must stay valid until the launched work ends.
 *  - Streams: fa_fwd launches on the legacy default stream; the _ex forms
 *    take a cudaStream_t (passed as void*, NULL = legacy default stream).
 *    Launches are asynchronous.
 *  - Errors: argument errors are reported synchronously and launch nothing.
 *    Every wait inside a kernel is bounded; a wait that runs out makes the
 *    kernel write FA_ERR_TIMEOUT into the status word and return, so no call
 *    can hang the device.  fa_check_status() reads that word.  Nothing aborts,
 *    traps or throws across this interface.
 */
#ifndef FA_B200_FA_H
#define FA_B200_FA_H

#include <stddef.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_NULL = -1,      /* a required pointer is NULL */
  FA_ERR_SHAPE = -2,     /* B, Hq, Hkv, N or d <= 0, scale not finite and > 0, or sizes overflow */
  FA_ERR_HEADS = -3,     /* Hq is not a multiple of Hkv */
  FA_ERR_HEADDIM = -4,   /* d not supported: the bf16 kernel takes d in {64, 128}, fp32 d in {64, 128} */
  FA_ERR_ALIGN = -5,     /* a pointer is not 16-byte aligned (tensor-memory-access rule) */
  FA_ERR_ARCH = -6,      /* no CUDA device, or the current device is not sm_100 */
  FA_ERR_LAUNCH = -7,    /* the CUDA launch itself failed */
  FA_ERR_TIMEOUT = -8,   /* a bounded in-kernel wait ran out (reported by fa_check_status) */
  FA_ERR_DTYPE = -9,     /* unknown dtype code */
  FA_ERR_CUDA = -10,     /* another CUDA runtime error (copy, query, driver entry point) */
  FA_ERR_WORKSPACE = -11 /* workspace missing, misaligned or smaller than required */
} fa_status;

/* dtype codes for fa_fwd_ex */
#define FA_DTYPE_BF16 0
#define FA_DTYPE_F32 1

/*
 * Attention forward, bf16 in / bf16 out, fp32 LSE, on the tensor cores.
 *  q, k, v, o: bf16 device buffers in the layout above; lse: fp32 device.
 *  B, Hq, Hkv, N, d: batch, query heads, kv heads, sequence length, head dim
 *  (d in {64, 128}).  scale: multiplies Q.K (the pages use 1/sqrt(d)).
 *  causal: 0 or 1.  seqlens: NULL or device int32[B].
 * Returns FA_OK once the kernel is launched on the legacy default stream, or
 * an fa_status code.  Device-side waits that run out are recorded in the
 * library's own status word: read it with fa_check_status(NULL, stream).
 */
FA_API int fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
           int Hkv, int N, int d, float scale, int causal, const int *seqlens);

/*
 * Same operation with an explicit element type and stream.
 *  dtype: FA_DTYPE_BF16 (tensor-core kernel) or FA_DTYPE_F32 (fp32 check
 *         mode: q, k, v, o are fp32, plain CUDA-core arithmetic).
 *  stream: cudaStream_t or NULL.
 *  status_dev: NULL (use the library's status word) or a device int the
 *         kernel sets to FA_ERR_TIMEOUT when a bounded wait runs out; the
 *         caller zeroes it before the call and reads it with fa_check_status.
 */
FA_API int fa_fwd_ex(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
              int Hkv, int N, int d, float scale, int causal, const int *seqlens, int dtype,
              void *stream, int *status_dev);

/*
 * fp32 check mode: same operation with fp32 q, k, v, o.  The online-softmax
 * recurrence runs in fp32 on CUDA cores with accurate exp2f, for comparisons
 * at 1e-5.  Same stream and status rules as fa_fwd.
 */
FA_API int fa_fwd_f32(const float *q, const float *k, const float *v, float *o, float *lse, int B,
               int Hq, int Hkv, int N, int d, float scale, int causal, const int *seqlens);

/*
 * End-to-end call on HOST buffers: copies q, k, v (and seqlens) from host to
 * the caller's device buffers, runs the bf16 forward and copies o and lse
 * back, then waits.  The work runs in up to 8 slices so that copies overlap
 * the forward: runs of consecutive (batch, kv head) pairs, or of whole
 * batches when seqlens is given.  The copies go on two streams the library
 * creates once per device; the forward runs on `stream`, which first waits
 * for them.  Before the first copy the copy stream waits for work already
 * queued on `stream`.  Calls from several host threads on one device are
 * served one at a time.
 *  q_h, k_h, v_h, o_h, lse_h, seqlens_h: host buffers (pinned memory gives
 *  asynchronous copies; seqlens_h may be NULL).
 *  q_d, k_d, v_d, o_d, lse_d, seqlens_d: device buffers of the same sizes
 *  (seqlens_d only when seqlens_h is given).
 * Returns FA_OK when everything, including the device work, has finished
 * without error; a bounded wait that ran out is returned as FA_ERR_TIMEOUT.
 */
FA_API int fa_fwd_hostio(const void *q_h, const void *k_h, const void *v_h, void *o_h, float *lse_h,
                  const int *seqlens_h, void *q_d, void *k_d, void *v_d, void *o_d, float *lse_d,
                  int *seqlens_d, int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                  void *stream);

/*
 * fa_fwd_hostio without the final wait, for a stream of steps on host
 * buffers.  Same arguments, same work, ordered on `stream`.  It returns FA_OK
 * once everything is queued, or an error before anything is queued.
 * Completion: synchronise `stream` (fa_check_status reads the status word
 * then).  Host buffers must stay valid and unchanged until then.
 *
 * Chaining.  A call that follows another fa_fwd_hostio_async call with the
 * same device buffers, the same B, Hq, Hkv, N, d and the same stream, without
 * key lengths, is chained to it.  Its copy into the device buffers for a
 * slice waits only for the previous call's forward of that slice, not for
 * all of the previous call's work, so its copies in overlap the previous
 * call's last forward and copies out.  Between two chained calls, no other
 * work may read or write q_d, k_d or v_d; o_d and lse_d follow stream order.
 * Any other call waits for all earlier work on `stream` before it overwrites
 * the device buffers.
 */
FA_API int fa_fwd_hostio_async(const void *q_h, const void *k_h, const void *v_h, void *o_h,
                               float *lse_h, const int *seqlens_h, void *q_d, void *k_d, void *v_d,
                               void *o_d, float *lse_d, int *seqlens_d, int B, int Hq, int Hkv,
                               int N, int d, float scale, int causal, void *stream);

/*
 * Attention backward by recomputation: the gradients of sum(dout * O) for
 * O = fa_fwd(q, k, v, ...), rebuilt from q, k, v, o, dout and the forward's
 * LSE without any stored probability matrix (interview notes "Why is
 * FlashAttention faster", section on memory: training stores less by
 * recomputing; exam explainer, "recomputation").
 *  q, o, dout, dq : [B, Hq, N, d] bf16     k, v, dk, dv : [B, Hkv, N, d] bf16
 *  lse : [B, Hq, N] fp32 from the forward with the same arguments.
 *  dk, dv sum over the query heads that share each kv head.  causal and
 *  seqlens as in fa_fwd.  d in {64, 128}.
 *  workspace: DEVICE buffer of at least fa_bwd_workspace_size(B, Hq, N)
 *  bytes, 16-byte aligned (per-row D = rowsum(dout * o) and LSE*log2(e)).
 * Three kernels: the per-row preprocess, then the dK/dV kernel (one CTA per
 * 128-key tile) on `stream` and the dQ kernel (one CTA per 128-row tile) on
 * a second stream the library creates once per device.  The dQ kernel
 * waits for the preprocess, and `stream` waits for the dQ kernel, so all the
 * work is ordered on `stream` as one call.
 */
FA_API size_t fa_bwd_workspace_size(int B, int Hq, int N);
FA_API int fa_bwd(const void *q, const void *k, const void *v, const void *o, const void *dout,
                  const float *lse, void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int N,
                  int d, float scale, int causal, const int *seqlens, void *workspace,
                  size_t workspace_bytes, void *stream, int *status_dev);

/*
 * FP8 forward: the same operation as fa_fwd on inputs stored as FP8 E4M3
 * codes with one scale per tensor (element value = code * descale).  The
 * news explainer "FlashAttention" (saiita), section on the second and third
 * generations, reports that the third generation reaches about 1.2 PFLOP/s
 * on H100 with FP8; it gives no details, so the format choices here are
 * this library's: E4M3 for Q, K, V and for the probabilities that enter
 * the P.V product (3 mantissa bits), fp32 scores, row sums and LSE, bf16 O.
 *  q  : [B, Hq, N, d] E4M3 codes      k : [B, Hkv, N, d] E4M3 codes
 *  vt : V transposed, [B, Hkv, d, ldvt] E4M3 codes (keys contiguous);
 *       ldvt >= N and a multiple of 16; columns N..ldvt-1 are never read
 *  o  : [B, Hq, N, d] bf16            lse : [B, Hq, N] fp32, natural log of
 *       the masked row sum of exp(scale * descale_q * descale_k * q.k)
 *  d must be 128.  descale_q, descale_k, descale_v: finite and > 0.
 *  seqlens, causal, GQA map: as fa_fwd.  All pointers DEVICE, 16-byte
 *  aligned (lse 4-byte), owned by the caller; nothing is allocated.
 * Returns FA_OK once launched on `stream` (NULL = legacy default stream);
 * bounded-wait time-outs reach status_dev (or the library's own word).
 * Errors: FA_ERR_NULL, FA_ERR_SHAPE (sizes, ldvt < N, a bad descale),
 * FA_ERR_HEADS, FA_ERR_HEADDIM (d != 128), FA_ERR_ALIGN (a pointer, or ldvt
 * not a multiple of 16), FA_ERR_ARCH, FA_ERR_CUDA, FA_ERR_LAUNCH.
 */
FA_API int fa_fwd_fp8(const void *q, const void *k, const void *vt, void *o, float *lse, int B,
                      int Hq, int Hkv, int N, int ldvt, int d, float scale, float descale_q,
                      float descale_k, float descale_v, int causal, const int *seqlens,
                      void *stream, int *status_dev);

/*
 * Packed variable-length forward: the tokens of B sequences are stored back
 * to back with no padding (the padding mask of the pages' statement, without
 * padded rows).  Same operation as fa_fwd per sequence, self-attention
 * (each sequence's queries attend to its own keys; causal is j <= i within
 * the sequence).
 *  q, o : [total, Hq, d] bf16      k, v : [total, Hkv, d] bf16
 *  lse  : [Hq, total] fp32
 *  cu_seqlens: DEVICE int32 [B+1], cu_seqlens[0] = 0, non-decreasing,
 *         cu_seqlens[B] = total; sequence b holds tokens
 *         [cu_seqlens[b], cu_seqlens[b+1]).
 *  max_seqlen: an upper bound on every sequence length (it sizes the work
 *         grid; rows past it would not be computed).
 *  d in {64, 128}.  Returns FA_OK once launched on `stream`, else fa_status.
 */
FA_API int fa_fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse,
                         const int *cu_seqlens, int B, int Hq, int Hkv, int total, int max_seqlen,
                         int d, float scale, int causal, void *stream, int *status_dev);

/*
 * Split-KV decode forward: Nq query rows per (batch, query head) against Nk
 * cached keys.  Same operation as fa_fwd with two differences of shape:
 *  q, o : [B, Hq, Nq, d] bf16      k, v : [B, Hkv, Nk, d] bf16 (the cache)
 *  lse  : [B, Hq, Nq] fp32
 *  seqlens_k: NULL or device int32[B], 0 <= seqlens_k[b] <= Nk, the number of
 *         valid cached keys of sequence b (keys past it are ignored).
 *  causal: 0/1; query i is position len_b - Nq + i of its sequence, so it sees
 *         keys j <= len_b - Nq + i (with Nq = 1: every valid key).
 *  Three kernels serve the call, chosen by G * Nq, the query rows per kv
 *  head (G = Hq / Hkv):
 *   - G * Nq <= 16: tensor cores, keys on the tensor-memory lanes.
 *   - 16 < G * Nq <= 128: tensor cores, query rows on the lanes.
 *     In both, the call's 128-key tiles of valid keys are divided evenly
 *     among persistent CTAs, whatever the lengths.
 *   - G * Nq > 128: CUDA cores, per key range of each (batch, kv head).
 *  num_splits: 0 for the automatic choice, or 1..128.
 *   - Tensor-core kernel: 0 gives one CTA per SM; n gives
 *     min(n * B * Hkv, 1024) CTAs, so each (batch, kv head) is processed by
 *     about n of them.
 *   - CUDA-core kernel: the number of key ranges per (batch, kv head); 0
 *     aims at about 16 CTAs per SM of a B200 with at least 256 keys per
 *     range.
 *  workspace: DEVICE buffer of at least fa_decode_workspace_size() bytes,
 *         16-byte aligned, owned by the caller.  It holds each CTA's partial
 *         output, row max and row sum, which a second kernel merges through
 *         their log-sum-exp.  It may be reused across calls that are ordered
 *         on one stream.
 * Reference: wiki note "FlashAttention", common misconceptions: generating a
 * single token is bound by reading the cached K/V, and needs decode-oriented
 * kernels; the merge is the same online-softmax update (section "what it
 * is") applied to whole key ranges.
 * Returns FA_OK when both kernels are launched on `stream`, FA_ERR_WORKSPACE
 * when the workspace is missing, misaligned or too small, or another
 * fa_status.  d must be 64 or 128.
 */
FA_API size_t fa_decode_workspace_size(int B, int Hq, int Hkv, int Nq, int Nk, int d,
                                       int num_splits);
FA_API int fa_fwd_decode(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                         int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                         const int *seqlens_k, int num_splits, void *workspace,
                         size_t workspace_bytes, void *stream, int *status_dev);

/*
 * fa_fwd_decode without a workspace argument, for callers that cannot
 * allocate device memory on the call path: code that runs where the
 * allocator must not be touched (an inference loop with a fixed memory
 * budget, a host framework that owns every device allocation, or a latency
 * path where cudaMalloc's implicit device synchronisation is not acceptable).
 * The pages have no counterpart to this call; it only changes where the
 * decode partials are kept.
 *
 * Same arguments and results as fa_fwd_decode, minus workspace and
 * workspace_bytes.  The partials go to one 8 MiB array that the library
 * defines in device memory; every GPU that loads the library holds it until
 * the process exits.  A shape whose partials need more than 8 MiB
 * (fa_decode_workspace_size() > 8388608) is rejected with FA_ERR_WORKSPACE;
 * nothing is launched then.  No call allocates or frees device memory.
 *
 * The first call on a device looks up the array's device address (with that
 * device current) and remembers it for the rest of the process; make that
 * first call before any stream capture.  The remembered address belongs to
 * the device's primary context: after cudaDeviceReset on that device it is
 * no longer valid, so do not call this entry point again in that process.
 * The array keeps the last call's contents: every call writes all
 * the partials it reads, so nothing needs clearing, but all calls share the
 * one array, so calls that overlap on the GPU (on different streams, or from
 * several host threads) race; order them on one stream.
 */
FA_API int fa_fwd_decode_noalloc(const void *q, const void *k, const void *v, void *o,
                                 float *lse, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                                 float scale, int causal, const int *seqlens_k, int num_splits,
                                 void *stream, int *status_dev);

/*
 * Waits for `stream` and reads a status word (status_dev, or the library's
 * own when NULL).  Returns FA_OK, FA_ERR_TIMEOUT, or FA_ERR_CUDA when the
 * stream reports an error.  Resets the library's own word to FA_OK.
 */
FA_API int fa_check_status(const int *status_dev, void *stream);

/*
 * Bounded-wait self test: launches one tiny kernel whose only work is to
 * wait on a shared-memory barrier that nothing ever arrives at, with a limit
 * of limit_ns nanoseconds.  The kernel must give up, write FA_ERR_TIMEOUT into
 * status_dev (a device int the caller zeroes) and return.  Proves that an
 * in-kernel wait cannot hang the device.  Returns the launch status.
 */
FA_API int fa_selftest_bounded_wait(int *status_dev, unsigned long long limit_ns, void *stream);

/*
 * Calibration, not part of the attention path: the throughput of the GPU's
 * exponential unit for ex2.approx.ftz.f32, the instruction the softmax
 * steps use.
 *  - One block of 1024 threads per SM runs 8 independent chains of
 *    x <- 2^(-|x|) each, for 2048 steps, and records its clock cycles and
 *    its SM.
 *  - The call waits for `stream` and writes to *ex2_per_clk (host) the
 *    median over SMs of exponentials per SM clock.
 *  - One exponential per score element is needed against 4d FLOPs of MMA,
 *    so this rate bounds the path at ex2_per_clk * 4d FLOP per clock per SM.
 *  - Its records live in a small static device array: calls that overlap on
 *    the GPU race.
 * Returns FA_OK, FA_ERR_NULL, FA_ERR_ARCH, FA_ERR_LAUNCH or FA_ERR_CUDA.
 */
FA_API int fa_measure_ex2_rate(float *ex2_per_clk, void *stream);

/* Human-readable text for an fa_status code (static storage). */
FA_API const char *fa_status_string(int status);

/* Library version, as major*10000 + minor*100 + patch. */
FA_API int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_FA_H */
