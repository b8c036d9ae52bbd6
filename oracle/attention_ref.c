/*
 * Exact attention forward, fp64, on the CPU.  TEST INFRASTRUCTURE ONLY.
 *
 * This is the oracle the CUDA path is checked against.  Only the tests, the
 * smoke check and the benchmark's CPU-baseline leg may call it; the product
 * path never does.  It shares no code, header or constant with the GPU
 * library.
 *
 * What it computes (the plain definition, no tiling, no online softmax):
 *   for each batch b and query head h, with kv head g = h / (Hq / Hkv):
 *     S[i][j] = scale * sum_c Q[b,h,i,c] * K[b,g,j,c]         (fp64)
 *     S[i][j] = -inf  if j >= len_b, or (causal and j > i)
 *     M_i     = max_j S[i][j]
 *     P[i][j] = exp(S[i][j] - M_i) / sum_j' exp(S[i][j'] - M_i)
 *     O[i]    = sum_j P[i][j] * V[b,g,j,:]
 *     LSE_i   = M_i + log(sum_j exp(S[i][j] - M_i))
 *   A row with no visible key gets O = 0 and LSE = -inf.
 *
 * Sources (page title, section):
 *   - "FlashAttention" wiki note (llm-wiki-maxwellmou), section "what it is":
 *     O = softmax(Q K^T / sqrt(d)) V; for one head S = Q K^T, P = softmax(S),
 *     output P V, with S and P both T x T.
 *   - "FlashAttention" explainer (liu-gong-zi), pseudo-code of standard
 *     attention: scores, softmax over each row, weighted sum of V.
 *   - "Why is FlashAttention faster" interview notes (arfxm), section on what
 *     standard attention stores: mask applied to the scores before softmax.
 *   - wiki note, same section: causal and padding masks and multiple heads
 *     are handled per tile; enable_gqa in the SDPA call (GQA head sharing).
 * Readings where the pages are silent: the mask is additive 0/-inf, causal is
 * top-left aligned (key j visible to query i iff j <= i), key padding masks
 * keys j >= len_b only (every query row is still computed), GQA groups are
 * contiguous (query heads [g*G, (g+1)*G) share kv head g), LSE is the
 * natural log.
 *
 * Queries and keys may have different lengths (Nq query rows against Nk keys,
 * the decode case the wiki note's "common misconceptions" section mentions):
 * with causal_bottom_right set, query i is the (len_b - Nq + i)-th position
 * of its sequence, so key j is visible iff j <= i + len_b - Nq; otherwise
 * causal stays top-left (j <= i).
 *
 * Backward (oracle_attention_bwd): the gradients of sum(dO * O) with
 * respect to Q, K and V, written out from the same definition by the chain
 * rule (the pages' training path recomputes these from the inputs instead of
 * storing P: interview notes, section on memory; exam explainer,
 * "recomputation"):
 *     dV[g]  += P^T dO                 (summed over the query heads of group g)
 *     dP      = dO V^T
 *     D_i     = sum_j P[i][j] dP[i][j]
 *     dS      = P * (dP - D)           (elementwise, D broadcast over j)
 *     dQ      = scale * dS K
 *     dK[g]  += scale * dS^T Q
 *
 * S and P are materialised per block of query rows, exactly as defined.
 * Blocks are independent and run on a pool of POSIX threads.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORACLE_IN_F64 = 0, ORACLE_IN_F32 = 1, ORACLE_IN_BF16 = 2, ORACLE_IN_E4M3 = 3 };

#define ORACLE_ROW_BLOCK 16

/*
 * One FP8 E4M3 code (the OCP 8-bit format with 4 exponent bits, bias 7, 3
 * mantissa bits, no infinities; S.1111.111 is NaN): normal values
 * (1 + m/8) * 2^(e-7), subnormals (e = 0) m * 2^-9.  Every code is exact in
 * fp64.
 */
static double e4m3_value(uint8_t c) {
  const int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
  double x;
  if (e == 15 && m == 7)
    x = NAN;
  else if (e == 0)
    x = ldexp((double)m, -9);
  else
    x = ldexp(1.0 + m / 8.0, e - 7);
  return s ? -x : x;
}

/* Decode one input element to fp64.  bf16, fp32 and e4m3 values widen exactly. */
static double in_at(const void *base, int kind, int64_t idx) {
  if (kind == ORACLE_IN_F64) return ((const double *)base)[idx];
  if (kind == ORACLE_IN_F32) return (double)((const float *)base)[idx];
  if (kind == ORACLE_IN_E4M3) return e4m3_value(((const uint8_t *)base)[idx]);
  uint32_t u = (uint32_t)((const uint16_t *)base)[idx] << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

typedef struct {
  const void *q, *k, *v;
  int in_kind, B, Hq, Hkv, Nq, N, d, causal, bottom_right, R, nblk;
  double scale;
  const int32_t *seqlens;
  const int64_t *rows;
  double *o, *lse, *p_out;
  int64_t total;
  int64_t next; /* shared task counter */
  int bad;
} job_t;

/* One task: one block of up to ORACLE_ROW_BLOCK query rows of one (b, h). */
static void run_block(const job_t *J, int64_t t, double *S, double *qrow) {
  const int N = J->N, d = J->d, R = J->R;
  const int64_t bh = t / J->nblk;
  const int blk = (int)(t % J->nblk);
  const int b = (int)(bh / J->Hq);
  const int h = (int)(bh % J->Hq);
  const int g = h / (J->Hq / J->Hkv);
  int len = J->seqlens ? J->seqlens[b] : N;
  if (len < 0) len = 0;
  if (len > N) len = N;
  const int64_t qbase = ((int64_t)b * J->Hq + h) * J->Nq * d;
  const int64_t off = J->bottom_right ? (int64_t)len - J->Nq : 0;
  const int64_t kvbase = ((int64_t)b * J->Hkv + g) * N * d;
  const int r0 = blk * ORACLE_ROW_BLOCK;
  const int r1 = (r0 + ORACLE_ROW_BLOCK < R) ? r0 + ORACLE_ROW_BLOCK : R;

  /* 1. S for this block of query rows, masked entries set to -inf. */
  for (int r = r0; r < r1; ++r) {
    const int64_t i = J->rows ? J->rows[bh * R + r] : r;
    double *Srow = S + (size_t)(r - r0) * N;
    for (int c = 0; c < d; ++c) qrow[c] = in_at(J->q, J->in_kind, qbase + i * d + c);
    for (int j = 0; j < N; ++j) {
      const int visible = (j < len) && (!J->causal || j <= i + off);
      if (!visible) {
        Srow[j] = -INFINITY;
        continue;
      }
      double acc = 0.0;
      for (int c = 0; c < d; ++c) acc += qrow[c] * in_at(J->k, J->in_kind, kvbase + (int64_t)j * d + c);
      Srow[j] = J->scale * acc;
    }
  }

  /* 2. P = softmax(S) row by row (in place over S), LSE from the same sum. */
  for (int r = r0; r < r1; ++r) {
    double *Srow = S + (size_t)(r - r0) * N;
    double m = -INFINITY;
    for (int j = 0; j < N; ++j)
      if (Srow[j] > m) m = Srow[j];
    double *orow = J->o + (bh * R + r) * (int64_t)d;
    if (m == -INFINITY) {
      for (int j = 0; j < N; ++j) Srow[j] = 0.0;
      J->lse[bh * R + r] = -INFINITY;
    } else {
      double denom = 0.0;
      for (int j = 0; j < N; ++j) denom += exp(Srow[j] - m);
      for (int j = 0; j < N; ++j) Srow[j] = exp(Srow[j] - m) / denom;
      J->lse[bh * R + r] = m + log(denom);
    }
    if (J->p_out) memcpy(J->p_out + (bh * R + r) * (int64_t)N, Srow, sizeof(double) * (size_t)N);

    /* 3. O = P V. */
    for (int c = 0; c < d; ++c) orow[c] = 0.0;
    for (int j = 0; j < N; ++j) {
      const double p = Srow[j];
      if (p == 0.0) continue;
      for (int c = 0; c < d; ++c) orow[c] += p * in_at(J->v, J->in_kind, kvbase + (int64_t)j * d + c);
    }
  }
}

static void *worker(void *arg) {
  job_t *J = (job_t *)arg;
  double *S = (double *)malloc(sizeof(double) * (size_t)ORACLE_ROW_BLOCK * (size_t)J->N);
  double *qrow = (double *)malloc(sizeof(double) * (size_t)J->d);
  if (!S || !qrow) {
    __atomic_store_n(&J->bad, 1, __ATOMIC_RELAXED);
  } else {
    for (;;) {
      const int64_t t = __atomic_fetch_add(&J->next, 1, __ATOMIC_RELAXED);
      if (t >= J->total) break;
      run_block(J, t, S, qrow);
    }
  }
  free(S);
  free(qrow);
  return NULL;
}

/*
 * q: [B, Hq, Nq, d]; k, v: [B, Hkv, Nk, d]; element type given by in_kind.
 * seqlens: int32 [B] key lengths (0 <= len_b <= Nk) or NULL for Nk.
 * causal: 0/1; causal_bottom_right: 0 = top-left (j <= i), 1 = bottom-right
 *       (j <= i + len_b - Nq).
 * rows: int64 [B*Hq, R] query rows to compute per (b, h), or NULL for all Nq
 *       (then R must equal Nq).
 * o: fp64 [B*Hq, R, d]; lse: fp64 [B*Hq, R].
 * p_out: optional fp64 [B*Hq, R, Nk], the probability rows P[i][:].
 * nthreads: worker threads (>= 1); tasks are independent blocks of rows, so
 *           the result does not depend on it.
 * Returns 0, or -1 on a bad argument or an allocation failure.
 */
int oracle_attention_fwd_general(const void *q, const void *k, const void *v, int in_kind, int B,
                                 int Hq, int Hkv, int Nq, int Nk, int d, double scale, int causal,
                                 int causal_bottom_right, const int32_t *seqlens,
                                 const int64_t *rows, int R, double *o, double *lse,
                                 double *p_out, int nthreads) {
  if (!q || !k || !v || !o || !lse) return -1;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nk <= 0 || d <= 0 || R <= 0) return -1;
  if (Hq % Hkv != 0) return -1;
  if (!rows && R != Nq) return -1;
  if (in_kind < ORACLE_IN_F64 || in_kind > ORACLE_IN_E4M3) return -1;
  job_t J;
  memset(&J, 0, sizeof J);
  J.q = q; J.k = k; J.v = v; J.in_kind = in_kind;
  J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.Nq = Nq; J.N = Nk; J.d = d; J.causal = causal;
  J.bottom_right = causal_bottom_right; J.R = R;
  J.scale = scale; J.seqlens = seqlens; J.rows = rows; J.o = o; J.lse = lse; J.p_out = p_out;
  J.nblk = (R + ORACLE_ROW_BLOCK - 1) / ORACLE_ROW_BLOCK;
  J.total = (int64_t)B * Hq * J.nblk;
  if (nthreads < 1) nthreads = 1;
  if ((int64_t)nthreads > J.total) nthreads = (int)J.total;
  pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
  if (!th) return -1;
  int started = 0;
  for (int t = 1; t < nthreads; ++t) {
    if (pthread_create(&th[t], NULL, worker, &J) != 0) break;
    ++started;
  }
  worker(&J);
  for (int t = 1; t <= started; ++t) pthread_join(th[t], NULL);
  free(th);
  return J.bad ? -1 : 0;
}

/* ------------------------------------------------------------------------- */
/* Backward                                                                  */
/* ------------------------------------------------------------------------- */

typedef struct {
  const void *q, *k, *v, *dout;
  int in_kind, B, Hq, Hkv, N, d, causal;
  double scale;
  const int32_t *seqlens;
  double *dq, *dk, *dv;
  int64_t total;
  int64_t next;
  int bad;
} bwd_job_t;

/* One task: one (batch, kv head) group: every query head of the group, every
 * query row; the group's dK and dV rows are written by this task only. */
static void run_bwd_group(const bwd_job_t *J, int64_t t, double *S, double *dP, double *qrow,
                          double *dorow) {
  const int N = J->N, d = J->d;
  const int b = (int)(t / J->Hkv), g = (int)(t % J->Hkv);
  const int G = J->Hq / J->Hkv;
  int len = J->seqlens ? J->seqlens[b] : N;
  if (len < 0) len = 0;
  if (len > N) len = N;
  const int64_t kvbase = ((int64_t)b * J->Hkv + g) * N * d;
  double *dkg = J->dk + kvbase, *dvg = J->dv + kvbase;
  for (int64_t e = 0; e < (int64_t)N * d; ++e) dkg[e] = dvg[e] = 0.0;
  for (int hh = 0; hh < G; ++hh) {
    const int h = g * G + hh;
    const int64_t qbase = ((int64_t)b * J->Hq + h) * N * d;
    for (int i = 0; i < N; ++i) {
      for (int c = 0; c < d; ++c) {
        qrow[c] = in_at(J->q, J->in_kind, qbase + (int64_t)i * d + c);
        dorow[c] = in_at(J->dout, J->in_kind, qbase + (int64_t)i * d + c);
      }
      /* S row, P row (softmax), dP row */
      double m = -INFINITY;
      for (int j = 0; j < N; ++j) {
        const int visible = (j < len) && (!J->causal || j <= i);
        if (!visible) {
          S[j] = -INFINITY;
          continue;
        }
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += qrow[c] * in_at(J->k, J->in_kind, kvbase + (int64_t)j * d + c);
        S[j] = J->scale * acc;
        if (S[j] > m) m = S[j];
      }
      double *dqrow = J->dq + qbase + (int64_t)i * d;
      for (int c = 0; c < d; ++c) dqrow[c] = 0.0;
      if (m == -INFINITY) continue; /* no visible key: every gradient of the row is 0 */
      double denom = 0.0;
      for (int j = 0; j < N; ++j) denom += exp(S[j] - m);
      double D = 0.0;
      for (int j = 0; j < N; ++j) {
        S[j] = exp(S[j] - m) / denom; /* P[i][j] */
        double acc = 0.0;
        if (S[j] != 0.0)
          for (int c = 0; c < d; ++c) acc += dorow[c] * in_at(J->v, J->in_kind, kvbase + (int64_t)j * d + c);
        dP[j] = acc;
        D += S[j] * dP[j];
      }
      for (int j = 0; j < N; ++j) {
        const double p = S[j];
        if (p == 0.0) continue;
        const double ds = p * (dP[j] - D);
        for (int c = 0; c < d; ++c) {
          dqrow[c] += J->scale * ds * in_at(J->k, J->in_kind, kvbase + (int64_t)j * d + c);
          dkg[(int64_t)j * d + c] += J->scale * ds * qrow[c];
          dvg[(int64_t)j * d + c] += p * dorow[c];
        }
      }
    }
  }
}

static void *bwd_worker(void *arg) {
  bwd_job_t *J = (bwd_job_t *)arg;
  double *S = (double *)malloc(sizeof(double) * (size_t)J->N);
  double *dP = (double *)malloc(sizeof(double) * (size_t)J->N);
  double *qrow = (double *)malloc(sizeof(double) * (size_t)J->d);
  double *dorow = (double *)malloc(sizeof(double) * (size_t)J->d);
  if (!S || !dP || !qrow || !dorow) {
    __atomic_store_n(&J->bad, 1, __ATOMIC_RELAXED);
  } else {
    for (;;) {
      const int64_t t = __atomic_fetch_add(&J->next, 1, __ATOMIC_RELAXED);
      if (t >= J->total) break;
      run_bwd_group(J, t, S, dP, qrow, dorow);
    }
  }
  free(S);
  free(dP);
  free(qrow);
  free(dorow);
  return NULL;
}

/*
 * Gradients of sum(dout * O) for O = attention(q, k, v) as defined above.
 * q, dout: [B, Hq, N, d]; k, v: [B, Hkv, N, d]; element type in_kind.
 * dq: fp64 [B, Hq, N, d]; dk, dv: fp64 [B, Hkv, N, d].
 * Returns 0, or -1 on a bad argument or an allocation failure.
 */
int oracle_attention_bwd(const void *q, const void *k, const void *v, const void *dout,
                         int in_kind, int B, int Hq, int Hkv, int N, int d, double scale,
                         int causal, const int32_t *seqlens, double *dq, double *dk, double *dv,
                         int nthreads) {
  if (!q || !k || !v || !dout || !dq || !dk || !dv) return -1;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || d <= 0 || Hq % Hkv != 0) return -1;
  if (in_kind < ORACLE_IN_F64 || in_kind > ORACLE_IN_E4M3) return -1;
  bwd_job_t J;
  memset(&J, 0, sizeof J);
  J.q = q; J.k = k; J.v = v; J.dout = dout; J.in_kind = in_kind;
  J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.N = N; J.d = d; J.causal = causal; J.scale = scale;
  J.seqlens = seqlens; J.dq = dq; J.dk = dk; J.dv = dv;
  J.total = (int64_t)B * Hkv;
  if (nthreads < 1) nthreads = 1;
  if ((int64_t)nthreads > J.total) nthreads = (int)J.total;
  pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
  if (!th) return -1;
  int started = 0;
  for (int t = 1; t < nthreads; ++t) {
    if (pthread_create(&th[t], NULL, bwd_worker, &J) != 0) break;
    ++started;
  }
  bwd_worker(&J);
  for (int t = 1; t <= started; ++t) pthread_join(th[t], NULL);
  free(th);
  return J.bad ? -1 : 0;
}

/* Square case (Nq = Nk = N, causal top-left): the problem the pages state. */
int oracle_attention_fwd(const void *q, const void *k, const void *v, int in_kind, int B, int Hq,
                         int Hkv, int N, int d, double scale, int causal,
                         const int32_t *seqlens, const int64_t *rows, int R, double *o,
                         double *lse, double *p_out, int nthreads) {
  return oracle_attention_fwd_general(q, k, v, in_kind, B, Hq, Hkv, N, N, d, scale, causal, 0,
                                      seqlens, rows, R, o, lse, p_out, nthreads);
}
