/*
 * attn_fp64.c -- dense fp64 attention oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call this
 * file; only the tests, the smoke check and the CPU-baseline leg of the benchmark use
 * it.  It shares no code, header, table or constant with the CUDA library.
 *
 * What it computes is the plain definition of scaled dot-product attention, one query
 * row at a time, materialising the whole score row exactly as the "direct" reference
 * programs on the pages do:
 *   - "Online Softmax Without the Attention Matrix" notebook (the dense line of the
 *     worked example: max, exp(s - max), weighted sum / sum);
 *   - nx_flashattn_scale.nx, the "DIRECT softmax reference" loop (score row, max,
 *     exp/sum, per-dimension weighted sum divided by the sum);
 *   - oxios flash_attention.rs, FlashAttention::naive_attention (full score matrix,
 *     max-subtracted softmax, then weights x values).
 * The method (tiled online softmax) reaches this result exactly up to rounding
 * ("Module 16: Efficient and Long Attention", section 16.2: the result is exactly
 * standard attention up to rounding), so the oracle is this definition, in fp64.
 *
 * Per query row i of head (b, hq), with key/value head kv = hq / (Hq / Hkv):
 *   1. s_j = scale * sum_c q[i,c] * k[j,c]          for every key j < Nk
 *   2. if softcap > 0:  s_j = softcap * tanh(s_j / softcap)
 *                                       (Module 16, section 16.5, logit soft-capping)
 *   3. with the query's position in the key sequence p = i + (Nk - Nq):
 *      s_j = -inf  if (causal and j > p)
 *                  or (window > 0 and p - j >= window and j >= n_sink)
 *                   (Module 16, 16.2 "Measured": the causal mask uses positions in the
 *                    full sequence; 16.3: a local layer sees the W most recent tokens;
 *                    16.6: the first tokens, the attention sinks, are kept alongside the
 *                    sliding window -- they are exempt from the window, not from the
 *                    causal mask, and n_sink = 0 is the plain window).
 *      With Nq == Nk (self-attention) p = i; with fewer queries than keys the queries
 *      are the last Nq positions of the key sequence (cross-attention / decode).
 *   4. m = max_j s_j,  p_j = exp(s_j - m),  l = sum_j p_j,
 *      O[i,c] = sum_j p_j v[j,c] / l,   LSE[i] = m + ln(l)
 *      A row with no valid key (m = -inf) gets O = 0 and LSE = -inf: the oxios
 *      `attention` routine only divides when its running sum is positive and
 *      otherwise leaves the zero output.
 *
 * Inputs are read in their stored type (fp64, fp32 or bf16 bit patterns) and upcast to
 * fp64 exactly; `scale` and `softcap` arrive as doubles (callers pass the exact value
 * of the fp32 argument the GPU library receives).  No blocking, fusion or reordering:
 * the dot product runs over c in order and both sums over j in order.  Rows are split
 * across POSIX threads; each row is computed by one thread alone, so the result does
 * not depend on the thread count.
 *
 * Layout: q, o  [B, Hq, Nq, d] row-major;  k, v [B, Hkv, Nk, d];  lse [B, Hq, Nq].
 * Parity of every function here is pinned by tests/test_oracle_pins.py.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORACLE_F64 = 0, ORACLE_F32 = 1, ORACLE_BF16 = 2 };

static double load_elem(const void* base, int dtype, int64_t idx) {
  if (dtype == ORACLE_F64) return ((const double*)base)[idx];
  if (dtype == ORACLE_F32) return (double)((const float*)base)[idx];
  /* bf16: the 16 stored bits are the top half of an IEEE binary32 */
  uint32_t bits = (uint32_t)((const uint16_t*)base)[idx] << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

typedef struct {
  const void *q, *k, *v;
  int dtype;
  int64_t B, Hq, Hkv, Nq, Nk, d;
  double scale;
  int causal;
  int64_t window;
  int64_t n_sink;
  double softcap;
  const int64_t* rows; /* NULL: every row in order */
  int64_t nrows;
  double* o;
  double* lse;
  int nthreads;
  int tid;
  int status;
} job_t;

/* One query row: steps 1-4 above, written out. */
static void attend_row(const job_t* J, int64_t row, double* s, double* o_row, double* lse) {
  const int64_t Nq = J->Nq, N = J->Nk, d = J->d;
  const int64_t i = row % Nq;
  const int64_t bh = row / Nq;
  const int64_t b = bh / J->Hq, hq = bh % J->Hq;
  const int64_t group = J->Hq / J->Hkv;
  const int64_t kv = hq / group;
  const int64_t q_off = ((b * J->Hq + hq) * Nq + i) * d;
  const int64_t kv_base = (b * J->Hkv + kv) * N * d;
  const int64_t pos = i + (N - Nq); /* position of query i in the key sequence */

  for (int64_t j = 0; j < N; ++j) {
    double dot = 0.0;
    for (int64_t c = 0; c < d; ++c)
      dot += load_elem(J->q, J->dtype, q_off + c) * load_elem(J->k, J->dtype, kv_base + j * d + c);
    double sj = J->scale * dot;
    if (J->softcap > 0.0) sj = J->softcap * tanh(sj / J->softcap);
    if (J->causal && j > pos) sj = -INFINITY;
    if (J->window > 0 && pos - j >= J->window && j >= J->n_sink) sj = -INFINITY;
    s[j] = sj;
  }

  double m = -INFINITY;
  for (int64_t j = 0; j < N; ++j)
    if (s[j] > m) m = s[j];
  for (int64_t c = 0; c < d; ++c) o_row[c] = 0.0;
  if (m == -INFINITY) { /* no valid key in this row */
    *lse = -INFINITY;
    return;
  }
  double l = 0.0;
  for (int64_t j = 0; j < N; ++j) {
    double p = exp(s[j] - m);
    l += p;
    if (p != 0.0)
      for (int64_t c = 0; c < d; ++c) o_row[c] += p * load_elem(J->v, J->dtype, kv_base + j * d + c);
  }
  for (int64_t c = 0; c < d; ++c) o_row[c] = o_row[c] / l;
  *lse = m + log(l);
}

static void* worker(void* arg) {
  job_t* J = (job_t*)arg;
  double* s = (double*)malloc(sizeof(double) * (size_t)(J->Nk > 0 ? J->Nk : 1));
  if (!s) {
    J->status = -2;
    return NULL;
  }
  /* interleaved rows: causal rows grow with i, so striding balances the threads */
  for (int64_t r = J->tid; r < J->nrows; r += J->nthreads) {
    int64_t row = J->rows ? J->rows[r] : r;
    attend_row(J, row, s, J->o + r * J->d, J->lse + r);
  }
  free(s);
  return NULL;
}

/*
 * oracle_attn_fp64 -- O and LSE for the listed query rows.
 *   rows[r] is a flat row index (b*Hq + hq)*Nq + i; rows == NULL means all B*Hq*Nq rows.
 *   o receives nrows*d doubles, lse nrows doubles, in the order of `rows`.
 *   n_sink >= 0 keys at the start of the key sequence are exempt from the window.
 * Returns 0, or -1 for bad arguments, -2 when memory or threads could not be had.
 */
int oracle_attn_fp64(const void* q, const void* k, const void* v, int dtype, int64_t B, int64_t Hq,
                     int64_t Hkv, int64_t Nq, int64_t Nk, int64_t d, double scale, int causal, int64_t window,
                     int64_t n_sink, double softcap, const int64_t* rows, int64_t nrows, double* o, double* lse,
                     int nthreads) {
  if (B < 0 || Hq < 0 || Hkv <= 0 || Nq < 0 || Nk < 0 || d <= 0 || (Hq % Hkv) != 0 || n_sink < 0) return -1;
  if (dtype != ORACLE_F64 && dtype != ORACLE_F32 && dtype != ORACLE_BF16) return -1;
  int64_t total = B * Hq * Nq;
  if (!rows) nrows = total;
  if (nrows <= 0) return 0;
  if (!q || !k || !v || !o || !lse) return -1;
  if (rows)
    for (int64_t r = 0; r < nrows; ++r)
      if (rows[r] < 0 || rows[r] >= total) return -1;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 512) nthreads = 512;
  if ((int64_t)nthreads > nrows) nthreads = (int)nrows;

  job_t* jobs = (job_t*)calloc((size_t)nthreads, sizeof(job_t));
  pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
  if (!jobs || !th) {
    free(jobs);
    free(th);
    return -2;
  }
  int rc = 0;
  int started = 0;
  for (int t = 0; t < nthreads; ++t) {
    job_t J = {q, k, v, dtype, B, Hq, Hkv, Nq, Nk, d, scale, causal, window, n_sink, softcap,
               rows, nrows, o, lse, nthreads, t, 0};
    jobs[t] = J;
  }
  for (int t = 1; t < nthreads; ++t) {
    if (pthread_create(&th[t], NULL, worker, &jobs[t]) != 0) {
      rc = -2;
      break;
    }
    started = t;
  }
  if (rc == 0) worker(&jobs[0]);
  for (int t = 1; t <= started; ++t) pthread_join(th[t], NULL);
  for (int t = 0; t < nthreads && rc == 0; ++t)
    if (jobs[t].status) rc = jobs[t].status;
  free(jobs);
  free(th);
  return rc;
}
