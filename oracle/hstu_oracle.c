/*
 * hstu_oracle.c — plain, slow, fp64 CPU oracle for jagged target-aware HSTU pointwise
 * (SiLU) attention.  TEST INFRASTRUCTURE ONLY: it exists to check the CUDA library, and
 * only the tests, the package's smoke() check and bench.py's CPU-baseline leg may load it.
 * It shares no code, header or table with the CUDA path.
 *
 * Definition followed (page titles and sections):
 *   - "DLRMv3: MLPerf Inference generative recommendation benchmark" (winzheng.jp review),
 *     section "model selection", time/position-encoding paragraph: the attention is
 *     Mask(SiLU(Q K^T)) V with no relative bias.
 *   - same section, FLOP-formula paragraph: the history (UIH) encoding is shared by every
 *     candidate of a request; K/V of the history is reused across timestamps (cached mode).
 *   - infolabhq.com multi-stage sequence model page, offline user model section (the user
 *     side never depends on a candidate) and its "Target-Aware Multi-Head Attention"
 *     section (each layer weighs the history against the candidate being scored).
 *   - voagi.com TorchRec tutorial, section 2.1: jagged = concatenated rows + lengths.
 *   alpha (score scale) and N (normaliser) are explicit arguments; the pages print neither.
 *
 * Readings taken where the pages are silent:
 *   - a history token attends to history tokens at or before itself (causal, self included);
 *   - a candidate attends to every history token of its user and to itself, never to other
 *     candidates; history tokens never attend to candidates;
 *   - the mask is applied after the SiLU: a masked pair contributes exactly nothing;
 *   - N is one scalar per call.
 *
 * Arithmetic: inputs are float32 (bf16 inputs widen to float32 exactly); every product,
 * sum, exp and division is done in IEEE double, with keys visited in ascending order, so
 * the result is deterministic and independent of the thread count.
 *
 *     out[i,h,:] = (1/N) * sum_{j in A(i), ascending} silu(alpha * sum_c q[i,h,c] k[j,h,c]) v[j,h,:]
 *     silu(x)    = x / (1 + exp(-x))
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* SiLU, the Sigmoid Linear Unit, from its definition x * sigmoid(x). */
static double silu(double x) { return x / (1.0 + exp(-x)); }

/*
 * May the query at position i see the key at position j?  U is the history length.
 * History token (i < U): the history tokens at or before it.  Candidate (i >= U): every
 * history token, and itself.
 */
static int visible(int32_t i, int32_t j, int32_t U) {
  if (i < U) return j <= i;
  return j < U || j == i;
}

/*
 * One output row.  qrow: d floats of the query; kseg/vseg: first row of the user's K/V
 * segment (row stride H*d floats, already offset to head h); i: the query's position in
 * the segment of length L; U: history length; res: d doubles.  Returns the multiply-adds
 * performed (2*d per visible key: d for the score, d for the weighted value).
 */
static int64_t one_row(const float* qrow, const float* kseg, const float* vseg, int64_t stride,
                       int32_t d, int32_t i, int32_t L, int32_t U, double alpha, double N,
                       double* res) {
  int64_t macs = 0;
  for (int32_t c = 0; c < d; ++c) res[c] = 0.0;
  for (int32_t j = 0; j < L; ++j) {
    if (!visible(i, j, U)) continue;
    const float* krow = kseg + (int64_t)j * stride;
    const float* vrow = vseg + (int64_t)j * stride;
    double s = 0.0;
    for (int32_t c = 0; c < d; ++c) s += (double)qrow[c] * (double)krow[c];
    double p = silu(alpha * s);
    for (int32_t c = 0; c < d; ++c) res[c] += p * (double)vrow[c];
    macs += 2 * (int64_t)d;
  }
  for (int32_t c = 0; c < d; ++c) res[c] /= N;
  return macs;
}

/*
 * One output row of the relative-attention-bias variant.  The DLRMv3 review (section "model
 * selection", time/position-encoding paragraph) prints the original HSTU attention, whose
 * relative bias DLRMv3 drops, as Mask(SiLU(Q K^T) + bias) V.  Reading taken here, literally:
 * each visible pair gets silu(alpha * s) plus a bias that depends only on the relative
 * position i - j of query and key, read from the head's table rab_h[0 .. R-1] and clipped at
 * its last entry; masked pairs contribute nothing.  Same arguments as one_row plus rab_h, R.
 */
static void one_row_rab(const float* qrow, const float* kseg, const float* vseg, int64_t stride,
                        int32_t d, int32_t i, int32_t L, int32_t U, double alpha, double N,
                        const float* rab_h, int32_t R, double* res) {
  for (int32_t c = 0; c < d; ++c) res[c] = 0.0;
  for (int32_t j = 0; j < L; ++j) {
    if (!visible(i, j, U)) continue;
    const float* krow = kseg + (int64_t)j * stride;
    const float* vrow = vseg + (int64_t)j * stride;
    double s = 0.0;
    for (int32_t c = 0; c < d; ++c) s += (double)qrow[c] * (double)krow[c];
    int32_t rel = i - j;
    if (rel > R - 1) rel = R - 1;
    double p = silu(alpha * s) + (double)rab_h[rel];
    for (int32_t c = 0; c < d; ++c) res[c] += p * (double)vrow[c];
  }
  for (int32_t c = 0; c < d; ++c) res[c] /= N;
}

/* Checks one user's lengths; returns 0 if consistent. */
static int user_ok(const int32_t* off, const int32_t* nt, const int32_t* cl, int32_t b,
                   int64_t total) {
  int32_t L = off[b + 1] - off[b];
  int32_t T = nt ? nt[b] : 0;
  int32_t c = cl ? cl[b] : 0;
  if (off[b] < 0 || L < 0 || off[b + 1] > total) return 1;
  if (T < 0 || T > L) return 1;
  if (c < 0 || c > L - T) return 1;
  return 0;
}

int hstu_oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/*
 * Selected output rows.  For n in [0, nrows): user row_user[n], query row row_local[n]
 * (0-based among that user's query rows; in cached mode the query rows are the new tokens
 * and the position is cached_len[b] + row_local[n]).  q holds the query rows (q_new in
 * cached mode, packed per user as in the library); k, v the full segments.
 * out: [nrows, H, d] doubles.  *macs (optional) receives the multiply-adds performed.
 * Returns 0, or -1 on inconsistent offsets / out-of-range rows.
 */
int hstu_oracle_rows(const float* q, const float* k, const float* v,
                     const int32_t* seq_offsets, const int32_t* num_targets,
                     const int32_t* cached_len, int32_t B, int32_t H, int32_t d,
                     int64_t total_kv, int64_t total_q, double alpha, double N,
                     const int32_t* row_user, const int32_t* row_local, int64_t nrows,
                     double* out, int64_t* macs) {
  if (B < 0 || H <= 0 || d <= 0 || !(N != 0.0)) return -1;
  if (seq_offsets[0] != 0 || seq_offsets[B] != total_kv) return -1;
  /* query-row start of every user */
  int64_t* qstart = (int64_t*)malloc(sizeof(int64_t) * (size_t)(B + 1));
  if (!qstart) return -1;
  qstart[0] = 0;
  for (int32_t b = 0; b < B; ++b) {
    if (user_ok(seq_offsets, num_targets, cached_len, b, total_kv)) { free(qstart); return -1; }
    int32_t L = seq_offsets[b + 1] - seq_offsets[b];
    int32_t c = cached_len ? cached_len[b] : 0;
    qstart[b + 1] = qstart[b] + (L - c);
  }
  if (qstart[B] != total_q) { free(qstart); return -1; }
  for (int64_t n = 0; n < nrows; ++n) {
    int32_t b = row_user[n];
    if (b < 0 || b >= B) { free(qstart); return -1; }
    int32_t L = seq_offsets[b + 1] - seq_offsets[b];
    int32_t c = cached_len ? cached_len[b] : 0;
    if (row_local[n] < 0 || row_local[n] >= L - c) { free(qstart); return -1; }
  }
  const int64_t stride = (int64_t)H * d;
  int64_t total_macs = 0;
  int64_t units = nrows * H;
#pragma omp parallel for schedule(dynamic, 16) reduction(+ : total_macs)
  for (int64_t u = 0; u < units; ++u) {
    int64_t n = u / H;
    int32_t h = (int32_t)(u % H);
    int32_t b = row_user[n];
    int32_t L = seq_offsets[b + 1] - seq_offsets[b];
    int32_t T = num_targets ? num_targets[b] : 0;
    int32_t c = cached_len ? cached_len[b] : 0;
    int32_t r = row_local[n];
    const float* qrow = q + (qstart[b] + r) * stride + (int64_t)h * d;
    const float* kseg = k + (int64_t)seq_offsets[b] * stride + (int64_t)h * d;
    const float* vseg = v + (int64_t)seq_offsets[b] * stride + (int64_t)h * d;
    total_macs += one_row(qrow, kseg, vseg, stride, d, c + r, L, L - T, alpha, N,
                          out + n * stride + (int64_t)h * d);
  }
  free(qstart);
  if (macs) *macs = total_macs;
  return 0;
}

/*
 * Every output row of a full forward pass: out[t, h, :] for all rows t in [0, total), in
 * the jagged [total, H, d] layout.  Returns 0, or -1 on inconsistent offsets.
 */
int hstu_oracle_fwd(const float* q, const float* k, const float* v,
                    const int32_t* seq_offsets, const int32_t* num_targets,
                    int32_t B, int32_t H, int32_t d, int64_t total, double alpha, double N,
                    double* out, int64_t* macs) {
  if (B < 0 || H <= 0 || d <= 0 || !(N != 0.0)) return -1;
  if (seq_offsets[0] != 0 || seq_offsets[B] != total) return -1;
  for (int32_t b = 0; b < B; ++b)
    if (user_ok(seq_offsets, num_targets, NULL, b, total)) return -1;
  int32_t* owner = (int32_t*)malloc(sizeof(int32_t) * (size_t)(total > 0 ? total : 1));
  if (!owner) return -1;
  for (int32_t b = 0; b < B; ++b)
    for (int32_t t = seq_offsets[b]; t < seq_offsets[b + 1]; ++t) owner[t] = b;
  const int64_t stride = (int64_t)H * d;
  int64_t total_macs = 0;
  int64_t units = total * H;
#pragma omp parallel for schedule(dynamic, 16) reduction(+ : total_macs)
  for (int64_t u = 0; u < units; ++u) {
    int64_t t = u / H;
    int32_t h = (int32_t)(u % H);
    int32_t b = owner[t];
    int32_t L = seq_offsets[b + 1] - seq_offsets[b];
    int32_t T = num_targets ? num_targets[b] : 0;
    int32_t i = (int32_t)(t - seq_offsets[b]);
    const float* kseg = k + (int64_t)seq_offsets[b] * stride + (int64_t)h * d;
    const float* vseg = v + (int64_t)seq_offsets[b] * stride + (int64_t)h * d;
    total_macs += one_row(q + t * stride + (int64_t)h * d, kseg, vseg, stride, d, i, L, L - T,
                          alpha, N, out + t * stride + (int64_t)h * d);
  }
  free(owner);
  if (macs) *macs = total_macs;
  return 0;
}

/*
 * Streaming variant: the query rows are the new tokens only (positions cached_len[b] ..
 * L_b - 1 of user b, packed per user in q_new); keys/values are the full segments.
 * out: [total_q, H, d].  Returns 0, or -1 on inconsistent offsets.
 */
int hstu_oracle_fwd_cached(const float* q_new, const float* k, const float* v,
                           const int32_t* seq_offsets, const int32_t* num_targets,
                           const int32_t* cached_len, int32_t B, int32_t H, int32_t d,
                           int64_t total_kv, int64_t total_q, double alpha, double N,
                           double* out, int64_t* macs) {
  if (B < 0) return -1;
  int64_t nrows = total_q;
  int32_t* ru = (int32_t*)malloc(sizeof(int32_t) * (size_t)(nrows > 0 ? nrows : 1));
  int32_t* rl = (int32_t*)malloc(sizeof(int32_t) * (size_t)(nrows > 0 ? nrows : 1));
  if (!ru || !rl) { free(ru); free(rl); return -1; }
  int64_t n = 0;
  for (int32_t b = 0; b < B; ++b) {
    int32_t L = seq_offsets[b + 1] - seq_offsets[b];
    int32_t c = cached_len ? cached_len[b] : 0;
    for (int32_t r = 0; r < L - c; ++r) {
      if (n >= nrows) { free(ru); free(rl); return -1; }
      ru[n] = b; rl[n] = r; ++n;
    }
  }
  int rc = (n == nrows) ? hstu_oracle_rows(q_new, k, v, seq_offsets, num_targets, cached_len, B,
                                           H, d, total_kv, total_q, alpha, N, ru, rl, nrows, out,
                                           macs)
                        : -1;
  free(ru);
  free(rl);
  return rc;
}

/*
 * Selected rows of the relative-attention-bias variant (one_row_rab); arguments as
 * hstu_oracle_rows plus rab [H, R] (R >= 1).  Returns 0, or -1 on inconsistent input.
 */
int hstu_oracle_rows_rab(const float* q, const float* k, const float* v,
                         const int32_t* seq_offsets, const int32_t* num_targets,
                         const int32_t* cached_len, const float* rab, int32_t R, int32_t B,
                         int32_t H, int32_t d, int64_t total_kv, int64_t total_q, double alpha,
                         double N, const int32_t* row_user, const int32_t* row_local,
                         int64_t nrows, double* out) {
  if (B < 0 || H <= 0 || d <= 0 || R <= 0 || !rab || !(N != 0.0)) return -1;
  if (seq_offsets[0] != 0 || seq_offsets[B] != total_kv) return -1;
  int64_t* qstart = (int64_t*)malloc(sizeof(int64_t) * (size_t)(B + 1));
  if (!qstart) return -1;
  qstart[0] = 0;
  for (int32_t b = 0; b < B; ++b) {
    if (user_ok(seq_offsets, num_targets, cached_len, b, total_kv)) { free(qstart); return -1; }
    int32_t L = seq_offsets[b + 1] - seq_offsets[b];
    int32_t c = cached_len ? cached_len[b] : 0;
    qstart[b + 1] = qstart[b] + (L - c);
  }
  if (qstart[B] != total_q) { free(qstart); return -1; }
  for (int64_t n = 0; n < nrows; ++n) {
    int32_t b = row_user[n];
    if (b < 0 || b >= B) { free(qstart); return -1; }
    int32_t L = seq_offsets[b + 1] - seq_offsets[b];
    int32_t c = cached_len ? cached_len[b] : 0;
    if (row_local[n] < 0 || row_local[n] >= L - c) { free(qstart); return -1; }
  }
  const int64_t stride = (int64_t)H * d;
  int64_t units = nrows * H;
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t u = 0; u < units; ++u) {
    int64_t n = u / H;
    int32_t h = (int32_t)(u % H);
    int32_t b = row_user[n];
    int32_t L = seq_offsets[b + 1] - seq_offsets[b];
    int32_t T = num_targets ? num_targets[b] : 0;
    int32_t c = cached_len ? cached_len[b] : 0;
    int32_t r = row_local[n];
    const float* qrow = q + (qstart[b] + r) * stride + (int64_t)h * d;
    const float* kseg = k + (int64_t)seq_offsets[b] * stride + (int64_t)h * d;
    const float* vseg = v + (int64_t)seq_offsets[b] * stride + (int64_t)h * d;
    one_row_rab(qrow, kseg, vseg, stride, d, c + r, L, L - T, alpha, N, rab + (int64_t)h * R, R,
                out + n * stride + (int64_t)h * d);
  }
  free(qstart);
  return 0;
}

/*
 * ---------------------------------------------------------------------------------------------
 * Backward pass.  The pages print no backward pass; the training story they tell (the scaling
 * section of the infolabhq.com multi-stage page) needs one.  It is derived here from the
 * forward definition above by the chain rule, for a scalar loss whose gradient with respect to
 * out is dout:
 *
 *   for every user, head, query position i and visible key j in A(i):
 *     s   = sum_c q[i,c] k[j,c],   x = alpha * s
 *     p   = silu(x)                        dv[j,:] += p * dout[i,:] / N
 *     g   = sum_c dout[i,c] v[j,c] / N     (gradient of the loss with respect to p)
 *     ds  = g * silu'(x) * alpha           (gradient with respect to s)
 *                                          dq[i,:] += ds * k[j,:]
 *                                          dk[j,:] += ds * q[i,:]
 *   silu'(x) = sigma(x) * (1 + x * (1 - sigma(x))),  sigma(x) = 1 / (1 + exp(-x))
 *
 * Masked pairs contribute nothing to any gradient.  Order: queries i ascending, and within a
 * query its keys j ascending, for every sum, so dq[i] adds keys in ascending order and dk[j],
 * dv[j] add queries in ascending order.
 * ---------------------------------------------------------------------------------------------
 */

/* Derivative of silu(x) = x * sigma(x): sigma(x) + x * sigma(x) * (1 - sigma(x)). */
static double dsilu(double x) {
  double sg = 1.0 / (1.0 + exp(-x));
  return sg * (1.0 + x * (1.0 - sg));
}

/*
 * Gradients of one user and head.  qs, ks, vs, dos: first row of the user's segment (row
 * stride `stride` floats, already offset to the head); dqs, dks, dvs: the same for the
 * doubles written (zeroed here first).  L: segment length; U: history length.
 */
static void bwd_user_head(const float* qs, const float* ks, const float* vs, const float* dos,
                          int64_t stride, int32_t d, int32_t L, int32_t U, double alpha, double N,
                          double* dqs, double* dks, double* dvs) {
  for (int32_t t = 0; t < L; ++t)
    for (int32_t c = 0; c < d; ++c) {
      dqs[(int64_t)t * stride + c] = 0.0;
      dks[(int64_t)t * stride + c] = 0.0;
      dvs[(int64_t)t * stride + c] = 0.0;
    }
  for (int32_t i = 0; i < L; ++i) {
    const float* qi = qs + (int64_t)i * stride;
    const float* doi = dos + (int64_t)i * stride;
    double* dqi = dqs + (int64_t)i * stride;
    for (int32_t j = 0; j < L; ++j) {
      if (!visible(i, j, U)) continue;
      const float* kj = ks + (int64_t)j * stride;
      const float* vj = vs + (int64_t)j * stride;
      double* dkj = dks + (int64_t)j * stride;
      double* dvj = dvs + (int64_t)j * stride;
      double s = 0.0, g = 0.0;
      for (int32_t c = 0; c < d; ++c) s += (double)qi[c] * (double)kj[c];
      for (int32_t c = 0; c < d; ++c) g += (double)doi[c] * (double)vj[c];
      g /= N;
      double x = alpha * s;
      double p = silu(x);
      double ds = g * dsilu(x) * alpha;
      for (int32_t c = 0; c < d; ++c) {
        dvj[c] += p * (double)doi[c] / N;
        dqi[c] += ds * (double)kj[c];
        dkj[c] += ds * (double)qi[c];
      }
    }
  }
}

/*
 * Full backward pass: dq, dk, dv [total, H, d] doubles from q, k, v, dout [total, H, d].
 * Returns 0, or -1 on inconsistent offsets.
 */
int hstu_oracle_bwd(const float* q, const float* k, const float* v, const float* dout,
                    const int32_t* seq_offsets, const int32_t* num_targets, int32_t B, int32_t H,
                    int32_t d, int64_t total, double alpha, double N, double* dq, double* dk,
                    double* dv) {
  if (B < 0 || H <= 0 || d <= 0 || !(N != 0.0)) return -1;
  if (seq_offsets[0] != 0 || seq_offsets[B] != total) return -1;
  for (int32_t b = 0; b < B; ++b)
    if (user_ok(seq_offsets, num_targets, NULL, b, total)) return -1;
  const int64_t stride = (int64_t)H * d;
  int64_t units = (int64_t)B * H;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t u = 0; u < units; ++u) {
    int32_t b = (int32_t)(u / H);
    int32_t h = (int32_t)(u % H);
    int32_t L = seq_offsets[b + 1] - seq_offsets[b];
    int32_t T = num_targets ? num_targets[b] : 0;
    int64_t o = (int64_t)seq_offsets[b] * stride + (int64_t)h * d;
    bwd_user_head(q + o, k + o, v + o, dout + o, stride, d, L, L - T, alpha, N, dq + o, dk + o,
                  dv + o);
  }
  return 0;
}

/*
 * Selected rows of the backward pass, for checks at sizes where the full pass is too slow.
 * For n in [0, nrows): user row_user[n], position row_local[n] of that user's segment; writes
 * dq of that query row and dk, dv of that key row ([nrows, H, d] doubles each), each summed in
 * the same order as hstu_oracle_bwd, so the rows equal the full pass's rows exactly.
 * Returns 0, or -1 on inconsistent offsets or rows.
 */
int hstu_oracle_bwd_rows(const float* q, const float* k, const float* v, const float* dout,
                         const int32_t* seq_offsets, const int32_t* num_targets, int32_t B,
                         int32_t H, int32_t d, int64_t total, double alpha, double N,
                         const int32_t* row_user, const int32_t* row_local, int64_t nrows,
                         double* dq, double* dk, double* dv) {
  if (B < 0 || H <= 0 || d <= 0 || !(N != 0.0)) return -1;
  if (seq_offsets[0] != 0 || seq_offsets[B] != total) return -1;
  for (int32_t b = 0; b < B; ++b)
    if (user_ok(seq_offsets, num_targets, NULL, b, total)) return -1;
  for (int64_t n = 0; n < nrows; ++n) {
    int32_t b = row_user[n];
    if (b < 0 || b >= B) return -1;
    if (row_local[n] < 0 || row_local[n] >= seq_offsets[b + 1] - seq_offsets[b]) return -1;
  }
  const int64_t stride = (int64_t)H * d;
  int64_t units = nrows * H;
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t u = 0; u < units; ++u) {
    int64_t n = u / H;
    int32_t h = (int32_t)(u % H);
    int32_t b = row_user[n];
    int32_t L = seq_offsets[b + 1] - seq_offsets[b];
    int32_t U = L - (num_targets ? num_targets[b] : 0);
    int32_t r = row_local[n];
    int64_t o = (int64_t)seq_offsets[b] * stride + (int64_t)h * d;
    const float *qs = q + o, *ks = k + o, *vs = v + o, *dos = dout + o;
    double* dqn = dq + n * stride + (int64_t)h * d;
    double* dkn = dk + n * stride + (int64_t)h * d;
    double* dvn = dv + n * stride + (int64_t)h * d;
    for (int32_t c = 0; c < d; ++c) dqn[c] = dkn[c] = dvn[c] = 0.0;
    /* dq of query row r: its visible keys, ascending */
    const float* qi = qs + (int64_t)r * stride;
    const float* doi = dos + (int64_t)r * stride;
    for (int32_t j = 0; j < L; ++j) {
      if (!visible(r, j, U)) continue;
      const float* kj = ks + (int64_t)j * stride;
      const float* vj = vs + (int64_t)j * stride;
      double s = 0.0, g = 0.0;
      for (int32_t c = 0; c < d; ++c) s += (double)qi[c] * (double)kj[c];
      for (int32_t c = 0; c < d; ++c) g += (double)doi[c] * (double)vj[c];
      g /= N;
      double ds = g * dsilu(alpha * s) * alpha;
      for (int32_t c = 0; c < d; ++c) dqn[c] += ds * (double)kj[c];
    }
    /* dk, dv of key row r: the queries that see it, ascending */
    const float* kr = ks + (int64_t)r * stride;
    const float* vr = vs + (int64_t)r * stride;
    for (int32_t i = 0; i < L; ++i) {
      if (!visible(i, r, U)) continue;
      const float* qi2 = qs + (int64_t)i * stride;
      const float* doi2 = dos + (int64_t)i * stride;
      double s = 0.0, g = 0.0;
      for (int32_t c = 0; c < d; ++c) s += (double)qi2[c] * (double)kr[c];
      for (int32_t c = 0; c < d; ++c) g += (double)doi2[c] * (double)vr[c];
      g /= N;
      double x = alpha * s;
      double p = silu(x);
      double ds = g * dsilu(x) * alpha;
      for (int32_t c = 0; c < d; ++c) {
        dvn[c] += p * (double)doi2[c] / N;
        dkn[c] += ds * (double)qi2[c];
      }
    }
  }
  return 0;
}
