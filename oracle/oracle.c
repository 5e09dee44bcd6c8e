/*
 * oracle.c -- plain, slow, fp64 CPU oracle for the REINFORCE Zero token-logprob /
 * loss / gradient path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may load, link or call this
 * library: only the test suite, the package smoke check and the benchmark's CPU-baseline
 * leg use it.  It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (sources are the pages' sections; readings are listed beside each step):
 *
 *   "vLLM says aligned kernels make asynchronous RL stable at lag 64" (ainewsbites.com),
 *   section "REINFORCE Zero removes the mismatch first":
 *     - the learner computes its own probability of every sampled token
 *       (token logprob = log-softmax of the LM-head logits, gathered at the token);
 *     - the ratio is the learner probability divided by the recorded rollout probability,
 *       with no clipping:  w_t = exp(lp_t - lp_rollout_t);
 *     - a response's advantage is r_i less the average r over the responses of its group;
 *     - the per-token terms of a response are combined by a mean over that response's
 *       tokens; there is no value model and no gate rejects any response;
 *     - the objective is plain REINFORCE (importance weighted).
 *
 * Definitions written out (everything in fp64, inputs widened exactly):
 *   z[t,v]  = sum_k H[t,k] * W[v,k]                      (k in increasing order)
 *   lse[t]  = m + log(sum_v exp(z[t,v] - m)),  m = max_v z[t,v]
 *   lp[t]   = z[t,y_t] - lse[t]
 *   A_i     = r_i - (1/|g|) sum_{j in g} r_j,  g = group of response i
 *   L_i     = off[i+1] - off[i]
 *   w_t     = exp(lp[t] - lp_rollout[t])                 (no clipping)
 *   loss    = -(1/N) sum_i (A_i / L_i) sum_{t in i} w_t,  N = number of responses
 *   kappa_t = -A_i * w_t / (N * L_i)                     (= d loss / d lp_t)
 *   dZ[t,v] = kappa_t * ([v == y_t] - exp(z[t,v] - lse[t]))
 *   dH[t,:] = sum_v dZ[t,v] W[v,:];   dW[v,:] = sum_t dZ[t,v] H[t,:]
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   temperature 1 and no LM-head bias; the group mean includes the response itself and
 *   is not divided by a standard deviation; the per-response token means are averaged
 *   over the N responses of the call; the loss is the ratio surrogate to be minimised,
 *   whose exact gradient equals the "ratio held constant" REINFORCE gradient.
 *
 * Matrices H and W can be passed either as bf16 bit patterns (uint16) or as fp64; the
 * bf16 path widens each element exactly.  OpenMP parallelism is only over independent
 * rows (token rows for lp/dH, vocabulary rows for dW): no reduction crosses threads.
 *
 * Return codes: 0 = ok, 1 = invalid argument (out-of-range id / group / offsets, empty
 * segment), 2 = out of memory.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* exact widening of a bf16 bit pattern */
static inline double bf16_bits_to_f64(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* element i of a matrix stored either as bf16 bits (is_bf16 != 0) or as fp64 */
static inline double elem(const void *p, size_t i, int is_bf16) {
  return is_bf16 ? bf16_bits_to_f64(((const uint16_t *)p)[i]) : ((const double *)p)[i];
}

/* z[v] = sum_k H[t,k] W[v,k], k ascending */
static void logits_row(const void *H, const void *W, int is_bf16, int64_t t, int32_t d, int32_t V,
                       double *z) {
  for (int32_t v = 0; v < V; ++v) {
    double acc = 0.0;
    for (int32_t k = 0; k < d; ++k)
      acc += elem(H, (size_t)t * d + k, is_bf16) * elem(W, (size_t)v * d + k, is_bf16);
    z[v] = acc;
  }
}

/* log-sum-exp of z[0..V) with the maximum taken out first */
static double logsumexp(const double *z, int32_t V) {
  double m = -INFINITY;
  for (int32_t v = 0; v < V; ++v)
    if (z[v] > m) m = z[v];
  double s = 0.0;
  for (int32_t v = 0; v < V; ++v) s += exp(z[v] - m);
  return m + log(s);
}

/*
 * Token logprobs for the rows listed in rows[0..nrows) (rows == NULL: rows 0..nrows).
 * lp[j], lse[j] refer to the j-th listed row.  Either output may be NULL.
 */
int oracle_lp_rows(const void *H, const void *W, int is_bf16, const int32_t *ids, int64_t n,
                   int32_t d, int32_t V, const int64_t *rows, int64_t nrows, double *lp,
                   double *lse) {
  if (d <= 0 || V <= 0 || n < 0 || nrows < 0) return 1;
  for (int64_t j = 0; j < nrows; ++j) {
    int64_t t = rows ? rows[j] : j;
    if (t < 0 || t >= n || ids[t] < 0 || ids[t] >= V) return 1;
  }
  int err = 0;
#pragma omp parallel
  {
    double *z = (double *)malloc(sizeof(double) * (size_t)V);
    if (!z) {
#pragma omp atomic write
      err = 2;
    } else {
#pragma omp for schedule(dynamic, 1)
      for (int64_t j = 0; j < nrows; ++j) {
        int64_t t = rows ? rows[j] : j;
        logits_row(H, W, is_bf16, t, d, V, z);
        double l = logsumexp(z, V);
        if (lse) lse[j] = l;
        if (lp) lp[j] = z[ids[t]] - l;
      }
      free(z);
    }
  }
  return err;
}

/* A_i = r_i - mean of r over the responses sharing group_ids[i] (mean includes i). */
int oracle_advantages(const double *rewards, const int32_t *gid, int32_t R, int32_t G,
                      double *A) {
  if (R <= 0 || G <= 0) return 1;
  double *sum = (double *)calloc((size_t)G, sizeof(double));
  int64_t *cnt = (int64_t *)calloc((size_t)G, sizeof(int64_t));
  if (!sum || !cnt) {
    free(sum);
    free(cnt);
    return 2;
  }
  int err = 0;
  for (int32_t i = 0; i < R; ++i) {
    if (gid[i] < 0 || gid[i] >= G) {
      err = 1;
      break;
    }
    sum[gid[i]] += rewards[i];
    cnt[gid[i]] += 1;
  }
  if (!err)
    for (int32_t i = 0; i < R; ++i) A[i] = rewards[i] - sum[gid[i]] / (double)cnt[gid[i]];
  free(sum);
  free(cnt);
  return err;
}

/* Segment checks: off[0] = 0, off[R] = n, every L_i = off[i+1]-off[i] >= 1. */
static int check_offsets(const int64_t *off, int32_t R, int64_t n) {
  if (off[0] != 0 || off[R] != n) return 1;
  for (int32_t i = 0; i < R; ++i)
    if (off[i + 1] <= off[i]) return 1;
  return 0;
}

/*
 * Loss stage from per-token logprobs: w_t, kappa_t and the scalar loss.
 * w / kappa may be NULL.  The loss is accumulated response by response in index order.
 */
int oracle_loss_from_lp(const double *lp, const double *lp_rollout, const double *rewards,
                        const int64_t *off, const int32_t *gid, int64_t n, int32_t R, int32_t G,
                        double *w_out, double *kappa_out, double *loss_out) {
  if (n <= 0 || R <= 0) return 1;
  if (check_offsets(off, R, n)) return 1;
  double *A = (double *)malloc(sizeof(double) * (size_t)R);
  if (!A) return 2;
  int err = oracle_advantages(rewards, gid, R, G, A);
  if (err) {
    free(A);
    return err;
  }
  const double N = (double)R;
  double loss = 0.0;
  for (int32_t i = 0; i < R; ++i) {
    const double L = (double)(off[i + 1] - off[i]);
    double wsum = 0.0;
    for (int64_t t = off[i]; t < off[i + 1]; ++t) {
      const double w = exp(lp[t] - lp_rollout[t]); /* unclipped ratio */
      wsum += w;
      if (w_out) w_out[t] = w;
      if (kappa_out) kappa_out[t] = -A[i] * w / (N * L);
    }
    loss += A[i] * (wsum / L);
  }
  *loss_out = -loss / N;
  free(A);
  return 0;
}

/*
 * dH rows for the listed token rows, given lse and kappa of those rows:
 *   dH[j,:] = sum_v kappa * ([v == y] - exp(z[v] - lse)) * W[v,:]
 */
int oracle_dh_rows(const void *H, const void *W, int is_bf16, const int32_t *ids, int64_t n,
                   int32_t d, int32_t V, const int64_t *rows, int64_t nrows,
                   const double *lse_rows, const double *kappa_rows, double *dH_rows) {
  for (int64_t j = 0; j < nrows; ++j) {
    int64_t t = rows ? rows[j] : j;
    if (t < 0 || t >= n || ids[t] < 0 || ids[t] >= V) return 1;
  }
  int err = 0;
#pragma omp parallel
  {
    double *z = (double *)malloc(sizeof(double) * (size_t)V);
    if (!z) {
#pragma omp atomic write
      err = 2;
    } else {
#pragma omp for schedule(dynamic, 1)
      for (int64_t j = 0; j < nrows; ++j) {
        int64_t t = rows ? rows[j] : j;
        double *out = dH_rows + (size_t)j * d;
        for (int32_t k = 0; k < d; ++k) out[k] = 0.0;
        logits_row(H, W, is_bf16, t, d, V, z);
        for (int32_t v = 0; v < V; ++v) {
          const double dz = kappa_rows[j] * ((v == ids[t] ? 1.0 : 0.0) - exp(z[v] - lse_rows[j]));
          for (int32_t k = 0; k < d; ++k) out[k] += dz * elem(W, (size_t)v * d + k, is_bf16);
        }
      }
      free(z);
    }
  }
  return err;
}

/*
 * dW rows vocab_rows[0..nv) (NULL: rows 0..nv), tokens summed in index order:
 *   dW[v,:] = sum_t kappa_t * ([v == y_t] - exp(z[t,v] - lse_t)) * H[t,:]
 * z[t,v] is recomputed per (t, v) with the same k-ordered dot product as the forward.
 */
int oracle_dw_rows(const void *H, const void *W, int is_bf16, const int32_t *ids, int64_t n,
                   int32_t d, int32_t V, const double *lse, const double *kappa,
                   const int64_t *vocab_rows, int64_t nv, double *dW_rows) {
  for (int64_t t = 0; t < n; ++t)
    if (ids[t] < 0 || ids[t] >= V) return 1;
  for (int64_t j = 0; j < nv; ++j) {
    int64_t v = vocab_rows ? vocab_rows[j] : j;
    if (v < 0 || v >= V) return 1;
  }
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t j = 0; j < nv; ++j) {
    const int64_t v = vocab_rows ? vocab_rows[j] : j;
    double *out = dW_rows + (size_t)j * d;
    for (int32_t k = 0; k < d; ++k) out[k] = 0.0;
    for (int64_t t = 0; t < n; ++t) {
      double z = 0.0;
      for (int32_t k = 0; k < d; ++k)
        z += elem(H, (size_t)t * d + k, is_bf16) * elem(W, (size_t)v * d + k, is_bf16);
      const double dz = kappa[t] * ((v == ids[t] ? 1.0 : 0.0) - exp(z - lse[t]));
      for (int32_t k = 0; k < d; ++k) out[k] += dz * elem(H, (size_t)t * d + k, is_bf16);
    }
  }
  return 0;
}

/*
 * The whole path: lp, lse, w, kappa, loss, dH [n,d], dW [V,d] (all fp64 outputs).
 * Any of lp/lse/w/kappa/dH/dW may be NULL; loss must not be NULL.
 */
int oracle_loss_fwd_bwd(const void *H, const void *W, int is_bf16, const int32_t *ids,
                        const double *lp_rollout, const double *rewards, const int64_t *off,
                        const int32_t *gid, int64_t n, int32_t R, int32_t G, int32_t d, int32_t V,
                        double *loss, double *dH, double *dW, double *lp_out, double *lse_out,
                        double *w_out, double *kappa_out) {
  if (n <= 0 || R <= 0 || G <= 0 || d <= 0 || V <= 0 || !loss) return 1;
  double *lp = (double *)malloc(sizeof(double) * (size_t)n);
  double *lse = (double *)malloc(sizeof(double) * (size_t)n);
  double *kappa = (double *)malloc(sizeof(double) * (size_t)n);
  int err = (!lp || !lse || !kappa) ? 2 : 0;
  if (!err) err = oracle_lp_rows(H, W, is_bf16, ids, n, d, V, NULL, n, lp, lse);
  if (!err) err = oracle_loss_from_lp(lp, lp_rollout, rewards, off, gid, n, R, G, w_out, kappa, loss);
  if (!err && dH) err = oracle_dh_rows(H, W, is_bf16, ids, n, d, V, NULL, n, lse, kappa, dH);
  if (!err && dW) err = oracle_dw_rows(H, W, is_bf16, ids, n, d, V, lse, kappa, NULL, V, dW);
  if (!err) {
    if (lp_out) memcpy(lp_out, lp, sizeof(double) * (size_t)n);
    if (lse_out) memcpy(lse_out, lse, sizeof(double) * (size_t)n);
    if (kappa_out) memcpy(kappa_out, kappa, sizeof(double) * (size_t)n);
  }
  free(lp);
  free(lse);
  free(kappa);
  return err;
}

/* Number of OpenMP threads a parallel region of this library uses. */
int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ------------------------------------------------------------------------------------
 * Variants of the loss stage (the baselines the pages contrast REINFORCE Zero with) and
 * diagnostics of the ratio.  Readings, as the pages give no formulas:
 *   - truncated IS (the clipped-weight baseline, which the page says biases the gradient;
 *     [A] section "REINFORCE Zero removes the mismatch first"): w -> min(w, clip_max) in the
 *     coefficient of each token's gradient, held constant;
 *   - sequence gate (the standard-kernel baseline on OSWorld, [A] section "Zero mismatch
 *     expands to newer models"): response i is kept iff gate_lo <= exp(mean_t (lp - lp_rollout))
 *     <= gate_hi over its counted tokens; a rejected response contributes nothing but its
 *     reward still enters its group's mean, and N still counts it;
 *   - token mask: only tokens with mask 1 count; L_i is the number of counted tokens of
 *     response i (a response with none contributes nothing);
 *   - n_resp_total > 0 replaces N (responses of the whole data-parallel batch).
 * kappa_t = -A_i * s_i * m_t * g(w_t) / (N * L_i) and loss = sum_t kappa_t.
 * ------------------------------------------------------------------------------------ */
#define ORACLE_CLIP 1
#define ORACLE_GATE 2
#define ORACLE_MASK 4

int oracle_loss_from_lp_ex(const double *lp, const double *lp_rollout, const double *rewards,
                           const int64_t *off, const int32_t *gid, int64_t n, int32_t R, int32_t G,
                           int32_t flags, double clip_max, double gate_lo, double gate_hi,
                           const uint8_t *mask, int32_t n_resp_total, double *w_out, double *kappa_out,
                           double *loss_out) {
  if (n <= 0 || R <= 0) return 1;
  if (check_offsets(off, R, n)) return 1;
  double *A = (double *)malloc(sizeof(double) * (size_t)R);
  if (!A) return 2;
  int err = oracle_advantages(rewards, gid, R, G, A);
  if (err) {
    free(A);
    return err;
  }
  const double N = n_resp_total > 0 ? (double)n_resp_total : (double)R;
  double loss = 0.0;
  for (int32_t i = 0; i < R; ++i) {
    double L = 0.0, logsum = 0.0;
    for (int64_t t = off[i]; t < off[i + 1]; ++t) {
      const int counted = (flags & ORACLE_MASK) ? (mask[t] != 0) : 1;
      if (counted) {
        L += 1.0;
        logsum += lp[t] - lp_rollout[t];
      }
    }
    int keep = L > 0.0;
    if (keep && (flags & ORACLE_GATE)) {
      const double g = exp(logsum / L); /* geometric-mean ratio of the response */
      keep = (g >= gate_lo && g <= gate_hi);
    }
    double wsum = 0.0;
    for (int64_t t = off[i]; t < off[i + 1]; ++t) {
      const int counted = (flags & ORACLE_MASK) ? (mask[t] != 0) : 1;
      double w = exp(lp[t] - lp_rollout[t]);
      if (w_out) w_out[t] = w;
      if ((flags & ORACLE_CLIP) && w > clip_max) w = clip_max;
      const double k = (keep && counted) ? -A[i] * w / (N * L) : 0.0;
      if (kappa_out) kappa_out[t] = k;
      if (keep && counted) wsum += w;
    }
    if (keep) loss += A[i] * (wsum / L);
  }
  *loss_out = -loss / N;
  free(A);
  return 0;
}

static int cmp_double(const void *a, const void *b) {
  const double x = *(const double *)a, y = *(const double *)b;
  return (x > y) - (x < y);
}

/*
 * Diagnostics of the ratio over the counted tokens (mask may be NULL), [A] sections
 * "Asynchronous training has two different gaps" (importance-weight deviation, peak vs
 * median) and "Reported results include 2.40 times higher throughput" (rollout-to-learner
 * KL).  stats: [0] k1 = mean(lp_rollout - lp); [1] k2 = mean((lp - lp_rollout)^2 / 2);
 * [2] k3 = mean(w - 1 - (lp - lp_rollout)); [3] min w; [4] max w; [5] max |w - 1|;
 * [6] lower median of |w - 1| (element of rank floor((m - 1) / 2) of the m counted tokens
 * in ascending order); [7] [5] / [6]; [8] m.  resp_mean_w (may be NULL): per response,
 * the mean of w over its counted tokens (0 when it has none).
 */
int oracle_ratio_stats(const double *lp, const double *lp_rollout, const int64_t *off, int64_t n, int32_t R,
                       const uint8_t *mask, double *stats, double *resp_mean_w) {
  if (n <= 0 || R <= 0 || check_offsets(off, R, n)) return 1;
  double *dev = (double *)malloc(sizeof(double) * (size_t)n);
  if (!dev) return 2;
  int64_t m = 0;
  double k1 = 0, k2 = 0, k3 = 0, wmin = INFINITY, wmax = -INFINITY, dmax = 0;
  for (int32_t i = 0; i < R; ++i) {
    double ws = 0.0;
    int64_t c = 0;
    for (int64_t t = off[i]; t < off[i + 1]; ++t) {
      if (mask && !mask[t]) continue;
      const double x = lp[t] - lp_rollout[t];
      const double w = exp(x);
      k1 += -x;
      k2 += 0.5 * x * x;
      k3 += w - 1.0 - x;
      if (w < wmin) wmin = w;
      if (w > wmax) wmax = w;
      const double d = fabs(w - 1.0);
      if (d > dmax) dmax = d;
      dev[m++] = d;
      ws += w;
      ++c;
    }
    if (resp_mean_w) resp_mean_w[i] = c ? ws / (double)c : 0.0;
  }
  if (m == 0) {
    free(dev);
    return 1;
  }
  qsort(dev, (size_t)m, sizeof(double), cmp_double);
  const double med = dev[(m - 1) / 2];
  stats[0] = k1 / (double)m;
  stats[1] = k2 / (double)m;
  stats[2] = k3 / (double)m;
  stats[3] = wmin;
  stats[4] = wmax;
  stats[5] = dmax;
  stats[6] = med;
  stats[7] = med > 0 ? dmax / med : INFINITY;
  stats[8] = (double)m;
  free(dev);
  return 0;
}
