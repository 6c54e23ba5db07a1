/*
 * gdpa_oracle.c -- plain fp64 CPU oracle for Generalized Dot-Product Attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file: only the tests, the package's smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code, header or constant with the CUDA
 * library (pffn_attention_b200/csrc); the two meet only in the seeded inputs.
 *
 * What it computes (the definition, written out, no blocking or fusion):
 *
 *   For every sample b, head h, query i < Lq_b and key j < Lk_b:
 *     vis(i,j) = (wl < 0 || j >= i - wl) && (wr < 0 || j <= i + wr)
 *     s_ij     = scale * sum_d Q[i,h,d] K[j,h,d] + beta_hj
 *     beta_hj  = 0 | bias[h][j] | log sigmoid(G[h][j])      (none/add/gate)
 *     p_ij     = silu(s_ij) | s_ij | softmax_j(s_ij) | gelu(s_ij)
 *                over visible j, else 0;  gelu(x) = x Phi(x), Phi the standard
 *                normal distribution function, 0.5 (1 + erf(x / sqrt 2))
 *     O_i      = sum_j p_ij V_j
 *     LSE_i    = log sum_{visible j} exp(s_ij)               (softmax only)
 *
 * Sources, by page and section:
 *   - Kunlun paper review (liuzhao09.github.io), §2.3 "GDPA" and Fig. 2:
 *     the personalised FFN recast as attention with the sequence as query and
 *     context-generated K, V; step order QK^T / tau, then an activation that
 *     may be element-wise (non-softmax), GELU named as the example, then
 *     Attn x V; tau is a free temperature, passed here as scale = 1/tau.
 *   - Kunlun reproduction notes (daiwk.github.io), "Core equations":
 *     A = softmax(QK^T / sqrt(d) + log sigma(G)) -- the gate enters the scores
 *     additively as log sigma(G), after the scaling.
 *   - Kunlun paper review, §2.5 "Sliding Window": each query attends only to
 *     keys within a local band; here a general (left, right) band over local
 *     indices.
 *   - Kunlun Breakdown (machinelearningatscale), "The Core Architecture and
 *     Mechanics": the sequence is the query and context-generated weights are
 *     key and value, fused into one FlashAttention-style operator.
 *
 * The backward pass is the chain rule of the definition above, per element:
 *   dV_j  = sum_i p_ij dO_i
 *   dP_ij = dO_i . V_j
 *   dS_ij = p_ij (dP_ij - delta_i), delta_i = sum_j p_ij dP_ij       (softmax)
 *         = dP_ij (sigma(s) + s sigma(s)(1 - sigma(s)))              (SiLU)
 *         = dP_ij                                                    (identity)
 *         = dP_ij (Phi(s) + s phi(s)), phi(x) = exp(-x^2/2) / sqrt(2 pi)  (GELU)
 *   dQ_i  = scale sum_j dS_ij K_j,  dK_j = scale sum_i dS_ij Q_i
 *   dbias_hj = sum_i dS_ij  (add)  or  sum_i dS_ij (1 - sigma(G_hj))  (gate)
 *
 * Rows with no visible key: O = 0 and LSE = -inf; they add nothing to any
 * gradient.  Everything is fp64; the inputs are the exact bf16 values widened.
 * OpenMP runs the independent (sample, head) units in parallel; each unit is
 * computed start to finish by one thread in the order written here.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_PHI_SILU = 0, ORACLE_PHI_SOFTMAX = 1, ORACLE_PHI_IDENTITY = 2, ORACLE_PHI_GELU = 3 };
enum { ORACLE_BIAS_NONE = 0, ORACLE_BIAS_ADD = 1, ORACLE_BIAS_GATE = 2 };

typedef struct {
  int B, H, D;
  int64_t total_q, total_kv;
  int phi;
  double scale;
  int window_left, window_right; /* -1 = unbounded on that side */
  int bias_kind;
} oracle_params;

static int is_visible(int64_t i, int64_t j, int wl, int wr) {
  if (wl >= 0 && j < i - wl) return 0;
  if (wr >= 0 && j > i + wr) return 0;
  return 1;
}

static double sigmoid(double x) {
  if (x >= 0.0) return 1.0 / (1.0 + exp(-x));
  double e = exp(x);
  return e / (1.0 + e);
}

/* Standard normal distribution function and density (GELU and its derivative). */
static double normal_cdf(double x) { return 0.5 * (1.0 + erf(x / sqrt(2.0))); }
static double normal_pdf(double x) {
  return exp(-0.5 * x * x) / sqrt(2.0 * 3.14159265358979323846);
}

/* log sigma(g), written so that neither branch overflows. */
static double log_sigmoid(double g) {
  if (g >= 0.0) return -log1p(exp(-g));
  return g - log1p(exp(g));
}

static double score_bias(const oracle_params* p, const double* bias, int h,
                         int64_t kv_row) {
  if (p->bias_kind == ORACLE_BIAS_NONE) return 0.0;
  double g = bias[(int64_t)h * p->total_kv + kv_row];
  return p->bias_kind == ORACLE_BIAS_ADD ? g : log_sigmoid(g);
}

static int check_params(const oracle_params* p, const int32_t* qo,
                        const int32_t* ko) {
  if (!p || p->B < 0 || p->H <= 0 || p->D <= 0) return 1;
  if (p->phi < 0 || p->phi > 3 || p->bias_kind < 0 || p->bias_kind > 2) return 1;
  if (qo[0] != 0 || ko[0] != 0) return 1;
  for (int b = 0; b < p->B; ++b)
    if (qo[b + 1] < qo[b] || ko[b + 1] < ko[b]) return 1;
  if (qo[p->B] != p->total_q || ko[p->B] != p->total_kv) return 1;
  return 0;
}

/* Scores s_ij (and visibility) for one query row of one (sample, head). */
static void row_scores(const oracle_params* p, const double* q, const double* k,
                       const double* bias, int h, int64_t q_row, int64_t kv_base,
                       int64_t i, int64_t Lk, double* s, unsigned char* vis) {
  const int H = p->H, D = p->D;
  const double* qi = q + (q_row * H + h) * D;
  for (int64_t j = 0; j < Lk; ++j) {
    vis[j] = (unsigned char)is_visible(i, j, p->window_left, p->window_right);
    if (!vis[j]) { s[j] = 0.0; continue; }
    const double* kj = k + ((kv_base + j) * H + h) * D;
    double dot = 0.0;
    for (int d = 0; d < D; ++d) dot += qi[d] * kj[d];
    s[j] = p->scale * dot + score_bias(p, bias, h, kv_base + j);
  }
}

/* p_ij from s_ij for one row; returns the row's LSE (softmax) or 0. */
static double row_probs(const oracle_params* p, const double* s,
                        const unsigned char* vis, int64_t Lk, double* pr) {
  if (p->phi == ORACLE_PHI_SOFTMAX) {
    double m = -INFINITY;
    for (int64_t j = 0; j < Lk; ++j)
      if (vis[j] && s[j] > m) m = s[j];
    if (m == -INFINITY) {
      for (int64_t j = 0; j < Lk; ++j) pr[j] = 0.0;
      return -INFINITY;
    }
    double l = 0.0;
    for (int64_t j = 0; j < Lk; ++j)
      if (vis[j]) l += exp(s[j] - m);
    for (int64_t j = 0; j < Lk; ++j) pr[j] = vis[j] ? exp(s[j] - m) / l : 0.0;
    return m + log(l);
  }
  for (int64_t j = 0; j < Lk; ++j) {
    if (!vis[j]) { pr[j] = 0.0; continue; }
    if (p->phi == ORACLE_PHI_SILU)
      pr[j] = s[j] * sigmoid(s[j]);
    else if (p->phi == ORACLE_PHI_GELU)
      pr[j] = s[j] * normal_cdf(s[j]);
    else
      pr[j] = s[j];
  }
  return 0.0;
}

int gdpa_oracle_forward(const oracle_params* p, const double* q, const double* k,
                        const double* v, const int32_t* q_offsets,
                        const int32_t* kv_offsets, const double* bias, double* o,
                        double* lse) {
  if (check_params(p, q_offsets, kv_offsets)) return 1;
  if (p->bias_kind != ORACLE_BIAS_NONE && !bias) return 1;
  const int H = p->H, D = p->D;
  const int64_t units = (int64_t)p->B * H;
  int err = 0;
#pragma omp parallel
  {
    int64_t maxk = 0;
    for (int b = 0; b < p->B; ++b) {
      int64_t L = kv_offsets[b + 1] - kv_offsets[b];
      if (L > maxk) maxk = L;
    }
    double* s = (double*)malloc(sizeof(double) * (size_t)(maxk + 1));
    double* pr = (double*)malloc(sizeof(double) * (size_t)(maxk + 1));
    unsigned char* vis = (unsigned char*)malloc((size_t)(maxk + 1));
    if (!s || !pr || !vis) {
#pragma omp atomic write
      err = 1;
    }
#pragma omp for schedule(dynamic, 1)
    for (int64_t u = 0; u < units; ++u) {
      if (err) continue;
      const int b = (int)(u / H), h = (int)(u % H);
      const int64_t q0 = q_offsets[b], Lq = q_offsets[b + 1] - q0;
      const int64_t k0 = kv_offsets[b], Lk = kv_offsets[b + 1] - k0;
      for (int64_t i = 0; i < Lq; ++i) {
        row_scores(p, q, k, bias, h, q0 + i, k0, i, Lk, s, vis);
        double row_lse = row_probs(p, s, vis, Lk, pr);
        double* oi = o + ((q0 + i) * H + h) * D;
        for (int d = 0; d < D; ++d) {
          double acc = 0.0;
          for (int64_t j = 0; j < Lk; ++j)
            acc += pr[j] * v[((k0 + j) * H + h) * D + d];
          oi[d] = acc;
        }
        if (lse) lse[(int64_t)h * p->total_q + q0 + i] = row_lse;
      }
    }
    free(s);
    free(pr);
    free(vis);
  }
  return err;
}

int gdpa_oracle_backward(const oracle_params* p, const double* q, const double* k,
                         const double* v, const double* dout,
                         const int32_t* q_offsets, const int32_t* kv_offsets,
                         const double* bias, double* dq, double* dk, double* dv,
                         double* dbias) {
  if (check_params(p, q_offsets, kv_offsets)) return 1;
  if (p->bias_kind != ORACLE_BIAS_NONE && !bias) return 1;
  const int H = p->H, D = p->D;
  const int64_t units = (int64_t)p->B * H;
  memset(dq, 0, sizeof(double) * (size_t)(p->total_q * H * D));
  memset(dk, 0, sizeof(double) * (size_t)(p->total_kv * H * D));
  memset(dv, 0, sizeof(double) * (size_t)(p->total_kv * H * D));
  if (dbias) memset(dbias, 0, sizeof(double) * (size_t)(p->total_kv * H));
  int err = 0;
#pragma omp parallel
  {
    int64_t maxk = 0;
    for (int b = 0; b < p->B; ++b) {
      int64_t L = kv_offsets[b + 1] - kv_offsets[b];
      if (L > maxk) maxk = L;
    }
    double* s = (double*)malloc(sizeof(double) * (size_t)(maxk + 1));
    double* pr = (double*)malloc(sizeof(double) * (size_t)(maxk + 1));
    double* dp = (double*)malloc(sizeof(double) * (size_t)(maxk + 1));
    double* ds = (double*)malloc(sizeof(double) * (size_t)(maxk + 1));
    unsigned char* vis = (unsigned char*)malloc((size_t)(maxk + 1));
    if (!s || !pr || !dp || !ds || !vis) {
#pragma omp atomic write
      err = 1;
    }
#pragma omp for schedule(dynamic, 1)
    for (int64_t u = 0; u < units; ++u) {
      if (err) continue;
      const int b = (int)(u / H), h = (int)(u % H);
      const int64_t q0 = q_offsets[b], Lq = q_offsets[b + 1] - q0;
      const int64_t k0 = kv_offsets[b], Lk = kv_offsets[b + 1] - k0;
      for (int64_t i = 0; i < Lq; ++i) {
        row_scores(p, q, k, bias, h, q0 + i, k0, i, Lk, s, vis);
        row_probs(p, s, vis, Lk, pr);
        const double* doi = dout + ((q0 + i) * H + h) * D;
        const double* qi = q + ((q0 + i) * H + h) * D;
        double delta = 0.0;
        for (int64_t j = 0; j < Lk; ++j) {
          dp[j] = 0.0;
          if (!vis[j]) continue;
          const double* vj = v + ((k0 + j) * H + h) * D;
          for (int d = 0; d < D; ++d) dp[j] += doi[d] * vj[d];
          delta += pr[j] * dp[j];
        }
        for (int64_t j = 0; j < Lk; ++j) {
          if (!vis[j]) { ds[j] = 0.0; continue; }
          if (p->phi == ORACLE_PHI_SOFTMAX) {
            ds[j] = pr[j] * (dp[j] - delta);
          } else if (p->phi == ORACLE_PHI_SILU) {
            double sg = sigmoid(s[j]);
            ds[j] = dp[j] * (sg + s[j] * sg * (1.0 - sg));
          } else if (p->phi == ORACLE_PHI_GELU) {
            ds[j] = dp[j] * (normal_cdf(s[j]) + s[j] * normal_pdf(s[j]));
          } else {
            ds[j] = dp[j];
          }
        }
        double* dqi = dq + ((q0 + i) * H + h) * D;
        for (int64_t j = 0; j < Lk; ++j) {
          if (!vis[j]) continue;
          const double* kj = k + ((k0 + j) * H + h) * D;
          double* dkj = dk + ((k0 + j) * H + h) * D;
          double* dvj = dv + ((k0 + j) * H + h) * D;
          for (int d = 0; d < D; ++d) {
            dvj[d] += pr[j] * doi[d];
            dqi[d] += p->scale * ds[j] * kj[d];
            dkj[d] += p->scale * ds[j] * qi[d];
          }
          if (dbias && p->bias_kind != ORACLE_BIAS_NONE) {
            double g = bias[(int64_t)h * p->total_kv + k0 + j];
            double w = p->bias_kind == ORACLE_BIAS_ADD ? 1.0 : 1.0 - sigmoid(g);
            dbias[(int64_t)h * p->total_kv + k0 + j] += ds[j] * w;
          }
        }
      }
    }
    free(s);
    free(pr);
    free(dp);
    free(ds);
    free(vis);
  }
  return err;
}

int gdpa_oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
