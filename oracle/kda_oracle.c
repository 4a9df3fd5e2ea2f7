/*
 * kda_oracle.c -- plain fp64 CPU oracle for chunked Kimi Delta Attention (KDA) prefill.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code, header or
 * constant with the CUDA library; the product path never calls it.
 *
 * Everything is fp64, row-major, one (sequence, value-head) unit at a time:
 *   q, k : [L][Dk]    v : [L][Dv]    g : [L][Dk] (already-activated natural-log decay)
 *   beta : [L]        S0, S : [Dv][Dk] (state, rows = value dim, cols = key dim)
 *   out  : [L][Dv]
 *
 * Sources (pages on the subject):
 *  - "FlashKDA" README (CANNBot-DSL samples/flash_kda), section 功能说明: the chunk
 *    equations gamma_t = exp(sum_{i<=t} g_i), K~ = gamma*K, K- = gamma^-1*K,
 *    Q~ = scale*(gamma*Q), T = stril(diag(beta) K~ K-^T), A^-1 = (I+T)^-1,
 *    U = A^-1 diag(beta) V, W = A^-1 diag(beta) K~, then the inter-chunk state pass.
 *  - Same README, parameter table (参数说明): raw q/k are L2-normalised in the op,
 *    beta arrives as logits (sigmoid in the op), the gate is activated from A_log
 *    (per value head), dt_bias [Nv, D] and lower_bound in [-5, 0]; state is [Dv, Dk].
 *  - vLLM PR 43195 summary ("KDA chunk prefill decay uses exp2"), 功能与动机: the KDA
 *    recurrence decays the state as state *= exp(g).
 *  - FLA PR 656 "[kda] add recursive block intra", review of chunk_intra.py: the
 *    intra-chunk q.k matrix keeps its diagonal (row >= col) while the k.k matrix is
 *    strictly lower (row > col) and beta-scaled.
 *
 * Readings where the pages are silent:
 *  - gate:  g = lower_bound * sigmoid(exp(A_log) * (g_raw + dt_bias))   [parity unpinned:
 *           the pages name the inputs and the bound, not the formula]
 *  - L2 normalise: x / sqrt(sum x^2 + 1e-6)
 *  - the per-token recurrence, with decay applied before the delta-rule update:
 *           S_t = S_{t-1} Diag(exp(g_t)) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *           o_t = scale * S_t q_t
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

/* sigmoid(x) = 1 / (1 + e^-x) */
static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* Gate activation (FlashKDA README, 参数说明: the raw gate is activated from A_log, dt_bias and
 * lower_bound; the formula itself is the reading documented in the module header).
 * graw: [n][D], dt_bias: [D], out g: [n][D]. */
void kda_oracle_gate(int n, int D, const double* graw, const double* dt_bias, double A_log,
                     double lower_bound, double* g) {
  const double a = exp(A_log);
  for (int t = 0; t < n; ++t)
    for (int d = 0; d < D; ++d) {
      const double x = graw[(size_t)t * D + d] + dt_bias[d];
      g[(size_t)t * D + d] = lower_bound * sigmoid(a * x);
    }
}

/* beta = sigmoid(logit) (FlashKDA parameter table: beta arrives as write logits). */
void kda_oracle_beta(int n, const double* logit, double* beta) {
  for (int t = 0; t < n; ++t)
    beta[t] = sigmoid(logit[t]);
}

/* Row-wise L2 normalise, y = x / sqrt(sum x^2 + eps) (FlashKDA: in-op q/k normalise). */
void kda_oracle_l2norm(int n, int D, const double* x, double eps, double* y) {
  for (int t = 0; t < n; ++t) {
    double ss = 0.0;
    for (int d = 0; d < D; ++d) ss += x[(size_t)t * D + d] * x[(size_t)t * D + d];
    const double inv = 1.0 / sqrt(ss + eps);
    for (int d = 0; d < D; ++d) y[(size_t)t * D + d] = x[(size_t)t * D + d] * inv;
  }
}

/* Token-by-token recurrence: the definition of the method. */
void kda_oracle_recurrent(int L, int Dk, int Dv, const double* q, const double* k,
                          const double* v, const double* g, const double* beta, double scale,
                          const double* S0, double* out, double* S) {
  double* decay = (double*)malloc(sizeof(double) * Dk);
  double* pred = (double*)malloc(sizeof(double) * Dv);
  memcpy(S, S0, sizeof(double) * (size_t)Dv * Dk);
  for (int t = 0; t < L; ++t) {
    const double* kt = k + (size_t)t * Dk;
    const double* qt = q + (size_t)t * Dk;
    const double* vt = v + (size_t)t * Dv;
    /* S <- S Diag(exp(g_t)) */
    for (int j = 0; j < Dk; ++j) decay[j] = exp(g[(size_t)t * Dk + j]);
    for (int i = 0; i < Dv; ++i)
      for (int j = 0; j < Dk; ++j) S[(size_t)i * Dk + j] *= decay[j];
    /* S <- S (I - beta k k^T) + beta v k^T  ==  S + beta (v - S k) k^T */
    for (int i = 0; i < Dv; ++i) {
      double acc = 0.0;
      for (int j = 0; j < Dk; ++j) acc += S[(size_t)i * Dk + j] * kt[j];
      pred[i] = acc;
    }
    for (int i = 0; i < Dv; ++i) {
      const double c = beta[t] * (vt[i] - pred[i]);
      for (int j = 0; j < Dk; ++j) S[(size_t)i * Dk + j] += c * kt[j];
    }
    /* o_t = scale * S_t q_t */
    for (int i = 0; i < Dv; ++i) {
      double acc = 0.0;
      for (int j = 0; j < Dk; ++j) acc += S[(size_t)i * Dk + j] * qt[j];
      out[(size_t)t * Dv + i] = scale * acc;
    }
  }
  free(decay);
  free(pred);
}

/* X = (I + T)^-1 for strictly lower-triangular T [n][n], by forward substitution. */
void kda_oracle_unit_lower_inverse(int n, const double* T, double* X) {
  memset(X, 0, sizeof(double) * (size_t)n * n);
  for (int c = 0; c < n; ++c) {
    X[(size_t)c * n + c] = 1.0;
    for (int r = c + 1; r < n; ++r) {
      double acc = 0.0;
      for (int s = c; s < r; ++s)
        acc += T[(size_t)r * n + s] * X[(size_t)s * n + c];
      X[(size_t)r * n + c] = -acc;
    }
  }
}

/* Chunked (WY / UT) form with chunk size C, following the FlashKDA chunk equations.
 * Within a chunk of n rows, with G the inclusive cumulative sum of g and gamma = exp(G):
 *   K~ = gamma*K, K- = K/gamma, Q~ = scale*gamma*Q,
 *   T = stril(diag(beta) K~ K-^T), A^-1 = (I+T)^-1, U = A^-1 diag(beta) V, W = A^-1 diag(beta) K~,
 *   Delta = U - W S0^T,  O = Q~ S0^T + tril(Q~ K-^T) Delta,
 *   S_next = S0 Diag(gamma_last) + Delta^T (K- Diag(gamma_last)).
 * The inter-chunk pass is not printed on the page; the last three lines follow from
 * substituting S_r = (S0 + sum_{j<=r} delta_j k-_j^T) Diag(gamma_r) into the recurrence. */
void kda_oracle_chunked(int L, int Dk, int Dv, int C, const double* q, const double* k,
                        const double* v, const double* g, const double* beta, double scale,
                        const double* S0, double* out, double* S) {
  double* G = (double*)malloc(sizeof(double) * (size_t)C * Dk);
  double* Kt = (double*)malloc(sizeof(double) * (size_t)C * Dk);
  double* Kb = (double*)malloc(sizeof(double) * (size_t)C * Dk);
  double* Qt = (double*)malloc(sizeof(double) * (size_t)C * Dk);
  double* T = (double*)malloc(sizeof(double) * (size_t)C * C);
  double* Ai = (double*)malloc(sizeof(double) * (size_t)C * C);
  double* Aqk = (double*)malloc(sizeof(double) * (size_t)C * C);
  double* U = (double*)malloc(sizeof(double) * (size_t)C * Dv);
  double* W = (double*)malloc(sizeof(double) * (size_t)C * Dk);
  double* Dl = (double*)malloc(sizeof(double) * (size_t)C * Dv);
  double* Sn = (double*)malloc(sizeof(double) * (size_t)Dv * Dk);
  memcpy(S, S0, sizeof(double) * (size_t)Dv * Dk);

  for (int c0 = 0; c0 < L; c0 += C) {
    const int n = (L - c0 < C) ? (L - c0) : C;
    /* G = inclusive cumulative sum of g inside the chunk; gamma = exp(G). */
    for (int j = 0; j < Dk; ++j) {
      double acc = 0.0;
      for (int r = 0; r < n; ++r) {
        acc += g[(size_t)(c0 + r) * Dk + j];
        G[(size_t)r * Dk + j] = acc;
      }
    }
    for (int r = 0; r < n; ++r)
      for (int j = 0; j < Dk; ++j) {
        const double gm = exp(G[(size_t)r * Dk + j]);
        Kt[(size_t)r * Dk + j] = gm * k[(size_t)(c0 + r) * Dk + j];
        Kb[(size_t)r * Dk + j] = k[(size_t)(c0 + r) * Dk + j] / gm;
        Qt[(size_t)r * Dk + j] = scale * gm * q[(size_t)(c0 + r) * Dk + j];
      }
    /* T = stril(diag(beta) K~ K-^T);  Aqk = tril(Q~ K-^T) (diagonal kept). */
    for (int r = 0; r < n; ++r)
      for (int s = 0; s < n; ++s) {
        double tk = 0.0, tq = 0.0;
        for (int j = 0; j < Dk; ++j) {
          tk += Kt[(size_t)r * Dk + j] * Kb[(size_t)s * Dk + j];
          tq += Qt[(size_t)r * Dk + j] * Kb[(size_t)s * Dk + j];
        }
        T[(size_t)r * n + s] = (s < r) ? beta[c0 + r] * tk : 0.0;
        Aqk[(size_t)r * n + s] = (s <= r) ? tq : 0.0;
      }
    kda_oracle_unit_lower_inverse(n, T, Ai);
    /* U = A^-1 diag(beta) V,  W = A^-1 diag(beta) K~ */
    for (int r = 0; r < n; ++r) {
      for (int i = 0; i < Dv; ++i) {
        double acc = 0.0;
        for (int s = 0; s < n; ++s)
          acc += Ai[(size_t)r * n + s] * beta[c0 + s] * v[(size_t)(c0 + s) * Dv + i];
        U[(size_t)r * Dv + i] = acc;
      }
      for (int j = 0; j < Dk; ++j) {
        double acc = 0.0;
        for (int s = 0; s < n; ++s)
          acc += Ai[(size_t)r * n + s] * beta[c0 + s] * Kt[(size_t)s * Dk + j];
        W[(size_t)r * Dk + j] = acc;
      }
    }
    /* Delta = U - W S0^T */
    for (int r = 0; r < n; ++r)
      for (int i = 0; i < Dv; ++i) {
        double acc = 0.0;
        for (int j = 0; j < Dk; ++j) acc += W[(size_t)r * Dk + j] * S[(size_t)i * Dk + j];
        Dl[(size_t)r * Dv + i] = U[(size_t)r * Dv + i] - acc;
      }
    /* O = Q~ S0^T + tril(Q~ K-^T) Delta */
    for (int r = 0; r < n; ++r)
      for (int i = 0; i < Dv; ++i) {
        double acc = 0.0;
        for (int j = 0; j < Dk; ++j) acc += Qt[(size_t)r * Dk + j] * S[(size_t)i * Dk + j];
        for (int s = 0; s < n; ++s) acc += Aqk[(size_t)r * n + s] * Dl[(size_t)s * Dv + i];
        out[(size_t)(c0 + r) * Dv + i] = acc;
      }
    /* S_next = S0 Diag(gamma_last) + Delta^T (K- Diag(gamma_last)) */
    for (int i = 0; i < Dv; ++i)
      for (int j = 0; j < Dk; ++j) {
        const double gl = exp(G[(size_t)(n - 1) * Dk + j]);
        double acc = 0.0;
        for (int r = 0; r < n; ++r) acc += Dl[(size_t)r * Dv + i] * Kb[(size_t)r * Dk + j];
        Sn[(size_t)i * Dk + j] = S[(size_t)i * Dk + j] * gl + acc * gl;
      }
    memcpy(S, Sn, sizeof(double) * (size_t)Dv * Dk);
  }
  free(G); free(Kt); free(Kb); free(Qt); free(T); free(Ai); free(Aqk);
  free(U); free(W); free(Dl); free(Sn);
}

/* One whole unit from raw (bf16-widened) inputs: activations, normalise, then the
 * recurrence (form 0) or the chunked form with chunk size C (form 1). */
void kda_oracle_unit(int form, int C, int L, int Dk, int Dv, const double* q_raw,
                     const double* k_raw, const double* v, const double* g_raw,
                     const double* beta_logit, const double* dt_bias, double A_log,
                     double lower_bound, double scale, const double* S0, double* out,
                     double* S) {
  double* qn = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * Dk);
  double* kn = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * Dk);
  double* g = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * Dk);
  double* beta = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
  kda_oracle_l2norm(L, Dk, q_raw, 1e-6, qn);
  kda_oracle_l2norm(L, Dk, k_raw, 1e-6, kn);
  kda_oracle_gate(L, Dk, g_raw, dt_bias, A_log, lower_bound, g);
  kda_oracle_beta(L, beta_logit, beta);
  if (form == 0)
    kda_oracle_recurrent(L, Dk, Dv, qn, kn, v, g, beta, scale, S0, out, S);
  else
    kda_oracle_chunked(L, Dk, Dv, C, qn, kn, v, g, beta, scale, S0, out, S);
  free(qn); free(kn); free(g); free(beta);
}
