/*
 * Agent Attention forward pass -- plain fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file; only the tests, the package's smoke check and the CPU
 * baseline leg of the benchmark use it.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * What it computes (per batch*head slice "bh"), written as the plain
 * definition, with no blocking, fusion or reordering:
 *
 *   agents   A = adaptive average pool of Q over its grid_h x grid_w token
 *              grid down to pool_h x pool_w agents.
 *              [Agent Attention: On the Integration of Softmax and Linear
 *               Attention (arXiv:2312.08874v3 summary), §4 "Efficiency":
 *               agents from pooling is the default; §6 Conclusion: A = f(Q).]
 *              Bin i along an axis of length G cut into P bins covers
 *              [floor(i*G/P), ceil((i+1)*G/P)); the divisor is the number of
 *              tokens in the bin (the usual adaptive-pool convention, the
 *              plainest reading of "pooling").
 *   aggregate V_A = softmax(A K^T * scale) V        (k x d)
 *   broadcast O   = softmax(Q A^T * scale) V_A      (N x d)
 *              [Agent Attention：Transformer计算量太大？试试这个'代理令牌'的
 *               轻量化方案 (jsqmd.com), §1, two-stage pseudocode: stage one
 *               aggregates K/V into the agents, stage two lets the queries
 *               read the agents, both softmaxes scaled by 1/sqrt(d);
 *               arXiv:2312.08874v3 summary §4 "Agent Attention": agent
 *               aggregation followed by agent broadcast.]
 *
 * Softmax is evaluated as exp(x - max) / sum exp(x - max), two passes per
 * row, in double precision.  Tokens are row-major on the grid
 * (n = y*grid_w + x); agent j = py*pool_w + px.
 *
 * All arrays are contiguous, row-major, double precision:
 *   q, k, v, o   [BH][N][d]
 *   a, va        [BH][n_agents][d]
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* start/end of adaptive bin i when an axis of length g is cut into p bins */
static int64_t bin_start(int64_t i, int64_t g, int64_t p) { return (i * g) / p; }
static int64_t bin_end(int64_t i, int64_t g, int64_t p) { return ((i + 1) * g + p - 1) / p; }

void oracle_agent_pool(const double* q, int64_t BH, int64_t N, int64_t d,
                       int64_t grid_h, int64_t grid_w, int64_t pool_h, int64_t pool_w,
                       double* a) {
  (void)N;
  int64_t n_agents = pool_h * pool_w;
#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t bh = 0; bh < BH; ++bh) {
    for (int64_t j = 0; j < n_agents; ++j) {
      int64_t py = j / pool_w, px = j % pool_w;
      int64_t y0 = bin_start(py, grid_h, pool_h), y1 = bin_end(py, grid_h, pool_h);
      int64_t x0 = bin_start(px, grid_w, pool_w), x1 = bin_end(px, grid_w, pool_w);
      double* out = a + (bh * n_agents + j) * d;
      for (int64_t c = 0; c < d; ++c) out[c] = 0.0;
      for (int64_t y = y0; y < y1; ++y)
        for (int64_t x = x0; x < x1; ++x) {
          const double* row = q + (bh * N + y * grid_w + x) * d;
          for (int64_t c = 0; c < d; ++c) out[c] += row[c];
        }
      double count = (double)((y1 - y0) * (x1 - x0));
      for (int64_t c = 0; c < d; ++c) out[c] /= count;
    }
  }
}

/* out[row] = softmax(scale * <x_row, keys_n>)_n  @ vals, for one row x_row.
 * keys: [n_keys][d], vals: [n_keys][d].  work: n_keys doubles. */
static void softmax_attend_row(const double* x_row, const double* keys, const double* vals,
                               int64_t n_keys, int64_t d, double scale, double* work,
                               double* out) {
  double mx = -INFINITY;
  for (int64_t n = 0; n < n_keys; ++n) {
    double s = 0.0;
    for (int64_t c = 0; c < d; ++c) s += x_row[c] * keys[n * d + c];
    s *= scale;
    work[n] = s;
    if (s > mx) mx = s;
  }
  double total = 0.0;
  for (int64_t n = 0; n < n_keys; ++n) {
    work[n] = exp(work[n] - mx);
    total += work[n];
  }
  for (int64_t c = 0; c < d; ++c) out[c] = 0.0;
  for (int64_t n = 0; n < n_keys; ++n) {
    double p = work[n] / total;
    for (int64_t c = 0; c < d; ++c) out[c] += p * vals[n * d + c];
  }
}

/* Agent aggregation: va[bh][j] = softmax_n(scale * A_j . K_n) @ V. */
void oracle_agent_aggregate(const double* a, const double* k, const double* v, int64_t BH,
                            int64_t N, int64_t d, int64_t n_agents, double scale, double* va) {
#pragma omp parallel
  {
    double* work = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
#pragma omp for collapse(2) schedule(dynamic, 1)
    for (int64_t bh = 0; bh < BH; ++bh)
      for (int64_t j = 0; j < n_agents; ++j)
        softmax_attend_row(a + (bh * n_agents + j) * d, k + bh * N * d, v + bh * N * d, N, d,
                           scale, work, va + (bh * n_agents + j) * d);
    free(work);
  }
}

/* Agent broadcast: o[bh][i] = softmax_j(scale * Q_i . A_j) @ V_A. */
void oracle_agent_broadcast(const double* q, const double* a, const double* va, int64_t BH,
                            int64_t N, int64_t d, int64_t n_agents, double scale, double* o) {
#pragma omp parallel
  {
    double* work = (double*)malloc(sizeof(double) * (size_t)(n_agents > 0 ? n_agents : 1));
#pragma omp for collapse(2) schedule(static)
    for (int64_t bh = 0; bh < BH; ++bh)
      for (int64_t i = 0; i < N; ++i)
        softmax_attend_row(q + (bh * N + i) * d, a + bh * n_agents * d, va + bh * n_agents * d,
                           n_agents, d, scale, work, o + (bh * N + i) * d);
    free(work);
  }
}

/* Whole forward pass.  If agents_or_null is NULL the agents are pooled from Q
 * (pool_h x pool_w of them); otherwise agents_or_null is [BH][n_agents][d]
 * (learnable agents, already expanded over the batch by the caller).
 * scratch_a and scratch_va must hold BH*n_agents*d doubles each. */
void oracle_agent_attn(const double* q, const double* k, const double* v,
                       const double* agents_or_null, int64_t BH, int64_t N, int64_t d,
                       int64_t grid_h, int64_t grid_w, int64_t pool_h, int64_t pool_w,
                       int64_t n_agents, double scale, double* scratch_a, double* scratch_va,
                       double* o) {
  const double* a = agents_or_null;
  if (a == NULL) {
    oracle_agent_pool(q, BH, N, d, grid_h, grid_w, pool_h, pool_w, scratch_a);
    a = scratch_a;
  }
  oracle_agent_aggregate(a, k, v, BH, N, d, n_agents, scale, scratch_va);
  oracle_agent_broadcast(q, a, scratch_va, BH, N, d, n_agents, scale, o);
}

/* Agent bias: the logits of both softmaxes get an additive bias.
 * [Agent Attention: On the Integration of Softmax and Linear Attention
 *  (arXiv:2312.08874v3 summary), §4 "Module Enhancements": the bias terms B1
 *  and B2 are incorporated into both attention operations; §6
 *  "Implementation Details": column, row and block components build the
 *  full bias.]
 *   aggregate: V_A[j] = softmax_n(scale * A_j . K_n + b1[h][j][n]) @ V
 *   broadcast: O[i]   = softmax_j(scale * Q_i . A_j + b2[h][j][i]) @ V_A
 * b1, b2: [H][n_agents][N] full bias matrices shared over the batch
 * (h = bh % H), either may be NULL for no bias.  How the full matrices are
 * built from their components is the caller's (oracle/__init__.py). */
static void softmax_attend_row_biased(const double* x_row, const double* keys,
                                      const double* vals, int64_t n_keys, int64_t d,
                                      double scale, const double* bias, int64_t bias_stride,
                                      double* work, double* out) {
  double mx = -INFINITY;
  for (int64_t n = 0; n < n_keys; ++n) {
    double s = 0.0;
    for (int64_t c = 0; c < d; ++c) s += x_row[c] * keys[n * d + c];
    s = s * scale + (bias ? bias[n * bias_stride] : 0.0);
    work[n] = s;
    if (s > mx) mx = s;
  }
  double total = 0.0;
  for (int64_t n = 0; n < n_keys; ++n) {
    work[n] = exp(work[n] - mx);
    total += work[n];
  }
  for (int64_t c = 0; c < d; ++c) out[c] = 0.0;
  for (int64_t n = 0; n < n_keys; ++n) {
    double p = work[n] / total;
    for (int64_t c = 0; c < d; ++c) out[c] += p * vals[n * d + c];
  }
}

void oracle_agent_attn_bias(const double* q, const double* k, const double* v,
                            const double* agents_or_null, const double* b1, const double* b2,
                            int64_t BH, int64_t H, int64_t N, int64_t d, int64_t grid_h,
                            int64_t grid_w, int64_t pool_h, int64_t pool_w, int64_t n_agents,
                            double scale, double* scratch_a, double* scratch_va, double* o) {
  const double* a = agents_or_null;
  if (a == NULL) {
    oracle_agent_pool(q, BH, N, d, grid_h, grid_w, pool_h, pool_w, scratch_a);
    a = scratch_a;
  }
#pragma omp parallel
  {
    double* work = (double*)malloc(sizeof(double) * (size_t)(N > n_agents ? N : n_agents));
#pragma omp for collapse(2) schedule(dynamic, 1)
    for (int64_t bh = 0; bh < BH; ++bh)
      for (int64_t j = 0; j < n_agents; ++j)
        softmax_attend_row_biased(a + (bh * n_agents + j) * d, k + bh * N * d, v + bh * N * d, N,
                                  d, scale, b1 ? b1 + ((bh % H) * n_agents + j) * N : NULL, 1,
                                  work, scratch_va + (bh * n_agents + j) * d);
#pragma omp for collapse(2) schedule(static)
    for (int64_t bh = 0; bh < BH; ++bh)
      for (int64_t i = 0; i < N; ++i)
        softmax_attend_row_biased(q + (bh * N + i) * d, a + bh * n_agents * d,
                                  scratch_va + bh * n_agents * d, n_agents, d, scale,
                                  b2 ? b2 + (bh % H) * n_agents * N + i : NULL, N, work,
                                  o + (bh * N + i) * d);
    free(work);
  }
}

/* Depth-wise 3x3 convolution of V over its token grid: the DWC term that the
 * full module adds to the attention output.
 * [Agent Attention: On the Integration of Softmax and Linear Attention
 *  (arXiv:2312.08874v3 summary), §4 "Module Enhancements": the full module
 *  adds a depth-wise convolution term whose cost is k^2 N C with k = 3.]
 * Each channel c of each head h has its own 3x3 kernel w[h][c][ty][tx] and an
 * optional bias[h][c]; positions outside the grid contribute zero (padding 1,
 * stride 1, so the output keeps the grid):
 *   out[bh][y*gw + x][c] = bias[h][c]
 *       + sum_{ty,tx in 0..2} w[h][c][ty][tx] * V[bh][(y+ty-1)*gw + (x+tx-1)][c]
 * with h = bh % H.  v, out: [BH][grid_h*grid_w][d]; w: [H][d][3][3];
 * bias_or_null: [H][d] or NULL. */
void oracle_dwc(const double* v, const double* w, const double* bias_or_null, int64_t BH,
                int64_t H, int64_t grid_h, int64_t grid_w, int64_t d, double* out) {
  const int64_t N = grid_h * grid_w;
#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t bh = 0; bh < BH; ++bh) {
    for (int64_t n = 0; n < N; ++n) {
      const int64_t h = bh % H, y = n / grid_w, x = n % grid_w;
      for (int64_t c = 0; c < d; ++c) {
        double acc = bias_or_null ? bias_or_null[h * d + c] : 0.0;
        for (int64_t ty = 0; ty < 3; ++ty) {
          for (int64_t tx = 0; tx < 3; ++tx) {
            const int64_t yy = y + ty - 1, xx = x + tx - 1;
            if (yy < 0 || yy >= grid_h || xx < 0 || xx >= grid_w) continue;
            acc += w[(h * d + c) * 9 + ty * 3 + tx] * v[(bh * N + yy * grid_w + xx) * d + c];
          }
        }
        out[(bh * N + n) * d + c] = acc;
      }
    }
  }
}

/* Backward pass of the forward pass above (pooled or given agents), for
 * finetuning.  [arXiv:2312.08874v3 summary, C.4 "AgentSD for finetuning":
 * agent attention is used during DreamBooth finetuning, i.e. gradients flow
 * through both softmax stages.]  The pages give no formulas; these are the
 * derivatives of the definition, written per stage:
 *   P1 = softmax_rows(s A K^T)  (k x N),  V_A = P1 V
 *   P2 = softmax_rows(s Q A^T)  (N x k),  O   = P2 V_A
 * given dO:
 *   dV_A = P2^T dO;  dP2 = dO V_A^T;  dS2 = P2 .* (dP2 - rowsum(dP2 .* P2))
 *   dQ  = s dS2 A;   dA  = s dS2^T Q
 *   dV  = P1^T dV_A; dP1 = dV_A V^T;  dS1 = P1 .* (dP1 - rowsum(dP1 .* P1))
 *   dK  = s dS1^T A; dA += s dS1 K
 *   pooled agents: dQ[n] += sum over the bins j holding token n of dA[j] / |bin j|
 * Outputs dq, dk, dv [BH][N][d]; dagents [BH][n_agents][d] (the gradient of
 * the agents themselves, before the pooling adjoint; may be NULL). */
void oracle_agent_attn_backward(const double* q, const double* k, const double* v,
                                const double* agents_or_null, const double* dout, int64_t BH,
                                int64_t N, int64_t d, int64_t grid_h, int64_t grid_w,
                                int64_t pool_h, int64_t pool_w, int64_t n_agents, double scale,
                                double* dq, double* dk, double* dv, double* dagents) {
  const int64_t K_ = n_agents;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t bh = 0; bh < BH; ++bh) {
    const double* Q = q + bh * N * d;
    const double* Kt = k + bh * N * d;
    const double* V = v + bh * N * d;
    const double* dO = dout + bh * N * d;
    double* A = (double*)malloc(sizeof(double) * (size_t)(K_ * d));
    double* VA = (double*)calloc((size_t)(K_ * d), sizeof(double));
    double* P1 = (double*)malloc(sizeof(double) * (size_t)(K_ * N));
    double* P2 = (double*)malloc(sizeof(double) * (size_t)(N * K_));
    double* dVA = (double*)calloc((size_t)(K_ * d), sizeof(double));
    double* dA = (double*)calloc((size_t)(K_ * d), sizeof(double));
    double* dS = (double*)malloc(sizeof(double) * (size_t)(N > K_ ? N : K_));
    if (agents_or_null) {
      for (int64_t i = 0; i < K_ * d; ++i) A[i] = agents_or_null[bh * K_ * d + i];
    } else {
      oracle_agent_pool(Q, 1, N, d, grid_h, grid_w, pool_h, pool_w, A);
    }
    /* forward: P1, V_A, P2 */
    for (int64_t j = 0; j < K_; ++j) {
      double mx = -INFINITY, tot = 0.0;
      for (int64_t n = 0; n < N; ++n) {
        double z = 0.0;
        for (int64_t c = 0; c < d; ++c) z += A[j * d + c] * Kt[n * d + c];
        P1[j * N + n] = z * scale;
        if (P1[j * N + n] > mx) mx = P1[j * N + n];
      }
      for (int64_t n = 0; n < N; ++n) tot += (P1[j * N + n] = exp(P1[j * N + n] - mx));
      for (int64_t n = 0; n < N; ++n) {
        P1[j * N + n] /= tot;
        for (int64_t c = 0; c < d; ++c) VA[j * d + c] += P1[j * N + n] * V[n * d + c];
      }
    }
    for (int64_t i = 0; i < N; ++i) {
      double mx = -INFINITY, tot = 0.0;
      for (int64_t j = 0; j < K_; ++j) {
        double t = 0.0;
        for (int64_t c = 0; c < d; ++c) t += Q[i * d + c] * A[j * d + c];
        P2[i * K_ + j] = t * scale;
        if (P2[i * K_ + j] > mx) mx = P2[i * K_ + j];
      }
      for (int64_t j = 0; j < K_; ++j) tot += (P2[i * K_ + j] = exp(P2[i * K_ + j] - mx));
      for (int64_t j = 0; j < K_; ++j) P2[i * K_ + j] /= tot;
    }
    /* broadcast stage */
    double* dQs = dq + bh * N * d;
    for (int64_t i = 0; i < N * d; ++i) dQs[i] = 0.0;
    for (int64_t i = 0; i < N; ++i) {
      double dot = 0.0;
      for (int64_t j = 0; j < K_; ++j) {
        double dp = 0.0;
        for (int64_t c = 0; c < d; ++c) dp += dO[i * d + c] * VA[j * d + c];
        dS[j] = dp;
        dot += dp * P2[i * K_ + j];
      }
      for (int64_t j = 0; j < K_; ++j) {
        const double p = P2[i * K_ + j];
        const double ds = p * (dS[j] - dot);
        for (int64_t c = 0; c < d; ++c) {
          dVA[j * d + c] += p * dO[i * d + c];
          dQs[i * d + c] += scale * ds * A[j * d + c];
          dA[j * d + c] += scale * ds * Q[i * d + c];
        }
      }
    }
    /* aggregation stage */
    double* dKs = dk + bh * N * d;
    double* dVs = dv + bh * N * d;
    for (int64_t i = 0; i < N * d; ++i) dKs[i] = dVs[i] = 0.0;
    for (int64_t j = 0; j < K_; ++j) {
      double dot = 0.0;
      for (int64_t n = 0; n < N; ++n) {
        double dp = 0.0;
        for (int64_t c = 0; c < d; ++c) dp += dVA[j * d + c] * V[n * d + c];
        dS[n] = dp;
        dot += dp * P1[j * N + n];
      }
      for (int64_t n = 0; n < N; ++n) {
        const double p = P1[j * N + n];
        const double ds = p * (dS[n] - dot);
        for (int64_t c = 0; c < d; ++c) {
          dVs[n * d + c] += p * dVA[j * d + c];
          dKs[n * d + c] += scale * ds * A[j * d + c];
          dA[j * d + c] += scale * ds * Kt[n * d + c];
        }
      }
    }
    if (dagents)
      for (int64_t i = 0; i < K_ * d; ++i) dagents[bh * K_ * d + i] = dA[i];
    /* pooling adjoint: each token of bin j receives dA[j] / |bin j| */
    if (!agents_or_null) {
      for (int64_t j = 0; j < K_; ++j) {
        const int64_t py = j / pool_w, px = j % pool_w;
        const int64_t y0 = bin_start(py, grid_h, pool_h), y1 = bin_end(py, grid_h, pool_h);
        const int64_t x0 = bin_start(px, grid_w, pool_w), x1 = bin_end(px, grid_w, pool_w);
        const double inv = 1.0 / (double)((y1 - y0) * (x1 - x0));
        for (int64_t y = y0; y < y1; ++y)
          for (int64_t x = x0; x < x1; ++x)
            for (int64_t c = 0; c < d; ++c)
              dQs[(y * grid_w + x) * d + c] += dA[j * d + c] * inv;
      }
    }
    free(A); free(VA); free(P1); free(P2); free(dVA); free(dA); free(dS);
  }
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
