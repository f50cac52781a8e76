/*
 * mhc_oracle.c -- plain fp64 CPU oracle for the mHC (manifold-constrained
 * hyper-connection) layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file; it exists so that the CUDA kernels can be checked against an
 * obviously correct, unfused, unreordered statement of the method.  Only the
 * tests, the package's smoke check and the CPU-baseline leg of the benchmark
 * load it.
 *
 * Every quantity is computed in double precision, per token, in the order the
 * method states it, with no blocking, fusion or reordering:
 *
 *   sources (web pages on mHC, by title and section):
 *   [P1]  chatgpz.de feed "DeepSeek-Forscher ..." -- sections
 *         "Von Residualverbindungen zu Hyperverbindungen" (the n-stream buffer,
 *         the three mappings, the update X_{l+1} = H_res X_l +
 *         H_post^T F(H_pre X_l)), "Vielfaeltig eingeschraenkte
 *         Hyperverbindungen" (H_res projected onto the doubly stochastic
 *         matrices by Sinkhorn-Knopp, 20 iterations; non-negative input and
 *         output maps), "Warum Hyperverbindungen instabil werden" (Amax gain
 *         from the maximum row and column sums of the composite map).
 *   [P5]  reportify.cn summary, paragraphs [10], [12], [15]-[21]
 *         (doubly stochastic constraint, non-negative maps, t_max = 20,
 *         fused RMSNorm/projection/gating, custom Sinkhorn backward,
 *         recompute of the mapping in the backward pass).
 *   The dynamic-mapping parameterisation (RMS normalisation of the flattened
 *   n*C stream, projection phi, scale alpha, bias b, H_pre = sigmoid,
 *   H_post = 2*sigmoid, H_res = Sinkhorn(exp(.))) is the problem statement
 *   this library implements; the pages only name "RMSNorm, projections and
 *   gating".
 *
 * Readings fixed here (the pages are silent on them):
 *   - flattening of a token's stream buffer: k = i*C + c (stream i, channel c);
 *   - logit column order: [pre 0..n-1 | post n..2n-1 | res 2n + i*n + j];
 *   - H_res[i][j] weights stream j into output stream i;
 *   - r = sqrt(mean_k x_k^2 + eps) over all n*C entries, no learnable gain;
 *   - one Sinkhorn iteration = normalise every row, then every column;
 *     M0 = exp(logits) exactly (no shift; fp64 range covers every input used);
 *   - Amax gain of P = H_L ... H_1 (layer 1 applied first):
 *     forward gain = max_i sum_j |P_ij|, backward gain = max_j sum_i |P_ij|.
 *
 * Layouts (row-major, C fastest):
 *   x, grad_x_next (G), grad_x : [T][n][C]      f_out, grad_h_in (g), h_in : [T][C]
 *   phi, grad_phi : [n*C][n*n+2n]   b, grad_b : [n*n+2n]
 *   H_pre, H_post : [T][n]          H_res : [T][n][n]
 *   red (the post half's reductions, backward in training order):
 *                   [T][n*n + n] = <G_i, x_j> (row-major i, j) then <G_i, f_out>
 *
 * Parity pins (tests/test_oracle_pins.py, fixtures in tests/golden/):
 * hand-worked and closed-form Sinkhorn cases, diagonal-scaling and
 * permutation invariants, the gate and RMS special cases, the standard
 * residual at n = 1, finite differences of every backward gradient (the whole
 * backward, the post half, and per-group alpha), three equal group scales
 * against one shared alpha, the split backward against the one-call backward,
 * and a hand-multiplied 2 x 2 depth product for the Amax gains.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double orc_sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }

/* Scale group of logit m: 0 = pre (m < n), 1 = post (m < 2n), 2 = res.
 * alpha is always passed as [alpha_pre, alpha_post, alpha_res]; one shared
 * alpha is the case of three equal entries. */
static int orc_group(int n, int m) { return m < n ? 0 : (m < 2 * n ? 1 : 2); }

/* Sinkhorn-Knopp [P1 "Vielfaeltig eingeschraenkte Hyperverbindungen";
 * P5 [10], [16]]: M0 = exp(logits), then `iters` times: divide each row by its
 * sum, then divide each column by its sum.  If `iterates` is non-NULL it
 * receives M0, M1, ..., M_{2*iters} (each n*n), the matrix after every single
 * normalisation, for the adjoint. */
static void orc_sk_forward(int n, int iters, const double *logits, double *out,
                           double *iterates) {
  const int nn = n * n;
  for (int e = 0; e < nn; ++e) out[e] = exp(logits[e]);
  if (iterates) memcpy(iterates, out, sizeof(double) * nn);
  for (int it = 0; it < iters; ++it) {
    for (int i = 0; i < n; ++i) {
      double s = 0.0;
      for (int j = 0; j < n; ++j) s += out[i * n + j];
      for (int j = 0; j < n; ++j) out[i * n + j] /= s;
    }
    if (iterates) memcpy(iterates + (size_t)(2 * it + 1) * nn, out, sizeof(double) * nn);
    for (int j = 0; j < n; ++j) {
      double s = 0.0;
      for (int i = 0; i < n; ++i) s += out[i * n + j];
      for (int i = 0; i < n; ++i) out[i * n + j] /= s;
    }
    if (iterates) memcpy(iterates + (size_t)(2 * it + 2) * nn, out, sizeof(double) * nn);
  }
}

/* Reverse mode of orc_sk_forward [P5 [19]: Sinkhorn iterations with their own
 * backward].  For a row normalisation A' = diag(1/s) A with s_i = sum_j A_ij:
 *   dA_ij = (dA'_ij - sum_l dA'_il A'_il) / s_i
 * and the transpose of that for a column normalisation.  At the start,
 * A0 = exp(z) so dz = dA0 * A0 elementwise.  `iterates` is as produced by
 * orc_sk_forward; dout is overwritten (used as scratch). */
static void orc_sk_backward(int n, int iters, const double *iterates, double *dout,
                            double *dlogits) {
  const int nn = n * n;
  double *dA = dout;
  for (int step = 2 * iters; step >= 1; --step) {
    const double *Ain = iterates + (size_t)(step - 1) * nn;   /* before the step */
    const double *Aout = iterates + (size_t)step * nn;        /* after the step */
    if (step % 2 == 1) { /* row normalisation */
      for (int i = 0; i < n; ++i) {
        double s = 0.0, d = 0.0;
        for (int j = 0; j < n; ++j) s += Ain[i * n + j];
        for (int j = 0; j < n; ++j) d += dA[i * n + j] * Aout[i * n + j];
        for (int j = 0; j < n; ++j) dA[i * n + j] = (dA[i * n + j] - d) / s;
      }
    } else { /* column normalisation */
      for (int j = 0; j < n; ++j) {
        double s = 0.0, d = 0.0;
        for (int i = 0; i < n; ++i) s += Ain[i * n + j];
        for (int i = 0; i < n; ++i) d += dA[i * n + j] * Aout[i * n + j];
        for (int i = 0; i < n; ++i) dA[i * n + j] = (dA[i * n + j] - d) / s;
      }
    }
  }
  for (int e = 0; e < nn; ++e) dlogits[e] = dA[e] * iterates[e];
}

/* Batched standalone Sinkhorn-Knopp: B independent n x n matrices. */
void orc_sinkhorn(int n, int iters, int64_t B, const double *logits, double *out) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < B; ++m)
    orc_sk_forward(n, iters, logits + m * n * n, out + m * n * n, NULL);
}

/* Reverse mode of the batched Sinkhorn-Knopp: dlogits = (d out / d logits)^T dout. */
void orc_sinkhorn_backward(int n, int iters, int64_t B, const double *logits,
                           const double *dout, double *dlogits) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < B; ++m) {
    const int nn = n * n;
    double *it = (double *)malloc(sizeof(double) * (size_t)(2 * iters + 1) * nn);
    double *tmp = (double *)malloc(sizeof(double) * (size_t)nn * 2);
    orc_sk_forward(n, iters, logits + m * nn, tmp, it);
    memcpy(tmp + nn, dout + m * nn, sizeof(double) * nn);
    orc_sk_backward(n, iters, it, tmp + nn, dlogits + m * nn);
    free(it);
    free(tmp);
  }
}

/* The dynamic mapping of one token: r, xhat = x / r, y = xhat . phi,
 * z = alpha * y + b.  The normalisation is applied first, as RMSNorm is
 * usually written. */
static void orc_logits(int n, int64_t C, double eps, const double *x, const double *phi,
                       const double *b, const double *alpha, double *r_out, double *y,
                       double *z) {
  const int64_t K = (int64_t)n * C;
  const int M = n * n + 2 * n;
  double ss = 0.0;
  for (int64_t k = 0; k < K; ++k) ss += x[k] * x[k];
  const double r = sqrt(ss / (double)K + eps);
  for (int m = 0; m < M; ++m) y[m] = 0.0;
  for (int64_t k = 0; k < K; ++k) {
    const double xh = x[k] / r;
    for (int m = 0; m < M; ++m) y[m] += xh * phi[k * M + m];
  }
  for (int m = 0; m < M; ++m) z[m] = alpha[orc_group(n, m)] * y[m] + b[m];
  *r_out = r;
}

/* Forward "pre" mapping for T tokens [P1 "Von Residualverbindungen zu
 * Hyperverbindungen"; P5 [12], [16]-[18]]:
 *   H_pre = sigmoid(z_pre), H_post = 2 sigmoid(z_post),
 *   H_res = Sinkhorn(exp(z_res)) with `iters` iterations,
 *   h_in[c] = sum_i H_pre[i] x[i][c].
 * z_out ([T][n*n+2n]) and r_out ([T]) may be NULL. */
void orc_pre(int n, int64_t T, int64_t C, int iters, double eps, const double *x,
             const double *phi, const double *b, const double *alpha, double *h_in, double *H_pre,
             double *H_post, double *H_res, double *z_out, double *r_out) {
  const int M = n * n + 2 * n;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    const double *xt = x + t * n * C;
    double y[16 * 16 + 32], z[16 * 16 + 32], r;
    orc_logits(n, C, eps, xt, phi, b, alpha, &r, y, z);
    for (int i = 0; i < n; ++i) {
      H_pre[t * n + i] = orc_sigmoid(z[i]);
      H_post[t * n + i] = 2.0 * orc_sigmoid(z[n + i]);
    }
    orc_sk_forward(n, iters, z + 2 * n, H_res + t * n * n, NULL);
    for (int64_t c = 0; c < C; ++c) {
      double acc = 0.0;
      for (int i = 0; i < n; ++i) acc += H_pre[t * n + i] * xt[i * C + c];
      h_in[t * C + c] = acc;
    }
    if (z_out) for (int m = 0; m < M; ++m) z_out[t * M + m] = z[m];
    if (r_out) r_out[t] = r;
  }
}

/* Post merge [P1 update equation; P5 [20]]:
 *   x_next[i][c] = sum_j H_res[i][j] x[j][c] + H_post[i] f_out[c]. */
void orc_post(int n, int64_t T, int64_t C, const double *x, const double *f_out,
              const double *H_post, const double *H_res, double *x_next) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    for (int i = 0; i < n; ++i) {
      for (int64_t c = 0; c < C; ++c) {
        double acc = 0.0;
        for (int j = 0; j < n; ++j) acc += H_res[t * n * n + i * n + j] * x[(t * n + j) * C + c];
        acc += H_post[t * n + i] * f_out[t * C + c];
        x_next[(t * n + i) * C + c] = acc;
      }
    }
  }
}

/* Backward of pre + post for T tokens, with the mapping recomputed from
 * (x, phi, b, alpha) [P5 [19], [21]].  The scalar being differentiated is
 *   L = sum G . x_next + sum g . h_in
 * with G = dL/dx_next, g = dL/dh_in given.  Hand-written reverse mode of the
 * program in orc_pre / orc_post.
 *
 * The derivatives of L with respect to the post merge's maps,
 *   dH_res[i][j] = <G_i, x_j>,   dH_post[i] = <G_i, f_out>,
 * are taken from `red` ([T][n*n + n]: dH_res then dH_post) when it is given,
 * and computed from G and f_out otherwise.  grad_f_out is written when the
 * pointer is non-null.
 *
 * Per-token output grad_x [T][n][C] is written.  grad_phi, grad_b and
 * grad_alpha (per scale group: pre, post, res) are ADDED to (the caller
 * zeroes them), token by token in
 * increasing t, so that a caller may run T in consecutive chunks. */
static void backward_core(int n, int64_t T, int64_t C, int iters, double eps, const double *x,
                          const double *phi, const double *b, const double *alpha,
                          const double *f_out,
                          const double *G, const double *g, const double *red, double *grad_x,
                          double *grad_phi, double *grad_b, double *grad_alpha,
                          double *grad_f_out) {
  const int M = n * n + 2 * n;
  const int nn = n * n;
  const int64_t K = (int64_t)n * C;
  double *dy_all = (double *)malloc(sizeof(double) * (size_t)T * M);
  double *dz_all = (double *)malloc(sizeof(double) * (size_t)T * M);
  double *y_all = (double *)malloc(sizeof(double) * (size_t)T * M);
  double *r_all = (double *)malloc(sizeof(double) * (size_t)T);

#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    const double *xt = x + t * K;
    const double *Gt = G + t * K;
    const double *gt = g + t * C;
    double *gx = grad_x + t * K;
    double y[16 * 16 + 32], z[16 * 16 + 32], dz[16 * 16 + 32], r;
    double hpre[16], spre[16], spost[16], hpost[16];
    double dhpre[16], dhpost[16], dhres[256], hres[256];
    double *iterates = (double *)malloc(sizeof(double) * (size_t)(2 * iters + 1) * nn);

    /* recompute the forward mapping */
    orc_logits(n, C, eps, xt, phi, b, alpha, &r, y, z);
    for (int i = 0; i < n; ++i) {
      spre[i] = orc_sigmoid(z[i]);
      spost[i] = orc_sigmoid(z[n + i]);
      hpre[i] = spre[i];
      hpost[i] = 2.0 * spost[i];
    }
    orc_sk_forward(n, iters, z + 2 * n, hres, iterates);

    /* post: x_next = H_res x + H_post^T f_out */
    if (grad_f_out != NULL) {
      for (int64_t c = 0; c < C; ++c) {
        double acc = 0.0;
        for (int i = 0; i < n; ++i) acc += hpost[i] * Gt[i * C + c];
        grad_f_out[t * C + c] = acc;
      }
    }
    if (red != NULL) {
      for (int e = 0; e < nn; ++e) dhres[e] = red[t * (nn + n) + e];
      for (int i = 0; i < n; ++i) dhpost[i] = red[t * (nn + n) + nn + i];
    } else {
      const double *ft = f_out + t * C;
      for (int i = 0; i < n; ++i) {
        double acc = 0.0;
        for (int64_t c = 0; c < C; ++c) acc += Gt[i * C + c] * ft[c];
        dhpost[i] = acc;
        for (int j = 0; j < n; ++j) {
          double a2 = 0.0;
          for (int64_t c = 0; c < C; ++c) a2 += Gt[i * C + c] * xt[j * C + c];
          dhres[i * n + j] = a2;
        }
      }
    }
    /* pre: h_in = H_pre x */
    for (int i = 0; i < n; ++i) {
      double acc = 0.0;
      for (int64_t c = 0; c < C; ++c) acc += gt[c] * xt[i * C + c];
      dhpre[i] = acc;
    }
    /* direct paths into x */
    for (int j = 0; j < n; ++j) {
      for (int64_t c = 0; c < C; ++c) {
        double acc = 0.0;
        for (int i = 0; i < n; ++i) acc += hres[i * n + j] * Gt[i * C + c];
        acc += hpre[j] * gt[c];
        gx[j * C + c] = acc;
      }
    }
    /* through the mapping: Sinkhorn adjoint and the gates */
    orc_sk_backward(n, iters, iterates, dhres, dz + 2 * n);
    for (int i = 0; i < n; ++i) {
      dz[i] = dhpre[i] * spre[i] * (1.0 - spre[i]);
      dz[n + i] = dhpost[i] * 2.0 * spost[i] * (1.0 - spost[i]);
    }
    /* z = alpha * y + b;  y = xhat . phi;  xhat = x / r */
    double dy[16 * 16 + 32];
    for (int m = 0; m < M; ++m) dy[m] = alpha[orc_group(n, m)] * dz[m];
    double dot = 0.0; /* sum_k dxhat_k x_k */
    for (int64_t k = 0; k < K; ++k) {
      double dxh = 0.0;
      for (int m = 0; m < M; ++m) dxh += phi[k * M + m] * dy[m];
      dot += dxh * xt[k];
      gx[k] += dxh / r;
    }
    for (int64_t k = 0; k < K; ++k) gx[k] -= dot * xt[k] / ((double)K * r * r * r);

    for (int m = 0; m < M; ++m) {
      dy_all[t * M + m] = dy[m];
      dz_all[t * M + m] = dz[m];
      y_all[t * M + m] = y[m];
    }
    r_all[t] = r;
    free(iterates);
  }

  /* parameter gradients: sums over tokens, in increasing t */
  for (int64_t t = 0; t < T; ++t) {
    double ga[3] = {0.0, 0.0, 0.0};
    for (int m = 0; m < M; ++m) {
      grad_b[m] += dz_all[t * M + m];
      ga[orc_group(n, m)] += dz_all[t * M + m] * y_all[t * M + m];
    }
    for (int g = 0; g < 3; ++g) grad_alpha[g] += ga[g];
  }
#pragma omp parallel for schedule(static)
  for (int64_t k = 0; k < K; ++k) {
    for (int64_t t = 0; t < T; ++t) {
      const double xh = x[t * K + k] / r_all[t];
      for (int m = 0; m < M; ++m) grad_phi[k * M + m] += xh * dy_all[t * M + m];
    }
  }
  free(dy_all);
  free(dz_all);
  free(y_all);
  free(r_all);
}

/* The whole layer backward in one call (grad_h_in given together with
 * grad_x_next): grad_x, grad_f_out and the parameter sums. */
void orc_backward(int n, int64_t T, int64_t C, int iters, double eps, const double *x,
                  const double *phi, const double *b, const double *alpha,
                  const double *f_out, const double *G, const double *g, double *grad_x,
                  double *grad_phi, double *grad_b, double *grad_alpha, double *grad_f_out) {
  backward_core(n, T, C, iters, eps, x, phi, b, alpha, f_out, G, g, NULL, grad_x, grad_phi, grad_b,
                grad_alpha, grad_f_out);
}

/* First half of the layer backward in training order [P5 [20]-[21]]: the
 * reverse of the post merge x_next = H_res x + H_post^T f_out alone, with the
 * forward's H_post given.  Writes
 *   grad_f_out[c] = sum_i H_post[i] G_i[c]
 *   red = [ dH_res[i][j] = <G_i, x_j>  (n*n) | dH_post[i] = <G_i, f_out>  (n) ]
 * per token; red is what the second half needs from grad_x_next besides G. */
void orc_post_backward(int n, int64_t T, int64_t C, const double *x, const double *f_out,
                       const double *H_post, const double *G, double *grad_f_out, double *red) {
  const int nn = n * n;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    const double *xt = x + t * n * C;
    const double *Gt = G + t * n * C;
    const double *ft = f_out + t * C;
    for (int64_t c = 0; c < C; ++c) {
      double acc = 0.0;
      for (int i = 0; i < n; ++i) acc += H_post[t * n + i] * Gt[i * C + c];
      grad_f_out[t * C + c] = acc;
    }
    for (int i = 0; i < n; ++i) {
      for (int j = 0; j < n; ++j) {
        double acc = 0.0;
        for (int64_t c = 0; c < C; ++c) acc += Gt[i * C + c] * xt[j * C + c];
        red[t * (nn + n) + i * n + j] = acc;
      }
      double acc = 0.0;
      for (int64_t c = 0; c < C; ++c) acc += Gt[i * C + c] * ft[c];
      red[t * (nn + n) + nn + i] = acc;
    }
  }
}

/* Second half of the layer backward in training order: given grad_h_in (from
 * F's backward), grad_x_next and the post half's reductions, recompute the
 * mapping and write grad_x plus the parameter sums (added to, as above). */
void orc_pre_backward(int n, int64_t T, int64_t C, int iters, double eps, const double *x,
                      const double *phi, const double *b, const double *alpha, const double *G,
                      const double *g, const double *red, double *grad_x, double *grad_phi,
                      double *grad_b, double *grad_alpha) {
  backward_core(n, T, C, iters, eps, x, phi, b, alpha, NULL, G, g, red, grad_x, grad_phi, grad_b,
                grad_alpha, NULL);
}

/* Composite residual map over depth and its Amax gain [P1 "Warum
 * Hyperverbindungen instabil werden", "Vielfaeltig eingeschraenkte
 * Hyperverbindungen"]: per token P = H_L ... H_1 (H[t][0] applied first),
 * gain_fwd = max_i sum_j |P_ij|, gain_bwd = max_j sum_i |P_ij|.
 * H is [T][L][n][n]. */
void orc_depth_amax(int n, int64_t T, int L, const double *H, double *gain_fwd,
                    double *gain_bwd) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    double P[256], Q[256];
    for (int i = 0; i < n; ++i)
      for (int j = 0; j < n; ++j) P[i * n + j] = (i == j) ? 1.0 : 0.0;
    for (int l = 0; l < L; ++l) {
      const double *Hl = H + ((size_t)t * L + l) * n * n;
      for (int i = 0; i < n; ++i)
        for (int j = 0; j < n; ++j) {
          double acc = 0.0;
          for (int k = 0; k < n; ++k) acc += Hl[i * n + k] * P[k * n + j];
          Q[i * n + j] = acc;
        }
      memcpy(P, Q, sizeof(double) * n * n);
    }
    double gf = 0.0, gb = 0.0;
    for (int i = 0; i < n; ++i) {
      double s = 0.0;
      for (int j = 0; j < n; ++j) s += fabs(P[i * n + j]);
      if (s > gf) gf = s;
    }
    for (int j = 0; j < n; ++j) {
      double s = 0.0;
      for (int i = 0; i < n; ++i) s += fabs(P[i * n + j]);
      if (s > gb) gb = s;
    }
    gain_fwd[t] = gf;
    gain_bwd[t] = gb;
  }
}

/* Number of OpenMP threads the oracle runs with (1 without OpenMP). */
int orc_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void orc_set_num_threads(int k) {
#ifdef _OPENMP
  extern void omp_set_num_threads(int);
  omp_set_num_threads(k);
#else
  (void)k;
#endif
}
