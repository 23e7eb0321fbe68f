/*
 * fp64 CPU oracle for the mHC / xHC residual-stream mixing.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg call this code; the CUDA library never links,
 * loads or calls it, and it shares no source with the CUDA path.
 *
 * Everything is double precision and written in the order the pages state
 * the method, with no blocking, fusion or reordering:
 *   - mHC: "mHC: Manifold-Constrained Hyper-Connections" (paper notes page),
 *     section 3 Eq.(3) (single-layer update), section 4.2 Eq.(7) (flatten,
 *     RMSNorm, projection, gates and biases), Eq.(8) (sigma, 2*sigma,
 *     Sinkhorn-Knopp), Eq.(9) (M0 = exp, M_t = T_r(T_c(M_{t-1})), t_max = 20),
 *     section 4.3.1 (F_pre and F_post,res apply steps).
 *   - xHC: "xHC: Expanded Hyper-Connections" (summary page), section
 *     "temporal feature augmentation" (causal depthwise convs, modified
 *     Gram-Schmidt), section "sparse residual stream architecture" (routing,
 *     dense read, sparse update + scatter), section "parameterisation"
 *     (gated projections, Sinkhorn on the active streams, H_post = 2*sigma);
 *     project page "default xHC configuration" table.
 *
 * Readings of points the pages leave open:
 *   RMSNorm: r = sqrt(sum(x^2)/(nC) + eps), no weight (folded into phi).
 *   vec(X): index i*C + c (streams outer).  phi columns: pre | post | res.
 *   mat(): row-major, H_res[i][j] = z[2n + i*n + j], weighting source stream
 *   j into destination stream i.  Each Sinkhorn iteration normalises columns
 *   first, then rows.  alpha multiplies the projected logits before +b.
 *
 * Parity pins: every function here is checked by tests/test_oracle_pins.py
 * against closed forms, invariants, hand-computed values and brute force.
 * The xHC parameter shapes (router columns, H_post k x Kr, routing weights)
 * are this project's reading of a text-only description: "parity unpinned"
 * beyond internal consistency for those choices.
 */
#include <math.h>
#include <stdint.h>
#ifdef _OPENMP
#include <omp.h>
#endif
#include <stdlib.h>
#include <string.h>

static double sigm(double z) { return 1.0 / (1.0 + exp(-z)); }

/* ---------------------------------------------------------------- Sinkhorn */

/* Eq.(8)-(9): M0 = exp(L) (n x n, row-major); then t_iters times
 * M <- T_r(T_c(M)): column normalisation followed by row normalisation.
 * If trace != NULL it receives M^(0..t_iters), (t_iters+1)*n*n doubles. */
void orc_sinkhorn(const double* L, int n, int t_iters, double* H, double* trace)
{
    double* M = (double*)malloc(sizeof(double) * n * n);
    for (int e = 0; e < n * n; ++e) M[e] = exp(L[e]);
    if (trace) memcpy(trace, M, sizeof(double) * n * n);
    for (int t = 1; t <= t_iters; ++t) {
        for (int j = 0; j < n; ++j) {            /* T_c: every column sums to 1 */
            double cs = 0.0;
            for (int i = 0; i < n; ++i) cs += M[i * n + j];
            for (int i = 0; i < n; ++i) M[i * n + j] /= cs;
        }
        for (int i = 0; i < n; ++i) {            /* T_r: every row sums to 1 */
            double rs = 0.0;
            for (int j = 0; j < n; ++j) rs += M[i * n + j];
            for (int j = 0; j < n; ++j) M[i * n + j] /= rs;
        }
        if (trace) memcpy(trace + (size_t)t * n * n, M, sizeof(double) * n * n);
    }
    memcpy(H, M, sizeof(double) * n * n);
    free(M);
}

/* ------------------------------------------------------------ mHC forward */

/* Eq.(7)-(9) for T tokens.  X [T][n][C]; phi [n*C][P], P = n*n + 2n;
 * alpha[3] = (pre, post, res); b[P].  Outputs (all nullable):
 * z [T][P] (gated logits), r [T] (RMS), H_pre [T][n], H_post [T][n],
 * H_res [T][n][n]. */
void orc_mhc_coeffs(const double* X, const double* phi, const double* alpha,
                    const double* b, int64_t T, int n, int C, int t_iters, double eps,
                    double* z_out, double* r_out, double* H_pre, double* H_post,
                    double* H_res)
{
    const int P = n * n + 2 * n;
    const int64_t K = (int64_t)n * C;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const double* x = X + t * K;                 /* vec(X_t), index i*C + c */
        double* xn = (double*)malloc(sizeof(double) * K);
        double z[8 * 8 + 16], d[8 * 8 + 16];
        double ss = 0.0;
        for (int64_t k = 0; k < K; ++k) ss += x[k] * x[k];
        const double r = sqrt(ss / (double)K + eps); /* RMSNorm over the nC vector */
        for (int64_t k = 0; k < K; ++k) xn[k] = x[k] / r;
        for (int p = 0; p < P; ++p) {                /* x' phi */
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += xn[k] * phi[k * P + p];
            d[p] = acc;
        }
        for (int p = 0; p < P; ++p) {                /* alpha * (x' phi) + b */
            const double a = p < n ? alpha[0] : (p < 2 * n ? alpha[1] : alpha[2]);
            z[p] = a * d[p] + b[p];
        }
        if (z_out) memcpy(z_out + t * P, z, sizeof(double) * P);
        if (r_out) r_out[t] = r;
        for (int i = 0; i < n; ++i) {
            if (H_pre) H_pre[t * n + i] = sigm(z[i]);
            if (H_post) H_post[t * n + i] = 2.0 * sigm(z[n + i]);
        }
        if (H_res) orc_sinkhorn(z + 2 * n, n, t_iters, H_res + t * n * n, NULL);
        free(xn);
    }
}

/* F_pre: x_in[t][c] = sum_i H_pre[t][i] * X[t][i][c]  (Eq.(3), H_pre x_l). */
void orc_mhc_apply_pre(const double* X, const double* H_pre, int64_t T, int n, int C,
                       double* x_in)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int c = 0; c < C; ++c) {
            double acc = 0.0;
            for (int i = 0; i < n; ++i) acc += H_pre[t * n + i] * X[(t * n + i) * C + c];
            x_in[t * C + c] = acc;
        }
}

/* F_post,res: X_next[t][i][c] = sum_j H_res[t][i][j] X[t][j][c] + H_post[t][i] F[t][c]
 * (Eq.(3): H_res x_l + H_post^T F). */
void orc_mhc_post(const double* X, const double* F, const double* H_post,
                  const double* H_res, int64_t T, int n, int C, double* X_next)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int i = 0; i < n; ++i)
            for (int c = 0; c < C; ++c) {
                double acc = 0.0;
                for (int j = 0; j < n; ++j)
                    acc += H_res[(t * n + i) * n + j] * X[(t * n + j) * C + c];
                acc += H_post[t * n + i] * F[t * C + c];
                X_next[(t * n + i) * C + c] = acc;
            }
}

/* ------------------------------------------------------ HC (tanh) variant */

/* Hyper-Connections coefficients, mHC paper section 3, Eq.(5), for T tokens.
 * RMSNorm acts on the last dimension: every stream b of X_t is normalised on its
 * own, x~_b = x_b / sqrt(mean_c x_b[c]^2 + eps) (no weight: it folds into theta).
 * The dynamic maps are linear projections of x~ followed by tanh, scaled by the
 * gate factor and shifted by the static map:
 *   H_pre[b]     = alpha[0] * tanh(theta_pre  . x~_b) + b_pre[b]
 *   H_post[b]    = alpha[1] * tanh(theta_post . x~_b) + b_post[b]
 *   H_res[a][b]  = alpha[2] * tanh(theta_res[a] . x~_b) + b_res[a][b]
 * (theta_res x~^T is n x n with entry [a][b] = theta_res[a] . x~_b).
 * X [T][n][C]; theta [n+2][C], rows pre, post, res_0 .. res_{n-1};
 * b [n*n + 2n] = b_pre | b_post | b_res (row-major); alpha[3] = (pre, post, res).
 * Outputs (nullable): H_pre [T][n], H_post [T][n], H_res [T][n][n]. */
void orc_hc_coeffs(const double* X, const double* theta, const double* alpha,
                   const double* b, int64_t T, int n, int C, double eps,
                   double* H_pre, double* H_post, double* H_res)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double* xn = (double*)malloc(sizeof(double) * (size_t)n * C);
        for (int s = 0; s < n; ++s) {                /* RMSNorm per stream */
            const double* x = X + (t * n + s) * (int64_t)C;
            double ss = 0.0;
            for (int c = 0; c < C; ++c) ss += x[c] * x[c];
            const double r = sqrt(ss / (double)C + eps);
            for (int c = 0; c < C; ++c) xn[(size_t)s * C + c] = x[c] / r;
        }
        for (int s = 0; s < n; ++s) {
            const double* xs = xn + (size_t)s * C;
            double proj[2 + 8];                      /* theta_q . x~_s, q = pre, post, res_0.. */
            for (int q = 0; q < n + 2; ++q) {
                double acc = 0.0;
                for (int c = 0; c < C; ++c) acc += theta[(size_t)q * C + c] * xs[c];
                proj[q] = acc;
            }
            if (H_pre) H_pre[t * n + s] = alpha[0] * tanh(proj[0]) + b[s];
            if (H_post) H_post[t * n + s] = alpha[1] * tanh(proj[1]) + b[n + s];
            if (H_res)
                for (int a = 0; a < n; ++a)
                    H_res[(t * n + a) * n + s] = alpha[2] * tanh(proj[2 + a]) + b[2 * n + a * n + s];
        }
        free(xn);
    }
}

/* Amax Gain Magnitude, mHC paper section 3.1, of the composite residual map of
 * Eq.(4).  For every token, the map from the input of layer 0 to the output of
 * layer d-1 is M_d = H_res[d-1] H_res[d-2] ... H_res[0] (x_d = M_d x_0 + terms of
 * the layer outputs).  The forward gain is the largest absolute row sum of M_d,
 * max_i |sum_j M_d[i][j]|; the backward gain the largest absolute column sum,
 * max_j |sum_i M_d[i][j]|.  H_res [L][T][n][n] (layer-major); gain [L][T][2] =
 * (forward, backward) for d = 1 .. L. */
void orc_amax_gain(const double* H_res, int L, int64_t T, int n, double* gain)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double M[64], P[64];
        for (int i = 0; i < n; ++i)
            for (int j = 0; j < n; ++j) M[i * n + j] = i == j ? 1.0 : 0.0;
        for (int l = 0; l < L; ++l) {
            const double* H = H_res + ((int64_t)l * T + t) * n * n;
            for (int i = 0; i < n; ++i)              /* M <- H_res[l] M */
                for (int j = 0; j < n; ++j) {
                    double acc = 0.0;
                    for (int k = 0; k < n; ++k) acc += H[i * n + k] * M[k * n + j];
                    P[i * n + j] = acc;
                }
            memcpy(M, P, sizeof(double) * n * n);
            double fwd = 0.0, bwd = 0.0;
            for (int i = 0; i < n; ++i) {
                double rs = 0.0;
                for (int j = 0; j < n; ++j) rs += M[i * n + j];
                if (fabs(rs) > fwd) fwd = fabs(rs);
            }
            for (int j = 0; j < n; ++j) {
                double cs = 0.0;
                for (int i = 0; i < n; ++i) cs += M[i * n + j];
                if (fabs(cs) > bwd) bwd = fabs(cs);
            }
            gain[((int64_t)l * T + t) * 2 + 0] = fwd;
            gain[((int64_t)l * T + t) * 2 + 1] = bwd;
        }
    }
}

/* ----------------------------------------------------------- mHC backward */

/* Reverse mode of orc_mhc_coeffs + orc_mhc_apply_pre + orc_mhc_post for T
 * tokens, with the gradient taken through all t_iters Sinkhorn iterations.
 * Inputs: the forward's inputs plus upstream gradients dXn [T][n][C] (of
 * X_next) and dxin [T][C] (of x_in).  Outputs: dX [T][n][C], dF [T][C],
 * dphi [n*C][P], dalpha[3], db[P] (the last three summed over tokens,
 * overwritten).  Derivation (per token):
 *   dH_post_i = <dXn_i, F>;  dF = sum_i H_post_i dXn_i
 *   dH_res_ij = <dXn_i, X_j>; dX_j += sum_i H_res_ij dXn_i
 *   dH_pre_i  = <dxin, X_i>;  dX_i += H_pre_i dxin
 *   sigma'/2sigma'; Sinkhorn reverse: for M' = A/rowsum: dA = (dM' - rowdot(dM',M'))/rowsum,
 *   for A = M/colsum: dM = (dA - coldot(dA,A))/colsum; dL = dM0 * M0.
 *   z = alpha*d/r + b with d = x phi (same value as alpha*(x/r)phi + b):
 *   dalpha += dz*d/r, db += dz, dd = alpha*dz/r, dr = -sum alpha*dz*d/r^2,
 *   dphi += x^T dd, dx += phi dd + dr * x/(nC r). */
void orc_mhc_backward(const double* X, const double* F, const double* phi,
                      const double* alpha, const double* b, const double* dXn,
                      const double* dxin, int64_t T, int n, int C, int t_iters, double eps,
                      double* dX, double* dF, double* dphi, double* dalpha, double* db)
{
    const int P = n * n + 2 * n;
    const int64_t K = (int64_t)n * C;
    const int nn = n * n;
    memset(dphi, 0, sizeof(double) * K * P);
    memset(dalpha, 0, sizeof(double) * 3);
    memset(db, 0, sizeof(double) * P);
    /* Tokens are split into fixed contiguous ranges, one per thread; each range
     * sums into its own partial dphi/dalpha/db, and the partials are added in
     * range order, so the result does not depend on scheduling. */
    int nthr = 1;
#ifdef _OPENMP
    nthr = omp_get_max_threads();
#endif
    if (nthr > T) nthr = T > 0 ? (int)T : 1;
    double* part = (double*)calloc((size_t)nthr * (K * P + 3 + P), sizeof(double));
#pragma omp parallel for schedule(static, 1) num_threads(nthr)
    for (int th = 0; th < nthr; ++th) {
    double* pphi = part + (size_t)th * (K * P + 3 + P);
    double* palpha = pphi + K * P;
    double* pdb = palpha + 3;
    const int64_t t_lo = T * th / nthr, t_hi = T * (th + 1) / nthr;
    for (int64_t t = t_lo; t < t_hi; ++t) {
        const double* x = X + t * K;
        const double* f = F + t * C;
        const double* gn = dXn + t * K;
        const double* gi = dxin + t * C;
        double* gx = dX + t * K;
        double* gf = dF + t * C;
        /* forward recompute */
        double ss = 0.0;
        for (int64_t k = 0; k < K; ++k) ss += x[k] * x[k];
        const double r = sqrt(ss / (double)K + eps);
        double d[8 * 8 + 16], z[8 * 8 + 16], dz[8 * 8 + 16];
        for (int p = 0; p < P; ++p) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += x[k] * phi[k * P + p];
            d[p] = acc;
        }
        double aseg[8 * 8 + 16];
        for (int p = 0; p < P; ++p) {
            aseg[p] = p < n ? alpha[0] : (p < 2 * n ? alpha[1] : alpha[2]);
            z[p] = aseg[p] * d[p] / r + b[p];
        }
        double hpre[8], hpost[8];
        for (int i = 0; i < n; ++i) { hpre[i] = sigm(z[i]); hpost[i] = 2.0 * sigm(z[n + i]); }
        double* tr = (double*)malloc(sizeof(double) * (t_iters + 1) * nn);
        double hres[64];
        orc_sinkhorn(z + 2 * n, n, t_iters, hres, tr);
        /* gradients of the apply steps */
        double dhpre[8], dhpost[8], dhres[64];
        for (int i = 0; i < n; ++i) {
            double a = 0.0, p2 = 0.0;
            for (int c = 0; c < C; ++c) { a += gn[i * C + c] * f[c]; p2 += gi[c] * x[i * C + c]; }
            dhpost[i] = a; dhpre[i] = p2;
            for (int j = 0; j < n; ++j) {
                double s2 = 0.0;
                for (int c = 0; c < C; ++c) s2 += gn[i * C + c] * x[j * C + c];
                dhres[i * n + j] = s2;
            }
        }
        for (int c = 0; c < C; ++c) {
            double a = 0.0;
            for (int i = 0; i < n; ++i) a += hpost[i] * gn[i * C + c];
            gf[c] = a;
        }
        for (int j = 0; j < n; ++j)
            for (int c = 0; c < C; ++c) {
                double a = hpre[j] * gi[c];
                for (int i = 0; i < n; ++i) a += hres[i * n + j] * gn[i * C + c];
                gx[j * C + c] = a;
            }
        /* gates */
        for (int i = 0; i < n; ++i) {
            const double s0 = sigm(z[i]), s1 = sigm(z[n + i]);
            dz[i] = dhpre[i] * s0 * (1.0 - s0);
            dz[n + i] = dhpost[i] * 2.0 * s1 * (1.0 - s1);
        }
        /* Sinkhorn reverse, iteration t_iters down to 1 */
        double g[64], A[64], ga[64];
        memcpy(g, dhres, sizeof(double) * nn);
        for (int it = t_iters; it >= 1; --it) {
            const double* Mp = tr + (size_t)(it - 1) * nn;   /* M^(it-1) */
            const double* Mo = tr + (size_t)it * nn;         /* M^(it) = T_r(A) */
            double cs[8], rs[8];
            for (int j = 0; j < n; ++j) { cs[j] = 0.0; for (int i = 0; i < n; ++i) cs[j] += Mp[i * n + j]; }
            for (int i = 0; i < n; ++i) for (int j = 0; j < n; ++j) A[i * n + j] = Mp[i * n + j] / cs[j];
            for (int i = 0; i < n; ++i) { rs[i] = 0.0; for (int j = 0; j < n; ++j) rs[i] += A[i * n + j]; }
            for (int i = 0; i < n; ++i) {                      /* through T_r */
                double dot = 0.0;
                for (int j = 0; j < n; ++j) dot += g[i * n + j] * Mo[i * n + j];
                for (int j = 0; j < n; ++j) ga[i * n + j] = (g[i * n + j] - dot) / rs[i];
            }
            for (int j = 0; j < n; ++j) {                      /* through T_c */
                double dot = 0.0;
                for (int i = 0; i < n; ++i) dot += ga[i * n + j] * A[i * n + j];
                for (int i = 0; i < n; ++i) g[i * n + j] = (ga[i * n + j] - dot) / cs[j];
            }
        }
        for (int e = 0; e < nn; ++e) dz[2 * n + e] = g[e] * tr[e];   /* d exp */
        free(tr);
        /* logits */
        double dr = 0.0, dd[8 * 8 + 16];
        for (int p = 0; p < P; ++p) {
            const int s = p < n ? 0 : (p < 2 * n ? 1 : 2);
            palpha[s] += dz[p] * d[p] / r;
            pdb[p] += dz[p];
            dd[p] = aseg[p] * dz[p] / r;
            dr -= aseg[p] * dz[p] * d[p] / (r * r);
        }
        for (int64_t k = 0; k < K; ++k) {
            double a = 0.0;
            for (int p = 0; p < P; ++p) {
                a += phi[k * P + p] * dd[p];
                pphi[k * P + p] += x[k] * dd[p];
            }
            gx[k] += a + dr * x[k] / ((double)K * r);
        }
    }
    }
    for (int th = 0; th < nthr; ++th) {
        const double* pphi = part + (size_t)th * (K * P + 3 + P);
        for (int64_t e = 0; e < K * P; ++e) dphi[e] += pphi[e];
        for (int s = 0; s < 3; ++s) dalpha[s] += pphi[K * P + s];
        for (int p = 0; p < P; ++p) db[p] += pphi[K * P + 3 + p];
    }
    free(part);
}

/* ---------------------------------------------------------------- xHC */

/* Stream routing + dense read.  X [T][N][C]; phi_read [N*C][R], R = 2N - m:
 * columns 0..N-1 give the H_pre logits, columns N..R-1 the route logits of
 * streams m..N-1.  alpha_read = (pre, route); b_read [R].
 * Outputs: x_in [T][C] = sum_i H_pre_i X_i; H_pre [T][N] = sigma;
 * score [T][N-m] = sigma(route logits); idx [T][k] = {0..m-1} and the k-m
 * routed streams with the highest score (ties: lower index), ascending;
 * w [T][k] = 1 for fixed streams, the score for routed ones. */
void orc_xhc_route(const double* X, const double* phi_read, const double* alpha_read,
                   const double* b_read, int64_t T, int N, int C, int k, int m, double eps,
                   double* x_in, double* H_pre, double* score, int32_t* idx, double* w)
{
    const int R = 2 * N - m;
    const int64_t K = (int64_t)N * C;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const double* x = X + t * K;
        double* xn = (double*)malloc(sizeof(double) * K);
        double z[96], sc[64];
        double ss = 0.0;
        for (int64_t q = 0; q < K; ++q) ss += x[q] * x[q];
        const double r = sqrt(ss / (double)K + eps);
        for (int64_t q = 0; q < K; ++q) xn[q] = x[q] / r;
        for (int p = 0; p < R; ++p) {
            double acc = 0.0;
            for (int64_t q = 0; q < K; ++q) acc += xn[q] * phi_read[q * R + p];
            z[p] = (p < N ? alpha_read[0] : alpha_read[1]) * acc + b_read[p];
        }
        double hp[64];
        for (int i = 0; i < N; ++i) { hp[i] = sigm(z[i]); if (H_pre) H_pre[t * N + i] = hp[i]; }
        for (int s = 0; s < N - m; ++s) { sc[s] = sigm(z[N + s]); if (score) score[t * (N - m) + s] = sc[s]; }
        int chosen[64] = {0};
        for (int q = 0; q < k - m; ++q) {            /* TopK by repeated arg-max */
            int best = -1;
            for (int s = 0; s < N - m; ++s)
                if (!chosen[s] && (best < 0 || sc[s] > sc[best])) best = s;
            chosen[best] = 1;
        }
        int slot = 0;
        for (int i = 0; i < m; ++i) { idx[t * k + slot] = i; w[t * k + slot] = 1.0; ++slot; }
        for (int s = 0; s < N - m; ++s)
            if (chosen[s]) { idx[t * k + slot] = m + s; w[t * k + slot] = sc[s]; ++slot; }
        for (int c = 0; c < C; ++c) {
            double acc = 0.0;
            for (int i = 0; i < N; ++i) acc += hp[i] * x[(int64_t)i * C + c];
            x_in[t * C + c] = acc;
        }
        free(xn);
    }
}

/* Causal depthwise convolutions: G[t][j][c] = sum_{s<kappa_j} w_j[s][c] * out[t-s][c],
 * zero where t-s falls before the start of t's sequence (sequences of seq_len
 * tokens laid end to end).  w: the r weight arrays concatenated, w_j [kappa_j][C]. */
void orc_xhc_conv(const double* out, const double* w, const int* kappa, int r,
                  int64_t T, int C, int64_t seq_len, double* G)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const int64_t pos = t % seq_len;
        int64_t off = 0;
        for (int j = 0; j < r; ++j) {
            for (int c = 0; c < C; ++c) {
                double acc = 0.0;
                for (int s = 0; s < kappa[j]; ++s)
                    if (pos - s >= 0) acc += w[off + (int64_t)s * C + c] * out[(t - s) * C + c];
                G[(t * r + j) * C + c] = acc;
            }
            off += (int64_t)kappa[j] * C;
        }
    }
}

/* Modified Gram-Schmidt over the Kr = r+1 components of each token:
 * v_1 = out; for j = 1..r: u = g_j, then for i = 1..j: u -= (<u,v_i>/<v_i,v_i>) v_i
 * (a zero v_i contributes nothing); v_{j+1} = u.  V [T][r+1][C].
 * If classical != 0 the coefficients use <g_j, v_i> instead of <u, v_i> (the
 * printed sum); the two agree in exact arithmetic. */
void orc_xhc_gs(const double* out, const double* G, int64_t T, int C, int r, int classical,
                double* V)
{
    const int Kr = r + 1;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double* v = V + t * Kr * C;
        for (int c = 0; c < C; ++c) v[c] = out[t * C + c];
        for (int j = 1; j <= r; ++j) {
            const double* g = G + (t * r + (j - 1)) * C;
            double* u = v + (int64_t)j * C;
            for (int c = 0; c < C; ++c) u[c] = g[c];
            for (int i = 0; i < j; ++i) {
                const double* vi = v + (int64_t)i * C;
                double num = 0.0, den = 0.0;
                for (int c = 0; c < C; ++c) {
                    num += (classical ? g[c] : u[c]) * vi[c];
                    den += vi[c] * vi[c];
                }
                const double coef = den > 0.0 ? num / den : 0.0;
                for (int c = 0; c < C; ++c) u[c] -= coef * vi[c];
            }
        }
    }
}

/* Sparse residual update + scatter, in place on X [T][N][C].
 * X_act = rows idx[t][0..k-1] of X_t (k x C, slot order = idx order);
 * r = RMS(vec X_act) over kC; d = vec(X_act) phi_act / r, phi_act [k*C][k*k + k*Kr]
 * with columns res (k*k, row-major) | post (k*Kr, row-major [j][c]);
 * alpha_act = (res, post); z = alpha*d + b_act;
 * H_res = Sinkhorn(mat z_res) (k x k), H_post = 2 sigma(z_post) (k x Kr);
 * X_act_new[j] = sum_l H_res[j][l] X_act[l] + w[t][j] * sum_c H_post[j][c] V[t][c];
 * X[idx[t][j]] = X_act_new[j]; other streams are untouched.
 * Optional outputs H_res_out [T][k][k], H_post_out [T][k][Kr]. */
void orc_xhc_sparse_update(double* X, const double* V, int Kr, const int32_t* idx,
                           const double* w, const double* phi_act, const double* alpha_act,
                           const double* b_act, int64_t T, int N, int C, int k, int t_iters,
                           double eps, double* H_res_out, double* H_post_out)
{
    const int Pa = k * k + k * Kr;
    const int64_t K = (int64_t)k * C;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double* xa = (double*)malloc(sizeof(double) * K);
        double* xn = (double*)malloc(sizeof(double) * K);
        double z[8 * 8 + 8 * 16], hres[64], hpost[8 * 16];
        for (int l = 0; l < k; ++l)
            memcpy(xa + (int64_t)l * C, X + (t * N + idx[t * k + l]) * (int64_t)C, sizeof(double) * C);
        double ss = 0.0;
        for (int64_t q = 0; q < K; ++q) ss += xa[q] * xa[q];
        const double r = sqrt(ss / (double)K + eps);
        for (int64_t q = 0; q < K; ++q) xn[q] = xa[q] / r;
        for (int p = 0; p < Pa; ++p) {
            double acc = 0.0;
            for (int64_t q = 0; q < K; ++q) acc += xn[q] * phi_act[q * Pa + p];
            z[p] = (p < k * k ? alpha_act[0] : alpha_act[1]) * acc + b_act[p];
        }
        orc_sinkhorn(z, k, t_iters, hres, NULL);
        for (int e = 0; e < k * Kr; ++e) hpost[e] = 2.0 * sigm(z[k * k + e]);
        if (H_res_out) memcpy(H_res_out + t * k * k, hres, sizeof(double) * k * k);
        if (H_post_out) memcpy(H_post_out + t * k * Kr, hpost, sizeof(double) * k * Kr);
        for (int j = 0; j < k; ++j) {
            double* dst = X + (t * N + idx[t * k + j]) * (int64_t)C;
            for (int c = 0; c < C; ++c) {
                double mix = 0.0, wb = 0.0;
                for (int l = 0; l < k; ++l) mix += hres[j * k + l] * xa[(int64_t)l * C + c];
                for (int q = 0; q < Kr; ++q) wb += hpost[j * Kr + q] * V[(t * Kr + q) * C + c];
                dst[c] = mix + w[t * k + j] * wb;
            }
        }
        free(xa);
        free(xn);
    }
}
