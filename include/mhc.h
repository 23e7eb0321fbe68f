/*
 * mhc.h -- C ABI of the B200 (sm_100a) residual-stream mixing library (libmhc.so).
 *
 * The library computes the per-token residual-stream mixing of one
 * Transformer sublayer as defined by
 *   [mHC]  "mHC: Manifold-Constrained Hyper-Connections" (paper notes page):
 *          section 3 Eq.(3) (single-layer update), section 4.2 Eq.(7)-(9)
 *          (coefficients), section 4.3.1 Eq.(10)-(19) and the F_pre /
 *          F_post,res apply kernels;
 *   [xHC]  "xHC: Expanded Hyper-Connections" (summary page): sections
 *          "temporal feature augmentation", "sparse residual stream
 *          architecture", "parameterisation"; and the xHC project page's
 *          "default xHC configuration" table.
 *
 * Common conventions (every entry point):
 *  - Pointers are DEVICE pointers owned by the caller unless marked "host".
 *    The library never allocates device memory and keeps no pointer after a
 *    call returns.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream).  Argument errors are detected on the host before any
 *    launch and return MHC_ERR_INVALID_ARG or MHC_ERR_UNSUPPORTED with nothing
 *    enqueued; a launch failure returns MHC_ERR_CUDA.  mhc_last_error() gives
 *    the message of the last failing call on the calling thread.
 *  - Layouts are row-major and dense.  The multi-stream state of T tokens is
 *    X[T][n][C] (each token's n*C row contiguous; vec(X_t) index = i*C + c).
 *  - dtype: MHC_BF16 (bfloat16 storage) or MHC_F32.  All arithmetic is fp32
 *    with fp32 accumulation; a bf16 output is rounded once, to nearest even,
 *    when stored.  Coefficients (H_*) are always fp32.
 *  - Alignment: every array pointer 16-byte aligned; C a multiple of 8.
 *  - Sizes: 1 <= n <= 8; T >= 0 (T == 0 enqueues nothing and returns MHC_OK);
 *    0 <= t_iters <= 1000; eps >= 0.
 */
#ifndef MHC_H
#define MHC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MHC_OK = 0,
    MHC_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size, forbidden aliasing */
    MHC_ERR_UNSUPPORTED = 2,  /* valid but outside what this library implements      */
    MHC_ERR_CUDA = 3,         /* a CUDA launch or runtime call failed                  */
    MHC_ERR_TIMEOUT = 4       /* a bounded on-device wait expired (see mhc_sync_status)*/
} mhc_status;

/* MHC_TF32_PAIR: only as the phi dtype of mhc_pre -- a tf32 projection matrix
 * ([mHC] Eq.(10)) in the exact bf16 pair layout written by mhc_phi_tf32_pair. */
typedef enum { MHC_F32 = 0, MHC_BF16 = 1, MHC_TF32_PAIR = 2 } mhc_dtype;

/* Message of the last failing call on this thread ("" if none).  Never NULL. */
const char* mhc_last_error(void);

/* Library ABI version (major*100 + minor). */
int mhc_version(void);

/*
 * mhc_pre -- the pre half of one mHC sublayer.   [mHC] Eq.(7), (8), (9); the
 * fused order of Eq.(14)-(19); F_pre := H_pre x_l (section 4.3.1).
 *
 * For every token t:
 *   x = vec(X_t) (length nC); s = sum(x^2); r = sqrt(s/(nC) + eps)
 *   z = alpha_seg * (x phi) / r + b            (P = n*n + 2n logits)
 *   H_pre  = sigmoid(z[0:n]);  H_post = 2*sigmoid(z[n:2n])
 *   H_res  = Sinkhorn-Knopp(z[2n:], row-major n x n): M = exp(z_res); t_iters times
 *            { normalise every column to sum 1; then every row }
 *   x_in[c] = sum_i H_pre[i] * X_t[i][c]
 *
 *   X      [T][n][C], dtype x_dt                       (read)
 *   phi    [P][n*C],  dtype phi_dt: the projection matrix of Eq.(7) stored
 *          transposed (the layout of a linear layer's weight): row p holds
 *          the weights of logit p over vec(X_t); rows are pre n | post n |
 *          res n*n, res row-major (read)
 *   alpha  HOST float[3] = (alpha_pre, alpha_post, alpha_res)
 *   b      [P] fp32                                    (read)
 *   x_in   [T][C], dtype x_dt                          (written)
 *   H_pre  [T][n] fp32, may be NULL                    (written)
 *   H_post [T][n] fp32                                 (written)
 *   H_res  [T][n][n] fp32 (H_res[t][i][j] weights source stream j into i) (written)
 * Supported (x_dt, phi_dt): (F32, F32), (BF16, BF16), (BF16, F32), and
 * (BF16, TF32_PAIR): phi is then the [2*RH][n*C] bf16 pair of a tf32 phi^T
 * from mhc_phi_tf32_pair (the pages' Eq.(10)-(11) dtypes), and the
 * projection is x . (hi + lo) = x . phi_tf32 with fp32 accumulation.
 * Outputs must not overlap any input.
 */
mhc_status mhc_pre(const void* X, mhc_dtype x_dt, const void* phi, mhc_dtype phi_dt,
                   const float* alpha, const float* b, int64_t T, int n, int C,
                   int t_iters, float eps, void* x_in, float* H_pre, float* H_post,
                   float* H_res, void* stream);

/*
 * mhc_phi_tf32_pair -- the projection matrix in tf32 ([mHC] section 4.3.1,
 * Eq.(10): phi is tfloat32 while x is bfloat16) as an exact pair of bf16 rows,
 * the phi operand of mhc_pre with phi_dt = MHC_TF32_PAIR.  Run once per update
 * of phi.
 *
 * Every element of phi is first rounded to tf32 (10 explicit mantissa bits,
 * round to nearest even; a no-op for values already in tf32), t; then
 * hi = bf16(t) (round to nearest even) and lo = t - hi, which is a bf16 value,
 * so hi + lo = t exactly for |t| >= 2^-116.
 *
 *   phi   [P][n*C] fp32, P = n*n + 2n: phi^T, as for mhc_pre (read)
 *   pair  [2*RH][n*C] bf16, RH = P rounded up to a multiple of 16: rows
 *         0..P-1 = hi, RH..RH+P-1 = lo, the other rows 0 (written;
 *         mhc_phi_tf32_pair_bytes(n, C) bytes, must not overlap phi)
 * 1 <= n <= 8, C a positive multiple of 8.
 */
size_t mhc_phi_tf32_pair_bytes(int n, int C);
mhc_status mhc_phi_tf32_pair(const float* phi, int n, int C, void* pair, void* stream);

/*
 * mhc_post -- the post half of one mHC sublayer.   [mHC] Eq.(3) and the fused
 * F_post,res := H_res x_l + H_post^T F kernel of section 4.3.1 (reads (n+1)C
 * and writes nC elements per token).
 *
 *   X_next[t][i][c] = sum_j H_res[t][i][j] * X[t][j][c] + H_post[t][i] * F_out[t][c]
 *
 *   X      [T][n][C], dtype dt (read)      F_out [T][C], dtype dt (read)
 *   H_post [T][n] fp32, H_res [T][n][n] fp32 (read; e.g. from mhc_pre)
 *   X_next [T][n][C], dtype dt (written).  X_next == X (in place) is allowed;
 *   any other overlap with an input is rejected.
 */
mhc_status mhc_post(const void* X, const void* F_out, mhc_dtype dt, const float* H_post,
                    const float* H_res, int64_t T, int n, int C, void* X_next, void* stream);

/*
 * hc_pre -- the pre half of one sublayer with the HC (tanh) parameterisation,
 * the unconstrained predecessor of mHC.   [mHC] section 3, Eq.(5) and Eq.(3).
 * The post half is mhc_post (same Eq.(3)).
 *
 * For every token t and stream s (RMSNorm over the last dimension: each
 * stream on its own):
 *   r_s = sqrt(sum_c X_t[s][c]^2 / C + eps);  g_{q,s} = theta[q] . X_t[s] / r_s
 *   H_pre[s]    = alpha_pre  * tanh(g_{0,s})   + b[s]
 *   H_post[s]   = alpha_post * tanh(g_{1,s})   + b[n + s]
 *   H_res[a][s] = alpha_res  * tanh(g_{2+a,s}) + b[2n + a*n + s]
 *   x_in[c] = sum_s H_pre[s] * X_t[s][c]
 *
 *   X      [T][n][C], dtype x_dt                        (read)
 *   theta  [n+2][C], dtype theta_dt: rows theta_pre, theta_post, theta_res[0..n-1] (read)
 *   alpha  HOST float[3] = (alpha_pre, alpha_post, alpha_res)
 *   b      [n*n + 2n] fp32 = b_pre | b_post | b_res (row-major)   (read)
 *   x_in   [T][C], dtype x_dt (written); H_pre [T][n] fp32, may be NULL;
 *   H_post [T][n] fp32; H_res [T][n][n] fp32 (H_res[t][a][s] weights source
 *   stream s into a) (written).
 * Supported (x_dt, theta_dt): (F32, F32), (BF16, BF16), (BF16, F32).  Outputs
 * must not overlap any input.  Errors as mhc_pre.
 */
mhc_status hc_pre(const void* X, mhc_dtype x_dt, const void* theta, mhc_dtype theta_dt,
                  const float* alpha, const float* b, int64_t T, int n, int C, float eps,
                  void* x_in, float* H_pre, float* H_post, float* H_res, void* stream);

/*
 * mhc_amax_gain -- the Amax Gain Magnitude of the composite residual map of a
 * stack of L layers.   [mHC] section 3 Eq.(4) and section 3.1.
 *
 * For every token t and depth d = 1..L, with M_d = H_res[d-1] ... H_res[0]
 * (newest layer on the left; x_d = M_d x_0 + terms of the layer outputs):
 *   forward gain  = max_i |sum_j M_d[i][j]|      (largest absolute row sum)
 *   backward gain = max_j |sum_i M_d[i][j]|      (largest absolute column sum)
 * products and sums in fp32.
 *
 *   H_res    [L][T][n][n] fp32, layer-major (e.g. the H_res of L mhc_pre or
 *            hc_pre calls stacked) (read)
 *   gain     [L][T][2] fp32 = (forward, backward), may be NULL (written)
 *   gain_max [L][2] fp32, the maxima over the tokens, may be NULL (written;
 *            zeroed by this call on `stream` first)
 * At least one output must be given; pointers 16-byte aligned; a NaN product
 * is skipped by the maxima.  n in [1, 8]; L, T >= 0.
 */
mhc_status mhc_amax_gain(const float* H_res, int L, int64_t T, int n, float* gain,
                         float* gain_max, void* stream);

/*
 * xhc_route -- stream routing and dense read of one xHC sublayer.
 * [xHC] "sparse residual stream architecture", steps 1 (routing: m fixed
 * streams with weight 1, k-m chosen by TopK over sigmoid scores derived from
 * the full N-stream state) and 2 (dense read over all N streams);
 * "parameterisation" (gated projection, alpha and bias).  For every token t:
 *   x = vec(X_t) (N*C); r = sqrt(sum(x^2)/(NC) + eps)
 *   z = alpha_seg * (x phi_read) / r + b_read      (R = 2N - m logits)
 *   H_pre[i] = sigmoid(z[i]), i < N;  score[s-m] = sigmoid(z[N + s - m]), s = m..N-1
 *   active = {0..m-1} and the k-m streams s >= m with the highest score (an exact
 *            tie goes to the lower index); idx[t] lists them in ascending order;
 *            w = 1 for fixed streams, the score for routed ones
 *   x_in[c] = sum_{i<N} H_pre[i] * X_t[i][c]
 *
 *   X        [T][N][C], dtype dt (read)
 *   phi_read [R][N*C], dtype dt: the router projection stored transposed; rows
 *            0..N-1 give the H_pre logits, rows N..R-1 the route logits (read)
 *   alpha_read HOST float[2] = (alpha_pre, alpha_route);  b_read [R] fp32 (read)
 *   x_in [T][C] dtype dt; H_pre [T][N] fp32 (may be NULL); score [T][N-m] fp32
 *   (may be NULL); idx [T][k] int32; w [T][k] fp32 (written)
 * N <= 32, 0 <= m <= k <= N.
 */
mhc_status xhc_route(const void* X, mhc_dtype dt, const void* phi_read, const float* alpha_read,
                     const float* b_read, int64_t T, int N, int C, int k, int m, float eps, void* x_in,
                     float* H_pre, float* score, int32_t* idx, float* w, void* stream);

/*
 * xhc_conv_gs -- temporal feature augmentation of the xHC write-back.
 * [xHC] "temporal feature augmentation": r causal depthwise convolutions of
 * the sublayer output and Gram-Schmidt orthogonalisation of the Kr = r + 1
 * components per token:
 *   a_0 = F_out[t]; a_j[c] = sum_{s<kappa_j} w_j[s][c] * F_out[t-s][c]
 *        (terms with t-s before the start of t's sequence are zero; sequences
 *        of seq_len tokens are laid end to end, seq_len = T for one sequence)
 *   v_0 = a_0; v_j = a_j - sum_{i<j} <a_j, v_i>/<v_i, v_i> v_i  (a zero v_i adds nothing)
 *
 *   F_out  [T][C], dtype dt (read)
 *   conv_w fp32, the r weight arrays w_j [kappa_j][C] concatenated (read)
 *   kappa  HOST int[r], 1 <= kappa_j <= 64;  1 <= r <= 4
 *   V      [T][Kr][C] fp32: V[t][j] = v_j (written; must not overlap an input)
 * The inner products are per token over the C channels.
 */
mhc_status xhc_conv_gs(const void* F_out, mhc_dtype dt, const float* conv_w, const int* kappa,
                       int r, int64_t T, int C, int64_t seq_len, float* V, void* stream);

/*
 * xhc_sparse_update -- sparse residual update and scatter of one xHC
 * sublayer.  [xHC] "sparse residual stream architecture" (step 3) and
 * "parameterisation": H_res and H_post are generated from the k active
 * streams only; H_res is Sinkhorn-normalised (k x k), H_post = 2 sigma (k x Kr).
 * For every token t, with X_act = rows idx[t][0..k-1] of X_t (slot order):
 *   r = sqrt(sum(X_act^2)/(kC) + eps)
 *   z = alpha * (vec(X_act) phi_act) / r + b_act   (alpha_act[0] on the k*k res
 *       logits, alpha_act[1] on the k*Kr post logits)
 *   H_res = Sinkhorn-Knopp(z[0:k*k] row-major, t_iters); H_post = 2 sigmoid(z[k*k:]) as [k][Kr]
 *   X[t][idx[t][j]] = sum_l H_res[j][l] X_act[l] + w[t][j] * sum_q H_post[j][q] V[t][q]
 * Streams not in idx[t] are not touched.
 *
 *   X       [T][N][C], dtype dt (read and written in place)
 *   V       [T][Kr][C] fp32 (read; e.g. from xhc_conv_gs)
 *   idx     [T][k] int32, distinct stream indices in [0, N) (e.g. from xhc_route);
 *           a token with an entry outside [0, N) is left unchanged and
 *           mhc_sync_status() then reports MHC_ERR_INVALID_ARG
 *   w       [T][k] fp32 routing weights (read)
 *   phi_act [k*k + k*Kr][k*C], dtype dt: the projection stored transposed
 *           (row p = weights of logit p over vec(X_act)); rows res | post (read)
 *   alpha_act HOST float[2] = (alpha_res, alpha_post);  b_act [k*k + k*Kr] fp32
 *   H_res   [T][k][k] fp32, may be NULL;  H_post [T][k][Kr] fp32, may be NULL (written)
 * This library: k <= 4, Kr <= 5, C % 64 == 0, N <= 64.
 */
mhc_status xhc_sparse_update(void* X, mhc_dtype dt, const float* V, int Kr, const int32_t* idx,
                             const float* w, const void* phi_act, const float* alpha_act,
                             const float* b_act, int64_t T, int N, int C, int k, int t_iters,
                             float eps, float* H_res, float* H_post, void* stream);

/*
 * mhc_backward -- gradients of one mHC sublayer (mhc_pre + mhc_post) with all
 * t_iters Sinkhorn-Knopp iterations unrolled.  [mHC] section 4.3.1 (the
 * backward of the projection and of the Sinkhorn kernel, which recomputes
 * the intermediates on chip).  The forward is recomputed from X; nothing from
 * a forward call is needed.
 *
 * Given upstream gradients dX_next (of X_next) and dx_in (of x_in):
 *   dX     [T][n][C], dtype dt    dL/dX (through x_in, X_next and the coefficients)
 *   dF_out [T][C],    dtype dt    dL/dF_out = sum_i H_post[i] dX_next[i]
 *   dphi   [P][n*C]   fp32        dL/dphi in phi's (transposed) layout, summed over tokens
 *   dalpha [3] fp32 (device), db [P] fp32 (device): summed over tokens
 * All three sums are overwritten, not accumulated; their summation order is
 * fixed, so results are bitwise reproducible.  Inputs: as mhc_pre/mhc_post
 * (phi [P][n*C] transposed, dtype dt; alpha HOST float[3]; b [P] fp32).
 *   workspace: device scratch of at least mhc_backward_workspace_bytes(T, n, C)
 *   bytes, 256-byte aligned, owned by the caller; its contents on entry are
 *   ignored and on exit undefined.
 * This library: n <= 4, C % 64 == 0, t_iters <= 100.  T == 0 zeroes the sums.
 */
size_t mhc_backward_workspace_bytes(int64_t T, int n, int C);
mhc_status mhc_backward(const void* X, const void* F_out, const void* phi, mhc_dtype dt,
                        const float* alpha, const float* b, const void* dX_next, const void* dx_in,
                        int64_t T, int n, int C, int t_iters, float eps, void* dX, void* dF_out,
                        float* dphi, float* dalpha, float* db, void* workspace,
                        size_t workspace_bytes, void* stream);

/*
 * mhc_backward_noalloc -- mhc_backward without a caller workspace.  The pages
 * have no counterpart to this entry point; it exists for callers that cannot
 * allocate device memory (code running while a CUDA graph is being captured,
 * a custom allocator's own callbacks, or an embedding runtime that owns all
 * allocations and forbids libraries to make any).
 *
 * Same arguments, results and restrictions as mhc_backward, minus the
 * workspace.  The scratch is a fixed MHC_NOALLOC_SCRATCH_BYTES (4 MiB) array
 * inside the library, held by every GPU that loads the library until the
 * process exits; batches whose mhc_backward_workspace_bytes(T, n, C) exceeds it
 * are rejected with MHC_ERR_UNSUPPORTED (at n = 4: T above about 4,600 at
 * C = 512, 2,000 at C = 2048, 1,024 at C = 4096).
 * No allocating routine is called.  The first call on each device looks up
 * the scratch address and should come before any stream capture.  Every call
 * on a device uses the same scratch: calls whose work overlaps on the GPU
 * race, so order them (one stream, or events).  Nothing in the scratch needs
 * to start at zero; it keeps the previous call's leftovers.
 */
#define MHC_NOALLOC_SCRATCH_BYTES (4u << 20)
mhc_status mhc_backward_noalloc(const void* X, const void* F_out, const void* phi, mhc_dtype dt,
                                const float* alpha, const float* b, const void* dX_next,
                                const void* dx_in, int64_t T, int n, int C, int t_iters, float eps,
                                void* dX, void* dF_out, float* dphi, float* dalpha, float* db,
                                void* stream);

/* Kernel selection for the projection of mhc_pre. */
typedef enum {
    MHC_PATH_AUTO = 0,    /* tensor cores where supported, else CUDA cores (default) */
    MHC_PATH_FMA = 1,     /* always the CUDA-core (FMA) projection                    */
    MHC_PATH_TENSOR = 2   /* always tensor cores; calls it cannot serve return        */
                          /* MHC_ERR_UNSUPPORTED                                       */
} mhc_path;

/*
 * mhc_set_path -- process-wide choice of the projection kernel of mhc_pre,
 * xhc_route and xhc_sparse_update, and of the dphi product of mhc_backward
 * (for comparisons and tests; both paths compute the same function).  The
 * tensor-core paths (TMA + tcgen05.mma) serve bf16 X, 1 <= T < 2^31, and:
 * mhc_pre with bf16 phi, C % 512 == 0 and n in [2, 8], or with the tf32 phi
 * pair and n in [1, 7]; xhc_route with C % 512 == 0 and N in {4, 8, 12, 16};
 * xhc_sparse_update with C % 512 == 0, k = 4 and Kr <= 4; mhc_backward's dphi
 * with n*C % 128 == 0.  Under MHC_PATH_TENSOR an mhc_pre, xhc_route or
 * xhc_sparse_update call outside that range returns MHC_ERR_UNSUPPORTED;
 * MHC_PATH_FMA selects the CUDA-core kernels everywhere.
 */
mhc_status mhc_set_path(mhc_path path);

/*
 * mhc_set_wait_limit -- number of polls after which a bounded on-device wait
 * gives up (default 2^26).  A kernel whose wait expires records it in the
 * device error word, stops, releases what it holds and returns; its outputs
 * are then undefined and mhc_sync_status() reports MHC_ERR_TIMEOUT.  Meant
 * for tests of that failure path; polls >= 1.
 */
mhc_status mhc_set_wait_limit(long long polls);

/*
 * mhc_sync_status -- wait for `stream`, then report and clear the device-side
 * error word: MHC_ERR_TIMEOUT if a kernel of this library gave up a bounded
 * wait since the last call, MHC_ERR_INVALID_ARG if a kernel met an
 * out-of-range stream index in device data, MHC_ERR_CUDA if a kernel found
 * its launch configuration inconsistent (shared memory smaller than its
 * layout, a tile shape it was not written for) and did no work, else MHC_OK
 * (or MHC_ERR_CUDA if the stream itself failed).
 */
mhc_status mhc_sync_status(void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MHC_H */
