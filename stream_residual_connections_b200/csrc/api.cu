// C ABI of libmhc: argument validation, dispatch, error reporting.
// Declarations and the contract of every entry point are in include/mhc.h.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace mhc {

static thread_local char g_msg[512] = "";

void set_error(const char* fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
    va_end(ap);
}

mhc_status cuda_status(cudaError_t e, const char* what)
{
    if (e == cudaSuccess) return MHC_OK;
    set_error("%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
    return MHC_ERR_CUDA;
}

mhc_status launch_status(const char* what) { return cuda_status(cudaGetLastError(), what); }

int g_pre_path = MHC_PATH_AUTO;

}  // namespace mhc

using namespace mhc;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t dt_size(mhc_dtype d) { return d == MHC_BF16 ? 2 : 4; }

bool valid_dt(mhc_dtype d) { return d == MHC_BF16 || d == MHC_F32; }

struct Range {
    uintptr_t lo, hi;
};
Range range_of(const void* p, size_t bytes)
{
    uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return Range{a, a + bytes};
}
bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi && a.hi > a.lo && b.hi > b.lo; }

#define REQUIRE(cond, code, ...)          \
    do {                                  \
        if (!(cond)) {                    \
            set_error(__VA_ARGS__);       \
            return code;                  \
        }                                 \
    } while (0)

#define REQUIRE_PTR(p, name)                                                              \
    do {                                                                                  \
        REQUIRE((p) != nullptr, MHC_ERR_INVALID_ARG, "%s: %s is NULL", fn, name);         \
        REQUIRE(aligned16(p), MHC_ERR_INVALID_ARG, "%s: %s is not 16-byte aligned", fn, name); \
    } while (0)

}  // namespace

extern "C" {

const char* mhc_last_error(void) { return g_msg; }

int mhc_version(void) { return 101; }

mhc_status mhc_pre(const void* X, mhc_dtype x_dt, const void* phi, mhc_dtype phi_dt,
                   const float* alpha, const float* b, int64_t T, int n, int C, int t_iters,
                   float eps, void* x_in, float* H_pre, float* H_post, float* H_res,
                   void* stream)
{
    const char* fn = "mhc_pre";
    g_msg[0] = 0;
    const bool pair = phi_dt == MHC_TF32_PAIR;
    REQUIRE(valid_dt(x_dt) && (valid_dt(phi_dt) || pair), MHC_ERR_INVALID_ARG, "%s: unknown dtype", fn);
    REQUIRE(n >= 1 && n <= 8, MHC_ERR_INVALID_ARG, "%s: n=%d outside [1, 8]", fn, n);
    REQUIRE(C > 0 && C % 8 == 0, MHC_ERR_INVALID_ARG, "%s: C=%d must be a positive multiple of 8", fn, C);
    REQUIRE(T >= 0, MHC_ERR_INVALID_ARG, "%s: T=%lld < 0", fn, (long long)T);
    REQUIRE(t_iters >= 0 && t_iters <= 1000, MHC_ERR_INVALID_ARG, "%s: t_iters=%d outside [0, 1000]", fn, t_iters);
    REQUIRE(eps >= 0.0f, MHC_ERR_INVALID_ARG, "%s: eps < 0", fn);
    REQUIRE(alpha != nullptr, MHC_ERR_INVALID_ARG, "%s: alpha (host float[3]) is NULL", fn);
    REQUIRE(!(x_dt == MHC_F32 && phi_dt == MHC_BF16), MHC_ERR_UNSUPPORTED,
            "%s: fp32 X with bf16 phi is not supported", fn);
    REQUIRE(!(x_dt == MHC_F32 && pair), MHC_ERR_UNSUPPORTED, "%s: the tf32 phi pair needs bf16 X", fn);
    if (T == 0) return MHC_OK;
    REQUIRE_PTR(X, "X");
    REQUIRE_PTR(phi, "phi");
    REQUIRE_PTR(b, "b");
    REQUIRE_PTR(x_in, "x_in");
    REQUIRE_PTR(H_post, "H_post");
    REQUIRE_PTR(H_res, "H_res");
    if (H_pre) REQUIRE(aligned16(H_pre), MHC_ERR_INVALID_ARG, "%s: H_pre is not 16-byte aligned", fn);
    const int P = n * n + 2 * n;
    const size_t es = dt_size(x_dt);
    const size_t phi_bytes = pair ? size_t(2 * tf32_pair_half_rows(n)) * n * C * 2 : size_t(n) * C * P * dt_size(phi_dt);
    const Range rX = range_of(X, size_t(T) * n * C * es), rphi = range_of(phi, phi_bytes),
                rb = range_of(b, size_t(P) * 4);
    const Range outs[4] = {range_of(x_in, size_t(T) * C * es), range_of(H_pre, H_pre ? size_t(T) * n * 4 : 0),
                           range_of(H_post, size_t(T) * n * 4), range_of(H_res, size_t(T) * n * n * 4)};
    for (int i = 0; i < 4; ++i) {
        REQUIRE(!overlap(outs[i], rX) && !overlap(outs[i], rphi) && !overlap(outs[i], rb),
                MHC_ERR_INVALID_ARG, "%s: an output overlaps an input", fn);
        for (int j = 0; j < i; ++j)
            REQUIRE(!overlap(outs[i], outs[j]), MHC_ERR_INVALID_ARG, "%s: outputs overlap", fn);
    }
    PreArgs a{X, x_dt, phi, phi_dt, {alpha[0], alpha[1], alpha[2]}, b, T, n, C, t_iters, eps,
              x_in, H_pre, H_post, H_res};
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool tc_ok = pre_tc_supported(a), wide_ok = pre_wide_supported(a);
    if (g_pre_path == MHC_PATH_TENSOR && !tc_ok && !wide_ok) {
        set_error("%s: the tensor-core path was forced but does not support this call "
                  "(needs bf16 X, bf16 phi with n in [2, 8] or the tf32 phi pair with n <= 7, "
                  "C %% 512 == 0)", fn);
        return MHC_ERR_UNSUPPORTED;
    }
    if (tc_ok && g_pre_path != MHC_PATH_FMA) return launch_pre_tc(a, s);
    if (wide_ok && g_pre_path != MHC_PATH_FMA) return launch_pre_wide(a, s);
    return launch_pre_fma(a, s);
}

mhc_status mhc_post(const void* X, const void* F_out, mhc_dtype dt, const float* H_post,
                    const float* H_res, int64_t T, int n, int C, void* X_next, void* stream)
{
    const char* fn = "mhc_post";
    g_msg[0] = 0;
    REQUIRE(valid_dt(dt), MHC_ERR_INVALID_ARG, "%s: unknown dtype", fn);
    REQUIRE(n >= 1 && n <= 8, MHC_ERR_INVALID_ARG, "%s: n=%d outside [1, 8]", fn, n);
    REQUIRE(C > 0 && C % 8 == 0, MHC_ERR_INVALID_ARG, "%s: C=%d must be a positive multiple of 8", fn, C);
    REQUIRE(T >= 0, MHC_ERR_INVALID_ARG, "%s: T=%lld < 0", fn, (long long)T);
    if (T == 0) return MHC_OK;
    REQUIRE_PTR(X, "X");
    REQUIRE_PTR(F_out, "F_out");
    REQUIRE_PTR(H_post, "H_post");
    REQUIRE_PTR(H_res, "H_res");
    REQUIRE_PTR(X_next, "X_next");
    const size_t es = dt_size(dt);
    const Range rXn = range_of(X_next, size_t(T) * n * C * es);
    REQUIRE(X_next == X || !overlap(rXn, range_of(X, size_t(T) * n * C * es)), MHC_ERR_INVALID_ARG,
            "%s: X_next partially overlaps X (only X_next == X is allowed)", fn);
    REQUIRE(!overlap(rXn, range_of(F_out, size_t(T) * C * es)) &&
                !overlap(rXn, range_of(H_post, size_t(T) * n * 4)) &&
                !overlap(rXn, range_of(H_res, size_t(T) * n * n * 4)),
            MHC_ERR_INVALID_ARG, "%s: X_next overlaps F_out or a coefficient array", fn);
    return launch_post(X, F_out, dt, H_post, H_res, T, n, C, X_next, static_cast<cudaStream_t>(stream));
}

mhc_status hc_pre(const void* X, mhc_dtype x_dt, const void* theta, mhc_dtype theta_dt, const float* alpha,
                  const float* b, int64_t T, int n, int C, float eps, void* x_in, float* H_pre, float* H_post,
                  float* H_res, void* stream)
{
    const char* fn = "hc_pre";
    g_msg[0] = 0;
    REQUIRE(valid_dt(x_dt) && valid_dt(theta_dt), MHC_ERR_INVALID_ARG, "%s: unknown dtype", fn);
    REQUIRE(n >= 1 && n <= 8, MHC_ERR_INVALID_ARG, "%s: n=%d outside [1, 8]", fn, n);
    REQUIRE(C > 0 && C % 8 == 0, MHC_ERR_INVALID_ARG, "%s: C=%d must be a positive multiple of 8", fn, C);
    REQUIRE(T >= 0, MHC_ERR_INVALID_ARG, "%s: T=%lld < 0", fn, (long long)T);
    REQUIRE(eps >= 0.0f, MHC_ERR_INVALID_ARG, "%s: eps < 0", fn);
    REQUIRE(alpha != nullptr, MHC_ERR_INVALID_ARG, "%s: alpha (host float[3]) is NULL", fn);
    REQUIRE(!(x_dt == MHC_F32 && theta_dt == MHC_BF16), MHC_ERR_UNSUPPORTED,
            "%s: fp32 X with bf16 theta is not supported", fn);
    if (T == 0) return MHC_OK;
    REQUIRE_PTR(X, "X");
    REQUIRE_PTR(theta, "theta");
    REQUIRE_PTR(b, "b");
    REQUIRE_PTR(x_in, "x_in");
    REQUIRE_PTR(H_post, "H_post");
    REQUIRE_PTR(H_res, "H_res");
    if (H_pre) REQUIRE(aligned16(H_pre), MHC_ERR_INVALID_ARG, "%s: H_pre is not 16-byte aligned", fn);
    const int P = n * n + 2 * n;
    const size_t es = dt_size(x_dt);
    const Range rX = range_of(X, size_t(T) * n * C * es), rth = range_of(theta, size_t(n + 2) * C * dt_size(theta_dt)),
                rb = range_of(b, size_t(P) * 4);
    const Range outs[4] = {range_of(x_in, size_t(T) * C * es), range_of(H_pre, H_pre ? size_t(T) * n * 4 : 0),
                           range_of(H_post, size_t(T) * n * 4), range_of(H_res, size_t(T) * n * n * 4)};
    for (int i = 0; i < 4; ++i) {
        REQUIRE(!overlap(outs[i], rX) && !overlap(outs[i], rth) && !overlap(outs[i], rb),
                MHC_ERR_INVALID_ARG, "%s: an output overlaps an input", fn);
        for (int j = 0; j < i; ++j)
            REQUIRE(!overlap(outs[i], outs[j]), MHC_ERR_INVALID_ARG, "%s: outputs overlap", fn);
    }
    HcArgs a{X, x_dt, theta, theta_dt, {alpha[0], alpha[1], alpha[2]}, b, T, n, C, eps, x_in, H_pre, H_post, H_res};
    return launch_hc_pre(a, static_cast<cudaStream_t>(stream));
}

size_t mhc_phi_tf32_pair_bytes(int n, int C)
{
    if (n < 1 || n > 8 || C <= 0) return 0;
    return size_t(2 * tf32_pair_half_rows(n)) * n * C * 2;
}

mhc_status mhc_phi_tf32_pair(const float* phi, int n, int C, void* pair, void* stream)
{
    const char* fn = "mhc_phi_tf32_pair";
    g_msg[0] = 0;
    REQUIRE(n >= 1 && n <= 8, MHC_ERR_INVALID_ARG, "%s: n=%d outside [1, 8]", fn, n);
    REQUIRE(C > 0 && C % 8 == 0, MHC_ERR_INVALID_ARG, "%s: C=%d must be a positive multiple of 8", fn, C);
    REQUIRE_PTR(phi, "phi");
    REQUIRE_PTR(pair, "pair");
    const int P = n * n + 2 * n;
    REQUIRE(!overlap(range_of(phi, size_t(P) * n * C * 4), range_of(pair, mhc_phi_tf32_pair_bytes(n, C))),
            MHC_ERR_INVALID_ARG, "%s: pair overlaps phi", fn);
    return launch_phi_tf32_pair(phi, n, C, pair, static_cast<cudaStream_t>(stream));
}

mhc_status mhc_amax_gain(const float* H_res, int L, int64_t T, int n, float* gain, float* gain_max, void* stream)
{
    const char* fn = "mhc_amax_gain";
    g_msg[0] = 0;
    REQUIRE(n >= 1 && n <= 8, MHC_ERR_INVALID_ARG, "%s: n=%d outside [1, 8]", fn, n);
    REQUIRE(L >= 0 && T >= 0, MHC_ERR_INVALID_ARG, "%s: L=%d, T=%lld must be >= 0", fn, L, (long long)T);
    REQUIRE(gain || gain_max, MHC_ERR_INVALID_ARG, "%s: neither gain nor gain_max given", fn);
    if (L == 0) return MHC_OK;
    // every argument is checked before anything is enqueued
    if (gain_max) REQUIRE(aligned16(gain_max), MHC_ERR_INVALID_ARG, "%s: gain_max is not 16-byte aligned", fn);
    if (T > 0) {
        REQUIRE_PTR(H_res, "H_res");
        if (gain) REQUIRE(aligned16(gain), MHC_ERR_INVALID_ARG, "%s: gain is not 16-byte aligned", fn);
        const Range rH = range_of(H_res, size_t(L) * T * n * n * 4);
        const Range rg = range_of(gain, gain ? size_t(L) * T * 2 * 4 : 0),
                    rm = range_of(gain_max, gain_max ? size_t(L) * 8 : 0);
        REQUIRE(!overlap(rg, rH) && !overlap(rm, rH) && !overlap(rg, rm), MHC_ERR_INVALID_ARG,
                "%s: an output overlaps H_res or the other output", fn);
    }
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (gain_max) {
        const mhc_status st = cuda_status(cudaMemsetAsync(gain_max, 0, size_t(L) * 2 * 4, s), fn);
        if (st != MHC_OK) return st;
    }
    if (T == 0) return MHC_OK;
    return launch_amax_gain(H_res, L, T, n, gain, gain_max, s);
}

mhc_status xhc_route(const void* X, mhc_dtype dt, const void* phi_read, const float* alpha_read,
                     const float* b_read, int64_t T, int N, int C, int k, int m, float eps, void* x_in,
                     float* H_pre, float* score, int32_t* idx, float* w, void* stream)
{
    const char* fn = "xhc_route";
    g_msg[0] = 0;
    REQUIRE(valid_dt(dt), MHC_ERR_INVALID_ARG, "%s: unknown dtype", fn);
    REQUIRE(C > 0 && C % 8 == 0, MHC_ERR_INVALID_ARG, "%s: C=%d must be a positive multiple of 8", fn, C);
    REQUIRE(T >= 0, MHC_ERR_INVALID_ARG, "%s: T=%lld < 0", fn, (long long)T);
    REQUIRE(N >= 1 && N <= 32, MHC_ERR_INVALID_ARG, "%s: N=%d outside [1, 32]", fn, N);
    REQUIRE(m >= 0 && m <= k && k <= N, MHC_ERR_INVALID_ARG, "%s: need 0 <= m <= k <= N (k=%d, m=%d)", fn, k, m);
    REQUIRE(eps >= 0.0f, MHC_ERR_INVALID_ARG, "%s: eps < 0", fn);
    REQUIRE(alpha_read != nullptr, MHC_ERR_INVALID_ARG, "%s: alpha_read (host float[2]) is NULL", fn);
    if (T == 0) return MHC_OK;
    REQUIRE_PTR(X, "X");
    REQUIRE_PTR(phi_read, "phi_read");
    REQUIRE(b_read != nullptr, MHC_ERR_INVALID_ARG, "%s: b_read is NULL", fn);
    REQUIRE_PTR(x_in, "x_in");
    REQUIRE(idx != nullptr && w != nullptr, MHC_ERR_INVALID_ARG, "%s: idx or w is NULL", fn);
    const int R = 2 * N - m;
    const size_t es = dt_size(dt);
    const Range ins[3] = {range_of(X, size_t(T) * N * C * es), range_of(phi_read, size_t(R) * N * C * es),
                          range_of(b_read, size_t(R) * 4)};
    const Range outs[5] = {range_of(x_in, size_t(T) * C * es), range_of(H_pre, H_pre ? size_t(T) * N * 4 : 0),
                           range_of(score, score ? size_t(T) * (N - m) * 4 : 0), range_of(idx, size_t(T) * k * 4),
                           range_of(w, size_t(T) * k * 4)};
    for (int o = 0; o < 5; ++o) {
        for (int i = 0; i < 3; ++i)
            REQUIRE(!overlap(outs[o], ins[i]), MHC_ERR_INVALID_ARG, "%s: an output overlaps an input", fn);
        for (int q = 0; q < o; ++q)
            REQUIRE(!overlap(outs[o], outs[q]), MHC_ERR_INVALID_ARG, "%s: outputs overlap", fn);
    }
    RouteArgs a{X, dt, phi_read, {alpha_read[0], alpha_read[1]}, b_read, T, N, C, k, m, eps, x_in, H_pre,
                score, idx, w};
    return launch_route(a, static_cast<cudaStream_t>(stream));
}

mhc_status xhc_conv_gs(const void* F_out, mhc_dtype dt, const float* conv_w, const int* kappa,
                       int r, int64_t T, int C, int64_t seq_len, float* V, void* stream)
{
    const char* fn = "xhc_conv_gs";
    g_msg[0] = 0;
    REQUIRE(valid_dt(dt), MHC_ERR_INVALID_ARG, "%s: unknown dtype", fn);
    REQUIRE(C > 0 && C % 8 == 0, MHC_ERR_INVALID_ARG, "%s: C=%d must be a positive multiple of 8", fn, C);
    REQUIRE(T >= 0, MHC_ERR_INVALID_ARG, "%s: T=%lld < 0", fn, (long long)T);
    REQUIRE(r >= 1 && r <= 4, MHC_ERR_INVALID_ARG, "%s: r=%d outside [1, 4]", fn, r);
    REQUIRE(kappa != nullptr, MHC_ERR_INVALID_ARG, "%s: kappa (host int[r]) is NULL", fn);
    int64_t wtot = 0;
    for (int j = 0; j < r; ++j) {
        REQUIRE(kappa[j] >= 1 && kappa[j] <= 64, MHC_ERR_INVALID_ARG, "%s: kappa[%d]=%d outside [1, 64]", fn, j, kappa[j]);
        wtot += int64_t(kappa[j]) * C;
    }
    if (T == 0) return MHC_OK;
    REQUIRE(seq_len >= 1, MHC_ERR_INVALID_ARG, "%s: seq_len=%lld < 1", fn, (long long)seq_len);
    REQUIRE_PTR(F_out, "F_out");
    REQUIRE_PTR(conv_w, "conv_w");
    REQUIRE_PTR(V, "V");
    const Range rV = range_of(V, size_t(T) * (r + 1) * C * 4);
    REQUIRE(!overlap(rV, range_of(F_out, size_t(T) * C * dt_size(dt))) &&
                !overlap(rV, range_of(conv_w, size_t(wtot) * 4)),
            MHC_ERR_INVALID_ARG, "%s: V overlaps an input", fn);
    return launch_conv_gs(F_out, dt, conv_w, kappa, r, T, C, seq_len, V, static_cast<cudaStream_t>(stream));
}

mhc_status xhc_sparse_update(void* X, mhc_dtype dt, const float* V, int Kr, const int32_t* idx,
                             const float* w, const void* phi_act, const float* alpha_act,
                             const float* b_act, int64_t T, int N, int C, int k, int t_iters,
                             float eps, float* H_res, float* H_post, void* stream)
{
    const char* fn = "xhc_sparse_update";
    g_msg[0] = 0;
    REQUIRE(valid_dt(dt), MHC_ERR_INVALID_ARG, "%s: unknown dtype", fn);
    REQUIRE(C > 0 && C % 8 == 0, MHC_ERR_INVALID_ARG, "%s: C=%d must be a positive multiple of 8", fn, C);
    REQUIRE(T >= 0, MHC_ERR_INVALID_ARG, "%s: T=%lld < 0", fn, (long long)T);
    REQUIRE(N >= 1 && N <= 64, MHC_ERR_INVALID_ARG, "%s: N=%d outside [1, 64]", fn, N);
    REQUIRE(k >= 1 && k <= N, MHC_ERR_INVALID_ARG, "%s: k=%d outside [1, N]", fn, k);
    REQUIRE(Kr >= 1, MHC_ERR_INVALID_ARG, "%s: Kr=%d < 1", fn, Kr);
    REQUIRE(t_iters >= 0 && t_iters <= 1000, MHC_ERR_INVALID_ARG, "%s: t_iters=%d outside [0, 1000]", fn, t_iters);
    REQUIRE(eps >= 0.0f, MHC_ERR_INVALID_ARG, "%s: eps < 0", fn);
    REQUIRE(alpha_act != nullptr, MHC_ERR_INVALID_ARG, "%s: alpha_act (host float[2]) is NULL", fn);
    REQUIRE(k <= 4 && Kr <= 5, MHC_ERR_UNSUPPORTED, "%s: k=%d, Kr=%d (this library: k <= 4, Kr <= 5)", fn, k, Kr);
    REQUIRE(C % 64 == 0, MHC_ERR_UNSUPPORTED, "%s: C=%d must be a multiple of 64", fn, C);
    if (T == 0) return MHC_OK;
    REQUIRE_PTR(X, "X");
    REQUIRE_PTR(V, "V");
    REQUIRE(idx != nullptr && w != nullptr, MHC_ERR_INVALID_ARG, "%s: idx or w is NULL", fn);
    REQUIRE_PTR(phi_act, "phi_act");
    REQUIRE(b_act != nullptr, MHC_ERR_INVALID_ARG, "%s: b_act is NULL", fn);
    const int Pa = k * k + k * Kr;
    const size_t es = dt_size(dt);
    const Range rX = range_of(X, size_t(T) * N * C * es);
    const Range ins[5] = {range_of(V, size_t(T) * Kr * C * 4), range_of(idx, size_t(T) * k * 4),
                          range_of(w, size_t(T) * k * 4), range_of(phi_act, size_t(Pa) * k * C * es),
                          range_of(b_act, size_t(Pa) * 4)};
    for (int i = 0; i < 5; ++i)
        REQUIRE(!overlap(rX, ins[i]), MHC_ERR_INVALID_ARG, "%s: X overlaps an input", fn);
    const Range outs[2] = {range_of(H_res, H_res ? size_t(T) * k * k * 4 : 0),
                           range_of(H_post, H_post ? size_t(T) * k * Kr * 4 : 0)};
    for (int o = 0; o < 2; ++o) {
        REQUIRE(!overlap(outs[o], rX), MHC_ERR_INVALID_ARG, "%s: a coefficient output overlaps X", fn);
        for (int i = 0; i < 5; ++i)
            REQUIRE(!overlap(outs[o], ins[i]), MHC_ERR_INVALID_ARG, "%s: a coefficient output overlaps an input", fn);
    }
    UpdateArgs a{X, dt, V, Kr, idx, w, phi_act, {alpha_act[0], alpha_act[1]}, b_act, T, N, C, k,
                 t_iters, eps, H_res, H_post};
    return launch_sparse_update(a, static_cast<cudaStream_t>(stream));
}

size_t mhc_backward_workspace_bytes(int64_t T, int n, int C)
{
    const size_t stride = backward_record_stride(n);
    if (T < 0 || C < 0 || stride == 0) return 0;
    const size_t P = size_t(n) * n + 2 * n;
    const int segs = backward_b3_segments(T);
    // per-token records, u and r; the dd^T bf16 pair of the tensor-core dphi product;
    // then the per-segment partial dphi sums
    const size_t floats = size_t(T) * stride + size_t(T) * P + size_t(T);
    const size_t head = ((floats * 4 + 255) / 256) * 256;
    const size_t ddt = ((size_t(64) * size_t(backward_ddt_pitch(T)) * 2 + 255) / 256) * 256;
    const size_t part = segs > 1 ? size_t(segs) * P * size_t(n) * size_t(C) * 4 : 0;
    return head + ddt + part + 256;
}

mhc_status mhc_backward(const void* X, const void* F_out, const void* phi, mhc_dtype dt, const float* alpha,
                        const float* b, const void* dX_next, const void* dx_in, int64_t T, int n, int C,
                        int t_iters, float eps, void* dX, void* dF_out, float* dphi, float* dalpha,
                        float* db, void* workspace, size_t workspace_bytes, void* stream)
{
    const char* fn = "mhc_backward";
    g_msg[0] = 0;
    REQUIRE(valid_dt(dt), MHC_ERR_INVALID_ARG, "%s: unknown dtype", fn);
    REQUIRE(n >= 1 && n <= 8, MHC_ERR_INVALID_ARG, "%s: n=%d outside [1, 8]", fn, n);
    REQUIRE(C > 0 && C % 8 == 0, MHC_ERR_INVALID_ARG, "%s: C=%d must be a positive multiple of 8", fn, C);
    REQUIRE(T >= 0, MHC_ERR_INVALID_ARG, "%s: T=%lld < 0", fn, (long long)T);
    REQUIRE(t_iters >= 0 && t_iters <= 1000, MHC_ERR_INVALID_ARG, "%s: t_iters=%d outside [0, 1000]", fn, t_iters);
    REQUIRE(eps >= 0.0f, MHC_ERR_INVALID_ARG, "%s: eps < 0", fn);
    REQUIRE(alpha != nullptr, MHC_ERR_INVALID_ARG, "%s: alpha (host float[3]) is NULL", fn);
    REQUIRE(n <= 4 && C % 64 == 0 && t_iters <= 100, MHC_ERR_UNSUPPORTED,
            "%s: this library needs n <= 4, C %% 64 == 0, t_iters <= 100", fn);
    const int P = n * n + 2 * n;
    REQUIRE_PTR(dphi, "dphi");
    REQUIRE(dalpha != nullptr && db != nullptr, MHC_ERR_INVALID_ARG, "%s: dalpha or db is NULL", fn);
    if (T == 0) {
        // empty batch: every gradient sum is zero
        cudaStream_t s = static_cast<cudaStream_t>(stream);
        mhc_status st = cuda_status(cudaMemsetAsync(dphi, 0, size_t(P) * n * C * 4, s), fn);
        if (st == MHC_OK) st = cuda_status(cudaMemsetAsync(dalpha, 0, 3 * 4, s), fn);
        if (st == MHC_OK) st = cuda_status(cudaMemsetAsync(db, 0, size_t(P) * 4, s), fn);
        return st;
    }
    REQUIRE_PTR(X, "X");
    REQUIRE_PTR(F_out, "F_out");
    REQUIRE_PTR(phi, "phi");
    REQUIRE(b != nullptr, MHC_ERR_INVALID_ARG, "%s: b is NULL", fn);
    REQUIRE_PTR(dX_next, "dX_next");
    REQUIRE_PTR(dx_in, "dx_in");
    REQUIRE_PTR(dX, "dX");
    REQUIRE_PTR(dF_out, "dF_out");
    REQUIRE(workspace != nullptr && (reinterpret_cast<uintptr_t>(workspace) & 255u) == 0, MHC_ERR_INVALID_ARG,
            "%s: workspace must be non-NULL and 256-byte aligned", fn);
    const size_t need = mhc_backward_workspace_bytes(T, n, C);
    REQUIRE(workspace_bytes >= need, MHC_ERR_INVALID_ARG, "%s: workspace of %zu bytes < %zu needed", fn,
            workspace_bytes, need);
    const size_t es = dt_size(dt);
    const Range ins[8] = {range_of(X, size_t(T) * n * C * es), range_of(F_out, size_t(T) * C * es),
                          range_of(phi, size_t(P) * n * C * es), range_of(b, size_t(P) * 4),
                          range_of(dX_next, size_t(T) * n * C * es), range_of(dx_in, size_t(T) * C * es),
                          range_of(workspace, need), range_of(alpha, 0)};
    const Range outs[5] = {range_of(dX, size_t(T) * n * C * es), range_of(dF_out, size_t(T) * C * es),
                           range_of(dphi, size_t(P) * n * C * 4), range_of(dalpha, 12), range_of(db, size_t(P) * 4)};
    for (int o = 0; o < 5; ++o) {
        for (int i = 0; i < 7; ++i)
            REQUIRE(!overlap(outs[o], ins[i]), MHC_ERR_INVALID_ARG, "%s: an output overlaps an input or the workspace", fn);
        for (int q = 0; q < o; ++q)
            REQUIRE(!overlap(outs[o], outs[q]), MHC_ERR_INVALID_ARG, "%s: outputs overlap", fn);
    }
    float* ws = static_cast<float*>(workspace);
    const size_t stride = backward_record_stride(n);
    const size_t head_floats = (((size_t(T) * stride + size_t(T) * P + size_t(T)) * 4 + 255) / 256) * 256 / 4;
    const size_t ddt_floats = ((size_t(64) * size_t(backward_ddt_pitch(T)) * 2 + 255) / 256) * 256 / 4;
    BwdArgs a{X, F_out, phi, dt, {alpha[0], alpha[1], alpha[2]}, b, dX_next, dx_in, T, n, C, t_iters, eps,
              dX, dF_out, dphi, dalpha, db, ws, ws + size_t(T) * stride, ws + size_t(T) * stride + size_t(T) * P,
              ws + head_floats + ddt_floats, ws + head_floats};
    return launch_backward(a, static_cast<cudaStream_t>(stream));
}

mhc_status mhc_set_path(mhc_path path)
{
    g_msg[0] = 0;
    REQUIRE(path == MHC_PATH_AUTO || path == MHC_PATH_FMA || path == MHC_PATH_TENSOR,
            MHC_ERR_INVALID_ARG, "mhc_set_path: unknown path %d", int(path));
    g_pre_path = path;
    return MHC_OK;
}

mhc_status mhc_set_wait_limit(long long polls)
{
    g_msg[0] = 0;
    REQUIRE(polls >= 1, MHC_ERR_INVALID_ARG, "mhc_set_wait_limit: polls must be >= 1");
    return cuda_status(cudaMemcpyToSymbol(g_wait_limit, &polls, sizeof(polls)), "mhc_set_wait_limit");
}

mhc_status mhc_sync_status(void* stream)
{
    g_msg[0] = 0;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_status(e, "mhc_sync_status");
    unsigned int flag = 0;
    e = cudaMemcpyFromSymbol(&flag, g_device_error, sizeof(flag));
    if (e != cudaSuccess) return cuda_status(e, "mhc_sync_status: read error word");
    if (flag) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
        if (e != cudaSuccess) return cuda_status(e, "mhc_sync_status: clear error word");
        if (flag & 1u) {
            set_error("a bounded on-device wait expired (error word 0x%x)", flag);
            return MHC_ERR_TIMEOUT;
        }
        if (flag & 4u) {
            set_error("a kernel's check of its own launch configuration failed; it did no work "
                      "(error word 0x%x)", flag);
            return MHC_ERR_CUDA;
        }
        set_error("a kernel met an out-of-range stream index; those tokens were left unchanged "
                  "(error word 0x%x)", flag);
        return MHC_ERR_INVALID_ARG;
    }
    return MHC_OK;
}

}  // extern "C"
