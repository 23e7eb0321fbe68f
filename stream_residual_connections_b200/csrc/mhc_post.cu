// mhc_post: the fused F_post,res apply step of one mHC sublayer.
//
// [mHC] section 3 Eq.(3) and section 4.3.1 (the post/res apply kernel fused
// with the residual merge: (n+1)C elements read, nC written per token):
//     X_next[t][i][:] = sum_j H_res[t][i][j] * X[t][j][:] + H_post[t][i] * F_out[t][:]
//
// Pure streaming, HBM-bound.  One thread owns one 16-byte column vector of a
// token across all n streams: it issues n+1 independent 16-byte loads (X rows
// and F_out), mixes them in fp32 registers with the token's n*n + n
// coefficients (read through L1, shared by the token's threads) and issues n
// 16-byte stores.  Loads and stores use the evict-first policy: every byte is
// touched once.  In-place use (X_next == X) is safe because each thread
// reads its whole column before writing it and no other thread touches it.
#include "common.cuh"
#include "internal.h"

namespace mhc {

template <int N, typename T, int ITEMS>
__global__ void __launch_bounds__(256)
post_kernel(const T* X, const T* __restrict__ F, const float* __restrict__ Hpost,
            const float* __restrict__ Hres, int64_t total, int CV, int C, T* Xn)
{
    constexpr int W = Vec<T>::W;
#pragma unroll
    for (int it = 0; it < ITEMS; ++it) {
        const int64_t w = (int64_t(blockIdx.x) * ITEMS + it) * blockDim.x + threadIdx.x;
        if (w >= total) return;
        const int64_t t = w / CV;
        const int c0 = int(w - t * CV) * W;
        float x[N][W], f[W];
#pragma unroll
        for (int j = 0; j < N; ++j) load16<true>(X + (t * N + j) * C + c0, x[j]);
        load16<true>(F + t * C + c0, f);
        float hr[N][N], hp[N];
#pragma unroll
        for (int i = 0; i < N; ++i) {
            hp[i] = __ldg(Hpost + t * N + i);
#pragma unroll
            for (int j = 0; j < N; ++j) hr[i][j] = __ldg(Hres + (t * N + i) * N + j);
        }
#pragma unroll
        for (int i = 0; i < N; ++i) {
            float o[W];
#pragma unroll
            for (int e = 0; e < W; ++e) {
                float acc = hp[i] * f[e];
#pragma unroll
                for (int j = 0; j < N; ++j) acc = fmaf(hr[i][j], x[j][e], acc);
                o[e] = acc;
            }
            store16<true>(Xn + (t * N + i) * C + c0, o);
        }
    }
}

template <int N, typename T>
static mhc_status launch_post_n(const void* X, const void* F, const float* Hpost,
                                const float* Hres, int64_t T_, int C, void* Xn, cudaStream_t s)
{
    constexpr int W = Vec<T>::W;
    constexpr int ITEMS = 1;
    const int CV = C / W;
    const int64_t total = T_ * CV;
    const int64_t blocks = (total + 256 * ITEMS - 1) / (256 * ITEMS);
    post_kernel<N, T, ITEMS><<<dim3(unsigned(blocks)), 256, 0, s>>>(
        static_cast<const T*>(X), static_cast<const T*>(F), Hpost, Hres, total, CV, C,
        static_cast<T*>(Xn));
    return launch_status("mhc_post kernel");
}

mhc_status launch_post(const void* X, const void* F, mhc_dtype dt, const float* Hpost,
                       const float* Hres, int64_t T_, int n, int C, void* Xn, cudaStream_t s)
{
#define MHC_POST_CASE(NN)                                                                   \
    case NN:                                                                                \
        return dt == MHC_BF16 ? launch_post_n<NN, bf16_t>(X, F, Hpost, Hres, T_, C, Xn, s) \
                              : launch_post_n<NN, float>(X, F, Hpost, Hres, T_, C, Xn, s);
    switch (n) {
        MHC_POST_CASE(1) MHC_POST_CASE(2) MHC_POST_CASE(3) MHC_POST_CASE(4)
        MHC_POST_CASE(5) MHC_POST_CASE(6) MHC_POST_CASE(7) MHC_POST_CASE(8)
        default: break;
    }
#undef MHC_POST_CASE
    set_error("mhc_post: n=%d not supported", n);
    return MHC_ERR_UNSUPPORTED;
}

}  // namespace mhc
