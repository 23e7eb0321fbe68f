// mhc_post: the fused F_post,res apply step of one mHC sublayer.
//
// [mHC] section 3 Eq.(3) and section 4.3.1 (the post/res apply kernel fused
// with the residual merge: (n+1)C elements read, nC written per token):
//     X_next[t][i][:] = sum_j H_res[t][i][j] * X[t][j][:] + H_post[t][i] * F_out[t][:]
//
// Pure streaming, HBM-bound.  One block per token; one thread owns one
// 16-byte column vector of the token across all n streams at a time: it
// issues n+1 independent 16-byte loads (X rows and F_out), mixes them in fp32
// registers with the token's n*n + n coefficients (uniform across the block)
// and issues n 16-byte stores.  Loads and stores use the evict-first policy: every byte is
// touched once.  In-place use (X_next == X) is safe because each thread
// reads its whole column before writing it and no other thread touches it.
#include "common.cuh"
#include "internal.h"

namespace mhc {

// One block per token: the token's coefficients are uniform across the block
// (one broadcast load each, 16-byte vectors where aligned), and each thread
// walks the token's column vectors with a stride of the block size.
template <int N>
__device__ __forceinline__ void load_coeffs(const float* __restrict__ Hpost, const float* __restrict__ Hres,
                                            int64_t t, float (&hp)[N], float (&hr)[N][N]) {
    if constexpr (N % 4 == 0) {
        const float4* h4 = reinterpret_cast<const float4*>(Hpost + t * N);
#pragma unroll
        for (int q = 0; q < N / 4; ++q) {
            const float4 v = __ldg(h4 + q);
            hp[4 * q] = v.x; hp[4 * q + 1] = v.y; hp[4 * q + 2] = v.z; hp[4 * q + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < N; ++i) hp[i] = __ldg(Hpost + t * N + i);
    }
    if constexpr ((N * N) % 4 == 0) {
        const float4* r4 = reinterpret_cast<const float4*>(Hres + t * N * N);
#pragma unroll
        for (int q = 0; q < N * N / 4; ++q) {
            const float4 v = __ldg(r4 + q);
            hr[(4 * q) / N][(4 * q) % N] = v.x;
            hr[(4 * q + 1) / N][(4 * q + 1) % N] = v.y;
            hr[(4 * q + 2) / N][(4 * q + 2) % N] = v.z;
            hr[(4 * q + 3) / N][(4 * q + 3) % N] = v.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < N; ++i)
#pragma unroll
            for (int j = 0; j < N; ++j) hr[i][j] = __ldg(Hres + (t * N + i) * N + j);
    }
}

template <int N, typename T>
__global__ void __launch_bounds__(256, (N <= 4 ? 4 : 2))
post_kernel(const T* X, const T* __restrict__ F, const float* __restrict__ Hpost,
            const float* __restrict__ Hres, int CV, int C, T* Xn)
{
    constexpr int W = Vec<T>::W;
    const int64_t t = blockIdx.x;
    float hp[N], hr[N][N];
    load_coeffs<N>(Hpost, Hres, t, hp, hr);
    for (int v = threadIdx.x; v < CV; v += blockDim.x) {
        const int c0 = v * W;
        float x[N][W], f[W];
#pragma unroll
        for (int j = 0; j < N; ++j) load16<true>(X + (t * N + j) * C + c0, x[j]);
        load16<true>(F + t * C + c0, f);
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
    const int CV = C / W;
    const int threads = CV >= 256 ? 256 : ((CV + 31) / 32) * 32;
    if (T_ > 0x7FFFFFFF) {
        set_error("mhc_post: T=%lld exceeds the grid limit", (long long)T_);
        return MHC_ERR_UNSUPPORTED;
    }
    post_kernel<N, T><<<dim3(unsigned(T_)), threads, 0, s>>>(
        static_cast<const T*>(X), static_cast<const T*>(F), Hpost, Hres, CV, C, static_cast<T*>(Xn));
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
