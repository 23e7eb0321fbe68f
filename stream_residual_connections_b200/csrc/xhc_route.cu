// xhc_route: stream routing and dense read of one xHC sublayer.
//
// [xHC] section "sparse residual stream architecture", steps 1-2, and
// "parameterisation":
//   x = vec(X_t) (N*C); r = sqrt(sum(x^2)/(NC) + eps)
//   z = alpha * (x phi_read) / r + b_read   (N pre logits | N-m route logits)
//   H_pre = sigma(z_pre); score_s = sigma(z_route[s-m]) for s = m..N-1
//   active = {0..m-1} U TopK_{k-m}(score) (ties to the lower index), ascending;
//   w = 1 for fixed streams, the score for routed ones
//   x_in = sum_{i<N} H_pre[i] X_t[i]        (dense read over all N streams)
//
// CUDA-core path: one warp per token.  Lanes walk the N*C row 8 elements at a
// time against the 2N-m rows of phi_read^T (16-byte loads), then a butterfly
// gives every lane all logits; lane i owns stream i: its gate, its score, its
// rank among the routed streams (shuffles), and a ballot orders the selected
// streams by index.  The dense read reuses the row while it is in L1/L2.
#include "common.cuh"
#include "internal.h"

namespace mhc {
namespace xroute {

template <int NMAX, typename TX>
__global__ void __launch_bounds__(256)
route_kernel(const TX* __restrict__ X, const TX* __restrict__ phiT, float a_pre, float a_route,
             const float* __restrict__ b, int64_t T, int N, int C, int k, int m, float eps,
             TX* __restrict__ x_in, float* __restrict__ Hpre, float* __restrict__ score,
             int32_t* __restrict__ idx, float* __restrict__ w)
{
    constexpr int PMAX = 2 * NMAX;
    constexpr int W = Vec<TX>::W;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = int64_t(blockIdx.x) * (blockDim.x >> 5) + warp;
    if (t >= T) return;
    const int P = 2 * N - m;
    const int64_t K = int64_t(N) * C;
    const TX* x = X + t * K;

    float acc[PMAX];
#pragma unroll
    for (int p = 0; p < PMAX; ++p) acc[p] = 0.0f;
    float ss = 0.0f;
    for (int64_t k0 = int64_t(lane) * W; k0 < K; k0 += 32 * W) {
        float xv[W];
        load16<false>(x + k0, xv);
#pragma unroll
        for (int e = 0; e < W; ++e) ss = fmaf(xv[e], xv[e], ss);
#pragma unroll
        for (int p = 0; p < PMAX; ++p) {
            if (p < P) {
                float pv[W];
                load16<false>(phiT + int64_t(p) * K + k0, pv);
#pragma unroll
                for (int e = 0; e < W; ++e) acc[p] = fmaf(xv[e], pv[e], acc[p]);
            }
        }
    }
#pragma unroll
    for (int p = 0; p < PMAX; ++p)
        if (p < P) acc[p] = warp_sum(acc[p]);
    ss = warp_sum(ss);
    const float inv_r = 1.0f / sqrtf(ss / float(K) + eps);

    // lane i owns stream i
    float zp = 0.0f, zr = 0.0f;
#pragma unroll
    for (int p = 0; p < PMAX; ++p) {
        if (p == lane) zp = acc[p];
        if (p == N + lane - m) zr = acc[p];
    }
    const bool stream = lane < N;
    const float hp = stream ? sigmoidf_(a_pre * zp * inv_r + __ldg(b + lane)) : 0.0f;
    const bool routed = stream && lane >= m;
    const float sc = routed ? sigmoidf_(a_route * zr * inv_r + __ldg(b + N + lane - m)) : -1.0f;
    int rank = 0;
    for (int s = m; s < N; ++s) {
        const float o = __shfl_sync(0xffffffffu, sc, s);
        if (routed && s != lane && (o > sc || (o == sc && s < lane))) ++rank;
    }
    const bool sel = stream && (lane < m || rank < k - m);
    const unsigned mask = __ballot_sync(0xffffffffu, sel);
    if (sel) {
        const int slot = __popc(mask & ((1u << lane) - 1u));
        idx[t * k + slot] = lane;
        w[t * k + slot] = lane < m ? 1.0f : sc;
    }
    if (stream && Hpre) Hpre[t * N + lane] = hp;
    if (routed && score) score[t * (N - m) + lane - m] = sc;

    // dense read: x_in = sum_i H_pre[i] X[i]  (gates gathered while the whole warp is converged)
    float hall[NMAX];
#pragma unroll
    for (int i = 0; i < NMAX; ++i) hall[i] = __shfl_sync(0xffffffffu, hp, i);
    for (int c0 = lane * W; c0 < C; c0 += 32 * W) {
        float o[W];
#pragma unroll
        for (int e = 0; e < W; ++e) o[e] = 0.0f;
#pragma unroll
        for (int i = 0; i < NMAX; ++i) {
            if (i >= N) break;
            const float h = hall[i];
            float xv[W];
            load16<false>(x + int64_t(i) * C + c0, xv);
#pragma unroll
            for (int e = 0; e < W; ++e) o[e] = fmaf(h, xv[e], o[e]);
        }
        store16<false>(x_in + t * C + c0, o);
    }
}

template <int NMAX>
static mhc_status launch_nmax(const RouteArgs& a, cudaStream_t s)
{
    const int64_t blocks = (a.T + 7) / 8;
    if (a.dt == MHC_BF16)
        route_kernel<NMAX, bf16_t><<<dim3(unsigned(blocks)), 256, 0, s>>>(
            static_cast<const bf16_t*>(a.X), static_cast<const bf16_t*>(a.phi), a.alpha[0], a.alpha[1], a.b,
            a.T, a.N, a.C, a.k, a.m, a.eps, static_cast<bf16_t*>(a.x_in), a.H_pre, a.score, a.idx, a.w);
    else
        route_kernel<NMAX, float><<<dim3(unsigned(blocks)), 256, 0, s>>>(
            static_cast<const float*>(a.X), static_cast<const float*>(a.phi), a.alpha[0], a.alpha[1], a.b,
            a.T, a.N, a.C, a.k, a.m, a.eps, static_cast<float*>(a.x_in), a.H_pre, a.score, a.idx, a.w);
    return launch_status("xhc_route kernel");
}

}  // namespace xroute

mhc_status launch_route(const RouteArgs& a, cudaStream_t s)
{
    // the tensor-core path (xhc_route_tc.cu) where it applies, unless the caller chose the
    // CUDA-core path with mhc_set_path
    const bool tc_ok = route_tc_supported(a);
    if (g_pre_path == MHC_PATH_TENSOR && !tc_ok) {
        set_error("xhc_route: the tensor-core path needs bf16, N in {4, 8, 12, 16} and C %% 512 == 0");
        return MHC_ERR_UNSUPPORTED;
    }
    if (tc_ok && g_pre_path != MHC_PATH_FMA) return launch_route_tc(a, s);
    if (a.N <= 8) return xroute::launch_nmax<8>(a, s);
    if (a.N <= 16) return xroute::launch_nmax<16>(a, s);
    return xroute::launch_nmax<32>(a, s);
}

}  // namespace mhc
