// mhc_pre, CUDA-core (FMA) path: one warp per token.
//
// [mHC] section 4.2 Eq.(7)-(9) in the fused order of section 4.3.1
// Eq.(14)-(19): the raw row is projected (Eq.14) while its sum of squares is
// taken in the same pass (Eq.15); the division by r, the gates and the biases
// follow on the P = n*n+2n logits (Eq.16-18); Sinkhorn-Knopp runs in registers
// (Eq.19); the F_pre contraction x_in = H_pre X closes the kernel.
//
// Each lane walks its share of the n*C row 8 (bf16) or 4 (fp32) elements at a
// time, reading the matching columns of every row of phi^T ([P][nC]) with
// 16-byte loads and keeping P fp32 accumulators.  A butterfly reduction gives every lane the full logits, so
// the small coefficient math runs redundantly per lane with no further
// communication.  The row is then re-read (now mostly from L2) for x_in.
//
// This path handles every n in [1, 8], both dtypes and any C % 8 == 0.  Its
// projection costs 2 n C P flops per token on the FMA pipe, which for n >= 4
// is more than the HBM time of the row; the tensor-core path is the fast one.
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace mhc {

// phi storage: float, bf16, or the exact bf16 pair of a tf32 phi (phi_tf32.cu:
// rows hi at p, lo at RH + p); PhiStore is the element type in memory.
struct Tf32Pair {};
template <typename TP> struct PhiStore { using type = TP; };
template <> struct PhiStore<Tf32Pair> { using type = bf16_t; };
template <typename TP> struct PhiVec { static constexpr int W = 16 / sizeof(typename PhiStore<TP>::type); };

// Weights of logit p at columns k..k+W-1 of vec(X) (W = one 16-byte load).
template <typename TP, int P>
__device__ __forceinline__ void load_phi(const typename PhiStore<TP>::type* phiT, int p, int64_t K, int64_t k,
                                         float (&pv)[PhiVec<TP>::W]) {
    if constexpr (std::is_same<TP, Tf32Pair>::value) {
        constexpr int RH = (P + 15) / 16 * 16;
        float lo[PhiVec<TP>::W];
        load16<false>(phiT + int64_t(p) * K + k, pv);
        load16<false>(phiT + int64_t(RH + p) * K + k, lo);
#pragma unroll
        for (int e = 0; e < PhiVec<TP>::W; ++e) pv[e] += lo[e];      // exact: the pair sums to the tf32 value
    } else {
        load16<false>(phiT + int64_t(p) * K + k, pv);
    }
}

template <int N, typename TX, typename TP>
__global__ void __launch_bounds__(256)
pre_fma_kernel(const TX* __restrict__ X, const typename PhiStore<TP>::type* __restrict__ phiT, float a0, float a1, float a2,
               const float* __restrict__ b, int64_t T, int C, int t_iters, float eps,
               TX* __restrict__ x_in, float* __restrict__ Hpre, float* __restrict__ Hpost,
               float* __restrict__ Hres, float* __restrict__ u_out, float* __restrict__ r_out)
{
    constexpr int P = N * N + 2 * N;
    constexpr int W = Vec<TX>::W;            // X elements per 16-byte load
    constexpr int PW = PhiVec<TP>::W;        // phi elements per 16-byte load
    static_assert(W % PW == 0, "a vector step of X must cover whole 16-byte loads of phi");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = int64_t(blockIdx.x) * (blockDim.x >> 5) + warp;
    if (t >= T) return;                       // whole warp leaves together
    const int64_t K = int64_t(N) * C;
    const TX* x = X + t * K;

    float acc[P];
#pragma unroll
    for (int p = 0; p < P; ++p) acc[p] = 0.0f;
    float ss = 0.0f;
    for (int64_t k0 = int64_t(lane) * W; k0 < K; k0 += 32 * W) {
        float xv[W];
        load16<false>(x + k0, xv);
#pragma unroll
        for (int e = 0; e < W; ++e) ss = fmaf(xv[e], xv[e], ss);
#pragma unroll
        for (int p = 0; p < P; ++p) {        // row p of phi^T: the weights of logit p
#pragma unroll
            for (int h = 0; h < W; h += PW) {
                float pv[PW];
                load_phi<TP, P>(phiT, p, K, k0 + h, pv);
#pragma unroll
                for (int e = 0; e < PW; ++e) acc[p] = fmaf(xv[h + e], pv[e], acc[p]);
            }
        }
    }
#pragma unroll
    for (int p = 0; p < P; ++p) acc[p] = warp_sum(acc[p]);
    ss = warp_sum(ss);

    // Eq.(15)-(16): r, then alpha * d / r + b.
    const float r = sqrtf(ss / float(K) + eps);
    const float inv_r = 1.0f / r;
    float hpre[N], hpost[N], m[N][N];
#pragma unroll
    for (int i = 0; i < N; ++i) {
        hpre[i] = sigmoidf_(a0 * acc[i] * inv_r + __ldg(b + i));               // Eq.(17)
        hpost[i] = 2.0f * sigmoidf_(a1 * acc[N + i] * inv_r + __ldg(b + N + i)); // Eq.(18)
    }
#pragma unroll
    for (int i = 0; i < N; ++i)
#pragma unroll
        for (int j = 0; j < N; ++j)
            m[i][j] = a2 * acc[2 * N + i * N + j] * inv_r + __ldg(b + 2 * N + i * N + j);
    sinkhorn_regs<N>(m, t_iters);                                               // Eq.(19)

    if (lane == 0) {
#pragma unroll
        for (int i = 0; i < N; ++i) {
            if (Hpre) Hpre[t * N + i] = hpre[i];
            if (Hpost) Hpost[t * N + i] = hpost[i];
#pragma unroll
            for (int j = 0; j < N; ++j) if (Hres) Hres[(t * N + i) * N + j] = m[i][j];
        }
        if (u_out) {
#pragma unroll
            for (int p = 0; p < P; ++p) u_out[t * P + p] = acc[p] * inv_r;
            r_out[t] = r;
        }
    }
    if (!x_in) return;

    // F_pre: x_in = sum_i H_pre[i] X[i].
    for (int c0 = lane * W; c0 < C; c0 += 32 * W) {
        float o[W];
#pragma unroll
        for (int e = 0; e < W; ++e) o[e] = 0.0f;
#pragma unroll
        for (int i = 0; i < N; ++i) {
            float xv[W];
            load16<false>(x + int64_t(i) * C + c0, xv);
#pragma unroll
            for (int e = 0; e < W; ++e) o[e] = fmaf(hpre[i], xv[e], o[e]);
        }
        store16<false>(x_in + t * C + c0, o);
    }
}

template <int N, typename TX, typename TP>
static mhc_status launch_pre_fma_n(const PreArgs& a, cudaStream_t s)
{
    const int warps = 8;
    const int64_t blocks = (a.T + warps - 1) / warps;
    pre_fma_kernel<N, TX, TP><<<dim3(unsigned(blocks)), warps * 32, 0, s>>>(
        static_cast<const TX*>(a.X), static_cast<const typename PhiStore<TP>::type*>(a.phi), a.alpha[0], a.alpha[1],
        a.alpha[2], a.b, a.T, a.C, a.t_iters, a.eps, a.skip_xin ? nullptr : static_cast<TX*>(a.x_in),
        a.H_pre, a.H_post, a.H_res, a.u_out, a.r_out);
    return launch_status("mhc_pre (fma) kernel");
}

template <int N>
static mhc_status dispatch_dtype(const PreArgs& a, cudaStream_t s)
{
    if (a.x_dt == MHC_F32 && a.phi_dt == MHC_F32) return launch_pre_fma_n<N, float, float>(a, s);
    if (a.x_dt == MHC_BF16 && a.phi_dt == MHC_BF16) return launch_pre_fma_n<N, bf16_t, bf16_t>(a, s);
    if (a.x_dt == MHC_BF16 && a.phi_dt == MHC_F32) return launch_pre_fma_n<N, bf16_t, float>(a, s);
    if (a.x_dt == MHC_BF16 && a.phi_dt == MHC_TF32_PAIR) return launch_pre_fma_n<N, bf16_t, Tf32Pair>(a, s);
    set_error("mhc_pre: dtype pair (x=%d, phi=%d) not supported", int(a.x_dt), int(a.phi_dt));
    return MHC_ERR_UNSUPPORTED;
}

mhc_status launch_pre_fma(const PreArgs& a, cudaStream_t s)
{
    switch (a.n) {
        case 1: return dispatch_dtype<1>(a, s);
        case 2: return dispatch_dtype<2>(a, s);
        case 3: return dispatch_dtype<3>(a, s);
        case 4: return dispatch_dtype<4>(a, s);
        case 5: return dispatch_dtype<5>(a, s);
        case 6: return dispatch_dtype<6>(a, s);
        case 7: return dispatch_dtype<7>(a, s);
        case 8: return dispatch_dtype<8>(a, s);
        default: break;
    }
    set_error("mhc_pre: n=%d not supported", a.n);
    return MHC_ERR_UNSUPPORTED;
}

}  // namespace mhc
