// hc_pre: the coefficients of the HC (tanh) parameterisation and the F_pre
// input, CUDA cores; and mhc_amax_gain, the Amax Gain Magnitude of a stack of
// residual maps.
//
// [mHC] section 3 Eq.(5): RMSNorm acts on the last dimension, so every stream s
// of the token is normalised on its own, x~_s = x_s / r_s with
// r_s = sqrt(mean_c x_s[c]^2 + eps); the dynamic maps are projections of x~_s by
// theta_pre, theta_post (1 x C) and the rows of theta_res (n x C), through tanh,
// times the gate factor, plus the static bias:
//   H_pre[s] = a_pre tanh(theta_pre . x~_s) + b_pre[s],
//   H_post[s] = a_post tanh(theta_post . x~_s) + b_post[s],
//   H_res[a][s] = a_res tanh(theta_res[a] . x~_s) + b_res[a][s];
// Eq.(3): x_in = H_pre x.  As in the mHC kernels the division by the norm comes
// after the projection: theta_q . x~_s = (theta_q . x_s) / r_s.
//
// One warp per token.  Per 16-byte step a lane loads the n+2 projection rows
// once (every stream uses them; 48 KB at n = 4, C = 4096 in bf16, so they stay in
// L1) and the n stream vectors, and keeps n (n+3) fp32 sums: per stream the n+2
// projections and the sum of squares.  A transposed butterfly (31 shuffles per
// 32 sums, instead of 5 per sum) leaves sum j on lane j mod 32; the lanes holding
// a projection form its coefficient.  The token's rows are read again (L1 / L2
// hits) for x_in.
//
// The Amax Gain Magnitude ([mHC] section 3.1) of the composite map of Eq.(4),
// M_d = H_res[d-1] ... H_res[0]: one thread per token carries M (n x n fp32) through
// the layers, and after each layer writes max_i |row sum i| (forward) and
// max_j |column sum j| (backward); the maxima over the tokens are reduced per warp
// and per block and reach the output through atomicMax on the bit patterns
// (non-negative floats order like their bits, so the result does not depend on
// the order).
#include "common.cuh"
#include "internal.h"

namespace mhc {
namespace hc {

template <int N, typename TX, typename TT>
__global__ void __launch_bounds__(256)
hc_pre_kernel(const TX* __restrict__ X, const TT* __restrict__ theta, float a0, float a1, float a2,
              const float* __restrict__ b, int64_t T, int C, float eps, TX* __restrict__ x_in,
              float* __restrict__ Hpre, float* __restrict__ Hpost, float* __restrict__ Hres)
{
    constexpr int Q = N + 2;                // projection rows: pre, post, res_0 .. res_{N-1}
    constexpr int S = N + 3;                // sums per stream: the Q projections, then sum x^2
    constexpr int V = N * S;
    constexpr int G = (V + 31) / 32;        // groups of 32 sums
    constexpr int W = Vec<TX>::W;           // X elements per 16-byte load
    constexpr int TW = 16 / int(sizeof(TT));  // theta elements per 16-byte load
    static_assert(W % TW == 0, "a step of X covers whole 16-byte loads of theta");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = int64_t(blockIdx.x) * (blockDim.x >> 5) + warp;
    if (t >= T) return;                     // whole warp leaves together
    const TX* x = X + t * N * int64_t(C);

    float acc[G * 32];
#pragma unroll
    for (int j = 0; j < G * 32; ++j) acc[j] = 0.0f;
    for (int c0 = lane * W; c0 < C; c0 += 32 * W) {
        float th[Q][W];
#pragma unroll
        for (int q = 0; q < Q; ++q)
#pragma unroll
            for (int h = 0; h < W; h += TW) {
                float tv[TW];
                load16<false>(theta + int64_t(q) * C + c0 + h, tv);
#pragma unroll
                for (int e = 0; e < TW; ++e) th[q][h + e] = tv[e];
            }
#pragma unroll
        for (int s = 0; s < N; ++s) {
            float xv[W];
            load16<false>(x + int64_t(s) * C + c0, xv);
#pragma unroll
            for (int e = 0; e < W; ++e) {
                acc[s * S + Q] = fmaf(xv[e], xv[e], acc[s * S + Q]);
#pragma unroll
                for (int q = 0; q < Q; ++q) acc[s * S + q] = fmaf(xv[e], th[q][e], acc[s * S + q]);
            }
        }
    }

    // transposed butterfly: at offset o a lane keeps the half of its sums selected
    // by bit o of its lane index and adds the partner's copy of that half
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float* v = acc + g * 32;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const bool up = (lane & o) != 0;
#pragma unroll
            for (int i = 0; i < o; ++i) {
                const float send = up ? v[i] : v[i + o];
                const float keep = up ? v[i + o] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
        }
    }
    // acc[g * 32] of lane l now holds sum j = 32 g + l

    const float inv_C = 1.0f / float(C);
    float coef[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const int j = g * 32 + lane;
        const int s = j / S, q = j % S;
        const int js = s * S + Q;           // where stream s's sum of squares lives
        float ss = 0.0f;
#pragma unroll
        for (int g2 = 0; g2 < G; ++g2) {
            const float v2 = __shfl_sync(0xffffffffu, acc[g2 * 32], js & 31);
            if ((js >> 5) == g2) ss = v2;
        }
        coef[g] = 0.0f;
        if (j < V && q < Q) {
            const float z = acc[g * 32] / sqrtf(ss * inv_C + eps);
            const float th = tanhf(z);
            if (q == 0) {
                coef[g] = a0 * th + b[s];
                if (Hpre) Hpre[t * N + s] = coef[g];
            } else if (q == 1) {
                Hpost[t * N + s] = a1 * th + b[N + s];
            } else {
                const int a = q - 2;
                Hres[(t * N + a) * N + s] = a2 * th + b[2 * N + a * N + s];
            }
        }
    }
    float hp[N];
#pragma unroll
    for (int s = 0; s < N; ++s) hp[s] = __shfl_sync(0xffffffffu, coef[(s * S) >> 5], (s * S) & 31);

    TX* out = x_in + t * int64_t(C);
    for (int c0 = lane * W; c0 < C; c0 += 32 * W) {
        float o[W];
#pragma unroll
        for (int e = 0; e < W; ++e) o[e] = 0.0f;
#pragma unroll
        for (int s = 0; s < N; ++s) {
            float xv[W];
            load16<false>(x + int64_t(s) * C + c0, xv);
#pragma unroll
            for (int e = 0; e < W; ++e) o[e] = fmaf(hp[s], xv[e], o[e]);
        }
        store16<true>(out + c0, o);
    }
}

template <int N, typename TX, typename TT>
static mhc_status launch_hc(const HcArgs& a, cudaStream_t s)
{
    const unsigned blocks = unsigned((a.T + 7) / 8);
    hc_pre_kernel<N, TX, TT><<<blocks, 256, 0, s>>>(
        static_cast<const TX*>(a.X), static_cast<const TT*>(a.theta), a.alpha[0], a.alpha[1], a.alpha[2], a.b,
        a.T, a.C, a.eps, static_cast<TX*>(a.x_in), a.H_pre, a.H_post, a.H_res);
    return launch_status("hc_pre");
}

template <typename TX, typename TT>
static mhc_status launch_hc_t(const HcArgs& a, cudaStream_t s)
{
    switch (a.n) {
        case 1: return launch_hc<1, TX, TT>(a, s);
        case 2: return launch_hc<2, TX, TT>(a, s);
        case 3: return launch_hc<3, TX, TT>(a, s);
        case 4: return launch_hc<4, TX, TT>(a, s);
        case 5: return launch_hc<5, TX, TT>(a, s);
        case 6: return launch_hc<6, TX, TT>(a, s);
        case 7: return launch_hc<7, TX, TT>(a, s);
        case 8: return launch_hc<8, TX, TT>(a, s);
        default: break;
    }
    set_error("hc_pre: n=%d not supported", a.n);
    return MHC_ERR_UNSUPPORTED;
}

// ------------------------------------------------------------------ Amax Gain

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

template <int N>
__device__ __forceinline__ void load_layer(const float* __restrict__ h, float (&Hl)[N * N]) {
    if constexpr ((N * N) % 4 == 0) {       // a token's n*n floats are 16-byte aligned
#pragma unroll
        for (int e = 0; e < N * N; e += 4) {
            const float4 v = __ldcs(reinterpret_cast<const float4*>(h + e));
            Hl[e] = v.x; Hl[e + 1] = v.y; Hl[e + 2] = v.z; Hl[e + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int e = 0; e < N * N; ++e) Hl[e] = __ldcs(h + e);
    }
}

// Persistent blocks walk groups of 256 tokens.  The maxima over tokens are
// reduced per warp (shuffles), then per block in shared memory (bmax [L][2], when
// it fits), and each block adds its L x 2 maxima to gmax with one global atomic
// per entry at the end, instead of one per warp and layer on the same few
// addresses.
template <int N>
__global__ void __launch_bounds__(256)
amax_gain_kernel(const float* __restrict__ H, int L, int64_t T, float* __restrict__ gain,
                 unsigned int* __restrict__ gmax, int block_max)
{
    extern __shared__ unsigned int bmax[];
    const bool use_b = gmax && block_max;
    if (use_b) {
        for (int i = threadIdx.x; i < 2 * L; i += blockDim.x) bmax[i] = 0u;
        __syncthreads();
    }
    for (int64_t base = int64_t(blockIdx.x) * blockDim.x; base < T; base += int64_t(gridDim.x) * blockDim.x) {
        const int64_t t = base + threadIdx.x;
        const bool live = t < T;           // idle threads still join the warp maxima
        float M[N][N];
#pragma unroll
        for (int i = 0; i < N; ++i)
#pragma unroll
            for (int j = 0; j < N; ++j) M[i][j] = i == j ? 1.0f : 0.0f;
        for (int l = 0; l < L; ++l) {
            float fw = 0.0f, bw = 0.0f;
            if (live) {
                float Hl[N * N];
                load_layer<N>(H + (int64_t(l) * T + t) * (N * N), Hl);
                float P[N][N];               // M <- H_res[l] M
#pragma unroll
                for (int i = 0; i < N; ++i)
#pragma unroll
                    for (int j = 0; j < N; ++j) {
                        float acc = 0.0f;
#pragma unroll
                        for (int k = 0; k < N; ++k) acc = fmaf(Hl[i * N + k], M[k][j], acc);
                        P[i][j] = acc;
                    }
#pragma unroll
                for (int i = 0; i < N; ++i)
#pragma unroll
                    for (int j = 0; j < N; ++j) M[i][j] = P[i][j];
#pragma unroll
                for (int i = 0; i < N; ++i) {
                    float rs = 0.0f, cs = 0.0f;
#pragma unroll
                    for (int j = 0; j < N; ++j) {
                        rs += M[i][j];
                        cs += M[j][i];
                    }
                    if (fabsf(rs) > fw) fw = fabsf(rs);
                    if (fabsf(cs) > bw) bw = fabsf(cs);
                }
                if (gain) *reinterpret_cast<float2*>(gain + (int64_t(l) * T + t) * 2) = make_float2(fw, bw);
            }
            if (gmax) {
                fw = warp_max(fw);
                bw = warp_max(bw);
                if ((threadIdx.x & 31) == 0) {
                    unsigned int* dst = use_b ? bmax : gmax;
                    atomicMax(dst + 2 * l, __float_as_uint(fw));
                    atomicMax(dst + 2 * l + 1, __float_as_uint(bw));
                }
            }
        }
    }
    if (use_b) {
        __syncthreads();
        for (int i = threadIdx.x; i < 2 * L; i += blockDim.x)
            if (bmax[i]) atomicMax(gmax + i, bmax[i]);
    }
}

}  // namespace hc

mhc_status launch_hc_pre(const HcArgs& a, cudaStream_t s)
{
    if (a.x_dt == MHC_BF16 && a.t_dt == MHC_BF16) return hc::launch_hc_t<bf16_t, bf16_t>(a, s);
    if (a.x_dt == MHC_F32 && a.t_dt == MHC_F32) return hc::launch_hc_t<float, float>(a, s);
    if (a.x_dt == MHC_BF16 && a.t_dt == MHC_F32) return hc::launch_hc_t<bf16_t, float>(a, s);
    set_error("hc_pre: fp32 X with bf16 theta is not supported");
    return MHC_ERR_UNSUPPORTED;
}

mhc_status launch_amax_gain(const float* H, int L, int64_t T, int n, float* gain, float* gain_max,
                            cudaStream_t s)
{
    unsigned int* gm = reinterpret_cast<unsigned int*>(gain_max);
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_status(e, "mhc_amax_gain: SM count");
    }
    // two resident blocks per SM, each walking groups of 256 tokens; the block
    // maxima live in shared memory up to L = 6144 layers (48 KB)
    const int64_t groups = (T + 255) / 256;
    const unsigned blocks = unsigned(groups < 2 * sms ? groups : 2 * sms);
    const int block_max = L <= 6144 ? 1 : 0;
    const size_t shm = gain_max && block_max ? size_t(L) * 2 * 4 : 0;
    switch (n) {
#define MHC_AMAX_CASE(K) \
        case K: hc::amax_gain_kernel<K><<<blocks, 256, shm, s>>>(H, L, T, gain, gm, block_max); break;
        MHC_AMAX_CASE(1) MHC_AMAX_CASE(2) MHC_AMAX_CASE(3) MHC_AMAX_CASE(4)
        MHC_AMAX_CASE(5) MHC_AMAX_CASE(6) MHC_AMAX_CASE(7) MHC_AMAX_CASE(8)
#undef MHC_AMAX_CASE
        default:
            set_error("mhc_amax_gain: n=%d not supported", n);
            return MHC_ERR_UNSUPPORTED;
    }
    return launch_status("mhc_amax_gain");
}

}  // namespace mhc
