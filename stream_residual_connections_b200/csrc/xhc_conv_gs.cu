// xhc_conv_gs: temporal feature augmentation of the xHC write-back.
//
// [xHC] section "temporal feature augmentation": r causal depthwise 1-D
// convolutions of the sublayer output (kernel sizes kappa_j) give the
// components g_j; together with out they are orthogonalised per token by
// (modified) Gram-Schmidt over the C channels:
//     a_0 = out[t],  a_j[c] = sum_{s < kappa_j} w_j[s][c] * out[t-s][c]   (zero before the sequence start)
//     V[t] = (v_0, ..., v_r),  v_j = a_j - sum_{i<j} <a_j, v_i>/<v_i, v_i> v_i
//
// The GPU forms the same vectors from the per-token Gram matrix G = A^T A
// (one reduction over C for all Kr(Kr+1)/2 inner products): with G = L D L^T
// (L unit lower triangular), V = A L^{-T}, which is exactly Gram-Schmidt's
// result in exact arithmetic (V^T V = D is diagonal and v_j - a_j lies in the
// span of a_0..a_{j-1}); a pivot D_j = 0 (a_j already in the span) gives
// v_j = 0 and contributes nothing afterwards, as in MGS.
//
// One block of 256 threads per tile of 8 consecutive tokens; a thread owns
// 8 channels at a time.  Pass 1 forms the components (each input row loaded
// once for all convolutions; rows and weights are L1/L2-resident) and
// accumulates the Gram partials, the block reduces them, pass 2 writes V in
// fp32 from the components kept in registers (C <= 2048) or recomputed.
#include "common.cuh"
#include "internal.h"

namespace mhc {

namespace convgs {

constexpr int THREADS = 256;
constexpr int TILE = 8;
constexpr int MAXR = 4;

template <typename TF>
__device__ __forceinline__ void load8(const TF* p, float (&v)[8]);
template <>
__device__ __forceinline__ void load8<bf16_t>(const bf16_t* p, float (&v)[8]) { load16<false>(p, v); }
template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&v)[8]) {
    float a[4], b[4];
    load16<false>(p, a);
    load16<false>(p + 4, b);
#pragma unroll
    for (int e = 0; e < 4; ++e) { v[e] = a[e]; v[4 + e] = b[e]; }
}

struct Params {
    int kap[MAXR];
    int64_t woff[MAXR];
};

// a[0..R][8] for token t, channels c..c+7.  Each of the max kappa input rows
// out[t-s] is loaded once and feeds every convolution that reaches it.
template <int R, typename TF>
__device__ __forceinline__ void components(const TF* __restrict__ F, const float* __restrict__ W,
                                           const Params& prm, int64_t t, int64_t pos, int C, int c,
                                           float (&a)[R + 1][8])
{
    load8<TF>(F + t * C + c, a[0]);
#pragma unroll
    for (int j = 0; j < R; ++j)
#pragma unroll
        for (int e = 0; e < 8; ++e) a[j + 1][e] = 0.0f;
    int kmax = 0;
#pragma unroll
    for (int j = 0; j < R; ++j) kmax = prm.kap[j] > kmax ? prm.kap[j] : kmax;
    for (int s = 0; s < kmax && s <= pos; ++s) {
        float f[8];
        if (s == 0) {
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = a[0][e];
        } else {
            load8<TF>(F + (t - s) * C + c, f);
        }
#pragma unroll
        for (int j = 0; j < R; ++j) {
            if (s < prm.kap[j]) {
                float w0[4], w1[4];
                const float* wp = W + prm.woff[j] + int64_t(s) * C + c;
                load16<false>(wp, w0);
                load16<false>(wp + 4, w1);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    a[j + 1][e] = fmaf(w0[e], f[e], a[j + 1][e]);
                    a[j + 1][4 + e] = fmaf(w1[e], f[4 + e], a[j + 1][4 + e]);
                }
            }
        }
    }
}

template <int R, typename TF>
__global__ void __launch_bounds__(THREADS, 2)
conv_gs_kernel(const TF* __restrict__ F, const float* __restrict__ W, Params prm, int64_t T, int C,
               int64_t seq_len, float* __restrict__ V)
{
    constexpr int KR = R + 1;
    constexpr int NG = KR * (KR + 1) / 2;
    __shared__ float red[THREADS / 32][NG];
    __shared__ float Gs[NG];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int CV = C / 8;
    // a thread that owns a single channel vector keeps its components between the
    // Gram pass and the output pass; otherwise the output pass recomputes them
    const bool one = CV <= THREADS;
    float keep[KR][8];
    for (int tt = 0; tt < TILE; ++tt) {
        const int64_t t = int64_t(blockIdx.x) * TILE + tt;
        if (t >= T) break;                       // uniform across the block
        const int64_t pos = t % seq_len;
        float g[NG];
#pragma unroll
        for (int q = 0; q < NG; ++q) g[q] = 0.0f;
        for (int v = threadIdx.x; v < CV; v += THREADS) {
            float a[KR][8];
            components<R, TF>(F, W, prm, t, pos, C, v * 8, a);
            if (one) {
#pragma unroll
                for (int i = 0; i < KR; ++i)
#pragma unroll
                    for (int e = 0; e < 8; ++e) keep[i][e] = a[i][e];
            }
            int q = 0;
#pragma unroll
            for (int i = 0; i < KR; ++i)
#pragma unroll
                for (int j = 0; j <= i; ++j, ++q)
#pragma unroll
                    for (int e = 0; e < 8; ++e) g[q] = fmaf(a[i][e], a[j][e], g[q]);
        }
#pragma unroll
        for (int q = 0; q < NG; ++q) {
            float x = warp_sum(g[q]);
            if (lane == 0) red[warp][q] = x;
        }
        __syncthreads();
        if (threadIdx.x < NG) {
            float x = 0.0f;
#pragma unroll
            for (int w = 0; w < THREADS / 32; ++w) x += red[w][threadIdx.x];
            Gs[threadIdx.x] = x;
        }
        __syncthreads();
        // G = L D L^T, then Li = L^{-1} (unit lower); v_j = a_j + sum_{i<j} Li[j][i] a_i
        float G[KR][KR], L[KR][KR], D[KR], Li[KR][KR];
        {
            int q = 0;
#pragma unroll
            for (int i = 0; i < KR; ++i)
#pragma unroll
                for (int j = 0; j <= i; ++j, ++q) { G[i][j] = Gs[q]; G[j][i] = Gs[q]; }
        }
#pragma unroll
        for (int j = 0; j < KR; ++j) {
            float d = G[j][j];
#pragma unroll
            for (int k = 0; k < j; ++k) d -= L[j][k] * L[j][k] * D[k];
            D[j] = d;
            L[j][j] = 1.0f;
#pragma unroll
            for (int i = j + 1; i < KR; ++i) {
                float x = G[i][j];
#pragma unroll
                for (int k = 0; k < j; ++k) x -= L[i][k] * L[j][k] * D[k];
                L[i][j] = d > 0.0f ? x / d : 0.0f;
            }
#pragma unroll
            for (int i = 0; i < j; ++i) L[i][j] = 0.0f;
        }
#pragma unroll
        for (int j = 0; j < KR; ++j) {
#pragma unroll
            for (int i = 0; i < KR; ++i) Li[j][i] = (i == j) ? 1.0f : 0.0f;
#pragma unroll
            for (int i = 0; i < j; ++i) {
                float x = 0.0f;
#pragma unroll
                for (int k = i; k < j; ++k) x -= L[j][k] * Li[k][i];
                Li[j][i] = x;
            }
        }
        for (int v = threadIdx.x; v < CV; v += THREADS) {
            float a[KR][8];
            if (one) {
#pragma unroll
                for (int i = 0; i < KR; ++i)
#pragma unroll
                    for (int e = 0; e < 8; ++e) a[i][e] = keep[i][e];
            } else {
                components<R, TF>(F, W, prm, t, pos, C, v * 8, a);
            }
#pragma unroll
            for (int j = 0; j < KR; ++j) {
                float o[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    float x = a[j][e];
#pragma unroll
                    for (int i = 0; i < j; ++i) x = fmaf(Li[j][i], a[i][e], x);
                    o[e] = x;
                }
                float* dst = V + (t * KR + j) * C + v * 8;
                const float lo[4] = {o[0], o[1], o[2], o[3]}, hi[4] = {o[4], o[5], o[6], o[7]};
                store16<true>(dst, lo);
                store16<true>(dst + 4, hi);
            }
        }
        __syncthreads();   // Gs is rewritten for the next token
    }
}

template <int R, typename TF>
static mhc_status launch_r(const void* F, const float* W, const Params& prm, int64_t T, int C,
                           int64_t seq_len, float* V, cudaStream_t s)
{
    const int64_t blocks = (T + TILE - 1) / TILE;
    conv_gs_kernel<R, TF><<<dim3(unsigned(blocks)), THREADS, 0, s>>>(
        static_cast<const TF*>(F), W, prm, T, C, seq_len, V);
    return launch_status("xhc_conv_gs kernel");
}

}  // namespace convgs

mhc_status launch_conv_gs(const void* F, mhc_dtype dt, const float* W, const int* kappa, int r,
                          int64_t T, int C, int64_t seq_len, float* V, cudaStream_t s)
{
    convgs::Params prm{};
    int64_t off = 0;
    for (int j = 0; j < r; ++j) {
        prm.kap[j] = kappa[j];
        prm.woff[j] = off;
        off += int64_t(kappa[j]) * C;
    }
#define MHC_CONV_CASE(RR)                                                                         \
    case RR:                                                                                      \
        return dt == MHC_BF16 ? convgs::launch_r<RR, bf16_t>(F, W, prm, T, C, seq_len, V, s)       \
                              : convgs::launch_r<RR, float>(F, W, prm, T, C, seq_len, V, s);
    switch (r) {
        MHC_CONV_CASE(1) MHC_CONV_CASE(2) MHC_CONV_CASE(3) MHC_CONV_CASE(4)
        default: break;
    }
#undef MHC_CONV_CASE
    set_error("xhc_conv_gs: r=%d not supported (1..4)", r);
    return MHC_ERR_UNSUPPORTED;
}

}  // namespace mhc
