// mhc_backward: gradients of one mHC sublayer (pre + post halves) with the
// Sinkhorn-Knopp iterations unrolled.
//
// [mHC] section 4.3.1: the backward of the projection kernel ("two matmuls"
// without re-loading x) and a Sinkhorn backward that recomputes the
// intermediates on chip and walks all iterations.  Per token, with
// u = (x phi)/r, z = alpha_seg * u + b (the forward's logits):
//   dH_post_i = <dX_next_i, F>,  dH_res_ij = <dX_next_i, X_j>,  dH_pre_i = <dx_in, X_i>
//   dF        = sum_i H_post_i dX_next_i
//   dz_pre = dH_pre * H_pre (1 - H_pre);  dz_post = dH_post * H_post (1 - H_post / 2)
//   dz_res = reverse of M <- T_r(T_c(M)), t_iters times, then * exp(z_res)
//   dd = alpha_seg * dz / r;  dr = -sum_p alpha_seg dz_p u_p / r
//   dX_j = sum_i H_res_ij dX_next_i + H_pre_j dx_in + (phi dd)_j + dr * X_j / (nC r)
//   dphi += x^T dd, db += dz, dalpha_seg += sum_{p in seg} dz_p u_p     (sums over tokens)
//
// Launches (all on the caller's stream, workspace from the caller):
//   B0  the forward projection recomputed by the mhc_pre kernels: u, r per token
//   B1  one block per token: the P dot products, dF, and the per-token
//       coefficient gradients (Sinkhorn forward trace kept in shared memory,
//       then walked backwards) -> workspace
//   B2  dX over 64-token x 64-channel tiles (all streams), phi^T chunk in
//       shared memory (read once per 64 tokens)
//   B3  dphi^T[p][k] = sum_t dd[t][p] x[t][k]: blocks of 64 columns x one of S
//       token segments (S = ceil(T / 512), at most 16), 64-token chunks staged
//       through registers; with S > 1 the per-segment sums go to the workspace
//       and B3R adds them in segment order (deterministic); db / dalpha by
//       per-output tree sums
#include "common.cuh"
#include "internal.h"

namespace mhc {
namespace bwd {

constexpr int MAX_TITERS = 100;    // Sinkhorn trace kept in shared memory

// per-token workspace record (floats): dd[P] dz[P] da[3] hpre[n] hres[n*n] cr
template <int N> struct WS {
    static constexpr int P = N * N + 2 * N;
    static constexpr int DD = 0, DZ = P, DA = 2 * P, HPRE = 2 * P + 3, HRES = HPRE + N,
                         CR = HRES + N * N, STRIDE = (CR + 1 + 3) / 4 * 4;
};

template <typename TX>
__device__ __forceinline__ void load8(const TX* p, float (&v)[8]);
template <>
__device__ __forceinline__ void load8<bf16_t>(const bf16_t* p, float (&v)[8]) { load16<false>(p, v); }
template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&v)[8]) {
    float a[4], b2[4];
    load16<false>(p, a);
    load16<false>(p + 4, b2);
#pragma unroll
    for (int e = 0; e < 4; ++e) { v[e] = a[e]; v[4 + e] = b2[e]; }
}
template <typename TX>
__device__ __forceinline__ void store8(TX* p, const float (&v)[8]);
template <>
__device__ __forceinline__ void store8<bf16_t>(bf16_t* p, const float (&v)[8]) { store16<false>(p, v); }
template <>
__device__ __forceinline__ void store8<float>(float* p, const float (&v)[8]) {
    const float a[4] = {v[0], v[1], v[2], v[3]}, b2[4] = {v[4], v[5], v[6], v[7]};
    store16<false>(p, a);
    store16<false>(p + 4, b2);
}

// ---------------------------------------------------------------- B1
#ifndef MHC_B1_THREADS
#define MHC_B1_THREADS 128
#endif
constexpr int B1_THREADS = MHC_B1_THREADS;   // small blocks: the per-token serial phases of
constexpr int B1_WARPS = B1_THREADS / 32;    // several blocks overlap on an SM

template <int N, typename TX>
__global__ void __launch_bounds__(B1_THREADS, 5)
b1_kernel(const TX* __restrict__ X, const TX* __restrict__ F, const TX* __restrict__ dXn,
          const TX* __restrict__ dxin, float a0, float a1, float a2, const float* __restrict__ b,
          int64_t T, int C, int t_iters, const float* __restrict__ uu, const float* __restrict__ rr,
          float* __restrict__ ws, TX* __restrict__ dF)
{
    using L = WS<N>;
    constexpr int P = L::P, NN = N * N;
    __shared__ float trace[MAX_TITERS + 1][NN];
    __shared__ float red[B1_WARPS][P];
    __shared__ float hp_s[N], ho_s[N], dot[P];
    const int64_t t = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float* rec = ws + t * L::STRIDE;

    // forward coefficients from the recomputed logits; thread 0 keeps the Sinkhorn trace
    if (tid == 0) {
        const float* u = uu + t * P;
        float m[N][N];
#pragma unroll
        for (int i = 0; i < N; ++i) {
            hp_s[i] = sigmoidf_(a0 * u[i] + b[i]);
            ho_s[i] = 2.0f * sigmoidf_(a1 * u[N + i] + b[N + i]);
#pragma unroll
            for (int j = 0; j < N; ++j) m[i][j] = a2 * u[2 * N + i * N + j] + b[2 * N + i * N + j];
        }
        // M0 = exp(z - column max) (the per-column factor cancels in the first T_c)
#pragma unroll
        for (int j = 0; j < N; ++j) {
            float mx = m[0][j];
#pragma unroll
            for (int i = 1; i < N; ++i) mx = fmaxf(mx, m[i][j]);
            if (t_iters == 0) mx = 0.0f;
#pragma unroll
            for (int i = 0; i < N; ++i) m[i][j] = expf(m[i][j] - mx);
        }
#pragma unroll
        for (int e = 0; e < NN; ++e) trace[0][e] = m[e / N][e % N];
        for (int it = 1; it <= t_iters; ++it) {
#pragma unroll
            for (int j = 0; j < N; ++j) {
                float s = 0.0f;
#pragma unroll
                for (int i = 0; i < N; ++i) s += m[i][j];
                const float inv = fast_rcp(s);
#pragma unroll
                for (int i = 0; i < N; ++i) m[i][j] *= inv;
            }
#pragma unroll
            for (int i = 0; i < N; ++i) {
                float s = 0.0f;
#pragma unroll
                for (int j = 0; j < N; ++j) s += m[i][j];
                const float inv = fast_rcp(s);
#pragma unroll
                for (int j = 0; j < N; ++j) m[i][j] *= inv;
            }
#pragma unroll
            for (int e = 0; e < NN; ++e) trace[it][e] = m[e / N][e % N];
        }
#pragma unroll
        for (int e = 0; e < NN; ++e) rec[L::HRES + e] = m[e / N][e % N];
#pragma unroll
        for (int i = 0; i < N; ++i) rec[L::HPRE + i] = hp_s[i];
    }
    __syncthreads();

    // dot products over C and dF
    float acc[P];
#pragma unroll
    for (int p = 0; p < P; ++p) acc[p] = 0.0f;
    const float* ho = ho_s;
    for (int c = tid * 8; c < C; c += B1_THREADS * 8) {
        float g[N][8], x[N][8], f[8], gi[8];
#pragma unroll
        for (int i = 0; i < N; ++i) {
            load8<TX>(dXn + (t * N + i) * C + c, g[i]);
            load8<TX>(X + (t * N + i) * C + c, x[i]);
        }
        load8<TX>(F + t * C + c, f);
        load8<TX>(dxin + t * C + c, gi);
        float df[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float s = 0.0f;
#pragma unroll
            for (int i = 0; i < N; ++i) s = fmaf(ho[i], g[i][e], s);
            df[e] = s;
        }
        store8<TX>(dF + t * C + c, df);
#pragma unroll
        for (int i = 0; i < N; ++i)
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                acc[i] = fmaf(gi[e], x[i][e], acc[i]);                 // dH_pre_i
                acc[N + i] = fmaf(g[i][e], f[e], acc[N + i]);          // dH_post_i
#pragma unroll
                for (int j = 0; j < N; ++j)
                    acc[2 * N + i * N + j] = fmaf(g[i][e], x[j][e], acc[2 * N + i * N + j]);   // dH_res_ij
            }
    }
#pragma unroll
    for (int p = 0; p < P; ++p) {
        const float v = warp_sum(acc[p]);
        if (lane == 0) red[warp][p] = v;
    }
    __syncthreads();
    if (tid < P) {
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < B1_WARPS; ++w) v += red[w][tid];
        dot[tid] = v;
    }
    __syncthreads();

    // coefficient gradients (thread 0)
    if (tid == 0) {
        const float* u = uu + t * P;
        const float r = rr[t];
        float dz[P];
#pragma unroll
        for (int i = 0; i < N; ++i) {
            dz[i] = dot[i] * hp_s[i] * (1.0f - hp_s[i]);
            dz[N + i] = dot[N + i] * ho_s[i] * (1.0f - 0.5f * ho_s[i]);
        }
        float g[N][N];
#pragma unroll
        for (int e = 0; e < NN; ++e) g[e / N][e % N] = dot[2 * N + e];
        for (int it = t_iters; it >= 1; --it) {
            float Mp[N][N], Mo[N][N], A[N][N], cs[N], rs[N], ga[N][N];
#pragma unroll
            for (int e = 0; e < NN; ++e) { Mp[e / N][e % N] = trace[it - 1][e]; Mo[e / N][e % N] = trace[it][e]; }
#pragma unroll
            for (int j = 0; j < N; ++j) {
                float s = 0.0f;
#pragma unroll
                for (int i = 0; i < N; ++i) s += Mp[i][j];
                cs[j] = s;
                const float inv = fast_rcp(s);
#pragma unroll
                for (int i = 0; i < N; ++i) A[i][j] = Mp[i][j] * inv;
            }
#pragma unroll
            for (int i = 0; i < N; ++i) {
                float s = 0.0f;
#pragma unroll
                for (int j = 0; j < N; ++j) s += A[i][j];
                rs[i] = s;
            }
#pragma unroll
            for (int i = 0; i < N; ++i) {                  // through T_r
                float d = 0.0f;
#pragma unroll
                for (int j = 0; j < N; ++j) d = fmaf(g[i][j], Mo[i][j], d);
                const float inv = fast_rcp(rs[i]);
#pragma unroll
                for (int j = 0; j < N; ++j) ga[i][j] = (g[i][j] - d) * inv;
            }
#pragma unroll
            for (int j = 0; j < N; ++j) {                  // through T_c
                float d = 0.0f;
#pragma unroll
                for (int i = 0; i < N; ++i) d = fmaf(ga[i][j], A[i][j], d);
                const float inv = fast_rcp(cs[j]);
#pragma unroll
                for (int i = 0; i < N; ++i) g[i][j] = (ga[i][j] - d) * inv;
            }
        }
#pragma unroll
        for (int e = 0; e < NN; ++e) dz[2 * N + e] = g[e / N][e % N] * trace[0][e];   // through exp
        float da[3] = {0.0f, 0.0f, 0.0f}, dr = 0.0f;
#pragma unroll
        for (int p = 0; p < P; ++p) {
            const int s = p < N ? 0 : (p < 2 * N ? 1 : 2);
            const float a = s == 0 ? a0 : (s == 1 ? a1 : a2);
            da[s] = fmaf(dz[p], u[p], da[s]);
            rec[L::DZ + p] = dz[p];
            rec[L::DD + p] = a * dz[p] / r;
            dr -= a * dz[p] * u[p] / r;
        }
        rec[L::DA + 0] = da[0]; rec[L::DA + 1] = da[1]; rec[L::DA + 2] = da[2];
        rec[L::CR] = dr / (float(N) * float(C) * r);
    }
}

// ---------------------------------------------------------------- B2
constexpr int B2_T = 64, B2_C = 64, B2_SUB = 16;   // tokens per block; per pass of the 128 threads

template <int N, typename TX>
__global__ void __launch_bounds__(128, 5)
b2_kernel(const TX* __restrict__ X, const TX* __restrict__ dXn, const TX* __restrict__ dxin,
          const TX* __restrict__ phiT, const float* __restrict__ ws, int64_t T, int C, TX* __restrict__ dX)
{
    using L = WS<N>;
    constexpr int P = L::P;
    __shared__ __align__(16) float sphi[P][N][B2_C];
    __shared__ float sdd[B2_T][P];
    __shared__ float sco[B2_T][N * N + 1];       // hres, cr
    __shared__ float shp[B2_T][N];
    const int64_t t0 = int64_t(blockIdx.x) * B2_T;
    const int c0 = blockIdx.y * B2_C;
    const int64_t K = int64_t(N) * C;
    const int tid = threadIdx.x;
    // channel c of the slice is stored at float4 slot (c / 8) for c % 8 < 4 and at slot
    // 8 + c / 8 otherwise, so the 8 lanes that read a thread's 8 channels read
    // 128 contiguous bytes (no bank conflict)
    for (int e = tid; e < P * N * B2_C; e += 128) {
        const int p = e / (N * B2_C), rem = e % (N * B2_C), j = rem / B2_C, c = rem % B2_C;
        const int cs = (c & 4) ? 32 + (c >> 3) * 4 + (c & 3) : (c >> 3) * 4 + (c & 3);
        sphi[p][j][cs] = to_f32(phiT[int64_t(p) * K + int64_t(j) * C + c0 + c]);
    }
    for (int e = tid; e < B2_T * P; e += 128) {
        const int tt = e / P, p = e % P;
        sdd[tt][p] = (t0 + tt < T) ? ws[(t0 + tt) * L::STRIDE + L::DD + p] : 0.0f;
    }
    for (int e = tid; e < B2_T * (N * N + 1); e += 128) {
        const int tt = e / (N * N + 1), q = e % (N * N + 1);          // hres (n*n) then cr
        sco[tt][q] = (t0 + tt < T) ? ws[(t0 + tt) * L::STRIDE + L::HRES + q] : 0.0f;
    }
    for (int e = tid; e < B2_T * N; e += 128) {
        const int tt = e / N, q = e % N;
        shp[tt][q] = (t0 + tt < T) ? ws[(t0 + tt) * L::STRIDE + L::HPRE + q] : 0.0f;
    }
    __syncthreads();
    const int v = tid % (B2_C / 8);
    for (int tt = tid / (B2_C / 8); tt < B2_T; tt += B2_SUB) {
    const int64_t t = t0 + tt;
    if (t >= T) break;
    const int c = c0 + v * 8;
    float g[N][8], x[N][8], gi[8];
#pragma unroll
    for (int i = 0; i < N; ++i) {
        load8<TX>(dXn + (t * N + i) * C + c, g[i]);
        load8<TX>(X + (t * N + i) * C + c, x[i]);
    }
    load8<TX>(dxin + t * C + c, gi);
    const float* hres = sco[tt];              // [N][N]
    const float cr = sco[tt][N * N];
    const float* hpre = shp[tt];
    float dd[P];                              // this token's dd in registers
#pragma unroll
    for (int p = 0; p < P; ++p) dd[p] = sdd[tt][p];
#pragma unroll
    for (int j = 0; j < N; ++j) {
        const float hpj = hpre[j];
        // (phi dd)_j for the thread's 8 channels: two 16-byte phi reads per logit
        float pr[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) pr[e] = 0.0f;
#pragma unroll
        for (int p = 0; p < P; ++p) {
            const float4 lo = *reinterpret_cast<const float4*>(&sphi[p][j][v * 4]);
            const float4 hi = *reinterpret_cast<const float4*>(&sphi[p][j][32 + v * 4]);
            pr[0] = fmaf(lo.x, dd[p], pr[0]); pr[1] = fmaf(lo.y, dd[p], pr[1]);
            pr[2] = fmaf(lo.z, dd[p], pr[2]); pr[3] = fmaf(lo.w, dd[p], pr[3]);
            pr[4] = fmaf(hi.x, dd[p], pr[4]); pr[5] = fmaf(hi.y, dd[p], pr[5]);
            pr[6] = fmaf(hi.z, dd[p], pr[6]); pr[7] = fmaf(hi.w, dd[p], pr[7]);
        }
        float o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float s = hpj * gi[e];
#pragma unroll
            for (int i = 0; i < N; ++i) s = fmaf(hres[i * N + j], g[i][e], s);
            o[e] = s + pr[e] + cr * x[j][e];
        }
        store8<TX>(dX + (t * N + j) * C + c, o);
    }
    }
}

// ---------------------------------------------------------------- B3
constexpr int B3_K = 64, B3_T = 64, B3_SEG_MIN = 512, B3_MAX_SEGS = 16;

// token segments of B3 for T tokens (the workspace holds S - 1 extra dphi copies
// when S > 1; see mhc_backward_workspace_bytes)
inline int b3_segments(int64_t T)
{
    const int64_t s = (T + B3_SEG_MIN - 1) / B3_SEG_MIN;
    return int(s < 1 ? 1 : (s > B3_MAX_SEGS ? B3_MAX_SEGS : s));
}

// block (k slab, segment): out[p][k0 + kk] = sum over the segment's tokens of
// dd[t][p] * x[t][k0 + kk]; out is dphi^T (one segment) or the segment's slice
// of the partial sums
template <int N, typename TX>
__global__ void __launch_bounds__(256)
b3_kernel(const TX* __restrict__ X, const float* __restrict__ ws, int64_t T, int C, int64_t seg_len,
          float* __restrict__ out)
{
    using L = WS<N>;
    constexpr int P = L::P;
    constexpr int PP = (P + 15) / 16 * 16;         // logits padded to 16 per row of sdd
    constexpr int PB = PP / 8;                     // logits per thread (8 logit blocks): even, so
    static_assert(PB % 2 == 0, "float2 reads of sdd stay 8-byte aligned");
    constexpr int XV = B3_T * (B3_K / 8);          // 8-element X vectors per chunk (2 per thread)
    constexpr int DV = B3_T * P;                   // dd values per chunk
    constexpr int DPT = (DV + 255) / 256;
    static_assert(256 == 32 * 8, "32 column pairs x 8 logit blocks");
    __shared__ __align__(16) float sx[B3_T][B3_K];
    __shared__ __align__(16) float sdd[B3_T][PP];
    const int64_t K = int64_t(N) * C;
    const int64_t k0 = int64_t(blockIdx.x) * B3_K;
    const int64_t ta = int64_t(blockIdx.y) * seg_len;
    const int64_t tb = ta + seg_len < T ? ta + seg_len : T;
    const int tid = threadIdx.x;
    const int kk = tid & 31;                       // columns kk and kk + 32 of the slab
    const int pb = tid >> 5;                       // logits [pb * PB, pb * PB + PB)
    float acc[2][PB];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int q = 0; q < PB; ++q) acc[h][q] = 0.0f;
    float xr[XV / 256][8], dr[DPT];
    auto fetch = [&](int64_t t0) {
#pragma unroll
        for (int u = 0; u < XV / 256; ++u) {
            const int e = tid + u * 256, tt = e / (B3_K / 8), vv = e % (B3_K / 8);
            if (t0 + tt < tb) load8<TX>(X + (t0 + tt) * K + k0 + vv * 8, xr[u]);
            else {
#pragma unroll
                for (int q = 0; q < 8; ++q) xr[u][q] = 0.0f;
            }
        }
#pragma unroll
        for (int u = 0; u < DPT; ++u) {
            const int e = tid + u * 256, tt = e / P, p = e % P;
            dr[u] = (e < DV && t0 + tt < tb) ? ws[(t0 + tt) * L::STRIDE + L::DD + p] : 0.0f;
        }
    };
    if (ta < tb) fetch(ta);
    for (int64_t t0 = ta; t0 < tb; t0 += B3_T) {
        __syncthreads();                           // the previous chunk is consumed
#pragma unroll
        for (int u = 0; u < XV / 256; ++u) {
            const int e = tid + u * 256, tt = e / (B3_K / 8), vv = e % (B3_K / 8);
#pragma unroll
            for (int q = 0; q < 8; ++q) sx[tt][vv * 8 + q] = xr[u][q];
        }
#pragma unroll
        for (int u = 0; u < DPT; ++u) {
            const int e = tid + u * 256;
            if (e < DV) sdd[e / P][e % P] = dr[u];
        }
        if (PP > P)
            for (int e = tid; e < B3_T * (PP - P); e += 256) sdd[e / (PP - P)][P + e % (PP - P)] = 0.0f;
        __syncthreads();
        if (t0 + B3_T < tb) fetch(t0 + B3_T);     // next chunk in flight during the products
#pragma unroll 4
        for (int tt = 0; tt < B3_T; ++tt) {
            const float x0 = sx[tt][kk], x1 = sx[tt][kk + 32];
            float dd[PB];
#pragma unroll
            for (int q = 0; q < PB; q += 2) {
                const float2 d2 = *reinterpret_cast<const float2*>(&sdd[tt][pb * PB + q]);
                dd[q] = d2.x;
                dd[q + 1] = d2.y;
            }
#pragma unroll
            for (int q = 0; q < PB; ++q) {
                acc[0][q] = fmaf(dd[q], x0, acc[0][q]);
                acc[1][q] = fmaf(dd[q], x1, acc[1][q]);
            }
        }
    }
    float* o = out + int64_t(blockIdx.y) * P * K;
#pragma unroll
    for (int q = 0; q < PB; ++q) {
        const int p = pb * PB + q;
        if (p < P) {
            o[int64_t(p) * K + k0 + kk] = acc[0][q];
            o[int64_t(p) * K + k0 + kk + 32] = acc[1][q];
        }
    }
}

// dphi^T[i] = sum_s part[s][i] in segment order
__global__ void __launch_bounds__(256)
b3r_kernel(const float* __restrict__ part, int segs, int64_t count, float* __restrict__ dphiT)
{
    const int64_t i = int64_t(blockIdx.x) * 256 + threadIdx.x;
    if (i >= count) return;
    float s = 0.0f;
    for (int q = 0; q < segs; ++q) s += part[int64_t(q) * count + i];
    dphiT[i] = s;
}

// one block per output: db[p] = sum_t dz[t][p]; dalpha[s] = sum_t da[t][s]
template <int N>
__global__ void __launch_bounds__(256)
bsum_kernel(const float* __restrict__ ws, int64_t T, float* __restrict__ db, float* __restrict__ dalpha)
{
    using L = WS<N>;
    constexpr int P = L::P;
    __shared__ float red[8];
    const int o = blockIdx.x;                 // 0..P-1: db, P..P+2: dalpha
    const int off = o < P ? L::DZ + o : L::DA + (o - P);
    float s = 0.0f;
    for (int64_t t = threadIdx.x; t < T; t += 256) s += ws[t * L::STRIDE + off];
    s = warp_sum(s);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        float v = 0.0f;
        for (int w = 0; w < 8; ++w) v += red[w];
        if (o < P) db[o] = v; else dalpha[o - P] = v;
    }
}

template <int N, typename TX>
static mhc_status run(const BwdArgs& a, cudaStream_t s)
{
    using L = WS<N>;
    constexpr int P = L::P;
    // B0: recompute u = (x phi)/r and r
    float* ws = a.records;
    {
        PreArgs pa{a.X, a.dt, a.phi, a.dt, {a.alpha[0], a.alpha[1], a.alpha[2]}, a.b, a.T, N, a.C,
                   a.t_iters, a.eps, nullptr, nullptr, nullptr, nullptr};
        pa.u_out = a.u_scratch;
        pa.r_out = a.r_scratch;
        pa.skip_xin = true;
        const mhc_status st = (pre_tc_supported(pa) && g_pre_path != MHC_PATH_FMA) ? launch_pre_tc(pa, s)
                                                                                    : launch_pre_fma(pa, s);
        if (st != MHC_OK) return st;
    }
    b1_kernel<N, TX><<<dim3(unsigned(a.T)), B1_THREADS, 0, s>>>(
        static_cast<const TX*>(a.X), static_cast<const TX*>(a.F), static_cast<const TX*>(a.dXn),
        static_cast<const TX*>(a.dxin), a.alpha[0], a.alpha[1], a.alpha[2], a.b, a.T, a.C, a.t_iters,
        a.u_scratch, a.r_scratch, ws, static_cast<TX*>(a.dF));
    mhc_status st = launch_status("mhc_backward B1 kernel");
    if (st != MHC_OK) return st;
    b2_kernel<N, TX><<<dim3(unsigned((a.T + B2_T - 1) / B2_T), unsigned(a.C / B2_C)), 128, 0, s>>>(
        static_cast<const TX*>(a.X), static_cast<const TX*>(a.dXn), static_cast<const TX*>(a.dxin),
        static_cast<const TX*>(a.phi), ws, a.T, a.C, static_cast<TX*>(a.dX));
    st = launch_status("mhc_backward B2 kernel");
    if (st != MHC_OK) return st;
    const int64_t K = int64_t(N) * a.C;
    int segs = b3_segments(a.T);
    int64_t seg_len = ((a.T + segs - 1) / segs + B3_T - 1) / B3_T * B3_T;
    if (backward_dphi_tc_supported(a) && g_pre_path != MHC_PATH_FMA) {
        // tensor cores: long token segments (a CTA's fixed costs -- TMEM, ring fill,
        // epilogue -- against its streaming), about two CTAs per SM in one wave; at most
        // the segments the workspace holds partials for
        static int sms = 0;
        if (!sms) {
            int dev = 0;
            cudaError_t e = cudaGetDevice(&dev);
            if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            if (e != cudaSuccess) return cuda_status(e, "mhc_backward: SM count");
        }
        const int64_t slabs = K / 128;
        const int64_t want = (2 * int64_t(sms) + slabs / 2) / slabs;
        const int segs_tc = int(want < 1 ? 1 : (want > segs ? segs : want));
        segs = segs_tc;
        seg_len = ((a.T + segs - 1) / segs + B3_T - 1) / B3_T * B3_T;
        st = launch_backward_dphi_tc(a, L::STRIDE, L::DD, segs, seg_len, s);
    } else {
        b3_kernel<N, TX><<<dim3(unsigned(K / B3_K), unsigned(segs)), 256, 0, s>>>(
            static_cast<const TX*>(a.X), ws, a.T, a.C, seg_len, segs > 1 ? a.dphi_part : a.dphi);
        st = launch_status("mhc_backward B3 kernel");
    }
    if (st != MHC_OK) return st;
    if (segs > 1) {
        const int64_t count = int64_t(P) * K;
        b3r_kernel<<<dim3(unsigned((count + 255) / 256)), 256, 0, s>>>(a.dphi_part, segs, count, a.dphi);
        st = launch_status("mhc_backward B3 reduction kernel");
        if (st != MHC_OK) return st;
    }
    bsum_kernel<N><<<dim3(unsigned(P + 3)), 256, 0, s>>>(ws, a.T, a.db, a.dalpha);
    return launch_status("mhc_backward reduction kernel");
}

}  // namespace bwd

int backward_b3_segments(int64_t T) { return bwd::b3_segments(T); }

size_t backward_record_stride(int n)
{
    size_t stride = 0;
    switch (n) {
        case 1: stride = bwd::WS<1>::STRIDE; break;
        case 2: stride = bwd::WS<2>::STRIDE; break;
        case 3: stride = bwd::WS<3>::STRIDE; break;
        case 4: stride = bwd::WS<4>::STRIDE; break;
        default: return 0;
    }
    return stride;
}

mhc_status launch_backward(const BwdArgs& a, cudaStream_t s)
{
#define MHC_BWD_CASE(NN)                                                                \
    case NN:                                                                            \
        return a.dt == MHC_BF16 ? bwd::run<NN, bf16_t>(a, s) : bwd::run<NN, float>(a, s);
    switch (a.n) {
        MHC_BWD_CASE(1) MHC_BWD_CASE(2) MHC_BWD_CASE(3) MHC_BWD_CASE(4)
        default: break;
    }
#undef MHC_BWD_CASE
    set_error("mhc_backward: n=%d not supported (1..4)", a.n);
    return MHC_ERR_UNSUPPORTED;
}

}  // namespace mhc
