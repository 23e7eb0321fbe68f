// xhc_sparse_update: sparse residual update + scatter of the xHC sublayer.
//
// [xHC] section "sparse residual stream architecture", step 3, and section
// "parameterisation": H_res (k x k, Sinkhorn on the active streams) and
// H_post (k x Kr, 2 sigma) are generated from the active state only:
//   X_act = rows idx[t][0..k-1] of X_t;  r = RMS(vec X_act) over kC
//   z = alpha * (vec X_act . phi_act^T) / r + b_act   (res k*k | post k*Kr)
//   X_act_new[j] = sum_l H_res[j][l] X_act[l] + w[t][j] * sum_q H_post[j][q] V[t][q]
//   X[t][idx[t][j]] = X_act_new[j]; the other streams pass through unchanged.
//
// One block of 256 threads per tile of 16 tokens.  Phase 1 projects the
// gathered rows on CUDA cores: K = kC is walked in chunks of 64 staged in
// shared memory (the X_act chunk of all 16 tokens and the phi_act^T chunk,
// double buffered; the next chunk's loads are in flight in registers while
// the current one is multiplied), 16 threads per token each owning up to 4
// logits; phi_act^T is stored as float4 per (k quad, logit), so the 16 threads
// of a token read consecutive 16-byte words.
// Phase 2: per-token coefficients (one thread per token).  Phase 3: the mix,
// reading X_act again (the block read it moments ago, so from L2) and V,
// writing the k updated rows in place.
//
// An idx entry outside [0, N) is reported in the device error word (bit 1)
// and that token is left unchanged.
#include "common.cuh"
#include "internal.h"

namespace mhc {
namespace xupd {

constexpr int THREADS = 256;
constexpr int TT = 16;        // tokens per block
constexpr int TPT = THREADS / TT;  // threads per token in the projection
constexpr int KCH = 64;       // K elements per staged chunk

template <typename TX>
__device__ __forceinline__ void load8(const TX* p, float (&v)[8]);
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
template <typename TX>
__device__ __forceinline__ void store8(TX* p, const float (&v)[8]);
template <>
__device__ __forceinline__ void store8<bf16_t>(bf16_t* p, const float (&v)[8]) { store16<false>(p, v); }
template <>
__device__ __forceinline__ void store8<float>(float* p, const float (&v)[8]) {
    const float a[4] = {v[0], v[1], v[2], v[3]}, b[4] = {v[4], v[5], v[6], v[7]};
    store16<false>(p, a);
    store16<false>(p + 4, b);
}

template <int K, int KR, typename TX>
__global__ void __launch_bounds__(THREADS)
update_kernel(TX* X, const float* __restrict__ V, const int32_t* __restrict__ idx,
              const float* __restrict__ w, const TX* __restrict__ phiT, float a_res, float a_post,
              const float* __restrict__ b, int64_t T, int N, int C, int t_iters, float eps,
              float* __restrict__ Hres_out, float* __restrict__ Hpost_out)
{
    constexpr int PA = K * K + K * KR;
    constexpr int PPT = (PA + TPT - 1) / TPT;     // logits per thread
    static_assert(PPT <= 4, "at most 64 logits");
    __shared__ __align__(16) float xs[2][TT][KCH];
    // phi_act^T chunk as float4 per (k quad, logit); logit p of k quad kq sits at
    // p ^ ((kq / 2) % 8) of a row padded to a multiple of 8, so that both the
    // stores (8 lanes: one logit, 8 k quads) and the reads (one k quad, 16
    // logits) touch distinct banks
    constexpr int PAP = (PA + 7) / 8 * 8;
    __shared__ __align__(16) float4 ps[2][KCH / 4][PAP];
    __shared__ float ssq[TT];
    __shared__ float logit[TT][PA];
    __shared__ float hres[TT][K][K];
    __shared__ float hpost[TT][K][KR];
    __shared__ int sidx[TT][K];
    __shared__ int sok[TT];

    const int64_t t0 = int64_t(blockIdx.x) * TT;
    const int tid = threadIdx.x;
    if (tid < TT) {
        const int64_t t = t0 + tid;
        int good = t < T;
        for (int l = 0; l < K; ++l) {
            int v = good ? idx[t * K + l] : 0;
            if (good && (v < 0 || v >= N)) { atomicOr(&g_device_error, 2u); good = 0; }
            sidx[tid][l] = v;
        }
        sok[tid] = good;
        ssq[tid] = 0.0f;
    }
    __syncthreads();

    // ---- phase 1: d[t][p] = sum_k xact[t][k] * phiT[p][k], and sum of squares
    const int64_t KT = int64_t(K) * C;
    const int nchunks = int((KT + KCH - 1) / KCH);
    const int my_t = tid / TPT, sub = tid % TPT;
    float acc[PPT];
#pragma unroll
    for (int q = 0; q < PPT; ++q) acc[q] = 0.0f;
    float ss = 0.0f;
    // chunk staging through registers: the loads of chunk ch+1 are in flight while
    // chunk ch is multiplied out of shared memory
    constexpr int XV = TT * (KCH / 8), PV = PA * (KCH / 8);       // 8-element vectors per chunk
    constexpr int XPT = (XV + THREADS - 1) / THREADS, PPV = (PV + THREADS - 1) / THREADS;
    float xr8[XPT][8], pr8[PPV][8];
    auto fetch = [&](int ch) {
        const int64_t k0 = int64_t(ch) * KCH;
#pragma unroll
        for (int u = 0; u < XPT; ++u) {
            const int e = tid + u * THREADS;
            if (e < XV) {
                // X_act chunk: TT tokens x KCH (a chunk never straddles two slots: C % KCH == 0)
                const int tt = e / (KCH / 8), v = e % (KCH / 8);
                const int64_t k = k0 + v * 8;
                const int l = int(k / C), c = int(k - int64_t(l) * C);
                if (sok[tt]) load8<TX>(X + ((t0 + tt) * N + sidx[tt][l]) * int64_t(C) + c, xr8[u]);
                else {
#pragma unroll
                    for (int q = 0; q < 8; ++q) xr8[u][q] = 0.0f;
                }
            }
        }
#pragma unroll
        for (int u = 0; u < PPV; ++u) {
            const int e = tid + u * THREADS;
            if (e < PV) load8<TX>(phiT + int64_t(e / (KCH / 8)) * KT + k0 + (e % (KCH / 8)) * 8, pr8[u]);
        }
    };
    auto put = [&](int buf) {
#pragma unroll
        for (int u = 0; u < XPT; ++u) {
            const int e = tid + u * THREADS;
            if (e < XV) {
                const int tt = e / (KCH / 8), v = e % (KCH / 8);
#pragma unroll
                for (int q = 0; q < 8; ++q) xs[buf][tt][v * 8 + q] = xr8[u][q];
            }
        }
#pragma unroll
        for (int u = 0; u < PPV; ++u) {
            const int e = tid + u * THREADS;
            if (e < PV) {
                const int p = e / (KCH / 8), v = e % (KCH / 8);
                ps[buf][2 * v][p ^ (v & 7)] = make_float4(pr8[u][0], pr8[u][1], pr8[u][2], pr8[u][3]);
                ps[buf][2 * v + 1][p ^ (v & 7)] = make_float4(pr8[u][4], pr8[u][5], pr8[u][6], pr8[u][7]);
            }
        }
    };
    fetch(0);
    put(0);
    __syncthreads();
    for (int ch = 0; ch < nchunks; ++ch) {
        const int buf = ch & 1;
        if (ch + 1 < nchunks) fetch(ch + 1);
        const float* xr = xs[buf][my_t];
#pragma unroll 4
        for (int kk = 0; kk < KCH; kk += 4) {
            const float4 x4 = *reinterpret_cast<const float4*>(xr + kk);
            if (sub == 0) {
                ss = fmaf(x4.x, x4.x, ss); ss = fmaf(x4.y, x4.y, ss);
                ss = fmaf(x4.z, x4.z, ss); ss = fmaf(x4.w, x4.w, ss);
            }
#pragma unroll
            for (int q = 0; q < PPT; ++q) {
                const int p = sub + q * TPT;
                if (p < PA) {
                    const float4 p4 = ps[buf][kk / 4][p ^ ((kk / 8) & 7)];
                    acc[q] = fmaf(x4.x, p4.x, acc[q]);
                    acc[q] = fmaf(x4.y, p4.y, acc[q]);
                    acc[q] = fmaf(x4.z, p4.z, acc[q]);
                    acc[q] = fmaf(x4.w, p4.w, acc[q]);
                }
            }
        }
        if (ch + 1 < nchunks) put(buf ^ 1);
        __syncthreads();
    }
#pragma unroll
    for (int q = 0; q < PPT; ++q) {
        const int p = sub + q * TPT;
        if (p < PA) logit[my_t][p] = acc[q];
    }
    if (sub == 0) ssq[my_t] = ss;
    __syncthreads();

    // ---- phase 2: coefficients, one thread per token
    if (tid < TT) {
        const int64_t t = t0 + tid;
        const float r = sqrtf(ssq[tid] / float(KT) + eps);
        const float inv_r = 1.0f / r;
        float m[K][K];
#pragma unroll
        for (int i = 0; i < K; ++i)
#pragma unroll
            for (int j = 0; j < K; ++j)
                m[i][j] = a_res * logit[tid][i * K + j] * inv_r + __ldg(b + i * K + j);
        sinkhorn_regs<K>(m, t_iters);
#pragma unroll
        for (int i = 0; i < K; ++i)
#pragma unroll
            for (int j = 0; j < K; ++j) hres[tid][i][j] = m[i][j];
#pragma unroll
        for (int e = 0; e < K * KR; ++e)
            hpost[tid][e / KR][e % KR] = 2.0f * sigmoidf_(a_post * logit[tid][K * K + e] * inv_r + __ldg(b + K * K + e));
        if (t < T) {
            if (Hres_out)
                for (int e = 0; e < K * K; ++e) Hres_out[t * K * K + e] = m[e / K][e % K];
            if (Hpost_out)
                for (int e = 0; e < K * KR; ++e) Hpost_out[t * K * KR + e] = hpost[tid][e / KR][e % KR];
        }
    }
    __syncthreads();

    // ---- phase 3: mix, write back, scatter
    const int CV = C / 8;
    for (int e = tid; e < TT * CV; e += THREADS) {
        const int tt = e / CV, v = e % CV;
        const int64_t t = t0 + tt;
        if (!sok[tt]) continue;
        const int c = v * 8;
        float xa[K][8], vb[KR][8];
#pragma unroll
        for (int l = 0; l < K; ++l) load8<TX>(X + (t * N + sidx[tt][l]) * int64_t(C) + c, xa[l]);
#pragma unroll
        for (int q = 0; q < KR; ++q) {
            float lo[4], hi[4];
            load16<true>(V + (t * KR + q) * int64_t(C) + c, lo);
            load16<true>(V + (t * KR + q) * int64_t(C) + c + 4, hi);
#pragma unroll
            for (int u = 0; u < 4; ++u) { vb[q][u] = lo[u]; vb[q][4 + u] = hi[u]; }
        }
#pragma unroll
        for (int j = 0; j < K; ++j) {
            const float wj = __ldg(w + t * K + j);
            float o[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                float wb = 0.0f;
#pragma unroll
                for (int q = 0; q < KR; ++q) wb = fmaf(hpost[tt][j][q], vb[q][u], wb);
                float mix = 0.0f;
#pragma unroll
                for (int l = 0; l < K; ++l) mix = fmaf(hres[tt][j][l], xa[l][u], mix);
                o[u] = fmaf(wj, wb, mix);
            }
            store8<TX>(X + (t * N + sidx[tt][j]) * int64_t(C) + c, o);
        }
    }
}

template <int K, int KR>
static mhc_status launch_kkr(const UpdateArgs& a, cudaStream_t s)
{
    const int64_t blocks = (a.T + TT - 1) / TT;
    if (a.dt == MHC_BF16)
        update_kernel<K, KR, bf16_t><<<dim3(unsigned(blocks)), THREADS, 0, s>>>(
            static_cast<bf16_t*>(a.X), a.V, a.idx, a.w, static_cast<const bf16_t*>(a.phi), a.alpha[0],
            a.alpha[1], a.b, a.T, a.N, a.C, a.t_iters, a.eps, a.H_res, a.H_post);
    else
        update_kernel<K, KR, float><<<dim3(unsigned(blocks)), THREADS, 0, s>>>(
            static_cast<float*>(a.X), a.V, a.idx, a.w, static_cast<const float*>(a.phi), a.alpha[0],
            a.alpha[1], a.b, a.T, a.N, a.C, a.t_iters, a.eps, a.H_res, a.H_post);
    return launch_status("xhc_sparse_update kernel");
}

template <int K>
static mhc_status launch_k(const UpdateArgs& a, cudaStream_t s)
{
    switch (a.Kr) {
        case 1: return launch_kkr<K, 1>(a, s);
        case 2: return launch_kkr<K, 2>(a, s);
        case 3: return launch_kkr<K, 3>(a, s);
        case 4: return launch_kkr<K, 4>(a, s);
        case 5: return launch_kkr<K, 5>(a, s);
        default: break;
    }
    set_error("xhc_sparse_update: Kr=%d not supported (1..5)", a.Kr);
    return MHC_ERR_UNSUPPORTED;
}

}  // namespace xupd

mhc_status launch_sparse_update(const UpdateArgs& a, cudaStream_t s)
{
    // the tensor-core path (xhc_update_tc.cu) where it applies, unless the caller chose
    // the CUDA-core path with mhc_set_path
    const bool tc_ok = update_tc_supported(a);
    if (g_pre_path == MHC_PATH_TENSOR && !tc_ok) {
        set_error("xhc_sparse_update: the tensor-core path needs bf16, k = 4, Kr <= 4 and C %% 512 == 0");
        return MHC_ERR_UNSUPPORTED;
    }
    if (tc_ok && g_pre_path != MHC_PATH_FMA) return launch_update_tc(a, s);
    switch (a.k) {
        case 1: return xupd::launch_k<1>(a, s);
        case 2: return xupd::launch_k<2>(a, s);
        case 3: return xupd::launch_k<3>(a, s);
        case 4: return xupd::launch_k<4>(a, s);
        default: break;
    }
    set_error("xhc_sparse_update: k=%d not supported (1..4)", a.k);
    return MHC_ERR_UNSUPPORTED;
}

}  // namespace mhc
