// mhc_pre, tensor-core path (sm_100a: TMA + tcgen05.mma + TMEM + a cluster
// of 8 CTAs sharing partial sums through distributed shared memory).
//
// [mHC] section 4.3.1, Eq.(14)-(19), and F_pre := H_pre x_l.  Per token tile
// of Mt <= 128 tokens, the 8 CTAs of a cluster split the C channels: CTA r
// owns channels [r*C/8, (r+1)*C/8) of every stream, i.e. a K-slice of
// n*C/8 elements of each token's n*C row.
//
//   warp 0   TMA producer: streams X[tile, stream i, 64-channel block] boxes
//            (Mt rows x 128 B, 128-byte swizzle) through a 4-stage ring.
//   warp 1   MMA issuer: D[Mt x NB] += X_chunk[Mt x 64] * phiT_chunk[NB x 64]^T
//            (tcgen05.mma kind::f16, M = 128, fp32 accumulator in TMEM,
//            double-buffered across tiles).  phiT (this CTA's K-slice of phi,
//            transposed to K-major) stays resident in shared memory.
//   warps 2-5 epilogue: the sum of squares of each row straight from the
//            ring stage (Eq.15), the partial logits from TMEM, an exchange of
//            the 8 partial (logits, sum of squares) rows through DSMEM, the
//            coefficients of 16 tokens per CTA (Eq.16-19, Sinkhorn in
//            registers), a DSMEM broadcast of H_pre, and x_in = H_pre X for
//            this CTA's channels (re-reading the tile's X slice, which the
//            cluster's recent loads keep in L2).
//
// HBM: X is read once by TMA; x_in and the coefficients are written once.
// phi is read once per CTA.  Every mbarrier wait is bounded (g_wait_limit);
// on expiry the kernel records MHC_ERR_TIMEOUT in the device error word,
// drains its own copies in flight, frees TMEM and returns.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace mhc {
namespace pretc {

using namespace sm100;

constexpr int CL = 8;            // CTAs per cluster (channel split)
constexpr int MROWS = 128;       // MMA M: token rows of one tile buffer
constexpr int KC = 64;           // K elements per chunk (one 128-byte row)
constexpr int STAGE_BYTES = MROWS * 128;
constexpr int STAGES = 4;
constexpr int NTHREADS = 192;    // 6 warps
constexpr int EPI_THREADS = 128; // warps 2..5
constexpr int TOK_PER_CTA = MROWS / CL;  // tokens whose coefficients a CTA computes

template <int N> struct Cfg {
    static constexpr int P = N * N + 2 * N;
    static constexpr int R = (P + 7) / 8 * 8;      // phiT rows stored per chunk
    static constexpr int NB = (P + 15) / 16 * 16;  // MMA N
    static constexpr int PS = P + 1;               // partial row: P logits + sum of squares
    static constexpr int TMEM_COLS = (2 * NB <= 32) ? 32 : (2 * NB <= 64 ? 64 : (2 * NB <= 128 ? 128 : 256));
};

struct Layout {
    uint32_t phi, ring, part, hpre, bars, slot, total;
};

template <int N>
__host__ __device__ inline Layout layout_for(int NQ) {
    using G = Cfg<N>;
    Layout L;
    L.phi = 0;
    L.ring = uint32_t(NQ) * G::R * 128;                      // multiple of 1024
    L.part = L.ring + STAGES * STAGE_BYTES;
    L.hpre = L.part + MROWS * G::PS * 4;
    L.bars = (L.hpre + MROWS * N * 4 + 15) / 16 * 16;
    L.slot = L.bars + (2 * STAGES + 8) * 8;
    L.total = L.slot + 16;
    return L;
}

template <int N>
__global__ void __cluster_dims__(CL, 1, 1) __launch_bounds__(NTHREADS, 1)
pre_tc_kernel(const __grid_constant__ CUtensorMap tmX, const bf16_t* __restrict__ X,
              const bf16_t* __restrict__ phi, float a0, float a1, float a2,
              const float* __restrict__ b, int64_t T, int C, int Mt, int num_tiles, int t_iters,
              float eps, bf16_t* __restrict__ x_in, float* __restrict__ Hpre,
              float* __restrict__ Hpost, float* __restrict__ Hres)
{
    using G = Cfg<N>;
    constexpr int P = G::P, R = G::R, NB = G::NB, PS = G::PS;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment for the 128-byte-swizzle atoms
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int Cs = C / CL;
    const int CB = Cs / KC;            // channel blocks per stream
    const int NQ = N * CB;             // K chunks of this CTA per tile
    const Layout L = layout_for<N>(NQ);
    uint8_t* sphi = smem + L.phi;
    uint8_t* sring = smem + L.ring;
    float* spart = reinterpret_cast<float*>(smem + L.part);
    float* shpre = reinterpret_cast<float*>(smem + L.hpre);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* tfull = bars + 2 * STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* part_ready = tempty + 2;
    uint64_t* hpre_ready = part_ready + 1;
    uint64_t* epi_sync = hpre_ready + 1;   // the 128 epilogue threads, twice per tile
    uint64_t* drain = epi_sync + 1;        // MMA completion on the abort path
    uint32_t* slot = reinterpret_cast<uint32_t*>(smem + L.slot);
    __shared__ int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int cluster_id = blockIdx.x / CL;
    const int nclusters = gridDim.x / CL;
    const int c0 = int(rank) * Cs;

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1 + EPI_THREADS / 32);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], EPI_THREADS / 32);
        }
        mbar_init(part_ready, CL);
        mbar_init(hpre_ready, CL);
        mbar_init(epi_sync, EPI_THREADS);
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(slot, G::TMEM_COLS);
    if (warp == 0 && lane == 0) tma_prefetch(&tmX);

    // Resident phiT: chunk q = (stream i, channel block cb) holds rows p < R of
    // phi[i*C + c0 + cb*64 + kk][p] at kk, 128-byte rows, 16-byte groups XOR-swizzled by row.
    for (int e = threadIdx.x; e < NQ * KC; e += NTHREADS) {
        const int q = e / KC, kk = e % KC;
        const int i = q / CB, cb = q % CB;
        const int64_t k = int64_t(i) * C + c0 + cb * KC + kk;
        uint8_t* rowbase = sphi + size_t(q) * R * 128;
        const int grp = kk >> 3, within = (kk & 7) * 2;
#pragma unroll 4
        for (int p = 0; p < R; ++p) {
            const bf16_t v = p < P ? phi[k * P + p] : bf16_t(0);
            *reinterpret_cast<bf16_t*>(rowbase + p * 128 + ((grp ^ (p & 7)) << 4) + within) = v;
        }
    }
    fence_proxy_async_smem();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *slot;
    cluster_sync();   // every CTA's barriers are initialised before any remote arrive

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            int inflight_s[STAGES], inflight_ph[STAGES], n_issued = 0;
            bool ok = true;
            for (int tile = cluster_id; tile < num_tiles && ok; tile += nclusters) {
                const int t0 = tile * Mt;
                for (int q = 0; q < NQ; ++q) {
                    if (!mbar_wait(&empty[s], ph ^ 1) || *(volatile int*)&s_abort) { ok = false; break; }
                    mbar_arrive_expect_tx(&full[s], uint32_t(Mt) * 128);
                    tma_load_3d(sring + s * STAGE_BYTES, &tmX, &full[s], c0 + (q % CB) * KC, q / CB, t0);
                    inflight_s[n_issued % STAGES] = s;
                    inflight_ph[n_issued % STAGES] = int(ph);
                    ++n_issued;
                    if (++s == STAGES) { s = 0; ph ^= 1; }
                }
            }
            if (!ok) {
                s_abort = 1;
                // drain this CTA's copies still in flight before the block can exit
                const int pending = n_issued < STAGES ? n_issued : STAGES;
                for (int j = 0; j < pending; ++j)
                    mbar_wait(&full[inflight_s[j]], uint32_t(inflight_ph[j]), 1ll << 22);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(MROWS, NB);
            const uint32_t ring_a = smem_u32(sring), phi_a = smem_u32(sphi);
            int s = 0, it = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int tile = cluster_id; tile < num_tiles && ok; tile += nclusters, ++it) {
                const int acc = it & 1;
                if (!mbar_wait(&tempty[acc], (uint32_t((it >> 1) & 1)) ^ 1)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem_base + uint32_t(acc * NB);
                for (int q = 0; q < NQ; ++q) {
                    if (!mbar_wait(&full[s], ph) || *(volatile int*)&s_abort) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < KC / 16; ++kk) {
                        const uint64_t ad = sdesc_k_sw128(ring_a + s * STAGE_BYTES + kk * 32);
                        const uint64_t bd = sdesc_k_sw128(phi_a + q * R * 128 + kk * 32);
                        mma_bf16(d, ad, bd, idesc, (q | kk) != 0);
                    }
                    mma_commit(&empty[s]);
                    if (++s == STAGES) { s = 0; ph ^= 1; }
                }
                if (ok) mma_commit(&tfull[acc]);
            }
            if (!ok) {
                s_abort = 1;
                mma_commit(drain);               // TMEM is freed only after issued MMAs finish
                mbar_wait(drain, 0, 1ll << 22);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int et = threadIdx.x - 64;          // 0..127
        const int qd = warp & 3;                  // TMEM lane quarter of this warp
        const int m = qd * 32 + lane;             // token row within the tile
        const float inv_K = 1.0f / float(N * C);
        int s = 0, it = 0;
        uint32_t ph = 0;
        for (int tile = cluster_id; tile < num_tiles; tile += nclusters, ++it) {
            const int64_t t0 = int64_t(tile) * Mt;
            bool ok = true;
            // Eq.(15): sum of squares of this row's K-slice, from the ring stages
            float ss = 0.0f;
            for (int q = 0; q < NQ; ++q) {
                if (!mbar_wait(&full[s], ph) || *(volatile int*)&s_abort) { ok = false; break; }
                const uint4* row = reinterpret_cast<const uint4*>(sring + s * STAGE_BYTES + m * 128);
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    const uint4 v = row[g];
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const float lo = bf16_lo(w[h]), hi = bf16_hi(w[h]);
                        ss = fmaf(lo, lo, ss);
                        ss = fmaf(hi, hi, ss);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
                if (++s == STAGES) { s = 0; ph ^= 1; }
            }
            const int acc = it & 1;
            if (ok && !mbar_wait(&tfull[acc], uint32_t((it >> 1) & 1))) ok = false;
            if (!ok) { s_abort = 1; break; }
            tc_fence_after();
            float d[NB];
            const uint32_t taddr = tmem_base + (uint32_t(qd * 32) << 16) + uint32_t(acc * NB);
#pragma unroll
            for (int c = 0; c < NB; c += 16) {
                float tmp[16];
                tmem_ld16(taddr + c, tmp);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) d[c + j] = tmp[j];
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);

            // share this CTA's partial logits and sum of squares with the cluster
#pragma unroll
            for (int p = 0; p < P; ++p) spart[m * PS + p] = d[p];
            spart[m * PS + P] = ss;
            asm volatile("fence.acq_rel.cluster;" ::: "memory");
            mbar_arrive(epi_sync);
            if (et == 0) {
                if (!mbar_wait(epi_sync, 0)) { s_abort = 1; break; }
                for (uint32_t r = 0; r < CL; ++r) mbar_arrive_cluster(mapa(smem_u32(part_ready), r));
            }
            if (!mbar_wait<true>(part_ready, uint32_t(it & 1))) { s_abort = 1; break; }

            // coefficients of 16 tokens: lane group of 8 = one token, one source CTA per lane
            {
                const int jj = et >> 3, src = et & 7;
                const int j = int(rank) * TOK_PER_CTA + jj;     // row within the tile
                const uint32_t pbase = mapa(smem_u32(spart + j * PS), uint32_t(src));
                float v[PS];
#pragma unroll
                for (int p = 0; p < PS; ++p) v[p] = ld_cluster_f32(pbase + p * 4);
#pragma unroll
                for (int p = 0; p < PS; ++p) {
                    v[p] += __shfl_xor_sync(0xffffffffu, v[p], 1);
                    v[p] += __shfl_xor_sync(0xffffffffu, v[p], 2);
                    v[p] += __shfl_xor_sync(0xffffffffu, v[p], 4);
                }
                const int64_t t = t0 + j;
                if (src == 0 && j < Mt && t < T) {
                    const float r = sqrtf(v[P] * inv_K + eps);                     // Eq.(15)
                    const float inv_r = 1.0f / r;
                    float hp[N], m2[N][N];
#pragma unroll
                    for (int i = 0; i < N; ++i) {
                        hp[i] = sigmoidf_(a0 * v[i] * inv_r + __ldg(b + i));                   // Eq.(17)
                        Hpost[t * N + i] = 2.0f * sigmoidf_(a1 * v[N + i] * inv_r + __ldg(b + N + i)); // Eq.(18)
                        if (Hpre) Hpre[t * N + i] = hp[i];
                    }
#pragma unroll
                    for (int i = 0; i < N; ++i)
#pragma unroll
                        for (int k = 0; k < N; ++k)
                            m2[i][k] = a2 * v[2 * N + i * N + k] * inv_r + __ldg(b + 2 * N + i * N + k);
                    sinkhorn_regs<N>(m2, t_iters);                                    // Eq.(19)
#pragma unroll
                    for (int i = 0; i < N; ++i)
#pragma unroll
                        for (int k = 0; k < N; ++k) Hres[(t * N + i) * N + k] = m2[i][k];
                    for (uint32_t rr = 0; rr < CL; ++rr) {
                        const uint32_t hb = mapa(smem_u32(shpre + j * N), rr);
#pragma unroll
                        for (int i = 0; i < N; ++i) st_cluster_f32(hb + i * 4, hp[i]);
                    }
                }
            }
            asm volatile("fence.acq_rel.cluster;" ::: "memory");
            mbar_arrive(epi_sync);
            if (et == 0) {
                if (!mbar_wait(epi_sync, 1)) { s_abort = 1; break; }
                for (uint32_t r = 0; r < CL; ++r) mbar_arrive_cluster(mapa(smem_u32(hpre_ready), r));
            }
            if (!mbar_wait<true>(hpre_ready, uint32_t(it & 1))) { s_abort = 1; break; }

            // F_pre: x_in[t][c] = sum_i H_pre[t][i] X[t][i][c] for this CTA's channels
            const int VPT = Cs / 8;                  // 16-byte vectors per token
            const int rows = int((T - t0) < int64_t(Mt) ? (T - t0) : int64_t(Mt));
            const int items = rows * VPT;
#pragma unroll 2
            for (int w = et; w < items; w += EPI_THREADS) {
                const int tok = w / VPT, v = w - tok * VPT;
                const int64_t t = t0 + tok;
                const int c = c0 + v * 8;
                float o[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) o[e] = 0.0f;
#pragma unroll
                for (int i = 0; i < N; ++i) {
                    float xv[8];
                    load16<false>(X + (t * N + i) * C + c, xv);
                    const float h = shpre[tok * N + i];
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[e] = fmaf(h, xv[e], o[e]);
                }
                store16<false>(x_in + t * C + c, o);
            }
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, G::TMEM_COLS);
    }
    cluster_sync();   // no CTA leaves while a peer may still touch its shared memory
}

// ------------------------------------------------------------------ host

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

template <int N>
static int smem_bytes(int C) { return int(layout_for<N>(N * (C / CL) / KC).total) + 1024; }

template <int N>
static bool fits(int C) { return C % (CL * KC) == 0 && smem_bytes<N>(C) <= 227 * 1024; }

template <int N>
static mhc_status launch_n(const PreArgs& a, cudaStream_t s)
{
    static int configured_smem = 0;
    static int max_clusters = 0;
    const int smem = smem_bytes<N>(a.C);
    auto kern = pre_tc_kernel<N>;
    if (smem > configured_smem) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return cuda_status(e, "mhc_pre (tc): set shared memory size");
        configured_smem = smem;
        max_clusters = 0;
    }
    if (max_clusters == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(CL * 64);
        cfg.blockDim = dim3(NTHREADS);
        cfg.dynamicSmemBytes = size_t(configured_smem);
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = CL; attr.val.clusterDim.y = 1; attr.val.clusterDim.z = 1;
        cfg.attrs = &attr; cfg.numAttrs = 1;
        int nc = 0;
        cudaError_t e = cudaOccupancyMaxActiveClusters(&nc, kern, &cfg);
        if (e != cudaSuccess || nc <= 0) return cuda_status(e != cudaSuccess ? e : cudaErrorInvalidConfiguration,
                                                             "mhc_pre (tc): cluster occupancy");
        max_clusters = nc;
    }
    // Token tiles of Mt <= 128 rows, sized so that every cluster gets the same number.
    const int64_t rounds = (a.T + int64_t(max_clusters) * MROWS - 1) / (int64_t(max_clusters) * MROWS);
    const int64_t per_round = (a.T + rounds - 1) / rounds;                     // tokens per round
    int Mt = int((per_round + max_clusters - 1) / max_clusters);
    if (Mt > MROWS) Mt = MROWS;
    const int64_t tiles64 = (a.T + Mt - 1) / Mt;
    const int nclusters = int(tiles64 < max_clusters ? tiles64 : max_clusters);

    EncodeTiledFn enc = encode_fn();
    if (!enc) {
        set_error("mhc_pre (tc): cuTensorMapEncodeTiled unavailable");
        return MHC_ERR_CUDA;
    }
    CUtensorMap map;
    const cuuint64_t dims[3] = {cuuint64_t(a.C), cuuint64_t(a.n), cuuint64_t(a.T)};
    const cuuint64_t strides[2] = {cuuint64_t(a.C) * 2, cuuint64_t(a.n) * a.C * 2};
    const cuuint32_t box[3] = {KC, 1, cuuint32_t(Mt)};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.X), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("mhc_pre (tc): cuTensorMapEncodeTiled failed (%d)", int(r));
        return MHC_ERR_CUDA;
    }
    kern<<<dim3(unsigned(nclusters * CL)), NTHREADS, size_t(smem), s>>>(
        map, static_cast<const bf16_t*>(a.X), static_cast<const bf16_t*>(a.phi), a.alpha[0], a.alpha[1],
        a.alpha[2], a.b, a.T, a.C, Mt, int(tiles64), a.t_iters, a.eps, static_cast<bf16_t*>(a.x_in),
        a.H_pre, a.H_post, a.H_res);
    return launch_status("mhc_pre (tc) kernel");
}

}  // namespace pretc

bool pre_tc_supported(const PreArgs& a)
{
    if (a.x_dt != MHC_BF16 || a.phi_dt != MHC_BF16 || a.T < 1 || a.T >= (int64_t(1) << 31)) return false;
    switch (a.n) {
        case 2: return pretc::fits<2>(a.C);
        case 3: return pretc::fits<3>(a.C);
        case 4: return pretc::fits<4>(a.C);
        default: return false;
    }
}

mhc_status launch_pre_tc(const PreArgs& a, cudaStream_t s)
{
    switch (a.n) {
        case 2: return pretc::launch_n<2>(a, s);
        case 3: return pretc::launch_n<3>(a, s);
        case 4: return pretc::launch_n<4>(a, s);
        default: break;
    }
    set_error("mhc_pre (tc): n=%d not supported", a.n);
    return MHC_ERR_UNSUPPORTED;
}

}  // namespace mhc
