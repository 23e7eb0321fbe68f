// mhc_pre for n = 5..8 streams, tensor-core path: a projection kernel
// (TMA + tcgen05.mma + TMEM, clusters of 8 CTAs) that writes the coefficients,
// then a streaming x_in pass.  The same kernel serves every n <= 7 when phi is
// given in tf32 ([mHC] Eq.(10)) as its exact bf16 pair (phi_tf32.cu): the stage
// then carries both halves of phiT and the epilogue adds their columns.
//
// [mHC] section 4.3.1, Eq.(14)-(19), and F_pre := H_pre x_l, as in
// mhc_pre_tc.cu.  With n >= 5 the projection has P = n^2 + 2n = 35..80
// outputs, too many for the pair layout of mhc_pre_tc.cu (one MMA with
// N = 2R + 128 <= 256), and a token is 10-16 KB per stream group, too much to
// keep a tile in L2 until its x_in re-read.  So:
//   * the projection streams one stream of a 128-token tile per ring stage,
//         [ phiT rows of stream i (R = P rounded up to 16) | X rows of stream i (128) ]
//     and one MMA per 16-wide K step, M = 128 tokens, N = R + 128, adds the
//     stream's contribution to the same P projection columns (every stream and
//     channel block accumulates into them: the projection sums over the whole
//     n*C row) and, in column R + m, to row m's sum of squares;
//   * x_in = H_pre X is a separate pass that streams X again (one block per
//     token, like mhc_post).
// The 8 CTAs of a cluster split the channels; TMEM lane quarter q of every CTA
// holds tokens 32q..32q+31 of the tile, whose partial rows (projections and sum
// of squares of this CTA's K-slice) go by st.async to the token's owner (16
// tokens per CTA).  The owner reduces the 8 partial rows (4 lanes per token),
// runs Eq.16-19 (Sinkhorn n x n in registers) and writes the coefficients;
// after reading the partial rows it tells every CTA of the cluster with a
// 4-byte st.async that completes transactions on that CTA's part_free barrier
// of the tile (two of them, alternating by tile); a CTA pushes the next tile's
// rows into the same buffer only after that phase.  Every remote store into a
// CTA is awaited by that CTA before it exits.
//
// Warp roles (6 warps): 0 TMA producer, 1 MMA issuer, 2-5 one TMEM lane
// quarter each (quarter = warp % 4); warps 2-3 also compute the coefficients.
// Every wait is bounded and warp-uniform.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace mhc {
namespace prewide {

using namespace sm100;

constexpr int CL = 8;
constexpr int MROWS = 128;       // tokens per tile (M)
constexpr int KC = 64;
constexpr int MAX_STAGES = 8;
constexpr int SMEM_LIMIT = 227 * 1024;
constexpr int NTHREADS = 192;
constexpr int EPI_WARP0 = 2, EPI_WARPS = 4;
constexpr int TOK_PER_CTA = MROWS / CL;   // 16 tokens whose coefficients a CTA computes
constexpr int LPT = 4;                    // coefficient lanes per token (warps 2-3)
constexpr int ACC_COLS = 256;
constexpr int TMEM_COLS = 512;
static_assert(TOK_PER_CTA * LPT == 64, "warps 2-3: one 4-lane group per token");

// SPLIT: phi is the exact bf16 pair of a tf32 phi (phi_tf32.cu): the stage holds
// hi rows [0, RH) and lo rows [RH, 2 RH), and logit p is column p + column RH + p.
template <int N, bool SPLIT> struct Cfg {
    static constexpr int P = N * N + 2 * N;
    static constexpr int RH = (P + 15) / 16 * 16;  // rows of one phiT half (M = 128 needs N % 16 == 0)
    static constexpr int R = SPLIT ? 2 * RH : RH;  // phiT rows per stage
    static constexpr int MMA_N = R + MROWS;
    static constexpr int STAGE_BYTES = MMA_N * 128;
    static constexpr int PS = P + 1;
    static constexpr int PSP = (PS + 3) / 4 * 4;
    static_assert(MMA_N <= ACC_COLS, "MMA N for M = 128");
};

enum Bar { B_FULL = 0, B_EMPTY = B_FULL + MAX_STAGES, B_TFULL = B_EMPTY + MAX_STAGES, B_TEMPTY = B_TFULL + 2,
           B_PART = B_TEMPTY + 2, B_FREE = B_PART + 1, B_DRAIN = B_FREE + 2, B_COUNT };
constexpr int SINK_FLOATS = 2 * CL * 2;   // [tile parity][owner rank][coefficient warp]: release tokens

struct Layout {
    uint32_t ring, part, bias, sink, bars, slot, total;
    int stages;
};

template <int N, bool SPLIT>
__host__ __device__ constexpr uint32_t fixed_bytes() {
    using G = Cfg<N, SPLIT>;
    return CL * TOK_PER_CTA * G::PSP * 4 + G::P * 4 + 16 + SINK_FLOATS * 4 + B_COUNT * 8 + 16;
}

template <int N, bool SPLIT>
__host__ __device__ constexpr int stages_fit() {
    constexpr int64_t room = int64_t(SMEM_LIMIT) - 1024 - fixed_bytes<N, SPLIT>();
    constexpr int64_t fit = room > 0 ? room / Cfg<N, SPLIT>::STAGE_BYTES : 0;
    return int(fit < MAX_STAGES ? fit : MAX_STAGES);
}

template <int N, bool SPLIT>
__host__ __device__ inline Layout layout_for() {
    using G = Cfg<N, SPLIT>;
    Layout L;
    L.ring = 0;
    L.stages = stages_fit<N, SPLIT>();
    L.part = L.ring + uint32_t(L.stages) * G::STAGE_BYTES;
    L.bias = L.part + CL * TOK_PER_CTA * G::PSP * 4;
    L.sink = (L.bias + G::P * 4 + 15) / 16 * 16;
    L.bars = L.sink + SINK_FLOATS * 4;
    L.slot = L.bars + B_COUNT * 8;
    L.total = L.slot + 16;
    return L;
}

template <int N, bool SPLIT>
__global__ void __cluster_dims__(CL, 1, 1) __launch_bounds__(NTHREADS, 1)
proj_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmPhi, float a0,
            float a1, float a2, const float* __restrict__ b, int64_t T, int C, int Mt, int num_tiles, int t_iters,
            float eps, float* __restrict__ Hpre, float* __restrict__ Hpost, float* __restrict__ Hres,
            float* __restrict__ hpre_alt, int64_t alt_stride)
{
    using G = Cfg<N, SPLIT>;
    constexpr int P = G::P, R = G::R, RH = G::RH, PS = G::PS, PSP = G::PSP, STAGE_BYTES = G::STAGE_BYTES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int Cs = C / CL;
    const int CB = Cs / KC;
    const int SPT = CB * N;            // ring stages per tile: (channel block, stream)
    const Layout L = layout_for<N, SPLIT>();
    const int STAGES = L.stages;
    uint8_t* sring = smem + L.ring;
    float* rpart = reinterpret_cast<float*>(smem + L.part);   // [CL][TOK_PER_CTA][PSP], pushed by the cluster
    float* sb = reinterpret_cast<float*>(smem + L.bias);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint64_t* full = bars + B_FULL;
    uint64_t* empty = bars + B_EMPTY;
    uint64_t* tfull = bars + B_TFULL;
    uint64_t* tempty = bars + B_TEMPTY;
    uint64_t* part_full = bars + B_PART;     // this CTA's tokens: all partial rows of a tile landed
    uint64_t* part_free = bars + B_FREE;     // [2] every owner has read its partial rows of a tile
    uint64_t* drain = bars + B_DRAIN;
    float* sink = reinterpret_cast<float*>(smem + L.sink);  // [2][CL][2] release tokens (never read)
    uint32_t* slot = reinterpret_cast<uint32_t*>(smem + L.slot);
    __shared__ int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int cluster_id = blockIdx.x / CL;
    const int nclusters = gridDim.x / CL;
    const int c0 = int(rank) * Cs;

    if (threadIdx.x == 0) {
        // launch self-check: the layout fits the dynamic shared memory this launch got
        // and the tile shape is one the kernel was written for (uniform over the grid)
        uint32_t dyn;
        asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
        const uint32_t need = uint32_t(smem - smem_raw) + L.total;
        const bool bad = need > dyn || STAGES < 2 || Mt < 8 || Mt > MROWS || (Mt & 7) || CB < 1 ||
                         Cs % KC || int(gridDim.x) % CL;
        s_abort = bad ? 1 : 0;
        if (bad) atomicOr(&g_device_error, 4u);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], EPI_WARPS);
        }
        mbar_init(part_full, 1);
        mbar_init(&part_free[0], 1);         // armed per tile; completed by 2 x CL 4-byte tokens
        mbar_init(&part_free[1], 1);
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (s_abort) return;                      // uniform over the grid: nothing allocated yet
    if (warp == 1) tmem_alloc(slot, TMEM_COLS);
    for (int p = threadIdx.x; p < P; p += NTHREADS) sb[p] = b[p];
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *slot;
    if (threadIdx.x == 0) {
        if (tmem_base != 0u) {                // 512 columns: the whole of this SM's TMEM
            atomicOr(&g_device_error, 4u);
            s_abort = 1;
        }
        tma_prefetch(&tmX);
        tma_prefetch(&tmPhi);
    }
    cluster_sync();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t keep = policy_evict_last();
            const uint64_t drop = policy_evict_first();
            const uint32_t tx = uint32_t(R + Mt) * 128;
            int s = 0, n_issued = 0;
            uint32_t ph = 0;
            int inflight_s[MAX_STAGES], inflight_ph[MAX_STAGES];
            bool ok = true;
            for (int tile = cluster_id; tile < num_tiles && ok; tile += nclusters) {
                const int t0 = tile * Mt;
                for (int q = 0; q < SPT; ++q) {
                    if (!mbar_wait(&empty[s], ph ^ 1) || *(volatile int*)&s_abort) { ok = false; break; }
                    mbar_arrive_expect_tx(&full[s], tx);
                    const int cc = c0 + (q / N) * KC, i = q % N;
                    uint8_t* st = sring + s * STAGE_BYTES;
                    tma_load_3d_hint(st, &tmPhi, &full[s], cc, 0, i, keep);           // phiT {64, R, 1}
                    tma_load_3d_hint(st + R * 128, &tmX, &full[s], cc, t0, i, drop);  // X {64, Mt, 1}
                    inflight_s[n_issued % MAX_STAGES] = s;
                    inflight_ph[n_issued % MAX_STAGES] = int(ph);
                    ++n_issued;
                    if (++s == STAGES) { s = 0; ph ^= 1; }
                }
            }
            if (!ok) {
                s_abort = 1;
                const int pending = n_issued < STAGES ? n_issued : STAGES;
                for (int j = 0; j < pending; ++j) {
                    const int kk = (n_issued - 1 - j) % MAX_STAGES;
                    mbar_wait(&full[inflight_s[kk]], uint32_t(inflight_ph[kk]), 1ll << 22);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(MROWS, G::MMA_N);
            const uint32_t ring_a = smem_u32(sring);
            int s = 0, it = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int tile = cluster_id; tile < num_tiles && ok; tile += nclusters, ++it) {
                const int acc = it & 1;
                if (!mbar_wait(&tempty[acc], (uint32_t((it >> 1) & 1)) ^ 1)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem_base + uint32_t(acc * ACC_COLS);
                for (int q = 0; q < SPT; ++q) {
                    if (!mbar_wait(&full[s], ph) || *(volatile int*)&s_abort) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < KC / 16; ++kk) {
                        const uint32_t base = ring_a + s * STAGE_BYTES + kk * 32;
                        const uint64_t ad = sdesc_k_sw128(base + R * 128);   // the stream's X rows
                        const uint64_t bd = sdesc_k_sw128(base);             // phiT rows, then X rows
                        mma_bf16(d, ad, bd, idesc, (q | kk) != 0);
                    }
                    mma_commit(&empty[s]);
                    if (++s == STAGES) { s = 0; ph ^= 1; }
                }
                if (ok) mma_commit(&tfull[acc]);
            }
            if (!ok) s_abort = 1;
            // TMEM is freed only after every issued MMA has finished, whatever the epilogue did
            mma_commit(drain);
            mbar_wait(drain, 0, 1ll << 22);
        }
    } else {
        // ------------------------------------------------------------ epilogue (warps 2-5)
        const int et = threadIdx.x - EPI_WARP0 * 32;    // 0..127
        const int qd = warp & 3;                        // TMEM lane quarter
        const int r = qd * 32 + lane;                   // TMEM row = token within the tile
        const float inv_K = 1.0f / float(N * C);
        constexpr uint32_t PART_BYTES = CL * TOK_PER_CTA * PSP * 4;
        constexpr uint32_t FREE_BYTES = CL * 2 * 4;     // one 4-byte token per owner and coefficient warp
        const uint32_t owner = uint32_t(r / TOK_PER_CTA);
        const uint32_t push_dst = mapa(smem_u32(rpart + (int(rank) * TOK_PER_CTA + r % TOK_PER_CTA) * PSP), owner);
        const uint32_t push_bar = mapa(smem_u32(part_full), owner);
        int it = 0;
        bool alive = !*(volatile int*)&s_abort;
        for (int tile = cluster_id; tile < num_tiles && alive; tile += nclusters, ++it) {
            const int64_t t0 = int64_t(tile) * Mt;
            const int acc = it & 1;
            if (et == 0) {
                // this tile's phases; pushes and tokens may land before or after.  The
                // previous phase of part_free[acc] (tile it-2) was awaited in iteration it-1.
                mbar_arrive_expect_tx(part_full, PART_BYTES);
                mbar_arrive_expect_tx(&part_free[acc], FREE_BYTES);
            }
            if (!warp_wait(&tfull[acc], uint32_t((it >> 1) & 1))) { s_abort = 1; alive = false; break; }
            tc_fence_after();
            float d[RH];
            const uint32_t taddr = tmem_base + (uint32_t(qd * 32) << 16) + uint32_t(acc * ACC_COLS);
#pragma unroll
            for (int c = 0; c < RH; c += 16) {
                float tmp[16];
                tmem_ld16(taddr + c, tmp);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) d[c + j] = tmp[j];
                if constexpr (SPLIT) {                  // x . lo, added to x . hi
                    tmem_ld16(taddr + RH + c, tmp);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) d[c + j] += tmp[j];
                }
            }
            float ss = 0.0f;
#pragma unroll
            for (int c = 0; c < 32; c += 16) {          // column R + r: X row r . X row r
                float tmp[16];
                tmem_ld16(taddr + R + qd * 32 + c, tmp);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) if (c + j == lane) ss = tmp[j];
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);

            // every owner is done with the partial rows of tile it-1
            if (it >= 1 && !warp_wait(&part_free[(it - 1) & 1], uint32_t(((it - 1) >> 1) & 1))) {
                s_abort = 1;
                alive = false;
                break;
            }
#pragma unroll
            for (int p = 0; p < PSP; p += 4) {
                float v4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) v4[e] = p + e < P ? d[p + e] : (p + e == P ? ss : 0.0f);
                st_async_f32x4(push_dst + p * 4, make_float4(v4[0], v4[1], v4[2], v4[3]), push_bar);
            }
            if (et < 64) {
                if (!warp_wait(part_full, uint32_t(it & 1))) { s_abort = 1; alive = false; break; }
                const int jj = et / LPT, g = et % LPT;
                const int j = int(rank) * TOK_PER_CTA + jj;     // token row within the tile
                constexpr int OWN = (PS + LPT - 1) / LPT;
                float own[OWN];
#pragma unroll
                for (int k = 0; k < OWN; ++k) {
                    const int p = g + LPT * k;
                    float s0 = 0.0f, s1 = 0.0f;
                    if (p < PS) {
#pragma unroll
                        for (int c = 0; c < CL; c += 2) {
                            s0 += rpart[(c * TOK_PER_CTA + jj) * PSP + p];
                            s1 += rpart[((c + 1) * TOK_PER_CTA + jj) * PSP + p];
                        }
                    }
                    own[k] = s0 + s1;
                }
                float v[PS];
#pragma unroll
                for (int p = 0; p < PS; ++p) v[p] = __shfl_sync(0xffffffffu, own[p / LPT], p % LPT, LPT);
                // this warp has read its partial rows: release them to every CTA of the cluster
                if (lane == 0) {
                    const uint32_t tok = smem_u32(sink + (acc * CL + int(rank)) * 2 + (warp - EPI_WARP0));
                    const uint32_t fb = smem_u32(&part_free[acc]);
                    for (uint32_t cr = 0; cr < CL; ++cr) st_async_f32(mapa(tok, cr), 0.0f, mapa(fb, cr));
                }
                const float rr_ = sqrtf(v[P] * inv_K + eps);                  // Eq.(15)
                const float inv_r = 1.0f / rr_;
                float m[N][N];
#pragma unroll
                for (int i = 0; i < N; ++i)
#pragma unroll
                    for (int k = 0; k < N; ++k)
                        m[i][k] = a2 * v[2 * N + i * N + k] * inv_r + sb[2 * N + i * N + k];   // Eq.(16)
                sinkhorn_regs<N>(m, t_iters);                                  // Eq.(19)
                const int64_t t = t0 + j;
                if (j < Mt && t < T) {
                    // lane g writes streams i = g, g + 4 (gates) and the matching rows of H_res
#pragma unroll
                    for (int i = 0; i < N; ++i) {
                        if (i % LPT != g) continue;
                        const float hp = sigmoidf_(a0 * v[i] * inv_r + sb[i]);                     // Eq.(17)
                        if (Hpre) Hpre[t * N + i] = hp;
                        if (hpre_alt) hpre_alt[t * alt_stride + i] = hp;
                        Hpost[t * N + i] = 2.0f * sigmoidf_(a1 * v[N + i] * inv_r + sb[N + i]);  // Eq.(18)
#pragma unroll
                        for (int k = 0; k < N; ++k) Hres[(t * N + i) * N + k] = m[i][k];
                    }
                }
            }
        }
        // the last tile's tokens: every remote store into this CTA lands before it exits
        if (alive && it >= 1) warp_wait(&part_free[(it - 1) & 1], uint32_t(((it - 1) >> 1) & 1));
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
    cluster_sync();
}

// x_in[t] = sum_i H_pre[t][i] X[t][i]: one block per token; H_pre from H_pre or,
// when the caller passed none, from the first N floats of the token's own x_in
// row (where the projection kernel parked it), read before the row is written.
template <int N>
__global__ void __launch_bounds__(256)
xin_kernel(const bf16_t* __restrict__ X, const float* __restrict__ Hpre, int64_t T, int C, bf16_t* x_in)
{
    __shared__ float h[N];
    const int64_t t = blockIdx.x;
    if (threadIdx.x < N)
        h[threadIdx.x] = Hpre ? Hpre[t * N + threadIdx.x]
                              : reinterpret_cast<const float*>(x_in + t * int64_t(C))[threadIdx.x];
    __syncthreads();
    for (int c = threadIdx.x * 8; c < C; c += 256 * 8) {
        uint4 raw[N];
#pragma unroll
        for (int i = 0; i < N; ++i) raw[i] = ldg16_raw_hint(X + (t * N + i) * int64_t(C) + c, policy_evict_first());
        float o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = 0.0f;
#pragma unroll
        for (int i = 0; i < N; ++i) {
            const uint32_t w4[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                o[2 * e] = fmaf(h[i], bf16_lo(w4[e]), o[2 * e]);
                o[2 * e + 1] = fmaf(h[i], bf16_hi(w4[e]), o[2 * e + 1]);
            }
        }
        store16<true>(x_in + t * C + c, o);
    }
}

// ------------------------------------------------------------------ host

template <int N, bool SPLIT>
static mhc_status launch_n(const PreArgs& a, cudaStream_t s)
{
    static int configured = 0, max_clusters = 0;
    auto kern = proj_kernel<N, SPLIT>;
    const int smem = int(layout_for<N, SPLIT>().total) + 1024;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return cuda_status(e, "mhc_pre (n > 4): set shared memory size");
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(CL * 64);
        cfg.blockDim = dim3(NTHREADS);
        cfg.dynamicSmemBytes = size_t(smem);
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = CL; attr.val.clusterDim.y = 1; attr.val.clusterDim.z = 1;
        cfg.attrs = &attr; cfg.numAttrs = 1;
        int nc = 0;
        e = cudaOccupancyMaxActiveClusters(&nc, kern, &cfg);
        if (e != cudaSuccess || nc <= 0)
            return cuda_status(e != cudaSuccess ? e : cudaErrorInvalidConfiguration, "mhc_pre (n > 4): cluster occupancy");
        max_clusters = nc;
        configured = 1;
    }
    // tiles of Mt <= 128 tokens (a multiple of 8): the busiest cluster's tokens plus a
    // per-tile overhead, minimised
    constexpr int TILE_COST = 32;
    int Mt = MROWS;
    int64_t best = -1;
    for (int m = MROWS; m >= 8; m -= 8) {
        const int64_t tiles = (a.T + m - 1) / m;
        const int64_t cost = (tiles + max_clusters - 1) / max_clusters * (m + TILE_COST);
        if (best < 0 || cost < best) { best = cost; Mt = m; }
    }
    const int64_t tiles64 = (a.T + Mt - 1) / Mt;
    const int nclusters = int(tiles64 < max_clusters ? tiles64 : max_clusters);
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) {
        set_error("mhc_pre (n > 4): cuTensorMapEncodeTiled unavailable");
        return MHC_ERR_CUDA;
    }
    using G = Cfg<N, SPLIT>;
    CUtensorMap mapX, mapPhi;
    {
        // X [T][n][C] viewed as {C, T, n}: a box {64, Mt, 1} holds one stream's rows
        const cuuint64_t dims[3] = {cuuint64_t(a.C), cuuint64_t(a.T), cuuint64_t(N)};
        const cuuint64_t strides[2] = {cuuint64_t(N) * a.C * 2, cuuint64_t(a.C) * 2};
        const cuuint32_t box[3] = {KC, cuuint32_t(Mt), 1};
        const cuuint32_t estr[3] = {1, 1, 1};
        CUresult r = enc(&mapX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.X), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            set_error("mhc_pre (n > 4): cuTensorMapEncodeTiled(X) failed (%d)", int(r));
            return MHC_ERR_CUDA;
        }
    }
    {
        // phiT [P][n*C] viewed as {C, P, n}: a box {64, R, 1} holds R rows (rows >= P
        // zero); the tf32 pair [2 RH][n*C] as {C, 2 RH, n}: one box holds both halves
        const cuuint64_t dims[3] = {cuuint64_t(a.C), cuuint64_t(SPLIT ? 2 * G::RH : G::P), cuuint64_t(N)};
        const cuuint64_t strides[2] = {cuuint64_t(N) * a.C * 2, cuuint64_t(a.C) * 2};
        const cuuint32_t box[3] = {KC, cuuint32_t(G::R), 1};
        const cuuint32_t estr[3] = {1, 1, 1};
        CUresult r = enc(&mapPhi, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.phi), dims, strides, box,
                         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            set_error("mhc_pre (n > 4): cuTensorMapEncodeTiled(phi) failed (%d)", int(r));
            return MHC_ERR_CUDA;
        }
    }
    // without a caller H_pre the gates wait in the first N floats of each x_in row
    // (a row holds 2C >= 4N bytes)
    float* alt = a.H_pre ? nullptr : static_cast<float*>(a.x_in);
    const int64_t alt_stride = a.C / 2;                         // floats per x_in row
    kern<<<dim3(unsigned(nclusters * CL)), NTHREADS, size_t(smem), s>>>(
        mapX, mapPhi, a.alpha[0], a.alpha[1], a.alpha[2], a.b, a.T, a.C, Mt, int(tiles64), a.t_iters, a.eps,
        a.H_pre, a.H_post, a.H_res, alt, alt_stride);
    mhc_status st = launch_status("mhc_pre (n > 4) projection kernel");
    if (st != MHC_OK) return st;
    xin_kernel<N><<<dim3(unsigned(a.T)), 256, 0, s>>>(static_cast<const bf16_t*>(a.X), a.H_pre, a.T, a.C,
                                                     static_cast<bf16_t*>(a.x_in));
    return launch_status("mhc_pre (n > 4) x_in kernel");
}

}  // namespace prewide

bool pre_wide_supported(const PreArgs& a)
{
    const bool shape = (a.phi_dt == MHC_BF16 && a.n >= 5 && a.n <= 8) ||
                       (a.phi_dt == MHC_TF32_PAIR && a.n >= 1 && a.n <= 7);   // 2 RH + 128 <= 256
    return a.x_dt == MHC_BF16 && shape && a.T >= 1 && a.T < (int64_t(1) << 31) &&
           a.C % (prewide::CL * prewide::KC) == 0 && !a.skip_xin && !a.u_out;
}

mhc_status launch_pre_wide(const PreArgs& a, cudaStream_t s)
{
    if (a.phi_dt == MHC_TF32_PAIR) {
        switch (a.n) {
            case 1: return prewide::launch_n<1, true>(a, s);
            case 2: return prewide::launch_n<2, true>(a, s);
            case 3: return prewide::launch_n<3, true>(a, s);
            case 4: return prewide::launch_n<4, true>(a, s);
            case 5: return prewide::launch_n<5, true>(a, s);
            case 6: return prewide::launch_n<6, true>(a, s);
            case 7: return prewide::launch_n<7, true>(a, s);
            default: break;
        }
    }
    switch (a.n) {
        case 5: return prewide::launch_n<5, false>(a, s);
        case 6: return prewide::launch_n<6, false>(a, s);
        case 7: return prewide::launch_n<7, false>(a, s);
        case 8: return prewide::launch_n<8, false>(a, s);
        default: break;
    }
    set_error("mhc_pre (n > 4): n=%d not supported", a.n);
    return MHC_ERR_UNSUPPORTED;
}

}  // namespace mhc
