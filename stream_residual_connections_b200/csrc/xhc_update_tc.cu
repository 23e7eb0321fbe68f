// xhc_sparse_update, tensor-core path (sm_100a: cp.async gather + TMA +
// tcgen05.mma + TMEM + a cluster of 8 CTAs sharing partial sums through
// distributed shared memory).
//
// [xHC] section "sparse residual stream architecture", step 3, and
// "parameterisation" (the same formulas as the CUDA-core path in
// xhc_update.cu), for k = 4 active streams and Kr <= 4:
//   X_act = rows idx[t][0..3] of X_t;  r = RMS(vec X_act) over 4C
//   z = alpha * (vec X_act . phi_act^T) / r + b_act   (res 16 | post 4 Kr)
//   H_res = Sinkhorn(mat(z_res)), H_post = 2 sigma(z_post)
//   X[t][idx[t][j]] = sum_l H_res[j][l] X_act[l] + w[t][j] sum_q H_post[j][q] V[t][q]
//
// The projection has the shape of xhc_route's with the 4 active rows as the 4
// streams of a group: per tile of 32 tokens the 8 CTAs of a cluster split the
// C channels; a ring stage holds one 64-channel block
//     [ phi_act^T rows of the 4 slots (R each) | the gathered X rows (4 x 32) ]
// and one tcgen05.mma per 16-wide K step (M = 128, N = 4R + 128) gives in TMEM
// row l*32 + t the projections of slot l's K-slice (columns [lR, lR + R)) and
// its sum of squares (column 4R + l*32 + t).  The X rows are gathered by
// cp.async (TMA tiles cannot follow idx), swizzled as the MMA expects; each
// gather thread waits for its copies and fences them into the async proxy
// before it arrives on the stage's barrier.
//
// Warp roles (16 warps):
//   0      phi_act^T TMA ({64, R, 4} boxes of phi_act^T viewed as {C, P, 4})
//   1      MMA issuer (fp32 accumulators in TMEM, double-buffered over tiles)
//   2-3    gather: cp.async of the 128 rows x 128 bytes of every stage; they
//          run at most LAG tiles ahead of the write-back (its re-read of the
//          gathered rows then hits L2)
//   4-7    one TMEM lane quarter each: push every row's partial projections
//          and sum of squares (st.async) to the token's owner CTA (4 tokens per
//          CTA); warps 4-5 of the owner reduce the 4 x 8 partial rows (16 lanes
//          per token), run the 4 x 4 Sinkhorn, form H_post and push H_res and
//          H_post to every CTA of the cluster
//   8-15   write-back of this CTA's channels: the gathered rows again (L2), V
//          (fp32) and w, mixed and stored in place
// An idx entry outside [0, N) is reported in the device error word (bit 1)
// and that token is left unchanged.  Every wait is bounded and warp-uniform.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace mhc {
namespace xutc {

using namespace sm100;

constexpr int K = 4;             // active streams (slots) per token
constexpr int CL = 8;
constexpr int MROWS = 128;       // 4 slots x 32 tokens
constexpr int MT = 32;
constexpr int KC = 64;
constexpr int MAX_STAGES = 8;
constexpr int SMEM_LIMIT = 227 * 1024;
constexpr int NTHREADS = 512;
constexpr int GATHER_WARP0 = 2, GATHER_THREADS = 64;
constexpr int EPI_WARP0 = 4, EPI_WARPS = 4;
constexpr int WB_WARP0 = 8, WB_WARPS = 8, WB_THREADS = WB_WARPS * 32;
constexpr int TOK_PER_CTA = MT / CL;
constexpr int LPT = 16;
constexpr int ACC_COLS = 256;
constexpr int TMEM_COLS = 512;
constexpr int LAG = 3;
constexpr int GD = 2;            // stages a gather thread keeps in flight before it arrives
static_assert(TOK_PER_CTA * LPT == 64, "warps 4-5: one 16-lane group per token");
static_assert(MROWS * 8 % GATHER_THREADS == 0, "16-byte gather chunks per thread");

template <int KR> struct Cfg {
    static constexpr int PA = K * K + K * KR;       // logits: res 16 | post 4 Kr
    static constexpr int R = (PA + 7) / 8 * 8;
    static constexpr int MMA_N = K * R + MROWS;
    static constexpr int STAGE_BYTES = MMA_N * 128;
    static constexpr int PHI_BYTES = K * R * 128;
    static constexpr int PS = R + 1;
    static constexpr int PSP = (PS + 3) / 4 * 4;
    static constexpr int CS = K * K + K * KR;       // coefficients pushed per token
    static_assert(MMA_N % 16 == 0 && MMA_N <= ACC_COLS, "MMA N for M = 128");
};

enum Bar { B_FULL = 0, B_EMPTY = B_FULL + MAX_STAGES, B_TFULL = B_EMPTY + MAX_STAGES, B_TEMPTY = B_TFULL + 2,
           B_PART = B_TEMPTY + 2, B_COEF, B_WB = B_COEF + 2, B_DRAIN, B_COUNT };

struct Layout {
    uint32_t ring, part, coef, bias, bars, slot, total;
    int stages;
};

template <int KR>
__host__ __device__ constexpr uint32_t fixed_bytes() {
    using G = Cfg<KR>;
    return CL * K * TOK_PER_CTA * G::PSP * 4 + 2 * MT * G::CS * 4 + G::PA * 4 + 16 + B_COUNT * 8 + 16;
}

template <int KR>
__host__ __device__ constexpr int stages_fit() {
    constexpr int64_t room = int64_t(SMEM_LIMIT) - 1024 - fixed_bytes<KR>();
    constexpr int64_t fit = room > 0 ? room / Cfg<KR>::STAGE_BYTES : 0;
    return int(fit < MAX_STAGES ? fit : MAX_STAGES);
}

template <int KR>
__host__ __device__ inline Layout layout_for() {
    using G = Cfg<KR>;
    Layout L;
    L.ring = 0;
    L.stages = stages_fit<KR>();
    L.part = L.ring + uint32_t(L.stages) * G::STAGE_BYTES;
    L.coef = L.part + CL * K * TOK_PER_CTA * G::PSP * 4;
    L.bias = L.coef + 2 * MT * G::CS * 4;
    L.bars = (L.bias + G::PA * 4 + 15) / 16 * 16;
    L.slot = L.bars + B_COUNT * 8;
    L.total = L.slot + 16;
    return L;
}

template <int KR>
__global__ void __cluster_dims__(CL, 1, 1) __launch_bounds__(NTHREADS, 1)
update_tc_kernel(const __grid_constant__ CUtensorMap tmPhi, bf16_t* X, const float* __restrict__ V,
                 const int32_t* __restrict__ idx, const float* __restrict__ w, float a_res, float a_post,
                 const float* __restrict__ b, int64_t T, int N, int C, int num_tiles, int t_iters, float eps,
                 float* __restrict__ Hres_out, float* __restrict__ Hpost_out)
{
    using G = Cfg<KR>;
    constexpr int R = G::R, PA = G::PA, PS = G::PS, PSP = G::PSP, CS = G::CS, STAGE_BYTES = G::STAGE_BYTES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int Cs = C / CL;
    const int CB = Cs / KC;            // ring stages per tile
    const Layout L = layout_for<KR>();
    const int STAGES = L.stages;
    uint8_t* sring = smem + L.ring;
    float* rpart = reinterpret_cast<float*>(smem + L.part);   // [CL][K][TOK_PER_CTA][PSP]
    float* scoef = reinterpret_cast<float*>(smem + L.coef);   // [2][MT][CS]: H_res (16), H_post (4 Kr)
    float* sb = reinterpret_cast<float*>(smem + L.bias);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint64_t* full = bars + B_FULL;
    uint64_t* empty = bars + B_EMPTY;
    uint64_t* tfull = bars + B_TFULL;
    uint64_t* tempty = bars + B_TEMPTY;
    uint64_t* part_full = bars + B_PART;
    uint64_t* coef_full = bars + B_COEF;
    uint64_t* wb_prog = bars + B_WB;
    uint64_t* drain = bars + B_DRAIN;
    uint32_t* slot = reinterpret_cast<uint32_t*>(smem + L.slot);
    __shared__ int s_abort;
    __shared__ int s_wb_done;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int cluster_id = blockIdx.x / CL;
    const int nclusters = gridDim.x / CL;
    const int c0 = int(rank) * Cs;

    if (threadIdx.x == 0) {
        s_abort = 0;
        s_wb_done = 0;
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1 + GATHER_THREADS);    // the phi TMA, then every gather thread
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], EPI_WARPS);
        }
        mbar_init(part_full, 1);
        mbar_init(&coef_full[0], 1);
        mbar_init(&coef_full[1], 1);
        mbar_init(wb_prog, WB_WARPS);
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(slot, TMEM_COLS);
    for (int p = threadIdx.x; p < PA; p += NTHREADS) sb[p] = b[p];
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *slot;
    if (threadIdx.x == 0) tma_prefetch(&tmPhi);
    cluster_sync();

    if (warp == 0) {
        // ------------------------------------------------------------ phi_act^T TMA
        if (lane == 0) {
            const uint64_t keep = policy_evict_last();
            int s = 0, n_issued = 0;
            uint32_t ph = 0;
            int inflight_s[MAX_STAGES], inflight_ph[MAX_STAGES];
            bool ok = true;
            for (int tile = cluster_id; tile < num_tiles && ok; tile += nclusters)
                for (int cb = 0; cb < CB; ++cb) {
                    if (!mbar_wait(&empty[s], ph ^ 1) || *(volatile int*)&s_abort) { ok = false; break; }
                    mbar_arrive_expect_tx(&full[s], uint32_t(G::PHI_BYTES));
                    tma_load_3d_hint(sring + s * STAGE_BYTES, &tmPhi, &full[s], c0 + cb * KC, 0, 0, keep);
                    inflight_s[n_issued % MAX_STAGES] = s;
                    inflight_ph[n_issued % MAX_STAGES] = int(ph);
                    ++n_issued;
                    if (++s == STAGES) { s = 0; ph ^= 1; }
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
                for (int cb = 0; cb < CB; ++cb) {
                    if (!mbar_wait(&full[s], ph) || *(volatile int*)&s_abort) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < KC / 16; ++kk) {
                        const uint32_t base = ring_a + s * STAGE_BYTES + kk * 32;
                        const uint64_t ad = sdesc_k_sw128(base + K * R * 128);   // the gathered X rows
                        const uint64_t bd = sdesc_k_sw128(base);                 // phi rows, then X rows
                        mma_bf16(d, ad, bd, idesc, (cb | kk) != 0);
                    }
                    mma_commit(&empty[s]);
                    if (++s == STAGES) { s = 0; ph ^= 1; }
                }
                if (ok) mma_commit(&tfull[acc]);
            }
            if (!ok) {
                s_abort = 1;
                mma_commit(drain);
                mbar_wait(drain, 0, 1ll << 22);
            }
        }
    } else if (warp >= GATHER_WARP0 && warp < GATHER_WARP0 + 2) {
        // ------------------------------------------------------------ gather (cp.async)
        const int gt = threadIdx.x - GATHER_WARP0 * 32;   // 0..63
        const uint64_t keep = policy_evict_last();
        constexpr int CPT = MROWS * 8 / GATHER_THREADS;   // 16-byte chunks per thread per stage
        int s = 0, it = 0;
        uint32_t ph = 0;
        int q[GD], nq = 0;                                // committed stages not yet arrived on
        bool ok = true;
        for (int tile = cluster_id; tile < num_tiles && ok; tile += nclusters, ++it) {
            const int64_t t0 = int64_t(tile) * MT;
            if (it >= LAG) {     // the write-back of tile it-LAG re-reads its rows from L2
                const int need = WB_WARPS * (it - LAG + 1);
                long long kk = 0;
                while (*(volatile int*)&s_wb_done < need && !*(volatile int*)&s_abort && kk < g_wait_limit) {
                    __nanosleep(64);
                    ++kk;
                }
                if (!__all_sync(0xffffffffu, kk < g_wait_limit && !*(volatile int*)&s_abort)) {
                    if (kk >= g_wait_limit) atomicOr(&g_device_error, 1u);
                    ok = false;
                    break;
                }
            }
            for (int cb = 0; cb < CB; ++cb) {
                if (!warp_wait(&empty[s], ph ^ 1) || *(volatile int*)&s_abort) { ok = false; break; }
                uint8_t* xs = sring + s * STAGE_BYTES + K * R * 128;
                const int cc = c0 + cb * KC;
#pragma unroll 4
                for (int u = 0; u < CPT; ++u) {
                    const int e = gt + u * GATHER_THREADS;      // chunk: row e / 8, 16-byte column e % 8
                    const int r = e >> 3, j = e & 7;
                    const int l = r >> 5, tt = r & 31;
                    const int64_t t = t0 + tt;
                    const bf16_t* src = X;
                    uint32_t nbytes = 0;
                    if (t < T) {
                        const int si = __ldg(idx + t * K + l);
                        if (si >= 0 && si < N) {
                            src = X + (t * N + si) * int64_t(C) + cc + j * 8;
                            nbytes = 16;
                        } else {
                            atomicOr(&g_device_error, 2u);
                        }
                    }
                    cp_async16(xs + r * 128 + ((j ^ (r & 7)) << 4), src, nbytes, keep);
                }
                cp_async_commit();
                q[nq++] = s;
                if (nq == GD) {
                    // the oldest stage's copies are done: make them visible to the tensor core
                    cp_async_wait_group<GD - 1>();
                    fence_proxy_async_smem();
                    mbar_arrive(&full[q[0]]);
#pragma unroll
                    for (int i = 0; i + 1 < GD; ++i) q[i] = q[i + 1];
                    --nq;
                }
                if (++s == STAGES) { s = 0; ph ^= 1; }
            }
        }
        cp_async_wait_group<0>();
        fence_proxy_async_smem();
        for (int i = 0; i < nq; ++i) mbar_arrive(&full[q[i]]);
        if (!ok) s_abort = 1;
    } else if (warp >= EPI_WARP0 && warp < EPI_WARP0 + EPI_WARPS) {
        // ------------------------------------------------------------ epilogue
        const int et = threadIdx.x - EPI_WARP0 * 32;
        const int qd = warp & 3;                        // TMEM lane quarter = slot
        const float inv_K = 1.0f / float(K * C);
        constexpr uint32_t PART_BYTES = CL * K * TOK_PER_CTA * PSP * 4;
        constexpr uint32_t COEF_BYTES = MT * CS * 4;
        const int tok = lane;
        const uint32_t owner = uint32_t(tok / TOK_PER_CTA);
        const uint32_t push_dst =
            mapa(smem_u32(rpart + ((int(rank) * K + qd) * TOK_PER_CTA + tok % TOK_PER_CTA) * PSP), owner);
        const uint32_t push_bar = mapa(smem_u32(part_full), owner);
        int it = 0;
        for (int tile = cluster_id; tile < num_tiles; tile += nclusters, ++it) {
            const int64_t t0 = int64_t(tile) * MT;
            const int acc = it & 1;
            const uint32_t par = uint32_t((it >> 1) & 1);
            if (et == 0) {
                mbar_arrive_expect_tx(part_full, PART_BYTES);
                mbar_arrive_expect_tx(&coef_full[acc], COEF_BYTES);
            }
            if (!warp_wait(&tfull[acc], par)) { s_abort = 1; break; }
            tc_fence_after();
            float d[R];
            const uint32_t taddr = tmem_base + (uint32_t(qd * 32) << 16) + uint32_t(acc * ACC_COLS);
            // columns [qd*R, qd*R + R) in loads of 16 (the last may run into the next
            // slot's block or the sum-of-squares block: still allocated)
#pragma unroll
            for (int c = 0; c < R; c += 16) {
                float tmp[16];
                tmem_ld16(taddr + qd * R + c, tmp);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) if (c + j < R) d[c + j] = tmp[j];
            }
            float ss = 0.0f;
#pragma unroll
            for (int c = 0; c < 32; c += 16) {
                float tmp[16];
                tmem_ld16(taddr + K * R + qd * 32 + c, tmp);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) if (c + j == lane) ss = tmp[j];
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);

            // the coefficients of tile it land in buffer it&1, last read by the
            // write-back of tile it-2
            if (it >= 1 && !warp_wait(wb_prog, uint32_t((it - 1) & 1))) { s_abort = 1; break; }
#pragma unroll
            for (int p = 0; p < PSP; p += 4) {
                float v4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) v4[e] = p + e < R ? d[p + e] : (p + e == R ? ss : 0.0f);
                st_async_f32x4(push_dst + p * 4, make_float4(v4[0], v4[1], v4[2], v4[3]), push_bar);
            }
            if (et < 64) {
                if (!warp_wait(part_full, uint32_t(it & 1))) { s_abort = 1; break; }
                const int jj = et / LPT, g = et % LPT;
                const int j = int(rank) * TOK_PER_CTA + jj;
                constexpr int OWN = (PS + LPT - 1) / LPT;
                float own[OWN];
#pragma unroll
                for (int kq = 0; kq < OWN; ++kq) {
                    const int p = g + LPT * kq;
                    float s0 = 0.0f, s1 = 0.0f;
                    if (p < PS) {
#pragma unroll
                        for (int c = 0; c < CL; ++c) {
#pragma unroll
                            for (int qq = 0; qq < K; qq += 2) {
                                s0 += rpart[((c * K + qq) * TOK_PER_CTA + jj) * PSP + p];
                                s1 += rpart[((c * K + qq + 1) * TOK_PER_CTA + jj) * PSP + p];
                            }
                        }
                    }
                    own[kq] = s0 + s1;
                }
                float v[PS];
#pragma unroll
                for (int p = 0; p < PS; ++p) v[p] = __shfl_sync(0xffffffffu, own[p / LPT], p % LPT, LPT);
                const float inv_r = 1.0f / sqrtf(v[R] * inv_K + eps);
                float m[K][K];
#pragma unroll
                for (int i = 0; i < K; ++i)
#pragma unroll
                    for (int jc = 0; jc < K; ++jc) m[i][jc] = a_res * v[i * K + jc] * inv_r + sb[i * K + jc];
                sinkhorn_regs<K>(m, t_iters);
                // lane g: H_res element g (row g / 4) and, for g < 4 Kr, H_post element g
                float hr = 0.0f, hp = 0.0f;
#pragma unroll
                for (int e = 0; e < K * K; ++e)
                    if (e == g) hr = m[e / K][e % K];
#pragma unroll
                for (int e = 0; e < K * KR; ++e)
                    if (e == g) hp = 2.0f * sigmoidf_(a_post * v[K * K + e] * inv_r + sb[K * K + e]);
                const uint32_t hoff = smem_u32(scoef + (acc * MT + j) * CS);
                const uint32_t hbar = smem_u32(&coef_full[acc]);
                for (uint32_t cr = 0; cr < CL; ++cr) {
                    const uint32_t dst = mapa(hoff, cr), bar = mapa(hbar, cr);
                    st_async_f32(dst + g * 4, hr, bar);
                    if (g < K * KR) st_async_f32(dst + (K * K + g) * 4, hp, bar);
                }
                const int64_t t = t0 + j;
                if (t < T) {
                    if (Hres_out) Hres_out[t * K * K + g] = hr;
                    if (Hpost_out && g < K * KR) Hpost_out[t * K * KR + g] = hp;
                }
            }
            if (!warp_wait(&coef_full[acc], par)) { s_abort = 1; break; }
        }
    } else {
        // ------------------------------------------------------------ write-back
        const int wt = (warp - WB_WARP0) * 32 + lane;
        const uint64_t drop = policy_evict_first();
        const int VPT = Cs / 8;
        int it = 0;
        for (int tile = cluster_id; tile < num_tiles; tile += nclusters, ++it) {
            if (!warp_wait_sleep(&coef_full[it & 1], uint32_t((it >> 1) & 1))) { s_abort = 1; break; }
            __syncwarp();
            if (lane == 0) mbar_arrive(wb_prog);
            const int64_t t0 = int64_t(tile) * MT;
            const float* cf = scoef + (it & 1) * MT * CS;
            const int rows = int((T - t0) < int64_t(MT) ? (T - t0) : int64_t(MT));
            const int items = rows * VPT;
            for (int wi = wt; wi < items; wi += WB_THREADS) {
                const int tk = wi / VPT;
                const int c = c0 + (wi - tk * VPT) * 8;
                const int64_t t = t0 + tk;
                int si[K];
                bool good = true;
#pragma unroll
                for (int l = 0; l < K; ++l) {
                    si[l] = __ldg(idx + t * K + l);
                    good = good && si[l] >= 0 && si[l] < N;
                }
                if (!good) continue;                    // reported by the gather; token unchanged
                float xa[K][8], vb[KR][8];
#pragma unroll
                for (int l = 0; l < K; ++l) {
                    const uint4 raw = ldg16_raw_hint(X + (t * N + si[l]) * int64_t(C) + c, drop);
                    const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) { xa[l][2 * e] = bf16_lo(w4[e]); xa[l][2 * e + 1] = bf16_hi(w4[e]); }
                }
#pragma unroll
                for (int qv = 0; qv < KR; ++qv) {
                    float lo[4], hi[4];
                    load16<true>(V + (t * KR + qv) * int64_t(C) + c, lo);
                    load16<true>(V + (t * KR + qv) * int64_t(C) + c + 4, hi);
#pragma unroll
                    for (int u = 0; u < 4; ++u) { vb[qv][u] = lo[u]; vb[qv][4 + u] = hi[u]; }
                }
                const float* co = cf + tk * CS;
#pragma unroll
                for (int jr = 0; jr < K; ++jr) {
                    const float wj = __ldg(w + t * K + jr);
                    float o[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        float wb = 0.0f;
#pragma unroll
                        for (int qv = 0; qv < KR; ++qv) wb = fmaf(co[K * K + jr * KR + qv], vb[qv][u], wb);
                        float mix = 0.0f;
#pragma unroll
                        for (int l = 0; l < K; ++l) mix = fmaf(co[jr * K + l], xa[l][u], mix);
                        o[u] = fmaf(wj, wb, mix);
                    }
                    store16<false>(X + (t * N + si[jr]) * int64_t(C) + c, o);
                }
            }
            __syncwarp();
            if (lane == 0) atomicAdd(&s_wb_done, 1);
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
    cluster_sync();
}

// ------------------------------------------------------------------ host

template <int KR>
static mhc_status launch_kr(const UpdateArgs& a, cudaStream_t s)
{
    static int configured = 0, max_clusters = 0;
    auto kern = update_tc_kernel<KR>;
    const int smem = int(layout_for<KR>().total) + 1024;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return cuda_status(e, "xhc_sparse_update (tc): set shared memory size");
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
            return cuda_status(e != cudaSuccess ? e : cudaErrorInvalidConfiguration,
                               "xhc_sparse_update (tc): cluster occupancy");
        max_clusters = nc;
        configured = 1;
    }
    const int64_t tiles64 = (a.T + MT - 1) / MT;
    const int nclusters = int(tiles64 < max_clusters ? tiles64 : max_clusters);
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) {
        set_error("xhc_sparse_update (tc): cuTensorMapEncodeTiled unavailable");
        return MHC_ERR_CUDA;
    }
    using G = Cfg<KR>;
    CUtensorMap mapPhi;
    {
        // phi_act^T [PA][k*C] viewed as {C, PA, k}: a box {64, R, 4} holds R rows (rows
        // >= PA zero-filled) of the 4 slots for one channel block
        const cuuint64_t dims[3] = {cuuint64_t(a.C), cuuint64_t(G::PA), cuuint64_t(K)};
        const cuuint64_t strides[2] = {cuuint64_t(K) * a.C * 2, cuuint64_t(a.C) * 2};
        const cuuint32_t box[3] = {KC, cuuint32_t(G::R), K};
        const cuuint32_t estr[3] = {1, 1, 1};
        CUresult r = enc(&mapPhi, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.phi), dims, strides, box,
                         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            set_error("xhc_sparse_update (tc): cuTensorMapEncodeTiled(phi_act) failed (%d)", int(r));
            return MHC_ERR_CUDA;
        }
    }
    kern<<<dim3(unsigned(nclusters * CL)), NTHREADS, size_t(smem), s>>>(
        mapPhi, static_cast<bf16_t*>(a.X), a.V, a.idx, a.w, a.alpha[0], a.alpha[1], a.b, a.T, a.N, a.C,
        int(tiles64), a.t_iters, a.eps, a.H_res, a.H_post);
    return launch_status("xhc_sparse_update (tc) kernel");
}

}  // namespace xutc

bool update_tc_supported(const UpdateArgs& a)
{
    return a.dt == MHC_BF16 && a.k == xutc::K && a.Kr >= 1 && a.Kr <= 4 && a.T >= 1 && a.T < (int64_t(1) << 31) &&
           a.C % (xutc::CL * xutc::KC) == 0;
}

mhc_status launch_update_tc(const UpdateArgs& a, cudaStream_t s)
{
    switch (a.Kr) {
        case 1: return xutc::launch_kr<1>(a, s);
        case 2: return xutc::launch_kr<2>(a, s);
        case 3: return xutc::launch_kr<3>(a, s);
        case 4: return xutc::launch_kr<4>(a, s);
        default: break;
    }
    set_error("xhc_sparse_update (tc): Kr=%d not supported", a.Kr);
    return MHC_ERR_UNSUPPORTED;
}

}  // namespace mhc
