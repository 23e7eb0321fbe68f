// xhc_route, tensor-core path (sm_100a: TMA + tcgen05.mma + TMEM + a cluster
// of 8 CTAs sharing partial sums through distributed shared memory).
//
// [xHC] section "sparse residual stream architecture", steps 1-2, and
// "parameterisation" (the same formulas as the CUDA-core path in
// xhc_route.cu):
//   x = vec(X_t) (N*C); r = sqrt(sum(x^2)/(NC) + eps)
//   z = alpha * (x phi_read) / r + b_read   (N pre logits | N-m route logits)
//   H_pre = sigma(z_pre); score_s = sigma(z_route[s-m]) for s = m..N-1
//   active = {0..m-1} U TopK_{k-m}(score) (ties to the lower index), ascending;
//   w = 1 for fixed streams, the score for routed ones
//   x_in = sum_{i<N} H_pre[i] X_t[i]
//
// Per tile of 32 tokens, the 8 CTAs of a cluster split the C channels: CTA r
// owns channels [r*C/8, (r+1)*C/8) of every stream.  A ring stage holds one
// 64-channel block of a group of 4 streams:
//     [ phi_read^T rows of the 4 streams (R rows each) | X rows of the 4 streams (32 each) ]
// (4R + 128 rows of 128 bytes, 128-byte swizzle).  One tcgen05.mma per 16-wide
// K step, M = 128 (the group's 4 x 32 X rows), N = 4R + 128 (B = the whole
// stage), gives in TMEM row q*32 + t (stream q of the group, token t) the
// projections of that stream's K-slice in columns [qR, qR + R) and its sum of
// squares in column 4R + q*32 + t (X row dotted with itself).  The groups and
// channel blocks accumulate into the same columns, so after the tile TMEM lane
// quarter q holds, for every token, the sums over streams q, q+4, q+8, ...
//
// Warp roles (16 warps), as in the mhc_pre tensor-core kernel:
//   0      TMA producer (a {64, R, 4} box of phi_read^T viewed as {C, 2N-m, N},
//          a {64, 32, 4} box of X viewed as {C, T, N}; L2 evict-last), at most
//          LAG tiles ahead of the x_in warps so that the x_in re-read hits L2;
//   1      MMA issuer (fp32 accumulators in TMEM, double-buffered over tiles);
//   4-7    one TMEM lane quarter each: push every row's partial projections
//          and sum of squares (st.async) to the CTA owning the token (4 tokens
//          per CTA); warps 4-5 of the owner reduce the 4 x 8 partial rows (16
//          lanes per token), form the gates and scores, take the TopK and push
//          H_pre to every CTA of the cluster;
//   2-3, 8-15  x_in = H_pre X for this CTA's channels (re-read from L2).
// Every wait is bounded and warp-uniform; on expiry the kernel records the
// timeout in the device error word, drains its copies and MMAs, frees TMEM
// and returns.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace mhc {
namespace xrtc {

using namespace sm100;

constexpr int CL = 8;            // CTAs per cluster (channel split)
constexpr int MROWS = 128;       // MMA M: 4 streams x 32 tokens
constexpr int MT = 32;           // tokens per tile
constexpr int KC = 64;           // channels per block (one 128-byte row)
constexpr int GS = 4;            // streams per MMA group
constexpr int MAX_STAGES = 8;
constexpr int SMEM_LIMIT = 227 * 1024;
constexpr int NTHREADS = 512;
constexpr int EPI_WARP0 = 4, EPI_WARPS = 4;
constexpr int XIN_WARPS = 10, XIN_THREADS = XIN_WARPS * 32;   // warps 2-3 and 8-15
constexpr int TOK_PER_CTA = MT / CL;     // tokens whose gates a CTA computes
constexpr int LPT = 16;                  // coefficient lanes per token (warps 4-5: 4 tokens)
constexpr int ACC_COLS = 256;
constexpr int TMEM_COLS = 512;
// The tiles loaded but not yet re-read by x_in wait in L2: 15 clusters x 32
// tokens x N*C*2 bytes per tile step (31 MB at N = 16, C = 2048).
constexpr int LAG = 3;
static_assert(TOK_PER_CTA * LPT == 64, "warps 4-5: one 16-lane group per token");

template <int N> struct Cfg {
    static_assert(N % GS == 0 && N <= 16, "groups of 4 streams; 4R + 128 <= 256");
    static constexpr int R = (2 * N + 7) / 8 * 8;   // phi_read^T rows per stream in a stage (>= 2N - m)
    static constexpr int NG = N / GS;               // stream groups
    static constexpr int MMA_N = GS * R + MROWS;
    static constexpr int STAGE_BYTES = MMA_N * 128;
    static constexpr int PS = R + 1;                // partial row: R projections + sum of squares
    static constexpr int PSP = (PS + 3) / 4 * 4;
    static constexpr int XU = N >= 16 ? 1 : 16 / N; // x_in vectors in flight per thread
    static_assert(MMA_N % 16 == 0 && MMA_N <= ACC_COLS, "MMA N for M = 128");
};

enum Bar { B_FULL = 0, B_EMPTY = B_FULL + MAX_STAGES, B_TFULL = B_EMPTY + MAX_STAGES, B_TEMPTY = B_TFULL + 2,
           B_PART = B_TEMPTY + 2, B_HPRE, B_XIN = B_HPRE + 2, B_DRAIN, B_COUNT };

struct Layout {
    uint32_t ring, part, hpre, bias, bars, slot, total;
    int stages;
};

// Bytes after the ring: partial rows [CL][GS][TOK_PER_CTA][PSP], H_pre
// [2][MT][N], b (at most 2N floats), barriers.
template <int N>
__host__ __device__ constexpr uint32_t fixed_bytes() {
    using G = Cfg<N>;
    return CL * GS * TOK_PER_CTA * G::PSP * 4 + 2 * MT * N * 4 + 2 * N * 4 + 16 + B_COUNT * 8 + 16;
}

template <int N>
__host__ __device__ constexpr int stages_fit() {
    constexpr int64_t room = int64_t(SMEM_LIMIT) - 1024 - fixed_bytes<N>();
    constexpr int64_t fit = room > 0 ? room / Cfg<N>::STAGE_BYTES : 0;
    return int(fit < MAX_STAGES ? fit : MAX_STAGES);
}

template <int N>
__host__ __device__ inline Layout layout_for() {
    using G = Cfg<N>;
    Layout L;
    L.ring = 0;
    L.stages = stages_fit<N>();
    L.part = L.ring + uint32_t(L.stages) * G::STAGE_BYTES;
    L.hpre = L.part + CL * GS * TOK_PER_CTA * G::PSP * 4;
    L.bias = L.hpre + 2 * MT * N * 4;
    L.bars = (L.bias + 2 * N * 4 + 15) / 16 * 16;
    L.slot = L.bars + B_COUNT * 8;
    L.total = L.slot + 16;
    return L;
}

template <int N>
__global__ void __cluster_dims__(CL, 1, 1) __launch_bounds__(NTHREADS, 1)
route_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmPhi,
                const bf16_t* __restrict__ X, float a_pre, float a_route, const float* __restrict__ b,
                int64_t T, int C, int k, int m, int num_tiles, float eps, bf16_t* __restrict__ x_in,
                float* __restrict__ Hpre, float* __restrict__ score, int32_t* __restrict__ idx,
                float* __restrict__ w)
{
    using G = Cfg<N>;
    constexpr int R = G::R, NG = G::NG, PS = G::PS, PSP = G::PSP, STAGE_BYTES = G::STAGE_BYTES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int P = 2 * N - m;           // logits in use (rows >= P of a stage are zero)
    const int Cs = C / CL;
    const int CB = Cs / KC;
    const int SPT = CB * NG;           // ring stages per tile
    const Layout L = layout_for<N>();
    const int STAGES = L.stages;
    uint8_t* sring = smem + L.ring;
    float* rpart = reinterpret_cast<float*>(smem + L.part);   // [CL][GS][TOK_PER_CTA][PSP], pushed by the cluster
    float* shpre = reinterpret_cast<float*>(smem + L.hpre);   // [2][MT][N]
    float* sb = reinterpret_cast<float*>(smem + L.bias);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint64_t* full = bars + B_FULL;
    uint64_t* empty = bars + B_EMPTY;
    uint64_t* tfull = bars + B_TFULL;
    uint64_t* tempty = bars + B_TEMPTY;
    uint64_t* part_full = bars + B_PART;
    uint64_t* hpre_full = bars + B_HPRE;
    uint64_t* xin_prog = bars + B_XIN;
    uint64_t* drain = bars + B_DRAIN;
    uint32_t* slot = reinterpret_cast<uint32_t*>(smem + L.slot);
    __shared__ int s_abort;
    __shared__ int s_xin_done;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int cluster_id = blockIdx.x / CL;
    const int nclusters = gridDim.x / CL;
    const int c0 = int(rank) * Cs;

    if (threadIdx.x == 0) {
        s_abort = 0;
        s_xin_done = 0;
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], EPI_WARPS);
        }
        mbar_init(part_full, 1);
        mbar_init(&hpre_full[0], 1);
        mbar_init(&hpre_full[1], 1);
        mbar_init(xin_prog, XIN_WARPS);
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(slot, TMEM_COLS);
    for (int p = threadIdx.x; p < P; p += NTHREADS) sb[p] = b[p];
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *slot;
    if (threadIdx.x == 0) {
        tma_prefetch(&tmX);
        tma_prefetch(&tmPhi);
    }
    cluster_sync();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t keep = policy_evict_last();
            int s = 0;
            uint32_t ph = 0;
            int inflight_s[MAX_STAGES], inflight_ph[MAX_STAGES], n_issued = 0;
            bool ok = true;
            int it = 0;
            for (int tile = cluster_id; tile < num_tiles && ok; tile += nclusters, ++it) {
                const int t0 = tile * MT;
                if (it >= LAG) {
                    const int need = XIN_WARPS * (it - LAG + 1);
                    long long kk = 0;
                    while (*(volatile int*)&s_xin_done < need && !*(volatile int*)&s_abort && kk < g_wait_limit) {
                        __nanosleep(64);
                        ++kk;
                    }
                    if (kk >= g_wait_limit) { atomicOr(&g_device_error, 1u); ok = false; break; }
                }
                for (int q = 0; q < SPT; ++q) {
                    if (!mbar_wait(&empty[s], ph ^ 1) || *(volatile int*)&s_abort) { ok = false; break; }
                    mbar_arrive_expect_tx(&full[s], uint32_t(STAGE_BYTES));
                    const int cc = c0 + (q / NG) * KC, grp = q % NG;
                    uint8_t* st = sring + s * STAGE_BYTES;
                    tma_load_3d_hint(st, &tmPhi, &full[s], cc, 0, GS * grp, keep);
                    tma_load_3d_hint(st + GS * R * 128, &tmX, &full[s], cc, t0, GS * grp, keep);
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
                        const uint64_t ad = sdesc_k_sw128(base + GS * R * 128);   // the group's X rows
                        const uint64_t bd = sdesc_k_sw128(base);                  // phi rows, then X rows
                        mma_bf16(d, ad, bd, idesc, (q | kk) != 0);
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
    } else if (warp >= EPI_WARP0 && warp < EPI_WARP0 + EPI_WARPS) {
        // ------------------------------------------------------------ epilogue
        const int et = threadIdx.x - EPI_WARP0 * 32;    // 0..127
        const int qd = warp & 3;                        // TMEM lane quarter = stream within the group
        const float inv_K = 1.0f / float(N * C);
        constexpr uint32_t PART_BYTES = CL * GS * TOK_PER_CTA * PSP * 4;
        constexpr uint32_t HPRE_BYTES = MT * N * 4;
        const int tok = lane;                           // TMEM row qd*32 + lane
        const uint32_t owner = uint32_t(tok / TOK_PER_CTA);
        const uint32_t push_dst =
            mapa(smem_u32(rpart + ((int(rank) * GS + qd) * TOK_PER_CTA + tok % TOK_PER_CTA) * PSP), owner);
        const uint32_t push_bar = mapa(smem_u32(part_full), owner);
        int it = 0;
        for (int tile = cluster_id; tile < num_tiles; tile += nclusters, ++it) {
            const int64_t t0 = int64_t(tile) * MT;
            const int acc = it & 1;
            const uint32_t par = uint32_t((it >> 1) & 1);
            if (et == 0) {
                mbar_arrive_expect_tx(part_full, PART_BYTES);
                mbar_arrive_expect_tx(&hpre_full[acc], HPRE_BYTES);
            }
            if (!warp_wait(&tfull[acc], par)) { s_abort = 1; break; }
            tc_fence_after();
            float d[R];
            const uint32_t taddr = tmem_base + (uint32_t(qd * 32) << 16) + uint32_t(acc * ACC_COLS);
            // columns [qd*R, qd*R + R) in loads of 16 (the last may run 8 columns into
            // the next stream's block or the sum-of-squares block: still allocated)
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
            for (int c = 0; c < 32; c += 16) {          // column 4R + row: X row . X row
                float tmp[16];
                tmem_ld16(taddr + GS * R + qd * 32 + c, tmp);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) if (c + j == lane) ss = tmp[j];
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);

            // H_pre of tile it lands in buffer it&1, last read by the x_in warps for tile it-2
            if (it >= 1 && !warp_wait(xin_prog, uint32_t((it - 1) & 1))) { s_abort = 1; break; }
#pragma unroll
            for (int p = 0; p < PSP; p += 4) {
                float v4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) v4[e] = p + e < R ? d[p + e] : (p + e == R ? ss : 0.0f);
                st_async_f32x4(push_dst + p * 4, make_float4(v4[0], v4[1], v4[2], v4[3]), push_bar);
            }
            if (et < 64) {
                if (!warp_wait(part_full, uint32_t(it & 1))) { s_abort = 1; break; }
                // 16 lanes per token: lane g sums entries p = g (mod 16) over the GS x CL
                // partial rows; the group exchanges the sums; lane g < N owns stream g.
                const int jj = et / LPT, g = et % LPT;
                const int j = int(rank) * TOK_PER_CTA + jj;     // token row within the tile
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
                            for (int q = 0; q < GS; q += 2) {
                                s0 += rpart[((c * GS + q) * TOK_PER_CTA + jj) * PSP + p];
                                s1 += rpart[((c * GS + q + 1) * TOK_PER_CTA + jj) * PSP + p];
                            }
                        }
                    }
                    own[kq] = s0 + s1;
                }
                float v[PS];
#pragma unroll
                for (int p = 0; p < PS; ++p) v[p] = __shfl_sync(0xffffffffu, own[p / LPT], p % LPT, LPT);
                const float inv_r = 1.0f / sqrtf(v[R] * inv_K + eps);
                // lane g: stream g's pre logit (entry g) and route logit (entry N + g - m)
                float zp = 0.0f, zr = 0.0f;
#pragma unroll
                for (int p = 0; p < R; ++p) {
                    if (p == g) zp = v[p];
                    if (p == N + g - m) zr = v[p];
                }
                const bool stream = g < N;
                const float hp = stream ? sigmoidf_(a_pre * zp * inv_r + sb[g < N ? g : 0]) : 0.0f;
                const bool routed = stream && g >= m;
                const float sc = routed ? sigmoidf_(a_route * zr * inv_r + sb[routed ? N + g - m : 0]) : -1.0f;
                int rk = 0;
                for (int s = m; s < N; ++s) {
                    const float o = __shfl_sync(0xffffffffu, sc, s, LPT);
                    if (routed && s != g && (o > sc || (o == sc && s < g))) ++rk;
                }
                const bool sel = stream && (g < m || rk < k - m);
                const unsigned bal = __ballot_sync(0xffffffffu, sel);
                const unsigned mine = (bal >> (lane & ~(LPT - 1))) & ((1u << LPT) - 1u);
                if (stream) {
                    // every CTA needs H_pre of every tile row for its x_in channels
                    const uint32_t hoff = smem_u32(shpre + (acc * MT + j) * N + g);
                    const uint32_t hbar = smem_u32(&hpre_full[acc]);
                    for (uint32_t cr = 0; cr < CL; ++cr) st_async_f32(mapa(hoff, cr), hp, mapa(hbar, cr));
                }
                const int64_t t = t0 + j;
                if (t < T) {
                    if (sel) {
                        const int sl = __popc(mine & ((1u << g) - 1u));
                        idx[t * k + sl] = g;
                        w[t * k + sl] = g < m ? 1.0f : sc;
                    }
                    if (stream && Hpre) Hpre[t * N + g] = hp;
                    if (routed && score) score[t * (N - m) + g - m] = sc;
                }
            }
            if (!warp_wait(&hpre_full[acc], par)) { s_abort = 1; break; }
        }
    } else {
        // ------------------------------------------------------------ x_in
        constexpr int XU = G::XU;
        const int xt = (warp < EPI_WARP0 ? warp - 2 : warp - (EPI_WARP0 + EPI_WARPS - 2)) * 32 + lane;   // 0..XIN_THREADS-1
        const uint64_t drop = policy_evict_first();
        const int VPT = Cs / 8;
        int it = 0;
        for (int tile = cluster_id; tile < num_tiles; tile += nclusters, ++it) {
            if (!warp_wait_sleep(&hpre_full[it & 1], uint32_t((it >> 1) & 1))) { s_abort = 1; break; }
            __syncwarp();
            if (lane == 0) mbar_arrive(xin_prog);
            const int64_t t0 = int64_t(tile) * MT;
            const float* hb = shpre + (it & 1) * MT * N;
            const int rows = int((T - t0) < int64_t(MT) ? (T - t0) : int64_t(MT));
            const int items = rows * VPT;
            for (int w0 = xt; w0 < items; w0 += XU * XIN_THREADS) {
                uint4 raw[XU][N];
                int tk[XU], cc[XU];
#pragma unroll
                for (int u = 0; u < XU; ++u) {
                    const int wi = w0 + u * XIN_THREADS;
                    const int wc = wi < items ? wi : items - 1;   // clamp; the store is skipped
                    tk[u] = wc / VPT;
                    cc[u] = c0 + (wc - tk[u] * VPT) * 8;
#pragma unroll
                    for (int i = 0; i < N; ++i)
                        raw[u][i] = ldg16_raw_hint(X + ((t0 + tk[u]) * N + i) * C + cc[u], drop);
                }
#pragma unroll
                for (int u = 0; u < XU; ++u) {
                    if (w0 + u * XIN_THREADS >= items) break;
                    float o[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[e] = 0.0f;
#pragma unroll
                    for (int i = 0; i < N; ++i) {
                        const float hh = hb[tk[u] * N + i];
                        const uint32_t w4[4] = {raw[u][i].x, raw[u][i].y, raw[u][i].z, raw[u][i].w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            o[2 * e] = fmaf(hh, bf16_lo(w4[e]), o[2 * e]);
                            o[2 * e + 1] = fmaf(hh, bf16_hi(w4[e]), o[2 * e + 1]);
                        }
                    }
                    store16<true>(x_in + (t0 + tk[u]) * C + cc[u], o);   // streaming: keep L2 for the tiles awaiting their re-read
                }
            }
            __syncwarp();
            if (lane == 0) atomicAdd(&s_xin_done, 1);
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

template <int N>
static int smem_bytes() { return int(layout_for<N>().total) + 1024; }

template <int N>
static mhc_status launch_n(const RouteArgs& a, cudaStream_t s)
{
    static int configured = 0, max_clusters = 0;
    auto kern = route_tc_kernel<N>;
    const int smem = smem_bytes<N>();
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return cuda_status(e, "xhc_route (tc): set shared memory size");
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
            return cuda_status(e != cudaSuccess ? e : cudaErrorInvalidConfiguration, "xhc_route (tc): cluster occupancy");
        max_clusters = nc;
        configured = 1;
    }
    const int64_t tiles64 = (a.T + MT - 1) / MT;
    const int nclusters = int(tiles64 < max_clusters ? tiles64 : max_clusters);

    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) {
        set_error("xhc_route (tc): cuTensorMapEncodeTiled unavailable");
        return MHC_ERR_CUDA;
    }
    using G = Cfg<N>;
    const int P = 2 * a.N - a.m;
    CUtensorMap mapX, mapPhi;
    {
        // X [T][N][C] viewed as {C, T, N}: a box {64, 32, 4} lands stream-major
        const cuuint64_t dims[3] = {cuuint64_t(a.C), cuuint64_t(a.T), cuuint64_t(a.N)};
        const cuuint64_t strides[2] = {cuuint64_t(a.N) * a.C * 2, cuuint64_t(a.C) * 2};
        const cuuint32_t box[3] = {KC, MT, GS};
        const cuuint32_t estr[3] = {1, 1, 1};
        CUresult r = enc(&mapX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.X), dims, strides, box,
                         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            set_error("xhc_route (tc): cuTensorMapEncodeTiled(X) failed (%d)", int(r));
            return MHC_ERR_CUDA;
        }
    }
    {
        // phi_read^T [2N-m][N*C] viewed as {C, 2N-m, N}: a box {64, R, 4} holds R rows
        // (rows >= 2N-m zero-filled) of 4 streams for one channel block
        const cuuint64_t dims[3] = {cuuint64_t(a.C), cuuint64_t(P), cuuint64_t(a.N)};
        const cuuint64_t strides[2] = {cuuint64_t(a.N) * a.C * 2, cuuint64_t(a.C) * 2};
        const cuuint32_t box[3] = {KC, cuuint32_t(G::R), GS};
        const cuuint32_t estr[3] = {1, 1, 1};
        CUresult r = enc(&mapPhi, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.phi), dims, strides,
                         box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            set_error("xhc_route (tc): cuTensorMapEncodeTiled(phi_read) failed (%d)", int(r));
            return MHC_ERR_CUDA;
        }
    }
    kern<<<dim3(unsigned(nclusters * CL)), NTHREADS, size_t(smem), s>>>(
        mapX, mapPhi, static_cast<const bf16_t*>(a.X), a.alpha[0], a.alpha[1], a.b, a.T, a.C, a.k, a.m,
        int(tiles64), a.eps, static_cast<bf16_t*>(a.x_in), a.H_pre, a.score, a.idx, a.w);
    return launch_status("xhc_route (tc) kernel");
}

}  // namespace xrtc

bool route_tc_supported(const RouteArgs& a)
{
    if (a.dt != MHC_BF16 || a.T < 1 || a.T >= (int64_t(1) << 31) || a.C % (xrtc::CL * xrtc::KC) != 0) return false;
    return a.N == 4 || a.N == 8 || a.N == 12 || a.N == 16;
}

mhc_status launch_route_tc(const RouteArgs& a, cudaStream_t s)
{
    switch (a.N) {
        case 4: return xrtc::launch_n<4>(a, s);
        case 8: return xrtc::launch_n<8>(a, s);
        case 12: return xrtc::launch_n<12>(a, s);
        case 16: return xrtc::launch_n<16>(a, s);
        default: break;
    }
    set_error("xhc_route (tc): N=%d not supported", a.N);
    return MHC_ERR_UNSUPPORTED;
}

}  // namespace mhc
