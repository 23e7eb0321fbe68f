// mhc_pre, tensor-core path (sm_100a: TMA + tcgen05.mma + TMEM + a cluster
// of 8 CTAs sharing partial sums through distributed shared memory).
//
// [mHC] section 4.3.1, Eq.(14)-(19), and F_pre := H_pre x_l.  Per token tile
// of Mt <= 64 tokens, the 8 CTAs of a cluster split the C channels: CTA r
// owns channels [r*C/8, (r+1)*C/8) of every stream, i.e. a K-slice of
// n*C/8 elements of each token's n*C row, and phi's matching K-slice stays
// resident in its shared memory for the whole (persistent) kernel.
//
// Warp roles (16 warps):
//   0      TMA producer: X[tile, stream i, 64-channel block] boxes (Mt rows x
//          128 B, 128-byte swizzle, L2 evict-last) through a 14-stage ring;
//          it runs at most LAG tiles ahead of the x_in warps, which keeps the
//          x_in re-read inside L2.
//   1      MMA issuer: D[128 x NB] += X_chunk[128 x 64] * phiT_chunk[NB x 64]^T
//          and S[128 x 64] += X_chunk * X_chunk[0..63]^T, whose diagonal is
//          each row's sum of squares (Eq.15) (tcgen05.mma kind::f16, fp32
//          accumulators in TMEM, double-buffered across tiles; rows >= Mt are
//          never read).  The MMA commit is the only consumer of a ring stage.
//   4-5    epilogue: each tile row's partial (logits, sum of squares) from TMEM
//          is pushed with st.async into the shared memory of the CTA that owns
//          the token (8 tokens per CTA); the owner reduces the 8 partial rows,
//          computes the coefficients (Eq.16-19, Sinkhorn in registers) and
//          pushes H_pre to every CTA of the cluster.  The pushes
//          complete transactions on the receivers' mbarriers, so no fence or
//          remote arrive sits on this path.
//   2-3, 6-15  x_in = H_pre X for this CTA's channels, re-reading the tile's
//          X slice from L2 (evict-first on this last read).
// The roles meet only through mbarriers and one progress counter, so the TMA
// ring keeps streaming while a tile's coefficients and x_in are produced.
//
// HBM: X is read once; x_in and the coefficients are written once; phi is
// read once per CTA.  Every wait is bounded (g_wait_limit); on expiry the
// kernel records the timeout in the device error word, drains its own copies
// and MMAs in flight, frees TMEM and returns.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace mhc {
namespace pretc {

using namespace sm100;

constexpr int CL = 8;            // CTAs per cluster (channel split)
constexpr int MROWS = 128;       // MMA M (TMEM lanes); a tile uses the first Mt <= MT_CAP rows
constexpr int MT_CAP = 64;       // token rows per tile: bounds the L2 footprint of the x_in re-read
constexpr int KC = 64;           // K elements per chunk (one 128-byte row)
constexpr int STAGE_BYTES = MT_CAP * 128;
constexpr int STAGES = 14;
constexpr int NTHREADS = 512;
constexpr int EPI_WARP0 = 4, EPI_WARPS = 2, EPI_THREADS = 64;   // TMEM lane quarters 0 and 1
constexpr int XIN_WARPS = 12, XIN_THREADS = 384;                 // warps 2-3 and 6-15
constexpr int TOK_PER_CTA = MT_CAP / CL;  // tokens whose coefficients a CTA computes
constexpr int XIN_UNROLL = 4;             // x_in vectors in flight per thread
constexpr int LAG = 2;                    // tiles the TMA stream may run ahead of x_in
static_assert(TOK_PER_CTA * 8 <= EPI_THREADS, "one 8-lane group per coefficient token");

template <int N> struct Cfg {
    static constexpr int P = N * N + 2 * N;
    static constexpr int R = (P + 7) / 8 * 8;      // phiT rows stored per chunk
    static constexpr int NB = (P + 15) / 16 * 16;  // MMA N
    static constexpr int PS = P + 1;               // partial row: P logits + sum of squares
    static constexpr int PSP = (PS + 3) / 4 * 4;   // ... padded to 16-byte multiples
    static constexpr int SQ_COL = 2 * NB;           // X X^T accumulators (2 x MT_CAP columns) after the logits
    static constexpr int TMEM_COLS = 256;
};

enum Bar { B_FULL = 0, B_EMPTY = B_FULL + STAGES, B_TFULL = B_EMPTY + STAGES, B_TEMPTY = B_TFULL + 2,
           B_PART = B_TEMPTY + 2, B_HPRE, B_XIN = B_HPRE + 2, B_PHI, B_DRAIN, B_COUNT };

struct Layout {
    uint32_t phi, ring, part, hpre, bias, bars, slot, total;
};

template <int N>
__host__ __device__ inline Layout layout_for(int NQ) {
    using G = Cfg<N>;
    Layout L;
    L.phi = 0;
    L.ring = uint32_t(NQ) * G::R * 128;                      // multiple of 1024
    L.part = L.ring + STAGES * STAGE_BYTES;
    L.hpre = L.part + CL * TOK_PER_CTA * G::PSP * 4;       // after [source CTA][token][PSP]
    L.bias = L.hpre + 2 * MT_CAP * N * 4;
    L.bars = (L.bias + G::P * 4 + 15) / 16 * 16;
    L.slot = L.bars + B_COUNT * 8;
    L.total = L.slot + 16;
    // The MMA reads 128 rows from a stage's base: the last stage's rows past
    // MT_CAP must still be inside this CTA's shared memory (their products land
    // in accumulator rows that are never read).
    const uint32_t mma_end = L.part + (MROWS - MT_CAP) * 128;
    if (L.total < mma_end) L.total = mma_end;
    return L;
}

template <int N>
__global__ void __cluster_dims__(CL, 1, 1) __launch_bounds__(NTHREADS, 1)
pre_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmPhi,
              const bf16_t* __restrict__ X, float a0, float a1, float a2,
              const float* __restrict__ b, int64_t T, int C, int Mt, int num_tiles, int t_iters,
              float eps, bf16_t* __restrict__ x_in, float* __restrict__ Hpre,
              float* __restrict__ Hpost, float* __restrict__ Hres, float* __restrict__ u_out,
              float* __restrict__ r_out)
{
    using G = Cfg<N>;
    constexpr int P = G::P, R = G::R, NB = G::NB, PS = G::PS, PSP = G::PSP;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment for the 128-byte-swizzle atoms
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int Cs = C / CL;
    const int CB = Cs / KC;            // channel blocks per stream
    const int NQ = N * CB;             // K chunks of this CTA per tile
    const Layout L = layout_for<N>(NQ);
    uint8_t* sphi = smem + L.phi;
    uint8_t* sring = smem + L.ring;
    float* rpart = reinterpret_cast<float*>(smem + L.part);   // [CL][TOK_PER_CTA][PSP], pushed by the cluster
    float* shpre = reinterpret_cast<float*>(smem + L.hpre);   // [2][MT_CAP][N]
    float* sb = reinterpret_cast<float*>(smem + L.bias);      // b, kept on chip for the coefficients
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint64_t* full = bars + B_FULL;
    uint64_t* empty = bars + B_EMPTY;
    uint64_t* tfull = bars + B_TFULL;
    uint64_t* tempty = bars + B_TEMPTY;
    uint64_t* part_full = bars + B_PART;     // this CTA's tokens: all CL partial rows landed
    uint64_t* hpre_full = bars + B_HPRE;     // [2] H_pre of every tile row landed (per tile parity)
    uint64_t* xin_prog = bars + B_XIN;
    uint64_t* phi_full = bars + B_PHI;
    uint64_t* drain = bars + B_DRAIN;
    uint32_t* slot = reinterpret_cast<uint32_t*>(smem + L.slot);
    __shared__ int s_abort;
    __shared__ int s_xin_done;   // x_in warp-tiles finished (monotonic)

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
        // one local arrival (with the expected byte count) per phase; the bytes
        // come from st.async pushes of the cluster
        mbar_init(part_full, 1);
        mbar_init(&hpre_full[0], 1);
        mbar_init(&hpre_full[1], 1);
        mbar_init(xin_prog, XIN_WARPS);
        mbar_init(phi_full, 1);
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(slot, G::TMEM_COLS);
    for (int p = threadIdx.x; p < P; p += NTHREADS) sb[p] = b[p];
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *slot;
    if (threadIdx.x == 0) {
        tma_prefetch(&tmX);
        tma_prefetch(&tmPhi);
        // Resident phiT: chunk q = (stream i, channel block cb) holds rows p < R of
        // phiT[p][i*C + c0 + cb*64 + 0..63] (rows >= P are zero-filled by the TMA).
        mbar_arrive_expect_tx(phi_full, uint32_t(NQ) * R * 128);
        for (int q = 0; q < NQ; ++q)
            tma_load_2d(sphi + size_t(q) * R * 128, &tmPhi, phi_full, (q / CB) * C + c0 + (q % CB) * KC, 0);
    }
    cluster_sync();   // every CTA's barriers are initialised before any remote arrive

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t keep = policy_evict_last();
            int s = 0;
            uint32_t ph = 0;
            int inflight_s[STAGES], inflight_ph[STAGES], n_issued = 0;
            bool ok = true;
            int it = 0;
            for (int tile = cluster_id; tile < num_tiles && ok; tile += nclusters, ++it) {
                const int t0 = tile * Mt;
                // keep the re-read of tile it-LAG in L2: do not run further ahead of x_in
                if (it >= LAG) {
                    const int need = XIN_WARPS * (it - LAG + 1);
                    long long k = 0;
                    while (*(volatile int*)&s_xin_done < need && !*(volatile int*)&s_abort && k < g_wait_limit) {
                        __nanosleep(64);
                        ++k;
                    }
                    if (k >= g_wait_limit) { atomicOr(&g_device_error, 1u); ok = false; break; }
                }
                for (int q = 0; q < NQ; ++q) {
                    if (!mbar_wait(&empty[s], ph ^ 1) || *(volatile int*)&s_abort) { ok = false; break; }
                    mbar_arrive_expect_tx(&full[s], uint32_t(Mt) * 128);
                    tma_load_3d_hint(sring + s * STAGE_BYTES, &tmX, &full[s], c0 + (q % CB) * KC, q / CB, t0, keep);
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
        if (lane == 1) mbar_wait(phi_full, 0, 1ll << 24);     // phiT copy settles before any exit
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(MROWS, NB);
            constexpr uint32_t idesc_sq = idesc_bf16_f32(MROWS, MT_CAP);   // X X^T, tile rows only
            const uint32_t ring_a = smem_u32(sring), phi_a = smem_u32(sphi);
            int s = 0, it = 0;
            uint32_t ph = 0;
            bool ok = mbar_wait(phi_full, 0);
            for (int tile = cluster_id; tile < num_tiles && ok; tile += nclusters, ++it) {
                const int acc = it & 1;
                if (!mbar_wait(&tempty[acc], (uint32_t((it >> 1) & 1)) ^ 1)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem_base + uint32_t(acc * NB);
                const uint32_t dsq = tmem_base + uint32_t(G::SQ_COL + acc * MT_CAP);
                for (int q = 0; q < NQ; ++q) {
                    if (!mbar_wait(&full[s], ph) || *(volatile int*)&s_abort) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < KC / 16; ++kk) {
                        const uint64_t ad = sdesc_k_sw128(ring_a + s * STAGE_BYTES + kk * 32);
                        const uint64_t bd = sdesc_k_sw128(phi_a + q * R * 128 + kk * 32);
                        mma_bf16(d, ad, bd, idesc, (q | kk) != 0);
                        // Eq.(15): the sums of squares are the diagonal of X X^T (B = the same rows)
                        mma_bf16(dsq, ad, ad, idesc_sq, (q | kk) != 0);
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

    } else if (warp == EPI_WARP0 || warp == EPI_WARP0 + 1) {
        // ------------------------------------------------------------ epilogue
        const int et = threadIdx.x - EPI_WARP0 * 32;    // 0..63
        const int qd = warp & 3;                        // TMEM lane quarter of this warp (0, 1)
        const int m = qd * 32 + lane;                   // token row within the tile
        const float inv_K = 1.0f / float(N * C);
        constexpr uint32_t PART_BYTES = CL * TOK_PER_CTA * PSP * 4;
        constexpr uint32_t HPRE_BYTES = MT_CAP * N * 4;
        // the partial row of tile row m goes to its owner CTA m / TOK_PER_CTA, slot (rank, m % TOK_PER_CTA)
        const uint32_t owner = uint32_t(m / TOK_PER_CTA);
        const uint32_t push_dst = mapa(smem_u32(rpart + (int(rank) * TOK_PER_CTA + m % TOK_PER_CTA) * PSP), owner);
        const uint32_t push_bar = mapa(smem_u32(part_full), owner);
        int it = 0;
        for (int tile = cluster_id; tile < num_tiles; tile += nclusters, ++it) {
            const int64_t t0 = int64_t(tile) * Mt;
            const int acc = it & 1;
            const uint32_t par = uint32_t((it >> 1) & 1);
            if (et == 0) {
                // expected bytes of this tile's phases; pushes may land before or after
                mbar_arrive_expect_tx(part_full, PART_BYTES);
                mbar_arrive_expect_tx(&hpre_full[acc], HPRE_BYTES);
            }
            if (!mbar_wait(&tfull[acc], par)) { s_abort = 1; break; }
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
            float ss = 0.0f;
            {
                const uint32_t qaddr = tmem_base + (uint32_t(qd * 32) << 16) +
                                       uint32_t(G::SQ_COL + acc * MT_CAP + qd * 32);
#pragma unroll
                for (int c = 0; c < 32; c += 16) {
                    float tmp[16];
                    tmem_ld16(qaddr + c, tmp);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) if (c + j == lane) ss = tmp[j];   // diagonal (m, m)
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);

            // H_pre of tile it lands in buffer it&1, last read by the x_in warps for
            // tile it-2: they must have moved on (they arrive after their tile it-1 wait)
            if (it >= 1 && !mbar_wait(xin_prog, uint32_t((it - 1) & 1))) { s_abort = 1; break; }
            // push (partial logits, sum of squares) of row m to its owner
#pragma unroll
            for (int p = 0; p < PSP; p += 4) {
                float4 w4;
                w4.x = p + 0 < P ? d[p + 0] : (p + 0 == P ? ss : 0.0f);
                w4.y = p + 1 < P ? d[p + 1] : (p + 1 == P ? ss : 0.0f);
                w4.z = p + 2 < P ? d[p + 2] : (p + 2 == P ? ss : 0.0f);
                w4.w = p + 3 < P ? d[p + 3] : (p + 3 == P ? ss : 0.0f);
                st_async_f32x4(push_dst + p * 4, w4, push_bar);
            }
            if (!mbar_wait(part_full, uint32_t(it & 1))) { s_abort = 1; break; }

            // Coefficients of this CTA's TOK_PER_CTA tokens: a group of 8 lanes per
            // token; lane g takes the partial row from CTA g, the group reduces, then
            // lane g < N carries row g of H_res through a row-parallel Sinkhorn.
            {
                const int jj = et >> 3, g = et & 7;
                const int j = int(rank) * TOK_PER_CTA + jj;     // row within the tile
                const float* src = rpart + (g * TOK_PER_CTA + jj) * PSP;
                float v[PSP];
#pragma unroll
                for (int p = 0; p < PSP; p += 4) {
                    const float4 f4 = *reinterpret_cast<const float4*>(src + p);
                    v[p] = f4.x; v[p + 1] = f4.y; v[p + 2] = f4.z; v[p + 3] = f4.w;
                }
#pragma unroll
                for (int p = 0; p < PS; ++p) {
                    v[p] += __shfl_xor_sync(0xffffffffu, v[p], 1);
                    v[p] += __shfl_xor_sync(0xffffffffu, v[p], 2);
                    v[p] += __shfl_xor_sync(0xffffffffu, v[p], 4);
                }
                const float r = sqrtf(v[P] * inv_K + eps);                     // Eq.(15)
                const float inv_r = 1.0f / r;
                // every lane of the group carries the whole n x n Sinkhorn (no shuffles in
                // the iterations); lane g < N then keeps stream g's gates and H_res row g
                float mres[N][N];
#pragma unroll
                for (int i = 0; i < N; ++i)
#pragma unroll
                    for (int k = 0; k < N; ++k)
                        mres[i][k] = a2 * v[2 * N + i * N + k] * inv_r + sb[2 * N + i * N + k];   // Eq.(16)
                sinkhorn_regs<N>(mres, t_iters);                                   // Eq.(19)
                float zpre = 0.0f, zpost = 0.0f, row[N];
#pragma unroll
                for (int k = 0; k < N; ++k) row[k] = 0.0f;
#pragma unroll
                for (int i = 0; i < N; ++i)
                    if (g == i) {
                        zpre = a0 * v[i] * inv_r + sb[i];
                        zpost = a1 * v[N + i] * inv_r + sb[N + i];
#pragma unroll
                        for (int k = 0; k < N; ++k) row[k] = mres[i][k];
                    }
                if (g < N) {
                    const float hp = sigmoidf_(zpre);                              // Eq.(17)
                    // every CTA needs H_pre of every tile row for its x_in channels
                    const uint32_t hoff = smem_u32(shpre + (acc * MT_CAP + j) * N + g);
                    const uint32_t hbar = smem_u32(&hpre_full[acc]);
                    for (uint32_t rr = 0; rr < CL; ++rr) st_async_f32(mapa(hoff, rr), hp, mapa(hbar, rr));
                    const int64_t t = t0 + j;
                    if (j < Mt && t < T) {
                        if (Hpost) Hpost[t * N + g] = 2.0f * sigmoidf_(zpost);     // Eq.(18)
                        if (Hpre) Hpre[t * N + g] = hp;
                        if (Hres) {
#pragma unroll
                            for (int k = 0; k < N; ++k) Hres[(t * N + g) * N + k] = row[k];
                        }
                    }
                }
                if (u_out && j < Mt && t0 + j < T) {       // the backward's recompute
#pragma unroll
                    for (int p = 0; p < P; ++p)
                        if ((p & 7) == g) u_out[(t0 + j) * P + p] = v[p] * inv_r;
                    if (g == 0) r_out[t0 + j] = r;
                }
            }
            // every owner has read its partial rows of this tile once this CTA holds the
            // tile's H_pre; only then may the next tile's partial rows be pushed
            if (!mbar_wait(&hpre_full[acc], par)) { s_abort = 1; break; }
        }
    } else {
        // ------------------------------------------------------------ x_in
        const int xt = (warp < EPI_WARP0 ? warp - 2 : warp - 4) * 32 + lane;   // 0..XIN_THREADS-1
        const uint64_t drop = policy_evict_first();
        const int VPT = Cs / 8;                          // 16-byte vectors per token
        int it = 0;
        for (int tile = cluster_id; tile < num_tiles; tile += nclusters, ++it) {
            if (!mbar_wait_sleep(&hpre_full[it & 1], uint32_t((it >> 1) & 1))) { s_abort = 1; break; }
            __syncwarp();
            if (lane == 0) mbar_arrive(xin_prog);
            const int64_t t0 = int64_t(tile) * Mt;
            const float* hb = shpre + (it & 1) * MT_CAP * N;
            const int rows = int((T - t0) < int64_t(Mt) ? (T - t0) : int64_t(Mt));
            const int items = x_in ? rows * VPT : 0;
            for (int w0 = xt; w0 < items; w0 += XIN_UNROLL * XIN_THREADS) {
                uint4 raw[XIN_UNROLL][N];
                int tok[XIN_UNROLL], cc[XIN_UNROLL];
#pragma unroll
                for (int u = 0; u < XIN_UNROLL; ++u) {
                    const int w = w0 + u * XIN_THREADS;
                    const int wc = w < items ? w : items - 1;   // clamp; the store is skipped
                    tok[u] = wc / VPT;
                    cc[u] = c0 + (wc - tok[u] * VPT) * 8;
#pragma unroll
                    for (int i = 0; i < N; ++i)
                        raw[u][i] = ldg16_raw_hint(X + ((t0 + tok[u]) * N + i) * C + cc[u], drop);
                }
#pragma unroll
                for (int u = 0; u < XIN_UNROLL; ++u) {
                    if (w0 + u * XIN_THREADS >= items) break;
                    float o[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[e] = 0.0f;
#pragma unroll
                    for (int i = 0; i < N; ++i) {
                        const float h = hb[tok[u] * N + i];
                        const uint32_t w4[4] = {raw[u][i].x, raw[u][i].y, raw[u][i].z, raw[u][i].w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            o[2 * e] = fmaf(h, bf16_lo(w4[e]), o[2 * e]);
                            o[2 * e + 1] = fmaf(h, bf16_hi(w4[e]), o[2 * e + 1]);
                        }
                    }
                    store16<false>(x_in + (t0 + tok[u]) * C + cc[u], o);
                }
            }
            __syncwarp();
            if (lane == 0) atomicAdd(&s_xin_done, 1);
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
    const int64_t rounds = (a.T + int64_t(max_clusters) * MT_CAP - 1) / (int64_t(max_clusters) * MT_CAP);
    const int64_t per_round = (a.T + rounds - 1) / rounds;                     // tokens per round
    int Mt = int((per_round + max_clusters - 1) / max_clusters);
    if (Mt > MT_CAP) Mt = MT_CAP;
    const int64_t tiles64 = (a.T + Mt - 1) / Mt;
    const int nclusters = int(tiles64 < max_clusters ? tiles64 : max_clusters);

    EncodeTiledFn enc = encode_fn();
    if (!enc) {
        set_error("mhc_pre (tc): cuTensorMapEncodeTiled unavailable");
        return MHC_ERR_CUDA;
    }
    using G = Cfg<N>;
    CUtensorMap mapX, mapPhi;
    {
        const cuuint64_t dims[3] = {cuuint64_t(a.C), cuuint64_t(a.n), cuuint64_t(a.T)};
        const cuuint64_t strides[2] = {cuuint64_t(a.C) * 2, cuuint64_t(a.n) * a.C * 2};
        const cuuint32_t box[3] = {KC, 1, cuuint32_t(Mt)};
        const cuuint32_t estr[3] = {1, 1, 1};
        CUresult r = enc(&mapX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.X), dims, strides,
                         box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            set_error("mhc_pre (tc): cuTensorMapEncodeTiled(X) failed (%d)", int(r));
            return MHC_ERR_CUDA;
        }
    }
    {
        const cuuint64_t K = cuuint64_t(a.n) * a.C;
        const cuuint64_t dims[2] = {K, cuuint64_t(G::P)};
        const cuuint64_t strides[1] = {K * 2};
        const cuuint32_t box[2] = {KC, cuuint32_t(G::R)};
        const cuuint32_t estr[2] = {1, 1};
        CUresult r = enc(&mapPhi, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a.phi), dims, strides,
                         box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            set_error("mhc_pre (tc): cuTensorMapEncodeTiled(phi) failed (%d)", int(r));
            return MHC_ERR_CUDA;
        }
    }
    kern<<<dim3(unsigned(nclusters * CL)), NTHREADS, size_t(smem), s>>>(
        mapX, mapPhi, static_cast<const bf16_t*>(a.X), a.alpha[0], a.alpha[1], a.alpha[2], a.b, a.T,
        a.C, Mt, int(tiles64), a.t_iters, a.eps, a.skip_xin ? nullptr : static_cast<bf16_t*>(a.x_in),
        a.H_pre, a.H_post, a.H_res, a.u_out, a.r_out);
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
