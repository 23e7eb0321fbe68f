// mhc_pre, tensor-core path (sm_100a: TMA + tcgen05.mma + TMEM + a cluster
// of 8 CTAs sharing partial sums through distributed shared memory).
//
// [mHC] section 4.3.1, Eq.(14)-(19), and F_pre := H_pre x_l.  Per token tile
// of Mt <= 64 tokens, the 8 CTAs of a cluster split the C channels: CTA r
// owns channels [r*C/8, (r+1)*C/8) of every stream, i.e. a K-slice of
// n*C/8 elements of each token's n*C row.
//
// Ring stage (one 64-channel block cb of the tile), per pair of streams
// (2p, 2p+1):  [ phiT rows of stream 2p | of stream 2p+1 ]  (2R rows)
//              [ X rows of stream 2p (Mt) | of stream 2p+1 (Mt) | unused ]  (128 rows)
// every row 128 bytes with the 128-byte swizzle.  One MMA per 16-wide K step
// and pair, D[128 x (2R+128)] += A * B^T with A = the pair's 128 X rows and
// B = the whole pair region, yields both products the coefficients need:
// columns [0, 2R) are the projections through phi (a row of stream 2p lands
// in columns [0, R), of stream 2p+1 in [R, 2R)), and column 2R+m is the dot
// product of X rows m and m, i.e. row m's sum of squares (Eq.15).  The pairs
// accumulate into the same columns, so after the tile TMEM row m < Mt holds
// the sums over streams 0, 2 of token m and row Mt+m those over streams 1, 3.
// phiT is streamed with X (it stays in L2), which leaves room for 4 stages.
// An odd n reads a zero-filled last stream (out of the tensor maps' range).
//
// Warp roles (16 warps):
//   0      TMA producer: per stage and pair, a {64, R, 2} box of phiT and a
//          {64, Mt, 2} box of X (L2 evict-last); it runs at most LAG tiles
//          ahead of the x_in warps, which keeps the x_in re-read in L2.
//   1      MMA issuer (tcgen05.mma kind::f16, fp32 accumulators in TMEM,
//          double-buffered across tiles).  The MMA commit is the only
//          consumer of a ring stage.
//   4-7    epilogue, one TMEM lane quarter each: every TMEM row (a token's
//          half: its projections and sum of squares) is pushed with st.async
//          into the shared memory of the CTA that owns the token (8 tokens per
//          CTA); warps 4-5 of the owner reduce the 2 x 8 partial rows, compute
//          the coefficients (Eq.16-19, Sinkhorn in registers) and push H_pre
//          to every CTA of the cluster.  The pushes complete transactions on
//          the receivers' mbarriers, so no fence or remote arrive sits on this
//          path.
//   2-3, 8-15  x_in = H_pre X for this CTA's channels, re-reading the tile's
//          X slice from L2 (evict-first on this last read).
// The roles meet only through mbarriers and one progress counter, so the TMA
// ring keeps streaming while a tile's coefficients and x_in are produced.
//
// HBM: X is read once; x_in and the coefficients are written once; phi is
// read from HBM about once (its re-reads hit L2).  Every wait is bounded
// (g_wait_limit); on expiry the kernel records the timeout in the device
// error word, drains its own copies and MMAs in flight, frees TMEM and returns.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace mhc {
namespace pretc {

using namespace sm100;

constexpr int CL = 8;            // CTAs per cluster (channel split)
constexpr int MROWS = 128;       // MMA M (TMEM lanes): two streams of up to MT_CAP tokens
constexpr int MT_CAP = 64;       // token rows per tile: bounds the L2 footprint of the x_in re-read
constexpr int KC = 64;           // channels per block (one 128-byte row)
constexpr int MAX_STAGES = 6;
constexpr int SMEM_LIMIT = 227 * 1024;
constexpr int NTHREADS = 512;
constexpr int EPI_WARP0 = 4, EPI_WARPS = 4;                       // TMEM lane quarters 0-3
constexpr int XIN_WARPS = 10, XIN_THREADS = XIN_WARPS * 32;       // warps 2-3 and 8-15
constexpr int TOK_PER_CTA = MT_CAP / CL;  // tokens whose coefficients a CTA computes
constexpr int XIN_UNROLL = 4;             // x_in vectors in flight per thread
// Tiles the TMA stream may run ahead of x_in.  With 15 clusters of 64-token
// tiles, LAG + 1 tiles of X (about 31 MB each at n = 4, C = 4096) wait in L2
// for their re-read: at LAG = 3 part of the re-read already misses L2 (about
// 60 of 256 MB, measured), yet the kernel is faster than at LAG = 2, where
// the ring idles while x_in catches up.
#ifndef MHC_PRE_LAG
#define MHC_PRE_LAG 3
#endif
constexpr int LAG = MHC_PRE_LAG;
constexpr int ACC_COLS = 256;             // TMEM columns per accumulator buffer
constexpr int TMEM_COLS = 512;
static_assert(TOK_PER_CTA * 8 == 64, "warps 4-5: one 8-lane group per coefficient token");

// SPLIT: phi is the exact bf16 pair of a tf32 phi (phi_tf32.cu), rows hi [0, RH) and
// lo [RH, 2 RH) per stream; a row's logit p is then column p + column RH + p of its half.
template <int N, bool SPLIT = false> struct Cfg {
    static constexpr int P = N * N + 2 * N;
    static constexpr int RH = (P + 15) / 16 * 16;   // rows of one half of the tf32 pair
    static constexpr int R = SPLIT ? 2 * RH : (P + 7) / 8 * 8;   // phiT rows per stream in a stage
    static constexpr int NP = (N + 1) / 2;          // stream pairs
    static constexpr int MMA_N = 2 * R + MROWS;     // B rows: the pair's phiT rows, then its X rows
    static constexpr int PAIR_BYTES = MMA_N * 128;
    static constexpr int STAGE_BYTES = NP * PAIR_BYTES;
    static constexpr int PS = P + 1;                // partial row: P projections + sum of squares
    static constexpr int PSP = (PS + 3) / 4 * 4;    // ... padded to 16-byte multiples
    static_assert(MMA_N % 16 == 0 && MMA_N <= ACC_COLS, "MMA N for M = 128");
};

enum Bar { B_FULL = 0, B_EMPTY = B_FULL + MAX_STAGES, B_TFULL = B_EMPTY + MAX_STAGES, B_TEMPTY = B_TFULL + 2,
           B_PART = B_TEMPTY + 2, B_HPRE, B_XIN = B_HPRE + 2, B_DRAIN, B_COUNT };

struct Layout {
    uint32_t ring, part, hpre, bias, bars, slot, total;
    int stages;
};

// Bytes after the ring: partial rows [CL][2 halves][TOK_PER_CTA][PSP], H_pre
// [2][MT_CAP][N], b, barriers.
template <int N, bool SPLIT = false>
__host__ __device__ constexpr uint32_t layout_fixed_bytes() {
    using G = Cfg<N, SPLIT>;
    return CL * 2 * TOK_PER_CTA * G::PSP * 4 + 2 * MT_CAP * N * 4 + G::P * 4 + 16 + B_COUNT * 8 + 16;
}

// Shared memory plan: the ring takes as many stages (up to MAX_STAGES) as the
// rest of the 227 KB leaves room for.
template <int N, bool SPLIT = false>
__host__ __device__ inline Layout layout_for() {
    using G = Cfg<N, SPLIT>;
    Layout L;
    L.ring = 0;
    {
        const int64_t room = int64_t(SMEM_LIMIT) - 1024 - layout_fixed_bytes<N, SPLIT>();
        const int64_t fit = room > 0 ? room / G::STAGE_BYTES : 0;
        L.stages = int(fit < MAX_STAGES ? fit : MAX_STAGES);
    }
    L.part = L.ring + uint32_t(L.stages) * G::STAGE_BYTES;
    L.hpre = L.part + CL * 2 * TOK_PER_CTA * G::PSP * 4;
    L.bias = L.hpre + 2 * MT_CAP * N * 4;
    L.bars = (L.bias + G::P * 4 + 15) / 16 * 16;
    L.slot = L.bars + B_COUNT * 8;
    L.total = L.slot + 16;
    return L;
}

// TMEM row r of a tile -> (half h, token) for rows r < 2 Mt; the unused rows
// r >= 2 Mt map one-to-one onto the slots of tokens Mt..MT_CAP-1, so that every
// owner receives the same number of bytes for every tile.
__device__ __forceinline__ void row_slot(int r, int Mt, int& h, int& tok) {
    if (r < 2 * Mt) {
        h = r >= Mt ? 1 : 0;
        tok = r - h * Mt;
    } else {
        const int k = r - 2 * Mt, spare = MT_CAP - Mt;     // spare >= 1 here
        h = k / spare;
        tok = Mt + k % spare;
    }
}

template <int N, bool SPLIT>
__global__ void __cluster_dims__(CL, 1, 1) __launch_bounds__(NTHREADS, 1)
pre_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmPhi,
              const bf16_t* __restrict__ X, float a0, float a1, float a2,
              const float* __restrict__ b, int64_t T, int C, int Mt, int num_tiles, int t_iters,
              float eps, bf16_t* __restrict__ x_in, float* __restrict__ Hpre,
              float* __restrict__ Hpost, float* __restrict__ Hres, float* __restrict__ u_out,
              float* __restrict__ r_out)
{
    using G = Cfg<N, SPLIT>;
    constexpr int P = G::P, R = G::R, NP = G::NP, PS = G::PS, PSP = G::PSP;
    constexpr int STAGE_BYTES = G::STAGE_BYTES, PAIR_BYTES = G::PAIR_BYTES;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment for the 128-byte-swizzle atoms
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int Cs = C / CL;
    const int CB = Cs / KC;            // channel blocks = ring stages per tile
    const Layout L = layout_for<N, SPLIT>();
    const int STAGES = L.stages;
    uint8_t* sring = smem + L.ring;
    float* rpart = reinterpret_cast<float*>(smem + L.part);   // [CL][2][TOK_PER_CTA][PSP], pushed by the cluster
    float* shpre = reinterpret_cast<float*>(smem + L.hpre);   // [2][MT_CAP][N]
    float* sb = reinterpret_cast<float*>(smem + L.bias);      // b, kept on chip for the coefficients
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint64_t* full = bars + B_FULL;
    uint64_t* empty = bars + B_EMPTY;
    uint64_t* tfull = bars + B_TFULL;
    uint64_t* tempty = bars + B_TEMPTY;
    uint64_t* part_full = bars + B_PART;     // this CTA's tokens: all partial rows landed
    uint64_t* hpre_full = bars + B_HPRE;     // [2] H_pre of every tile row landed (per tile parity)
    uint64_t* xin_prog = bars + B_XIN;
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
    cluster_sync();   // every CTA's barriers are initialised before any remote arrive

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t keep = policy_evict_last();
            const uint32_t stage_tx = uint32_t(NP) * uint32_t(2 * R + 2 * Mt) * 128;
            int s = 0;
            uint32_t ph = 0;
            int inflight_s[MAX_STAGES], inflight_ph[MAX_STAGES], n_issued = 0;
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
                for (int cb = 0; cb < CB; ++cb) {
                    if (!mbar_wait(&empty[s], ph ^ 1) || *(volatile int*)&s_abort) { ok = false; break; }
                    mbar_arrive_expect_tx(&full[s], stage_tx);
                    const int cc = c0 + cb * KC;
#pragma unroll
                    for (int p = 0; p < NP; ++p) {
                        uint8_t* pb = sring + s * STAGE_BYTES + p * PAIR_BYTES;
                        // phiT {64 channels, R rows, streams 2p..2p+1} of the {C, P, n} view
                        tma_load_3d_hint(pb, &tmPhi, &full[s], cc, 0, 2 * p, keep);
                        // X {64 channels, Mt tokens, streams 2p..2p+1} of the {C, T, n} view
                        tma_load_3d_hint(pb + 2 * R * 128, &tmX, &full[s], cc, t0, 2 * p, keep);
                    }
                    inflight_s[n_issued % MAX_STAGES] = s;
                    inflight_ph[n_issued % MAX_STAGES] = int(ph);
                    ++n_issued;
                    if (++s == STAGES) { s = 0; ph ^= 1; }
                }
            }
            if (!ok) {
                s_abort = 1;
                // drain this CTA's copies still in flight (the ring slots of the
                // last min(n_issued, STAGES) stages) before the block can exit
                const int pending = n_issued < STAGES ? n_issued : STAGES;
                for (int j = 0; j < pending; ++j) {
                    const int k = (n_issued - 1 - j) % MAX_STAGES;
                    mbar_wait(&full[inflight_s[k]], uint32_t(inflight_ph[k]), 1ll << 22);
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
                    for (int p = 0; p < NP; ++p) {
#pragma unroll
                        for (int kk = 0; kk < KC / 16; ++kk) {
                            const uint32_t pb = ring_a + s * STAGE_BYTES + p * PAIR_BYTES + kk * 32;
                            const uint64_t ad = sdesc_k_sw128(pb + 2 * R * 128);   // the pair's X rows
                            const uint64_t bd = sdesc_k_sw128(pb);                 // phiT rows, then X rows
                            mma_bf16(d, ad, bd, idesc, (cb | p | kk) != 0);
                        }
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

    } else if (warp >= EPI_WARP0 && warp < EPI_WARP0 + EPI_WARPS) {
        // ------------------------------------------------------------ epilogue
        const int et = threadIdx.x - EPI_WARP0 * 32;    // 0..127
        const int qd = warp & 3;                        // TMEM lane quarter of this warp
        const int r = qd * 32 + lane;                   // TMEM row (lane)
        const float inv_K = 1.0f / float(N * C);
        constexpr uint32_t PART_BYTES = CL * 2 * TOK_PER_CTA * PSP * 4;
        constexpr uint32_t HPRE_BYTES = MT_CAP * N * 4;
        int h, tok;
        row_slot(r, Mt, h, tok);
        // the partial row goes to the token's owner CTA, slot (rank, half, token % TOK_PER_CTA)
        const uint32_t owner = uint32_t(tok / TOK_PER_CTA);
        const uint32_t push_dst =
            mapa(smem_u32(rpart + ((int(rank) * 2 + h) * TOK_PER_CTA + tok % TOK_PER_CTA) * PSP), owner);
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
            if (!warp_wait(&tfull[acc], par)) { s_abort = 1; break; }
            tc_fence_after();
            // the row's projections: columns [h R, h R + P) of its half h (with the tf32
            // pair, column h R + RH + q adds the lo part of logit q)
            constexpr int DW = SPLIT ? G::RH : 2 * R;
            float d[DW];
            const uint32_t taddr = tmem_base + (uint32_t(qd * 32) << 16) + uint32_t(acc * ACC_COLS);
            if constexpr (SPLIT) {
#pragma unroll
                for (int q = 0; q < DW; ++q) d[q] = 0.0f;
            }
#pragma unroll
            for (int c = 0; c < 2 * R; c += 16) {
                float tmp[16];
                tmem_ld16(taddr + c, tmp);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    if constexpr (SPLIT) {
                        const int col = c + j, hc = col / R, q = (col % R) % G::RH;   // compile-time
                        if (hc == h) d[q] += tmp[j];
                    } else {
                        if (c + j < 2 * R) d[c + j] = tmp[j];
                    }
                }
            }
            float ss = 0.0f;
#pragma unroll
            for (int c = 0; c < 32; c += 16) {          // column 2R + r: X row r . X row r
                float tmp[16];
                tmem_ld16(taddr + 2 * R + qd * 32 + c, tmp);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) if (c + j == lane) ss = tmp[j];
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);

            // H_pre of tile it lands in buffer it&1, last read by the x_in warps for
            // tile it-2: they must have moved on (they arrive after their tile it-1 wait)
            if (it >= 1 && !warp_wait(xin_prog, uint32_t((it - 1) & 1))) { s_abort = 1; break; }
            // push (partial projections, sum of squares) of this row's half to its owner
#pragma unroll
            for (int p = 0; p < PSP; p += 4) {
                float w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int q = p + e;
                    if constexpr (SPLIT)
                        w[e] = q < P ? d[q] : (q == P ? ss : 0.0f);
                    else
                        w[e] = q < P ? (h ? d[R + q] : d[q]) : (q == P ? ss : 0.0f);   // q < P <= R
                }
                st_async_f32x4(push_dst + p * 4, make_float4(w[0], w[1], w[2], w[3]), push_bar);
            }
            if (et < 64) {
                if (!warp_wait(part_full, uint32_t(it & 1))) { s_abort = 1; break; }
                // Coefficients of this CTA's TOK_PER_CTA tokens: a group of 8 lanes per
                // token.  Lane g sums entries p = g (mod 8) over the 2 x CL partial
                // rows, then the group exchanges the sums (independent shuffles, no
                // reduction chain); lane g < N later carries row g of H_res.
                const int jj = et >> 3, g = et & 7;
                const int j = int(rank) * TOK_PER_CTA + jj;     // row within the tile
                constexpr int OWN = (PS + 7) / 8;               // entries summed per lane
                float own[OWN];
#pragma unroll
                for (int k = 0; k < OWN; ++k) {
                    const int p = g + 8 * k;
                    float s0 = 0.0f, s1 = 0.0f;
                    if (p < PS) {
#pragma unroll
                        for (int c = 0; c < CL; ++c) {
                            s0 += rpart[((c * 2 + 0) * TOK_PER_CTA + jj) * PSP + p];
                            s1 += rpart[((c * 2 + 1) * TOK_PER_CTA + jj) * PSP + p];
                        }
                    }
                    own[k] = s0 + s1;
                }
                float v[PSP];
#pragma unroll
                for (int p = 0; p < PS; ++p) v[p] = __shfl_sync(0xffffffffu, own[p >> 3], p & 7, 8);
                const float rr_ = sqrtf(v[P] * inv_K + eps);                   // Eq.(15)
                const float inv_r = 1.0f / rr_;
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
                    for (uint32_t cr = 0; cr < CL; ++cr) st_async_f32(mapa(hoff, cr), hp, mapa(hbar, cr));
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
                    if (g == 0) r_out[t0 + j] = rr_;
                }
            }
            // every owner has read its partial rows of this tile once this CTA holds the
            // tile's H_pre; only then may the next tile's partial rows be pushed
            if (!warp_wait(&hpre_full[acc], par)) { s_abort = 1; break; }
        }
    } else {
        // ------------------------------------------------------------ x_in
        const int xt = (warp < EPI_WARP0 ? warp - 2 : warp - (EPI_WARP0 + EPI_WARPS - 2)) * 32 + lane;
        const uint64_t drop = policy_evict_first();
        const int VPT = Cs / 8;                          // 16-byte vectors per token
        int it = 0;
        for (int tile = cluster_id; tile < num_tiles; tile += nclusters, ++it) {
            if (!warp_wait_sleep(&hpre_full[it & 1], uint32_t((it >> 1) & 1))) { s_abort = 1; break; }
            __syncwarp();
            if (lane == 0) mbar_arrive(xin_prog);
            const int64_t t0 = int64_t(tile) * Mt;
            const float* hb = shpre + (it & 1) * MT_CAP * N;
            const int rows = int((T - t0) < int64_t(Mt) ? (T - t0) : int64_t(Mt));
            const int items = x_in ? rows * VPT : 0;
            for (int w0 = xt; w0 < items; w0 += XIN_UNROLL * XIN_THREADS) {
                uint4 raw[XIN_UNROLL][N];
                int tk[XIN_UNROLL], cc[XIN_UNROLL];
#pragma unroll
                for (int u = 0; u < XIN_UNROLL; ++u) {
                    const int w = w0 + u * XIN_THREADS;
                    const int wc = w < items ? w : items - 1;   // clamp; the store is skipped
                    tk[u] = wc / VPT;
                    cc[u] = c0 + (wc - tk[u] * VPT) * 8;
#pragma unroll
                    for (int i = 0; i < N; ++i)
                        raw[u][i] = ldg16_raw_hint(X + ((t0 + tk[u]) * N + i) * C + cc[u], drop);
                }
#pragma unroll
                for (int u = 0; u < XIN_UNROLL; ++u) {
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
    cluster_sync();   // no CTA leaves while a peer may still touch its shared memory
}

// ------------------------------------------------------------------ host

template <int N, bool SPLIT>
static int smem_bytes() { return int(layout_for<N, SPLIT>().total) + 1024; }

template <int N, bool SPLIT>
static bool fits(int C)
{
    return C % (CL * KC) == 0 && layout_for<N, SPLIT>().stages >= 2 && smem_bytes<N, SPLIT>() <= SMEM_LIMIT;
}

template <int N, bool SPLIT>
static mhc_status launch_n(const PreArgs& a, cudaStream_t s)
{
    static int configured_smem = 0;
    static int max_clusters = 0;
    const int smem = smem_bytes<N, SPLIT>();
    auto kern = pre_tc_kernel<N, SPLIT>;
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
    // Token tiles of Mt rows, Mt a multiple of 8 (each stream's rows in a stage
    // then start on a 1024-byte swizzle atom) and at most MT_CAP.  A tile costs
    // its Mt tokens plus a fixed overhead worth about TILE_COST tokens (the MMAs
    // always cover 128 rows; the coefficient exchange; a shorter TMA box); take
    // the Mt that minimises the busiest cluster's cost (ties: the larger Mt).
    constexpr int TILE_COST = 32;
    int Mt = MT_CAP;
    int64_t best = -1;
    for (int m = MT_CAP; m >= 8; m -= 8) {
        const int64_t tiles = (a.T + m - 1) / m;
        const int64_t cost = (tiles + max_clusters - 1) / max_clusters * (m + TILE_COST);
        if (best < 0 || cost < best) { best = cost; Mt = m; }
    }
    const int64_t tiles64 = (a.T + Mt - 1) / Mt;
    const int nclusters = int(tiles64 < max_clusters ? tiles64 : max_clusters);

    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) {
        set_error("mhc_pre (tc): cuTensorMapEncodeTiled unavailable");
        return MHC_ERR_CUDA;
    }
    using G = Cfg<N, SPLIT>;
    CUtensorMap mapX, mapPhi;
    {
        // X [T][n][C] viewed as {C, T, n}: a box {64, Mt, 2} lands stream-major
        // (the Mt rows of stream 2p, then those of stream 2p+1)
        const cuuint64_t dims[3] = {cuuint64_t(a.C), cuuint64_t(a.T), cuuint64_t(a.n)};
        const cuuint64_t strides[2] = {cuuint64_t(a.n) * a.C * 2, cuuint64_t(a.C) * 2};
        const cuuint32_t box[3] = {KC, cuuint32_t(Mt), 2};
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
        // phiT [P][n*C] viewed as {C, P, n}: a box {64, R, 2} holds the R rows
        // (rows >= P zero-filled) of streams 2p and 2p+1 for one channel block; the
        // tf32 pair [2 RH][n*C] as {C, 2 RH, n}: both halves in the R = 2 RH rows
        const cuuint64_t dims[3] = {cuuint64_t(a.C), cuuint64_t(SPLIT ? 2 * G::RH : G::P), cuuint64_t(a.n)};
        const cuuint64_t strides[2] = {cuuint64_t(a.n) * a.C * 2, cuuint64_t(a.C) * 2};
        const cuuint32_t box[3] = {KC, cuuint32_t(G::R), 2};
        const cuuint32_t estr[3] = {1, 1, 1};
        CUresult r = enc(&mapPhi, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.phi), dims, strides,
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
    const bool split = a.phi_dt == MHC_TF32_PAIR;
    if (a.x_dt != MHC_BF16 || (a.phi_dt != MHC_BF16 && !split) || a.T < 1 || a.T >= (int64_t(1) << 31))
        return false;
    switch (a.n) {
        case 2: return split ? pretc::fits<2, true>(a.C) : pretc::fits<2, false>(a.C);
        case 3: return split ? pretc::fits<3, true>(a.C) : pretc::fits<3, false>(a.C);
        case 4: return split ? pretc::fits<4, true>(a.C) : pretc::fits<4, false>(a.C);
        default: return false;
    }
}

mhc_status launch_pre_tc(const PreArgs& a, cudaStream_t s)
{
    const bool split = a.phi_dt == MHC_TF32_PAIR;
    switch (a.n) {
        case 2: return split ? pretc::launch_n<2, true>(a, s) : pretc::launch_n<2, false>(a, s);
        case 3: return split ? pretc::launch_n<3, true>(a, s) : pretc::launch_n<3, false>(a, s);
        case 4: return split ? pretc::launch_n<4, true>(a, s) : pretc::launch_n<4, false>(a, s);
        default: break;
    }
    set_error("mhc_pre (tc): n=%d not supported", a.n);
    return MHC_ERR_UNSUPPORTED;
}

}  // namespace mhc
