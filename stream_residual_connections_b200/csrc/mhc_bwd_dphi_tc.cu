// mhc_backward, the dphi product on tensor cores:
//   dphi^T[p][k] = sum_t dd[t][p] x[t][k]     ([mHC] section 4.3.1: the backward of the
// Eq.(14)-(15) projection kernel; dd = alpha dz / r is the gradient of the projection).
//
// A contraction over tokens (K = tokens, M = logits, N = columns k of vec(X)):
//   A = dd^T as an exact-enough bf16 pair: rows 0..31 hold bf16(dd[.][p]) (p < P), rows
//       32..63 the remainder bf16(dd - hi), written by ddt_kernel from the B1 records
//       ([64][T8] bf16, token-contiguous: K-major); rows 64..127 are outside the tensor
//       map (TMA zero fill), so M = 128 with the hi and lo rows of logit p in D rows p
//       and 32 + p.  hi + lo carries dd to about 2^-17.
//   B = x, straight from X [T][nC]: a TMA box of 64 channels x 64 tokens is 64 rows of
//       128 bytes, channels contiguous, i.e. the 128-byte-swizzled MN-major layout; two
//       boxes side by side give N = 128 columns (the second box 8 KB on: the MN atom
//       stride), and the 8-token-row groups are 1 KB apart (the K group stride).
// One CTA per (128-column slab, token segment); D accumulates the segment's tokens in
// TMEM (128 columns) over a ring of 3 stages (16 KB of A + 16 KB of B each); at the end
// warps 4 and 5 (TMEM lanes 0-31 and 32-63) add each logit's hi and lo rows through
// shared memory and write the slab of dphi^T (one segment) or of the segment's partial
// sums, which the existing fixed-order reduction adds up.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace mhc {
namespace bwdtc {

using namespace sm100;

constexpr int KT = 64;                       // tokens per stage (4 MMAs of K = 16)
constexpr int NCH = 128;                     // columns per CTA (MMA N)
constexpr int MROWS = 128;                   // MMA M: dd^T pair rows (64 loaded, 64 zero)
constexpr int HALF = 32;                     // lo rows start here
constexpr int STAGES = 3;
constexpr int A_BYTES = MROWS * 128;         // 16 KB
constexpr int BOX_BYTES = KT * 128;          // 64 token rows x 64 channels: 8 KB
constexpr int B_BYTES = (NCH / 64) * BOX_BYTES;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NTHREADS = 192;                // warp 0 TMA, 1 MMA, 2-5 TMEM lane quarters
constexpr int TMEM_COLS = 128;
constexpr int LO_PITCH = NCH + 4;            // floats per row of the lo exchange (bank spread)
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
static_assert(HALF * LO_PITCH * 4 <= STAGE_BYTES, "the lo exchange reuses stage 0");

// 128-byte-swizzled MN-major operand: rows of 128 bytes run along M/N (64 bf16), the
// K index advances by row; lbo = byte stride between 64-element MN atoms, sbo = byte
// stride between groups of 8 K rows.
__device__ __forceinline__ uint64_t sdesc_mn_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    const uint64_t lo = uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t((lbo >> 4) & 0x3FFFu) << 16);
    const uint64_t hi = uint64_t((sbo >> 4) & 0x3FFFu) | (uint64_t(1) << 14) | (uint64_t(2) << 29);
    return lo | (hi << 32);
}

// kind::f16, D fp32, A and B bf16, A K-major, B MN-major ("transpose B").
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | (uint32_t(NCH >> 3) << 17) |
                           (uint32_t(MROWS >> 4) << 24);

// dd^T pair from the B1 records: thread per token, coalesced along t.
template <int N>
__global__ void __launch_bounds__(256)
ddt_kernel(const float* __restrict__ ws, int stride, int dd_off, int64_t T, int64_t pitch, bf16_t* __restrict__ ddt)
{
    constexpr int P = N * N + 2 * N;
    const int64_t t = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (t >= T) return;
#pragma unroll
    for (int p = 0; p < HALF; ++p) {
        float hi = 0.0f, lo = 0.0f;
        if (p < P) {
            const float d = ws[t * stride + dd_off + p];
            const __nv_bfloat16 h = __float2bfloat16_rn(d);
            hi = __bfloat162float(h);
            lo = d - hi;
        }
        const __nv_bfloat16 hb = __float2bfloat16_rn(hi), lb = __float2bfloat16_rn(lo);
        ddt[int64_t(p) * pitch + t] = *reinterpret_cast<const bf16_t*>(&hb);
        ddt[int64_t(HALF + p) * pitch + t] = *reinterpret_cast<const bf16_t*>(&lb);
    }
}

__global__ void __launch_bounds__(NTHREADS, 1)
dphi_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int64_t T,
            int64_t seg_len, int P, int64_t K, float* __restrict__ out_base, int64_t seg_stride)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* done = bars + 2 * STAGES;
    uint32_t* slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 1);
    __shared__ int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t k0 = int64_t(blockIdx.x) * NCH;
    const int64_t t_begin = int64_t(blockIdx.y) * seg_len;
    const int64_t t_end = (t_begin + seg_len < T) ? t_begin + seg_len : T;
    const int nst = t_end > t_begin ? int((t_end - t_begin + KT - 1) / KT) : 0;
    float* out = out_base + int64_t(blockIdx.y) * seg_stride;

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(slot, TMEM_COLS);
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *slot;

    if (warp == 0) {
        if (lane == 0 && nst > 0) {
            tma_prefetch(&tmA);
            tma_prefetch(&tmB);
            int s = 0;
            uint32_t ph = 0;
            int issued = 0;
            for (int j = 0; j < nst; ++j) {
                if (!mbar_wait(&empty[s], ph ^ 1) || *(volatile int*)&s_abort) {
                    s_abort = 1;
                    break;
                }
                uint8_t* st = smem + s * STAGE_BYTES;
                const int t = int(t_begin + int64_t(j) * KT);
                mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
                tma_load_2d(st, &tmA, &full[s], t, 0);                                   // dd^T rows
#pragma unroll
                for (int bx = 0; bx < NCH / 64; ++bx)
                    tma_load_2d(st + A_BYTES + bx * BOX_BYTES, &tmB, &full[s], int(k0) + 64 * bx, t);  // x
                ++issued;
                if (++s == STAGES) { s = 0; ph ^= 1; }
            }
            if (issued < nst) {
                // wait (bounded) for the loads in flight before the CTA may leave
                const int pending = issued < STAGES ? issued : STAGES;
                for (int q = 0; q < pending; ++q) {
                    const int j = issued - 1 - q;
                    mbar_wait(&full[j % STAGES], uint32_t((j / STAGES) & 1), 1ll << 22);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && nst > 0) {
            const uint32_t ring = smem_u32(smem);
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int j = 0; j < nst; ++j) {
                if (!mbar_wait(&full[s], ph) || *(volatile int*)&s_abort) { ok = false; break; }
                tc_fence_after();
                const uint32_t a0 = ring + s * STAGE_BYTES, b0 = a0 + A_BYTES;
#pragma unroll
                for (int kk = 0; kk < KT / 16; ++kk) {
                    const uint64_t ad = sdesc_k_sw128(a0 + kk * 32);                    // 16 tokens along a row
                    const uint64_t bd = sdesc_mn_sw128(b0 + kk * 2048, BOX_BYTES, 1024);  // 16 token rows
                    mma_bf16(tmem_base, ad, bd, IDESC, (j | kk) != 0);
                }
                mma_commit(&empty[s]);
                if (++s == STAGES) { s = 0; ph ^= 1; }
            }
            if (!ok) s_abort = 1;
            mma_commit(done);                       // every issued MMA has finished
        }
    } else {
        // epilogue: warp 4 = TMEM lanes 0-31 (hi rows), warp 5 = lanes 32-63 (lo rows)
        const int qd = warp & 3;
        if (qd <= 1) {
            bool ok = true;
            if (nst > 0) ok = warp_wait(done, 0);
            // warp-uniform: the TMEM loads below need every lane of the warp
            ok = __all_sync(0xffffffffu, ok && !*(volatile int*)&s_abort);
            float* lo_x = reinterpret_cast<float*>(smem);     // [32][LO_PITCH], stage 0 is free now
            const uint32_t taddr = tmem_base + (uint32_t(qd * 32) << 16);
            if (qd == 1 && nst > 0 && ok) {
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < NCH; c += 16) {
                    float v[16];
                    tmem_ld16(taddr + c, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; e += 4)
                        *reinterpret_cast<float4*>(lo_x + lane * LO_PITCH + c + e) =
                            make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                }
            }
            asm volatile("bar.sync 1, 64;" ::: "memory");     // warps 4 and 5
            if (qd == 0 && ok) {
                // the TMEM loads are warp-collective: every lane takes part, lanes < P store
                float* row = out + int64_t(lane) * K + k0;
                const bool mine = lane < P;
                if (nst > 0) tc_fence_after();
#pragma unroll
                for (int c = 0; c < NCH; c += 16) {
                    float v[16];
                    if (nst > 0) {
                        tmem_ld16(taddr + c, v);
                        tmem_wait_ld();
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] = 0.0f;
                    }
                    if (mine) {
#pragma unroll
                        for (int e = 0; e < 16; e += 4) {
                            float4 r = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                            if (nst > 0) {
                                const float4 l = *reinterpret_cast<const float4*>(lo_x + lane * LO_PITCH + c + e);
                                r.x += l.x; r.y += l.y; r.z += l.z; r.w += l.w;
                            }
                            *reinterpret_cast<float4*>(row + c + e) = r;
                        }
                    }
                }
            }
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace bwdtc

bool backward_dphi_tc_supported(const BwdArgs& a)
{
    return a.dt == MHC_BF16 && a.n >= 1 && a.n <= 4 && (int64_t(a.n) * a.C) % bwdtc::NCH == 0 && a.T >= 1 &&
           a.T < (int64_t(1) << 31) && a.ddt != nullptr;
}

mhc_status launch_backward_dphi_tc(const BwdArgs& a, int stride, int dd_off, int segs, int64_t seg_len,
                                   cudaStream_t s)
{
    using namespace bwdtc;
    const int P = a.n * a.n + 2 * a.n;
    const int64_t K = int64_t(a.n) * a.C;
    const int64_t pitch = backward_ddt_pitch(a.T);
    switch (a.n) {
        case 1: ddt_kernel<1><<<unsigned((a.T + 255) / 256), 256, 0, s>>>(a.records, stride, dd_off, a.T, pitch, static_cast<bf16_t*>(a.ddt)); break;
        case 2: ddt_kernel<2><<<unsigned((a.T + 255) / 256), 256, 0, s>>>(a.records, stride, dd_off, a.T, pitch, static_cast<bf16_t*>(a.ddt)); break;
        case 3: ddt_kernel<3><<<unsigned((a.T + 255) / 256), 256, 0, s>>>(a.records, stride, dd_off, a.T, pitch, static_cast<bf16_t*>(a.ddt)); break;
        case 4: ddt_kernel<4><<<unsigned((a.T + 255) / 256), 256, 0, s>>>(a.records, stride, dd_off, a.T, pitch, static_cast<bf16_t*>(a.ddt)); break;
        default: set_error("mhc_backward: n=%d not supported", a.n); return MHC_ERR_UNSUPPORTED;
    }
    mhc_status st = launch_status("mhc_backward dd^T pair kernel");
    if (st != MHC_OK) return st;

    static int configured = 0;
    if (!configured) {
        const cudaError_t e = cudaFuncSetAttribute(dphi_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return cuda_status(e, "mhc_backward dphi: set shared memory size");
        configured = 1;
    }
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) {
        set_error("mhc_backward: cuTensorMapEncodeTiled unavailable");
        return MHC_ERR_CUDA;
    }
    CUtensorMap mapA, mapB;
    {
        // dd^T pair [64][pitch] bf16 viewed as {T, 64}: a box {64 tokens, 128 rows}; rows
        // 64..127 and tokens >= T lie outside and read as zero
        const cuuint64_t dims[2] = {cuuint64_t(a.T), cuuint64_t(2 * HALF)};
        const cuuint64_t strides[1] = {cuuint64_t(pitch) * 2};
        const cuuint32_t box[2] = {KT, MROWS};
        const cuuint32_t estr[2] = {1, 1};
        const CUresult r = enc(&mapA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.ddt, dims, strides, box, estr,
                               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            set_error("mhc_backward: cuTensorMapEncodeTiled(dd^T) failed (%d)", int(r));
            return MHC_ERR_CUDA;
        }
    }
    {
        // X [T][nC] viewed as {nC, T}: a box {64 columns, 64 tokens}
        const cuuint64_t dims[2] = {cuuint64_t(K), cuuint64_t(a.T)};
        const cuuint64_t strides[1] = {cuuint64_t(K) * 2};
        const cuuint32_t box[2] = {64, KT};
        const cuuint32_t estr[2] = {1, 1};
        const CUresult r = enc(&mapB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a.X), dims, strides,
                               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            set_error("mhc_backward: cuTensorMapEncodeTiled(X) failed (%d)", int(r));
            return MHC_ERR_CUDA;
        }
    }
    float* out = segs > 1 ? a.dphi_part : a.dphi;
    const int64_t seg_stride = segs > 1 ? int64_t(P) * K : 0;
    dphi_kernel<<<dim3(unsigned(K / NCH), unsigned(segs)), NTHREADS, SMEM_BYTES, s>>>(mapA, mapB, a.T, seg_len, P, K,
                                                                                   out, seg_stride);
    return launch_status("mhc_backward dphi tensor-core kernel");
}

}  // namespace mhc
