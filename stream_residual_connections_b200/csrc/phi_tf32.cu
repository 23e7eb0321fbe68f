// The projection matrix in tf32 ([mHC] section 4.3.1, Eq.(10): phi is stored as
// tfloat32 while x is bfloat16, Eq.(11)) as an exact pair of bf16 rows.
//
// A tf32 value t has 11 significant bits.  hi = bf16(t) (round to nearest even,
// 8 significant bits) leaves t - hi, a multiple of t's last tf32 bit no larger
// than half of hi's last bf16 bit: at most 3 significant bits, so lo = t - hi is
// a bf16 value too and hi + lo = t exactly (for |t| >= 2^-116, i.e. away from the
// subnormal range).  Since a bf16 x is exact in tf32, x t = x hi + x lo: the
// product the pages take in tf32 is the sum of two bf16 x bf16 products, which
// the bf16 tensor-core MMA (kind::f16) forms with an fp32 accumulator.
//
// Layout of the pair ([2 RH][n C] bf16, RH = P rounded up to 16): rows 0..P-1
// hold hi of phi^T's rows, rows RH..RH+P-1 lo, the rest zero; so one TMA box of
// 2 RH rows brings both halves, and lo's columns start at the 16-aligned RH.
#include "common.cuh"
#include "internal.h"

namespace mhc {
namespace tf32 {

// fp32 -> tf32, round to nearest even on the 13 dropped mantissa bits (inf and
// NaN pass unchanged).
__device__ __forceinline__ float round_tf32(float v) {
    const uint32_t u = __float_as_uint(v);
    if ((u & 0x7F800000u) == 0x7F800000u) return v;
    return __uint_as_float((u + 0xFFFu + ((u >> 13) & 1u)) & 0xFFFFE000u);
}

__device__ __forceinline__ uint32_t bits_bf16(float v) {
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    return uint32_t(*reinterpret_cast<const uint16_t*>(&h));
}

// One thread writes 8 bf16 (16 bytes) of one row of the pair.
__global__ void __launch_bounds__(256)
pair_kernel(const float* __restrict__ phi, int P, int RH, int64_t K, bf16_t* __restrict__ pair)
{
    const int64_t K8 = K / 8;
    const int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= int64_t(2 * RH) * K8) return;
    const int r = int(idx / K8);
    const int64_t k = (idx - int64_t(r) * K8) * 8;
    const int half = r / RH, p = r - half * RH;
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    if (p < P) {
        const float4 a = *reinterpret_cast<const float4*>(phi + int64_t(p) * K + k);
        const float4 c = *reinterpret_cast<const float4*>(phi + int64_t(p) * K + k + 4);
        const float v[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float t = round_tf32(v[e]);
            const uint32_t hb = bits_bf16(t);
            const uint32_t ob = half ? bits_bf16(t - __uint_as_float(hb << 16)) : hb;
            w[e >> 1] |= ob << (16 * (e & 1));
        }
    }
    *reinterpret_cast<uint4*>(pair + int64_t(r) * K + k) = make_uint4(w[0], w[1], w[2], w[3]);
}

}  // namespace tf32

mhc_status launch_phi_tf32_pair(const float* phi, int n, int C, void* pair, cudaStream_t s)
{
    const int P = n * n + 2 * n;
    const int RH = tf32_pair_half_rows(n);
    const int64_t K = int64_t(n) * C;
    const int64_t items = int64_t(2 * RH) * (K / 8);
    tf32::pair_kernel<<<unsigned((items + 255) / 256), 256, 0, s>>>(phi, P, RH, K, static_cast<bf16_t*>(pair));
    return launch_status("mhc_phi_tf32_pair");
}

}  // namespace mhc
