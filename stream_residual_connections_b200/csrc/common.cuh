// Shared device/host helpers of libmhc (CUDA path only; nothing here is used
// by the CPU oracle).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "mhc.h"

namespace mhc {

using bf16_t = uint16_t;  // bfloat16 storage (raw bits)

// ------------------------------------------------------------ status plumbing
void set_error(const char* fmt, ...);
mhc_status cuda_status(cudaError_t e, const char* what);
mhc_status launch_status(const char* what);  // checks cudaGetLastError after a launch

// Device error word written by bounded waits that expire (bit 0 = timeout).
// libmhc is one translation unit (libmhc.cu), so these are defined here.
__device__ unsigned int g_device_error = 0u;
// Iteration cap of every bounded wait (device constant, settable for tests).
__constant__ long long g_wait_limit = 1ll << 26;

// -------------------------------------------------------------- conversions
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // RNE, lo in the low half
    return *reinterpret_cast<uint32_t*>(&v);
}

template <typename T> struct Vec;  // one 16-byte vector of a storage type
template <> struct Vec<float> { static constexpr int W = 4; };
template <> struct Vec<bf16_t> { static constexpr int W = 8; };

// Loads of 16 bytes widened to fp32.  `Stream` selects the evict-first
// (streaming) policy for data read exactly once.
template <bool Stream>
__device__ __forceinline__ void load16(const float* p, float (&v)[4]) {
    float4 a = Stream ? __ldcs(reinterpret_cast<const float4*>(p))
                      : *reinterpret_cast<const float4*>(p);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}
template <bool Stream>
__device__ __forceinline__ void load16(const bf16_t* p, float (&v)[8]) {
    uint4 a = Stream ? __ldcs(reinterpret_cast<const uint4*>(p))
                     : *reinterpret_cast<const uint4*>(p);
    v[0] = bf16_lo(a.x); v[1] = bf16_hi(a.x); v[2] = bf16_lo(a.y); v[3] = bf16_hi(a.y);
    v[4] = bf16_lo(a.z); v[5] = bf16_hi(a.z); v[6] = bf16_lo(a.w); v[7] = bf16_hi(a.w);
}
template <bool Stream>
__device__ __forceinline__ void store16(float* p, const float (&v)[4]) {
    float4 a = make_float4(v[0], v[1], v[2], v[3]);
    if (Stream) __stcs(reinterpret_cast<float4*>(p), a); else *reinterpret_cast<float4*>(p) = a;
}
template <bool Stream>
__device__ __forceinline__ void store16(bf16_t* p, const float (&v)[8]) {
    uint4 a = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                         pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
    if (Stream) __stcs(reinterpret_cast<uint4*>(p), a); else *reinterpret_cast<uint4*>(p) = a;
}

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(bf16_t v) { return __uint_as_float(uint32_t(v) << 16); }

__device__ __forceinline__ float sigmoidf_(float z) { return 1.0f / (1.0f + expf(-z)); }

// Approximate reciprocal: the PTX rcp.approx.ftz.f32 instruction (at most 1 ulp
// from 1/x for normal x, per the PTX ISA).  Operands here are sums of positive
// values of order one, far from the subnormal range that ftz flushes.
__device__ __forceinline__ float fast_rcp(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// Sinkhorn-Knopp on an N x N logit matrix held in registers ([mHC] Eq.(8)-(9)):
// M = exp(L); `iters` times normalise every column, then every row.  Each
// column is shifted by its maximum before exp when iters >= 1; the first
// column normalisation cancels any per-column factor, so the result is the
// same and exp cannot overflow.  The iterations form one dependent chain, so
// the normalisers use the approximate reciprocal: a correctly rounded one is
// a long sequence on this GPU (20 iterations measured ~4x slower), and the
// coefficients are only required to 1e-5.
template <int N>
__device__ __forceinline__ void sinkhorn_regs(float (&m)[N][N], int iters) {
#pragma unroll
    for (int j = 0; j < N; ++j) {
        float mx = m[0][j];
#pragma unroll
        for (int i = 1; i < N; ++i) mx = fmaxf(mx, m[i][j]);
        if (iters == 0) mx = 0.0f;
#pragma unroll
        for (int i = 0; i < N; ++i) m[i][j] = expf(m[i][j] - mx);
    }
    for (int it = 0; it < iters; ++it) {
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
    }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

}  // namespace mhc
