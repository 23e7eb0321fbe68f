// Internal launcher interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "mhc.h"

namespace mhc {

mhc_status launch_post(const void* X, const void* F, mhc_dtype dt, const float* Hpost,
                       const float* Hres, int64_t T, int n, int C, void* Xn, cudaStream_t s);

struct PreArgs {
    const void* X; mhc_dtype x_dt;
    const void* phi; mhc_dtype phi_dt;
    float alpha[3];
    const float* b;
    int64_t T; int n; int C; int t_iters; float eps;
    void* x_in; float* H_pre; float* H_post; float* H_res;
    // internal (the backward's recompute): u = (x phi)/r [T][P] and r [T] when
    // non-null; skip_xin leaves x_in unwritten; H_post / H_res may then be null
    float* u_out = nullptr; float* r_out = nullptr; bool skip_xin = false;
};

// CUDA-core (FMA) projection path: every n, dtype pair and C % 8 == 0.
mhc_status launch_pre_fma(const PreArgs& a, cudaStream_t s);

// Tensor-core path (TMA + tcgen05 + 8-CTA cluster): bf16 X and phi, n in
// {2, 3, 4}, C % 512 == 0 and phi's per-CTA slice resident in shared memory.
bool pre_tc_supported(const PreArgs& a);
mhc_status launch_pre_tc(const PreArgs& a, cudaStream_t s);
bool pre_wide_supported(const PreArgs& a);   // bf16 phi, n = 5..8; tf32 pair phi, n = 1..7 (mhc_pre_wide.cu)
mhc_status launch_pre_wide(const PreArgs& a, cudaStream_t s);

mhc_status launch_conv_gs(const void* F, mhc_dtype dt, const float* W, const int* kappa, int r,
                          int64_t T, int C, int64_t seq_len, float* V, cudaStream_t s);

struct UpdateArgs {
    void* X; mhc_dtype dt; const float* V; int Kr; const int32_t* idx; const float* w;
    const void* phi; float alpha[2]; const float* b;
    int64_t T; int N; int C; int k; int t_iters; float eps;
    float* H_res; float* H_post;
};
mhc_status launch_sparse_update(const UpdateArgs& a, cudaStream_t s);
bool update_tc_supported(const UpdateArgs& a);
mhc_status launch_update_tc(const UpdateArgs& a, cudaStream_t s);

struct RouteArgs {
    const void* X; mhc_dtype dt; const void* phi; float alpha[2]; const float* b;
    int64_t T; int N; int C; int k; int m; float eps;
    void* x_in; float* H_pre; float* score; int32_t* idx; float* w;
};
mhc_status launch_route(const RouteArgs& a, cudaStream_t s);
bool route_tc_supported(const RouteArgs& a);
mhc_status launch_route_tc(const RouteArgs& a, cudaStream_t s);

struct BwdArgs {
    const void* X; const void* F; const void* phi; mhc_dtype dt; float alpha[3]; const float* b;
    const void* dXn; const void* dxin; int64_t T; int n; int C; int t_iters; float eps;
    void* dX; void* dF; float* dphi; float* dalpha; float* db;
    float* records; float* u_scratch; float* r_scratch;   // carved from the caller's workspace
    float* dphi_part;                                     // [segments][P][nC] when segments > 1
    void* ddt = nullptr;                                  // dd^T bf16 pair [64][pitch] (dphi on tensor cores)
};
int backward_b3_segments(int64_t T);
inline int64_t backward_ddt_pitch(int64_t T) { return (T + 7) / 8 * 8; }   // 16-byte rows for TMA
bool backward_dphi_tc_supported(const BwdArgs& a);
mhc_status launch_backward_dphi_tc(const BwdArgs& a, int stride, int dd_off, int segs, int64_t seg_len,
                                   cudaStream_t s);
size_t backward_record_stride(int n);            // floats per token record (0: unsupported n)
mhc_status launch_backward(const BwdArgs& a, cudaStream_t s);

// tf32 phi as an exact pair of bf16 rows (phi_tf32.cu): [2 RH][n C], RH = P rounded up to 16.
inline int tf32_pair_half_rows(int n) { return (n * n + 2 * n + 15) / 16 * 16; }
mhc_status launch_phi_tf32_pair(const float* phi, int n, int C, void* pair, cudaStream_t s);

// HC (tanh) coefficients + F_pre input (hc_pre.cu); Amax Gain of a stack of H_res.
struct HcArgs {
    const void* X; mhc_dtype x_dt; const void* theta; mhc_dtype t_dt;
    float alpha[3]; const float* b;
    int64_t T; int n; int C; float eps;
    void* x_in; float* H_pre; float* H_post; float* H_res;
};
mhc_status launch_hc_pre(const HcArgs& a, cudaStream_t s);
mhc_status launch_amax_gain(const float* H, int L, int64_t T, int n, float* gain, float* gain_max,
                            cudaStream_t s);

// Which mhc_pre path to take (MHC_PRE_PATH_*), process-wide.
extern int g_pre_path;

}  // namespace mhc
