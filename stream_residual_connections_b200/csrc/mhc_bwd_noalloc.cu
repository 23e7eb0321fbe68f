// mhc_backward_noalloc: mhc_backward for callers that cannot allocate device
// memory -- code running inside a CUDA graph capture, a custom allocator's own
// callbacks, or an embedding runtime that owns every allocation and forbids
// libraries from making their own.  They cannot provide the workspace that
// mhc_backward takes, so this entry point uses a fixed scratch area compiled
// into the library instead, and calls no allocating routine at all.
//
// The scratch is a file-scope device array of MHC_NOALLOC_SCRATCH_BYTES
// (4 MiB).  Every GPU that loads the library holds one copy of it until the
// process exits.  Host code cannot use the array's name as a device address,
// so the first call on each device looks the address up (cudaGetSymbolAddress,
// with that device current) and remembers it; that first call should
// therefore come before any stream capture.  All calls on a device share the
// one array: calls whose work overlaps on the GPU (different streams, no
// ordering between them) race and give undefined results.  The scratch keeps
// whatever the previous call left there; nothing in it has to start at zero,
// because every value the backward reads from it is written earlier in the
// same call.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace mhc {

static __device__ __align__(256) unsigned char g_noalloc_scratch[MHC_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of this device's scratch array (set up on first use).
mhc_status noalloc_scratch(void** out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_status(e, "mhc_backward_noalloc: cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) {
        set_error("mhc_backward_noalloc: device ordinal %d out of range", dev);
        return MHC_ERR_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr)
            return cuda_status(e != cudaSuccess ? e : cudaErrorInvalidSymbol,
                               "mhc_backward_noalloc: cudaGetSymbolAddress of the scratch array");
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return MHC_OK;
}

}  // namespace
}  // namespace mhc

extern "C" mhc_status mhc_backward_noalloc(const void* X, const void* F_out, const void* phi, mhc_dtype dt,
                                           const float* alpha, const float* b, const void* dX_next,
                                           const void* dx_in, int64_t T, int n, int C, int t_iters,
                                           float eps, void* dX, void* dF_out, float* dphi, float* dalpha,
                                           float* db, void* stream)
{
    using namespace mhc;
    const size_t need = mhc_backward_workspace_bytes(T, n, C);
    if (T > 0 && (need == 0 || need > size_t(MHC_NOALLOC_SCRATCH_BYTES))) {
        set_error("mhc_backward_noalloc: T=%lld, n=%d needs %zu bytes of scratch; the built-in "
                  "scratch holds %zu (use mhc_backward with a workspace for larger batches)",
                  (long long)T, n, need, size_t(MHC_NOALLOC_SCRATCH_BYTES));
        return MHC_ERR_UNSUPPORTED;
    }
    void* scratch = nullptr;
    if (T > 0) {
        const mhc_status st = noalloc_scratch(&scratch);
        if (st != MHC_OK) return st;
    }
    return mhc_backward(X, F_out, phi, dt, alpha, b, dX_next, dx_in, T, n, C, t_iters, eps, dX, dF_out,
                        dphi, dalpha, db, scratch, T > 0 ? size_t(MHC_NOALLOC_SCRATCH_BYTES) : 0, stream);
}
