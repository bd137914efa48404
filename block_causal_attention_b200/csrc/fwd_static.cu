// bca_fwd_static_workspace: the forward with its scratch (the K-hat / V tile images
// that bca_fwd keeps in the caller's workspace) in a file-scope device array, for
// callers that may not allocate device memory.  It launches the same kernels as
// bca_fwd, through the same launcher, with the array as the workspace.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "kernels.hpp"
#include "plan.hpp"

namespace {

// The scratch.  In host code `g_static_ws` is only a host-side stand-in for the
// symbol, never a device address: the device address is looked up per device with
// cudaGetSymbolAddress below and passed to the kernels.
static __device__ __align__(256) uint8_t g_static_ws[BCA_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_ws_addr[kMaxDevices] = {};

// Device address of g_static_ws on the current device (looked up once per device).
int static_ws_address(int dev, void **out) {
    if (dev < 0 || dev >= kMaxDevices) return BCA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_ws_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || !p) return BCA_ERR_CUDA;
        g_ws_addr[dev] = p;
    }
    *out = g_ws_addr[dev];
    return BCA_OK;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int bca_fwd_static_workspace(bca_plan_t plan, const void *q, const void *k, const void *v,
                                        const void *k_cache, const void *v_cache, const float *q_gain,
                                        const float *k_gain, void *o, float *lse, void *stream) {
    if (!plan) return BCA_ERR_INVALID_ARGUMENT;
    bca::Plan &P = plan->plan;
    if (P.flags & BCA_PLAN_HOST_ONLY) return BCA_ERR_HOST_ONLY_PLAN;
    if (P.profiling) return BCA_ERR_INVALID_ARGUMENT;  // profiling would create CUDA events
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return BCA_ERR_CUDA;
    if (dev != P.device) return BCA_ERR_INVALID_ARGUMENT;
    if (P.nq == 0) return BCA_OK;
    if (bca::fwd_workspace_bytes(P) > (size_t)BCA_STATIC_WORKSPACE_BYTES) return BCA_ERR_TOO_LARGE;
    if (!q || !k || !v || !o || !lse) return BCA_ERR_INVALID_ARGUMENT;
    if (P.nc > 0 && (!k_cache || !v_cache)) return BCA_ERR_INVALID_ARGUMENT;
    if ((P.flags & BCA_NO_PROLOGUE) && (q_gain || k_gain)) return BCA_ERR_INVALID_ARGUMENT;
    const void *ptrs[] = {q, k, v, k_cache, v_cache, q_gain, k_gain, o, lse};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return BCA_ERR_MISALIGNED;
    void *ws = nullptr;
    int rc = static_ws_address(dev, &ws);
    if (rc != BCA_OK) return rc;
    bca::FwdIO io{q, k, v, k_cache, v_cache, q_gain, k_gain, o, lse, ws};
    return bca::launch_fwd(P, io, static_cast<cudaStream_t>(stream));
}
