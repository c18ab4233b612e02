// switch_route_noalloc: the routing step without a caller-supplied workspace.
//
// Some callers cannot allocate device memory when they route tokens: code
// that runs under a host framework which owns every device allocation and
// forbids new ones while it executes (an inference engine's plugin, a
// serving process that reserves all of its device memory at start-up), or a
// caller with no allocator to hand at that point.  For them the scratch that
// switch_route keeps in the workspace (status word, scan ticket, per-tile
// expert counts, per-tile probability sums, tile offsets, probability
// totals) lives here instead, in one file-scope device array that the
// library owns.
//
// The array is part of this library's device image: every GPU on which the
// library is used holds kNoAllocScratchBytes for it until the process exits.
// Host code never dereferences its name (on the host it only stands in for
// the symbol); its device address is looked up with cudaGetSymbolAddress on
// every call, with the calling device current, and passed to the kernels like
// any workspace pointer.
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace switchmoe {
namespace {

constexpr size_t kNoAllocScratchBytes = SWITCH_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_route_scratch[kNoAllocScratchBytes];

// Device address of the scratch array in the current device's context.  It
// is looked up on every call (cudaGetSymbolAddress allocates nothing and
// costs a few microseconds) rather than cached per device ordinal: a cached
// address would go stale if the caller reset the device or released and
// re-created its primary context, and the next call would then write through
// a dangling device pointer.
cudaError_t scratch_on_current_device(void **out) {
    void *p = nullptr;
    const cudaError_t err = cudaGetSymbolAddress(&p, g_route_scratch);
    if (err != cudaSuccess) return err;
    *out = p;
    return cudaSuccess;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace switchmoe

using namespace switchmoe;

extern "C" switch_status_t switch_route_noalloc(const switch_dims_t *dims, const void *x, const float *w_r,
                                                const float *logit_bias, int32_t *expert, float *gate,
                                                int32_t *slot, int32_t *counts, int32_t *slot_token, float *aux,
                                                switch_stream_t stream) {
    size_t full = 0;
    switch_status_t s = switch_workspace_size(dims, &full);  // validates dims
    if (s != SWITCH_OK) return s;
    const bool has_tokens = dims->T > 0;
    const void *required[] = {w_r, counts, slot_token, aux, has_tokens ? x : w_r,
                              has_tokens ? (const void *)expert : w_r, has_tokens ? (const void *)gate : w_r,
                              has_tokens ? (const void *)slot : w_r};
    for (const void *p : required)
        if (!p) return SWITCH_ERR_NULL;
    for (const void *p : required)
        if (!aligned16(p)) return SWITCH_ERR_ALIGN;
    for (const void *p : {(const void *)logit_bias, x, (const void *)expert, (const void *)gate, (const void *)slot})
        if (p && !aligned16(p)) return SWITCH_ERR_ALIGN;
    if (route_scratch_bytes(*dims) > kNoAllocScratchBytes) return SWITCH_ERR_TOO_LARGE;

    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return SWITCH_ERR_CUDA;
    if (major != 10) return SWITCH_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    if (scratch_on_current_device(&scratch) != cudaSuccess) return SWITCH_ERR_CUDA;

    // Only the routing sections of the workspace layout are carved; they all
    // lie inside the first route_scratch_bytes(dims) bytes.  The router's
    // first block clears the ticket and the status word, and every other
    // section is fully rewritten by the call, so the previous call's
    // contents never leak into this one.
    // The training and statistics flags would make the routers also write the
    // [T][N] probabilities or per-tile entropy sums into sections past the
    // routing scratch; routing here keeps neither, so both flags are cleared
    // for the carve and the launch.
    switch_dims_t route_dims = *dims;
    route_dims.flags &= ~(SWITCH_FLAG_TRAINING | SWITCH_FLAG_ROUTER_STATS);
    const Workspace ws = carve_workspace(route_dims, scratch);
    const cudaError_t err = launch_route(route_dims, x, w_r, logit_bias, expert, gate, slot, counts, slot_token, aux,
                                         ws, reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? SWITCH_OK : SWITCH_ERR_CUDA;
}

extern "C" switch_status_t switch_check_noalloc(switch_stream_t stream) {
    void *scratch = nullptr;
    if (scratch_on_current_device(&scratch) != cudaSuccess) return SWITCH_ERR_CUDA;
    return switch_check(scratch, kNoAllocScratchBytes, stream);
}

extern "C" switch_status_t switch_selftest_wait_timeout_noalloc(switch_stream_t stream) {
    void *scratch = nullptr;
    if (scratch_on_current_device(&scratch) != cudaSuccess) return SWITCH_ERR_CUDA;
    return switch_selftest_wait_timeout(scratch, kNoAllocScratchBytes, stream);
}
