// ss_fwd_noalloc: the selective-scan forward with its scratch in a static
// device array instead of caller memory (declaration and contract in
// include/selscan.h).
//
// Who needs it: a caller that may not allocate device memory at call time --
// code that runs under a memory budget it does not own, inside another
// library's allocator or a plugin host that hands out no device memory, or
// on a path where cudaMalloc / cudaFree are off limits because they
// synchronise the whole device.  The sequence-segmented launch shape needs
// scratch for the segments' end states, so without this entry such a caller
// would be left with the slower unsegmented shapes of ss_fwd.
//
// The scratch is this file's module-scope array.  Its device address is
// looked up once per device, under a lock, by the first call made with that
// device current (so that first call should not be made while a stream is
// being captured); later calls reuse the cached address and make no CUDA
// runtime call beyond the launches of ss_fwd_ws.  The cache is not refreshed:
// after cudaDeviceReset the cached address of that device is stale, and the
// header tells callers not to use this entry on that device again.  Nothing in the array has to
// start at zero: every word the kernels read in a call was first written by
// the segment kernel of that same call (end states and delta' sums of each
// segment), and the fix-up kernel starts its carried state at zero in
// registers.  One array serves every call on a device, so two calls whose
// kernels overlap on the GPU (different streams, or different host threads)
// race on it.

#include <cuda_runtime.h>

#include <mutex>

#include "selscan.h"

namespace {

constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[SS_NOALLOC_SCRATCH_BYTES];

// The device address of g_scratch on the current device; SS_ERR_CUDA if the
// runtime cannot give it.
ss_status scratch_for_current_device(void **out) {
    static std::mutex mu;
    static void *addr[kMaxDevices];
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SS_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return SS_ERR_CUDA;
        addr[dev] = p;
    }
    *out = addr[dev];
    return SS_OK;
}

}  // namespace

extern "C" ss_status ss_fwd_noalloc(const ss_desc *desc, const void *u, const void *delta,
                                    const float *A, const void *B, const void *C, const float *D,
                                    const void *z, const float *delta_bias, int delta_softplus,
                                    void *y, float *last_state, ss_stream_t stream) {
    ss_launch_config shape;
    const ss_status valid = ss_fwd_heuristic(desc, 0, &shape);  // the descriptor's own errors first
    if (valid != SS_OK) return valid;
    // Scratch of the launch shape ss_fwd_ws picks when given all the
    // workspace it can use (0 for a shape without segments).
    const size_t need = ss_fwd_workspace_bytes(desc, nullptr);
    if (need > (size_t)SS_NOALLOC_SCRATCH_BYTES) return SS_ERR_SCRATCH_LIMIT;
    void *scratch = nullptr;
    const ss_status st = scratch_for_current_device(&scratch);
    if (st != SS_OK) return st;
    return ss_fwd_ws(desc, u, delta, A, B, C, D, z, delta_bias, delta_softplus, y, last_state,
                     scratch, need > 0 ? (size_t)SS_NOALLOC_SCRATCH_BYTES : 0, stream);
}
