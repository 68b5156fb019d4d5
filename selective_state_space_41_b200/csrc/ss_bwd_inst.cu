// One launcher of the selective-scan backward kernel: compiled once per
// (SS_INST_TIN, SS_INST_TOUT, SS_INST_NMAX) with SS_INST_NAME as its name.
#include "ss_bwd_launch.h"

#if !defined(SS_INST_TIN) || !defined(SS_INST_TOUT) || !defined(SS_INST_NMAX) || !defined(SS_INST_NAME)
#error "compile with -DSS_INST_TIN=... -DSS_INST_TOUT=... -DSS_INST_NMAX=... -DSS_INST_NAME=..."
#endif

namespace selscan {

namespace {

template <bool kReset, bool kZ = true>
cudaError_t launch(dim3 grid, dim3 block, size_t smem, cudaStream_t s, const BwdParams &p) {
    constexpr int kMaxDevices = 64;
    static bool opted_in[kMaxDevices];
    auto kernel = ss_bwd_kernel<SS_INST_TIN, SS_INST_TOUT, SS_INST_NMAX, kReset, kZ>;
    if (smem > 48 * 1024) {  // above the default a kernel opts in to more dynamic shared memory, once per device
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= kMaxDevices || !opted_in[dev]) {
            e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMaxSmemBytes);
            if (e != cudaSuccess) return e;
            if (dev >= 0 && dev < kMaxDevices) opted_in[dev] = true;
        }
    }
    kernel<<<grid, block, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

// The instance that reads sequence starts when p.reset is given; without
// them, the one without the gate's sums when there is no z.
cudaError_t SS_INST_NAME(dim3 grid, dim3 block, size_t smem, cudaStream_t s, const BwdParams &p) {
    if (p.reset) return launch<true>(grid, block, smem, s, p);
    return p.z ? launch<false>(grid, block, smem, s, p) : launch<false, false>(grid, block, smem, s, p);
}

}  // namespace selscan
