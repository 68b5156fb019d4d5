// One launcher of the selective-scan kernel: compiled once per
// (SS_INST_TIN, SS_INST_TOUT, SS_INST_NMAX) with SS_INST_NAME as its name.
#include "ss_launch.h"

#if !defined(SS_INST_TIN) || !defined(SS_INST_TOUT) || !defined(SS_INST_NMAX) || !defined(SS_INST_NAME)
#error "compile with -DSS_INST_TIN=... -DSS_INST_TOUT=... -DSS_INST_NMAX=... -DSS_INST_NAME=..."
#endif

namespace selscan {

namespace {

constexpr int kMaxDevices = 64;

// Launch one instance; above the 48 KB default the kernel must opt in to
// more dynamic shared memory, once per device.
template <int kW>
auto kernel_for() {
    if constexpr (kW == 1) return ss_fwd_direct_kernel<SS_INST_TIN, SS_INST_TOUT, SS_INST_NMAX>;
    else return ss_fwd_kernel<SS_INST_TIN, SS_INST_TOUT, SS_INST_NMAX, kW>;
}

template <int kW>
cudaError_t launch_one(dim3 grid, dim3 block, size_t smem, cudaStream_t s, const FwdParams &p) {
    auto kernel = kernel_for<kW>();
    if (smem > 48 * 1024) {
        static bool opted_in[kMaxDevices];
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= kMaxDevices || !opted_in[dev]) {
            e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kMaxSmemBytes);
            if (e != cudaSuccess) return e;
            if (dev >= 0 && dev < kMaxDevices) opted_in[dev] = true;
        }
    }
    kernel<<<grid, block, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t SS_INST_NAME(int lanes, dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                         const FwdParams &p) {
    switch (lanes) {
        case 1: return launch_one<1>(grid, block, smem, s, p);
        case 2: return launch_one<2>(grid, block, smem, s, p);
        case 4: return launch_one<4>(grid, block, smem, s, p);
        case 8: return launch_one<8>(grid, block, smem, s, p);
        case 16: return launch_one<16>(grid, block, smem, s, p);
        case 32: return launch_one<32>(grid, block, smem, s, p);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace selscan
