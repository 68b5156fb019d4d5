// One launcher of the selective-scan kernel: compiled once per
// (SS_INST_TIN, SS_INST_TOUT, SS_INST_NMAX) with SS_INST_NAME as its name.
#include <type_traits>

#include "ss_launch.h"

#if !defined(SS_INST_TIN) || !defined(SS_INST_TOUT) || !defined(SS_INST_NMAX) || !defined(SS_INST_NAME)
#error "compile with -DSS_INST_TIN=... -DSS_INST_TOUT=... -DSS_INST_NMAX=... -DSS_INST_NAME=..."
#endif

namespace selscan {

namespace {

constexpr int kMaxDevices = 64;

// Launch one kernel instance; above the 48 KB default a kernel must opt in
// to more dynamic shared memory, once per device.
template <typename Kernel>
cudaError_t launch_kernel(Kernel kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                          const FwdParams &p, bool (&opted_in)[kMaxDevices]) {
    if (smem > 48 * 1024) {
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

template <int kW>
cudaError_t launch_scan(dim3 grid, dim3 block, size_t smem, cudaStream_t s, const FwdParams &p) {
    static bool opted_in[kMaxDevices];
    return launch_kernel(ss_fwd_kernel<SS_INST_TIN, SS_INST_TOUT, SS_INST_NMAX, kW>, grid, block, smem,
                         s, p, opted_in);
}

template <int kG>
cudaError_t launch_direct(dim3 grid, dim3 block, size_t smem, cudaStream_t s, const FwdParams &p) {
    if constexpr (SS_INST_NMAX / 2 / kG < 1) {
        return cudaErrorInvalidValue;  // fewer state pairs than lanes
    } else {
        if (p.delta_r) {  // the dt_proj form: bf16, 2 or 4 lanes, double-buffered stages
            if constexpr (std::is_same<SS_INST_TIN, __nv_bfloat16>::value && (kG == 2 || kG == 4) &&
                          direct_double_buffer(SS_INST_NMAX, kG)) {
                static bool opted_in_dt[kMaxDevices];
                return launch_kernel(ss_fwd_direct_kernel<SS_INST_TIN, SS_INST_TOUT, SS_INST_NMAX, kG, false, true>,
                                     grid, block, smem, s, p, opted_in_dt);
            } else {
                return cudaErrorInvalidValue;
            }
        }
        if (p.ckpt) {  // the instances that write the backward's checkpoints
            if (p.reset) {
                static bool opted_in_ck_reset[kMaxDevices];
                return launch_kernel(ss_fwd_direct_kernel<SS_INST_TIN, SS_INST_TOUT, SS_INST_NMAX, kG, true, false, true>,
                                     grid, block, smem, s, p, opted_in_ck_reset);
            }
            static bool opted_in_ck[kMaxDevices];
            return launch_kernel(ss_fwd_direct_kernel<SS_INST_TIN, SS_INST_TOUT, SS_INST_NMAX, kG, false, false, true>,
                                 grid, block, smem, s, p, opted_in_ck);
        }
        if (p.reset) {  // the instance that reads the sequence starts
            static bool opted_in_reset[kMaxDevices];
            return launch_kernel(ss_fwd_direct_kernel<SS_INST_TIN, SS_INST_TOUT, SS_INST_NMAX, kG, true>,
                                 grid, block, smem, s, p, opted_in_reset);
        }
        static bool opted_in[kMaxDevices];
        return launch_kernel(ss_fwd_direct_kernel<SS_INST_TIN, SS_INST_TOUT, SS_INST_NMAX, kG>, grid,
                             block, smem, s, p, opted_in);
    }
}

template <int kG>
cudaError_t launch_tmem(dim3 grid, dim3 block, size_t smem, cudaStream_t s, const FwdParams &p) {
    if constexpr (!std::is_same<SS_INST_TIN, __nv_bfloat16>::value || !tmem_supported(SS_INST_NMAX, kG)) {
        return cudaErrorInvalidValue;  // bf16 inputs and the splits it is built for only
    } else {
        if (p.reset) return cudaErrorInvalidValue;  // sequence starts: the shared-memory form
        static bool opted_in[kMaxDevices];
        return launch_kernel(ss_fwd_tmem_kernel<SS_INST_TOUT, SS_INST_NMAX, kG>, grid, block, smem, s, p,
                             opted_in);
    }
}

}  // namespace

cudaError_t SS_INST_NAME(int lanes, int split_states, dim3 grid, dim3 block, size_t smem,
                         cudaStream_t s, const FwdParams &p) {
    if (split_states == 2) {
        switch (lanes) {
            case 2: return launch_tmem<2>(grid, block, smem, s, p);
            case 4: return launch_tmem<4>(grid, block, smem, s, p);
            case 8: return launch_tmem<8>(grid, block, smem, s, p);
            default: return cudaErrorInvalidValue;
        }
    }
    if (lanes == 1 || split_states) {
        switch (lanes) {
            case 1: return launch_direct<1>(grid, block, smem, s, p);
            case 2: return launch_direct<2>(grid, block, smem, s, p);
            case 4: return launch_direct<4>(grid, block, smem, s, p);
            case 8: return launch_direct<8>(grid, block, smem, s, p);
            default: return cudaErrorInvalidValue;
        }
    }
    if (p.reset) return cudaErrorInvalidValue;  // the scan kernel does not read sequence starts
    switch (lanes) {
        case 2: return launch_scan<2>(grid, block, smem, s, p);
        case 4: return launch_scan<4>(grid, block, smem, s, p);
        case 8: return launch_scan<8>(grid, block, smem, s, p);
        case 16: return launch_scan<16>(grid, block, smem, s, p);
        case 32: return launch_scan<32>(grid, block, smem, s, p);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace selscan
