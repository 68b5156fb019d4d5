// One launcher of the selective-scan kernel: compiled once per
// (SS_INST_TIN, SS_INST_TOUT, SS_INST_NMAX) with SS_INST_NAME as its name.
#include "ss_launch.h"

#if !defined(SS_INST_TIN) || !defined(SS_INST_TOUT) || !defined(SS_INST_NMAX) || !defined(SS_INST_NAME)
#error "compile with -DSS_INST_TIN=... -DSS_INST_TOUT=... -DSS_INST_NMAX=... -DSS_INST_NAME=..."
#endif

namespace selscan {

cudaError_t SS_INST_NAME(int lanes, dim3 grid, dim3 block, cudaStream_t s, const FwdParams &p) {
    using Tin = SS_INST_TIN;
    using Tout = SS_INST_TOUT;
    constexpr int kN = SS_INST_NMAX;
    switch (lanes) {
        case 1: ss_fwd_kernel<Tin, Tout, kN, 1><<<grid, block, 0, s>>>(p); break;
        case 2: ss_fwd_kernel<Tin, Tout, kN, 2><<<grid, block, 0, s>>>(p); break;
        case 4: ss_fwd_kernel<Tin, Tout, kN, 4><<<grid, block, 0, s>>>(p); break;
        case 8: ss_fwd_kernel<Tin, Tout, kN, 8><<<grid, block, 0, s>>>(p); break;
        case 16: ss_fwd_kernel<Tin, Tout, kN, 16><<<grid, block, 0, s>>>(p); break;
        case 32: ss_fwd_kernel<Tin, Tout, kN, 32><<<grid, block, 0, s>>>(p); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace selscan
