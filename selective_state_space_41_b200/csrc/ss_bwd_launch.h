// Internal: one backward launcher per (input dtype, dtype of dy, state
// bucket), each defined in its own translation unit (ss_bwd_inst.cu).
#pragma once

#include <cuda_runtime.h>

#include "ss_bwd_kernel.cuh"

namespace selscan {

#define SS_DECLARE_BWD_LAUNCHER(NAME) \
    cudaError_t NAME(dim3 grid, dim3 block, size_t smem, cudaStream_t s, const BwdParams &p);

#define SS_FOR_EACH_BWD_NBUCKET(X, PREFIX) X(PREFIX##_n4) X(PREFIX##_n8) X(PREFIX##_n16) X(PREFIX##_n32) X(PREFIX##_n64)

SS_FOR_EACH_BWD_NBUCKET(SS_DECLARE_BWD_LAUNCHER, bwd_f32_f32)
SS_FOR_EACH_BWD_NBUCKET(SS_DECLARE_BWD_LAUNCHER, bwd_bf16_bf16)
SS_FOR_EACH_BWD_NBUCKET(SS_DECLARE_BWD_LAUNCHER, bwd_bf16_f32)

}  // namespace selscan
