// Internal: one launcher per (input dtype, output dtype, state bucket).  Each
// is defined in its own translation unit (ss_fwd_inst.cu compiled with
// SS_INST_* defines) so the kernel instances compile in parallel.
#pragma once

#include <cuda_runtime.h>

#include "ss_fwd_kernel.cuh"
#include "ss_fwd_tmem.cuh"

namespace selscan {

// lanes: lanes per row; split_states: the lanes split the row's states (direct
// kernel, 1/2/4 lanes; 2: its TMEM-fed form, bf16 inputs) rather than its
// steps (scan kernel, 2..32 lanes); one lane is the direct kernel either way.
#define SS_DECLARE_LAUNCHER(NAME)                                                            \
    cudaError_t NAME(int lanes, int split_states, dim3 grid, dim3 block, size_t smem, cudaStream_t s, \
                     const FwdParams &p);

#define SS_FOR_EACH_NBUCKET(X, PREFIX) X(PREFIX##_n4) X(PREFIX##_n8) X(PREFIX##_n16) X(PREFIX##_n32) X(PREFIX##_n64)

SS_FOR_EACH_NBUCKET(SS_DECLARE_LAUNCHER, launch_f32_f32)
SS_FOR_EACH_NBUCKET(SS_DECLARE_LAUNCHER, launch_bf16_bf16)
SS_FOR_EACH_NBUCKET(SS_DECLARE_LAUNCHER, launch_bf16_f32)

}  // namespace selscan
