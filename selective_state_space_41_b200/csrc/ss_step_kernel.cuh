// Single-step recurrent decoding: one step of the selective scan from a
// given state, the state updated in place.
//
// The recurrence is the sequential loop of the selective_scan_ref walkthrough
// ("Mamba代码实战：手把手教你用PyTorch复现选择性扫描核心逻辑（附避坑指南）", §2.2-§3.3)
// taken for one step l: delta' = softplus/exp(delta + bias),
// h_n <- exp(delta' A_n) h_n + delta' B_n u, y = sum_n C_n h_n + D u, times
// silu(z).  Decoding advances it one token at a time (the single-step use
// "告别‘炼丹’：从Mamba-minimal入手..." describes in §2.1), so the work per call
// is one read and one write of the (B, D, N) state: bound by memory and
// launch latency, not by the SFU.
//
// Thread mapping: T = (state bucket)/2 threads per row (b, d), each holding
// one state pair; the row's y is summed over its T threads by shuffles.
#pragma once

#include "ss_fwd_kernel.cuh"

namespace selscan {

struct StepParams {
    const void *u, *delta, *B, *C, *z;   // u, delta, z: (batch, dim); B, C: (batch, dstate)
    const float *A, *D, *delta_bias;
    float *state;                        // (batch, dim, dstate), read and written
    void *y;                             // (batch, dim)
    int64_t batch, dim;
    int dstate;
    int softplus;
};

template <typename Tin>
__device__ __forceinline__ float load_in(const void *p, int64_t i) {
    return static_cast<float>(static_cast<const Tin *>(p)[i]);
}

// kT threads per row (1..32, a power of two), 256 threads per block.
template <typename Tin, typename Tout, int kT>
__global__ void __launch_bounds__(256) ss_step_kernel(const StepParams p) {
    constexpr bool kFast = sizeof(Tin) == 2;
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t rows = p.batch * p.dim;
    const int64_t row = t / kT;                 // whole warps share rows (kT divides 32)
    const int q = (int)(t % kT);                // this thread's state pair
    const bool row_ok = row < rows;
    const int64_t rr = row_ok ? row : rows - 1;
    const int64_t b = rr / p.dim, d = rr % p.dim;
    const int N = p.dstate;

    const float x = load_in<Tin>(p.delta, rr) + (p.delta_bias ? p.delta_bias[d] : 0.f);
    const float dl = delta_transform<kFast>(x, p.softplus != 0);
    const float uv = load_in<Tin>(p.u, rr);
    const float du = dl * uv;
    float part = 0.f;
    const int n = 2 * q;
    for (int e = 0; e < 2; ++e) {
        const int m = n + e;
        if (m < N && row_ok) {
            const float a = sfu_exp2(dl * (p.A[d * N + m] * kLog2e));
            float *hp = p.state + rr * N + m;
            const float h = fmaf(a, *hp, du * load_in<Tin>(p.B, b * N + m));
            *hp = h;
            part = fmaf(load_in<Tin>(p.C, b * N + m), h, part);
        }
    }
#pragma unroll
    for (int off = kT / 2; off >= 1; off /= 2) part += __shfl_xor_sync(0xffffffffu, part, off, kT);
    if (row_ok && q == 0) {
        float yv = p.D ? fmaf(p.D[d], uv, part) : part;
        if (p.z) yv *= silu<kFast>(load_in<Tin>(p.z, rr));
        static_cast<Tout *>(p.y)[rr] = static_cast<Tout>(yv);
    }
}

}  // namespace selscan
