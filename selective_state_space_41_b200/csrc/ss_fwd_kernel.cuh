// Selective-scan forward kernels for sm_100a: the scan kernel (lanes split a
// row's steps; described here), the direct kernel (lanes split a row's
// states; used whenever the rows fill the GPU; its instances also read
// sequence starts, take delta from the dt_proj product on the tensor cores,
// or write the backward's checkpoints) and the two fix-up kernels of sequence
// segments (the carry fold and the correction of y), each with its own
// description further down.
//
// Computes, per row (b, d) of the (batch, dim) grid and per state n, the
// recurrence of the selective_scan_ref walkthrough ("Mamba代码实战：手把手教你用
// PyTorch复现选择性扫描核心逻辑（附避坑指南）", §2.2, §3.1-§3.3, §6):
//   delta' = softplus(delta + bias) | exp(delta + bias)
//   h_n   <- exp(delta' A[d,n]) h_n + delta' B[b,n,l] u        (h_n = 0 at l = 0)
//   y      = (sum_n C[b,n,l] h_n + D[d] u) * silu(z)
// without materialising the (B, D, L, N) tensors dA and dB that the page's
// reference builds (§3.1): every exp and product lives in registers.
//
// Work mapping.  A warp holds 32/W rows; the W lanes of a row split each
// chunk of W*K consecutive steps, K (8 or 16) steps per lane.  For every
// state n a lane runs its K steps from a zero state, recording the decays a_i
// and inputs b_i, then the W lanes combine their (prod a, h) pairs with a
// shuffle scan under the associative operator
// (a1, h1) . (a2, h2) = (a2 a1, a2 h1 + h2) (the operator of
// "手把手用PyTorch实现Mamba的SSM层" §3.2, for diagonal A).  The scan gives each
// lane its true incoming state; a second pass over the recorded (a_i, b_i)
// yields the states and y.  The state leaving the chunk goes to a per-row
// shared table for the next chunk.  With W = 1 the lane owns its row and runs
// the plain sequential recurrence, the states in registers.
//
// exp(delta' A) is ex2(delta' * (A log2 e)) on the SFU.  Two consecutive steps
// of one state share one packed sm_100 instruction (mul/fma .f32x2) for the
// exponent arguments, delta' u B, the chunk decay product and y; the state
// recurrence itself is sequential and stays scalar.  Every streamed operand
// (u, delta, z, B, C) reaches shared memory by cp.async one chunk ahead; B and
// C, shared by all rows of a batch entry, are converted once per block to fp32.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

#include "ss_tcgen05.cuh"

namespace selscan {

constexpr size_t kMaxSmemBytes = 227 * 1024;  // opt-in dynamic shared memory per block (sm_100)
constexpr float kLog2e = 1.4426950408889634f;

struct FwdParams {
    const void *u, *delta, *B, *C, *z;
    const float *A, *D, *delta_bias;
    void *y;
    float *last_state;
    const float *init_state;  // (batch, dim, dstate) state before step 0, or null (zero)
    // (batch, seqlen) bytes, or null: nonzero at (b, l) means a new sequence
    // starts at step l, so the state entering step l is zero (direct kernel
    // and fix-up only).
    const uint8_t *reset;
    int64_t batch, dim, seqlen;
    int dstate;
    int softplus;     // 1: softplus, 0: exp
    int vec;          // 1: every row of u/delta/z/B/C/y starts 16-byte aligned
    int64_t dtiles;   // row tiles per batch entry
    // Sequence segments (direct kernel only): nseg > 1 runs each segment of
    // seg_len steps from a zero state (the first one from init_state, if
    // given) and records, per (segment, row), the
    // end state (ws_hend, N floats) and the sum of delta' (ws_dsum) for the
    // fix-up kernel, which adds the carried state's share of y.  A segment
    // holding a reset records -1 as its delta' sum: it passes no state on.
    int64_t seg_len;
    int nseg;
    float *ws_hend, *ws_dsum;
    // Device status word (or null): a kernel whose bounded wait ran out
    // writes a nonzero code here (the kernels that use tensor memory).
    int *status;
    // The dt_proj form of delta (delta null, direct kernel, bf16):
    // delta[b, d, l] = sum_r W_dt[d, r] delta_r[b, r, l], delta_r (batch,
    // dt_rank, L) and W_dt (dim, dt_rank) in the input dtype.
    const void *delta_r, *W_dt;
    int dt_rank;
    // Elements between consecutive batch entries of B and C, and of delta_r
    // (direct kernel and fix-up); 0: contiguous, N L and dt_rank L.  The
    // x_proj output form passes B, C and delta_r as row ranges of one
    // (batch, dt_rank + 2 N, L) tensor, so all three step by its batch stride.
    int64_t bc_bstride = 0, dtr_bstride = 0;
    // Checkpoints for the backward (direct kernel; or null): the state
    // entering every step l = 8k, (batch, dim, ceil(L / 8), dstate) fp32 —
    // the state after step l - 1, before any sequence start at l zeroes it.
    // With sequence segments the fix-up adds the carried state's share to
    // the checkpoints of segments >= 1, as to y.
    float *ckpt;
};

// Steps between two checkpoints of the state (the backward's sub-chunk).
constexpr int kCkptStride = 8;

// ------------------------------------------------------------ element I/O
template <typename T>
struct Io;

template <>
struct Io<float> {
    static constexpr int kUnit = 4;  // elements per 16-byte unit
    __device__ __forceinline__ static float widen(const uint32_t *w, int i) { return __uint_as_float(w[i]); }
    __device__ __forceinline__ static uint32_t bits(const float *p, int64_t i) { return __float_as_uint(p[i]); }
};

template <>
struct Io<__nv_bfloat16> {
    static constexpr int kUnit = 8;  // two bf16 per 32-bit word, element 2j in the low half
    __device__ __forceinline__ static float widen(const uint32_t *w, int i) {
        return __uint_as_float((i & 1) ? (w[i >> 1] & 0xffff0000u) : (w[i >> 1] << 16));
    }
    __device__ __forceinline__ static uint32_t bits(const __nv_bfloat16 *p, int64_t i) {
        return reinterpret_cast<const unsigned short *>(p)[i];
    }
};

// Stores of y for steps [l0, l0 + K): streaming vector stores (16, 8 or 4
// bytes) when the run is complete and aligned, else element stores guarded
// by L.
template <int K>
__device__ __forceinline__ void store_run(float *row, int64_t l0, int64_t L, bool vec, const float (&v)[K]) {
    if (vec && l0 + K <= L) {
        if constexpr (K % 4 == 0) {
            float4 *p = reinterpret_cast<float4 *>(row + l0);
#pragma unroll
            for (int j = 0; j < K / 4; ++j) __stcs(p + j, make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
        } else if constexpr (K == 2) {
            __stcs(reinterpret_cast<float2 *>(row + l0), make_float2(v[0], v[1]));
        } else {
#pragma unroll
            for (int i = 0; i < K; ++i) row[l0 + i] = v[i];
        }
    } else {
#pragma unroll
        for (int i = 0; i < K; ++i)
            if (l0 + i < L) row[l0 + i] = v[i];
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

template <int K>
__device__ __forceinline__ void store_run(__nv_bfloat16 *row, int64_t l0, int64_t L, bool vec,
                                          const float (&v)[K]) {
    if (vec && l0 + K <= L) {
        if constexpr (K % 8 == 0) {
            uint4 *p = reinterpret_cast<uint4 *>(row + l0);
#pragma unroll
            for (int j = 0; j < K / 8; ++j) {
                uint4 q;
                q.x = pack_bf16x2(v[8 * j + 0], v[8 * j + 1]);
                q.y = pack_bf16x2(v[8 * j + 2], v[8 * j + 3]);
                q.z = pack_bf16x2(v[8 * j + 4], v[8 * j + 5]);
                q.w = pack_bf16x2(v[8 * j + 6], v[8 * j + 7]);
                __stcs(p + j, q);
            }
        } else if constexpr (K == 4) {
            __stcs(reinterpret_cast<uint2 *>(row + l0),
                   make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3])));
        } else if constexpr (K == 2) {
            __stcs(reinterpret_cast<unsigned int *>(row + l0), pack_bf16x2(v[0], v[1]));
        } else {
#pragma unroll
            for (int i = 0; i < K; ++i) row[l0 + i] = __float2bfloat16_rn(v[i]);
        }
    } else {
#pragma unroll
        for (int i = 0; i < K; ++i)
            if (l0 + i < L) row[l0 + i] = __float2bfloat16_rn(v[i]);
    }
}

// 2^x on the SFU (MUFU.EX2), flushing subnormal results to zero.
__device__ __forceinline__ float sfu_exp2(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}


// 1/x on the SFU (MUFU.RCP).
__device__ __forceinline__ float sfu_rcp(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}


// log1p(t) / t for t in [0, 1]: the degree-7 polynomial through that
// function's values at the 8 Chebyshev nodes of [0, 1] (Chebyshev
// interpolation, within a small factor of the minimax error: 2.2e-7 relative
// with exact coefficients, 2.8e-7 with these fp32 ones evaluated in fp32 by
// Horner's rule), the coefficients as immediates of the FMAs.
__device__ __forceinline__ float log1p_over_t(float t) {
    float q = fmaf(-0.00837115291506052f, t, 0.04349390044808388f);
    q = fmaf(q, t, -0.1068500280380249f);
    q = fmaf(q, t, 0.1768747717142105f);
    q = fmaf(q, t, -0.24474774301052094f);
    q = fmaf(q, t, 0.3327192962169647f);
    q = fmaf(q, t, -0.49997174739837646f);
    return fmaf(q, t, 0.9999997615814209f);
}

// delta' of §2.2: torch's softplus (beta 1, linear above 20) or exp.
// kFast (bf16 inputs, whose values carry 2^-9 relative rounding):
//   softplus(x) = max(x, 0) + log1p(t), t = exp(-|x|) = 2^(-|x| log2 e) in
//   (0, 1] on the SFU (one MUFU op), log1p(t) = t P(t) with the polynomial
//   above on the FMA pipe.  Above 20, t P(t) < 2.1e-9 is below half an ulp
//   of x, so the sum is exactly x: torch's linear region.  Relative error
//   below 2e-6 (the fp32 rounding of the exp argument dominates at large |x|).
// Otherwise (fp32 inputs): libm-accurate log1pf(expf(x)) and expf(x).
template <bool kFast>
__device__ __forceinline__ float delta_transform(float x, bool softplus) {
    if constexpr (kFast) {
        if (!softplus) return sfu_exp2(x * kLog2e);
        const float t = sfu_exp2(-fabsf(x) * kLog2e);
        return fmaxf(x, 0.f) + t * log1p_over_t(t);
    } else {
        if (softplus) return x > 20.f ? x : log1pf(expf(x));
        return expf(x);
    }
}

// silu(z) = z * sigmoid(z) = z / (1 + exp(-z)) (§3.3).  kFast: exp and the
// reciprocal on the SFU (relative error about 1e-6); otherwise libm expf and
// an IEEE division.
template <bool kFast>
__device__ __forceinline__ float silu(float z) {
    if constexpr (kFast) return z * sfu_rcp(1.f + sfu_exp2(-z * kLog2e));
    else return z / (1.f + expf(-z));
}

// ------------------------------------------------------------ async copies
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_addr(smem_dst)),
                 "l"(gmem_src));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::); }
// Wait until at most one (the most recent) committed group is still in flight.
__device__ __forceinline__ void cp_async_wait_one() { asm volatile("cp.async.wait_group 1;\n" ::); }

// One stage of the inclusive scan of (P, h) pairs over the W lanes of a row,
// under (P1, h1) . (P2, h2) = (P2 P1, P2 h1 + h2): take the pair `off` lanes
// up and fold it in.  shfl.up's predicate is false exactly for the lanes with
// no partner `off` lanes up inside the W-lane segment; those keep their pair.
template <int kW>
__device__ __forceinline__ void scan_stage(float &P, float &h, int off) {
    constexpr int kSeg = (32 - kW) << 8;  // segment mask of width W, clamp 0
    asm("{\n\t.reg .pred p;\n\t.reg .f32 pu, hu;\n\t"
        "shfl.sync.up.b32 pu|p, %0, %2, %3, -1;\n\t"
        "shfl.sync.up.b32 hu, %1, %2, %3, -1;\n\t"
        "@p fma.rn.f32 %1, %0, hu, %1;\n\t"
        "@p mul.rn.f32 %0, %0, pu;\n\t}"
        : "+f"(P), "+f"(h)
        : "r"(off), "n"(kSeg));
}

// The same stage for two independent (P, h) pairs (two states), so that the
// four shuffles are in flight together.
template <int kW>
__device__ __forceinline__ void scan_stage2(float &P0, float &h0, float &P1, float &h1, int off) {
    constexpr int kSeg = (32 - kW) << 8;
    asm("{\n\t.reg .pred p;\n\t.reg .f32 pu, hu, pv, hv;\n\t"
        "shfl.sync.up.b32 pu|p, %0, %4, %5, -1;\n\t"
        "shfl.sync.up.b32 hu, %1, %4, %5, -1;\n\t"
        "shfl.sync.up.b32 pv, %2, %4, %5, -1;\n\t"
        "shfl.sync.up.b32 hv, %3, %4, %5, -1;\n\t"
        "@p fma.rn.f32 %1, %0, hu, %1;\n\t"
        "@p mul.rn.f32 %0, %0, pu;\n\t"
        "@p fma.rn.f32 %3, %2, hv, %3;\n\t"
        "@p mul.rn.f32 %2, %2, pv;\n\t}"
        : "+f"(P0), "+f"(h0), "+f"(P1), "+f"(h1)
        : "r"(off), "n"(kSeg));
}

// Store v to a shared-memory float2 only on the lanes where `pred` holds,
// without a branch.
__device__ __forceinline__ void st_shared_f2_if(float *dst, float2 v, bool pred) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %3, 0;\n\t"
                 "@p st.shared.v2.f32 [%0], {%1, %2};\n\t}" ::"r"(smem_addr(dst)),
                 "f"(v.x), "f"(v.y), "r"((unsigned)pred)
                 : "memory");
}

// Store v to a shared float only on the lanes where `pred` holds, without a branch.
__device__ __forceinline__ void st_shared_f1_if(float *dst, float v, bool pred) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %2, 0;\n\t"
                 "@p st.shared.f32 [%0], %1;\n\t}" ::"r"(smem_addr(dst)),
                 "f"(v), "r"((unsigned)pred)
                 : "memory");
}

// ------------------------------------------------------------------- kernel
// Steps per lane per chunk for a lane count W: 8 for W <= 4 (two states per
// iteration of the state loop), 16 for W >= 8 (one state per iteration; the
// scan's cost is spread over twice the steps).
#ifndef SS_K_SMALL_W
#define SS_K_SMALL_W 8
#endif
#ifndef SS_K_LARGE_W
#define SS_K_LARGE_W 16
#endif
__host__ __device__ constexpr int items_for(int w) { return w <= 4 ? SS_K_SMALL_W : SS_K_LARGE_W; }
__host__ __device__ constexpr int chunk_len(int w) { return w * items_for(w); }

// Shared memory of one block, for a chunk of Lc = W K steps, the state bucket
// kNmax (states n >= N are zero rows, so they add nothing) and R rows:
//   F : float4, B and C of the chunk as fp32: float4 number
//       ((t kNmax + n) K/4 + q) W + s holds steps 4q..4q+3 of lane slot s for
//       state n of X = B (t = 0) or C (t = 1).  The W slots of a row read
//       consecutive float4s (no bank conflicts); rows that share a slot read
//       the same address (broadcast).
//   RB: Tin [2][kNmax][Lc], raw B and C in global order (cp.async target).
//   RU: Tin [2 buffers][3 (u, delta, z)][R][Lc], raw streams; within a row,
//       16-byte unit g of lane slot s sits at unit number g W + s, so each
//       lane reads its K steps without bank conflicts.  Double-buffered: the
//       next chunk lands while this one is read.
//   With W > 1: two per-row tables of kNmax + 2 floats (padding spreads the
//       rows over banks): A[d, n] log2(e), and the state entering the chunk.
__host__ __device__ constexpr size_t smem_bytes(size_t in_size, int nmax, int w, int warps) {
    const size_t rows = (size_t)warps * (size_t)(32 / w), lc = (size_t)chunk_len(w);
    return 2 * sizeof(float) * nmax * lc + 2 * in_size * nmax * lc + 6 * in_size * rows * lc +
           (w > 1 ? 2 * sizeof(float) * (size_t)(nmax + 2) * rows : 0);
}

// State bucket (compile-time state count) for a runtime state count.
__host__ __device__ constexpr int state_bucket(int n) {
    return n <= 4 ? 4 : n <= 8 ? 8 : n <= 16 ? 16 : n <= 32 ? 32 : 64;
}

#ifndef SS_MIN_BLOCKS_SMALL_N
#define SS_MIN_BLOCKS_SMALL_N 2
#endif
// Up to 256 threads per block.  For up to 32 states the register budget is
// capped at 128 per thread (two 256-thread blocks per SM); 64 states take up
// to 255.
template <int kNmax>
struct Occupancy {
    static constexpr int kMinBlocks = kNmax <= 32 ? SS_MIN_BLOCKS_SMALL_N : 1;
};

template <typename Tin, typename Tout, int kNmax, int kW>
__global__ void __launch_bounds__(256, Occupancy<kNmax>::kMinBlocks) ss_fwd_kernel(const FwdParams p) {
    static_assert(kW >= 1 && kW <= 32 && (32 % kW) == 0, "lanes per row must divide 32");
    constexpr int kK = items_for(kW);                    // steps per lane per chunk
    static_assert(kK == 8 || kK == 16, "8 or 16 steps per lane");
    constexpr int kJ = kK / 2;                           // step pairs per lane
    constexpr int kRowsPerWarp = 32 / kW;
    constexpr int kChunk = kW * kK;
    constexpr int kUnit = Io<Tin>::kUnit;                // elements per 16-byte unit
    constexpr int kUnitsPerRow = kChunk / kUnit;         // a power of two
    constexpr int kLaneUnits = kK / kUnit;               // 16-byte units per lane per stream
    constexpr int kLaneWords = kK * (int)sizeof(Tin) / 4;
#ifndef SS_SCAN_STATES
#define SS_SCAN_STATES 0
#endif
    constexpr int kS = SS_SCAN_STATES ? SS_SCAN_STATES : ((kW == 1 || kK == 16) ? 1 : 2);  // states per scan iteration
    constexpr bool kFast = sizeof(Tin) == 2;             // bf16 inputs: SFU transforms
    constexpr int kRowStride = kNmax + 2;                // per-row tables (W > 1)
    constexpr unsigned kFull = 0xffffffffu;

    const int tid = threadIdx.x;
    const int nthreads = blockDim.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int seg = lane % kW;  // this lane's slot among the row's W lanes
    const int N = p.dstate;
    const int rows = (nthreads >> 5) * kRowsPerWarp;
    const int rloc = warp * kRowsPerWarp + lane / kW;    // row within the block
    const int64_t b = blockIdx.x / p.dtiles;
    const int64_t d0 = (blockIdx.x % p.dtiles) * rows;
    const int64_t d_raw = d0 + rloc;
    // Rows past the end mirror the last row (valid addresses) and store nothing;
    // they must still run so that every lane takes part in the shuffles.
    const bool row_ok = d_raw < p.dim;
    const int64_t d = row_ok ? d_raw : p.dim - 1;
    const int64_t L = p.seqlen;
    const int64_t row = b * p.dim + d;
    const bool vec = p.vec != 0;
    const bool softplus = p.softplus != 0;
    const bool has_z = p.z != nullptr;

    extern __shared__ float4 smem[];
    float4 *F = smem;                                                       // 2 kNmax kChunk / 4
    Tin *RB = reinterpret_cast<Tin *>(smem + 2 * kNmax * (kChunk / 4));      // [2][kNmax][kChunk]
    Tin *RU = RB + 2 * kNmax * kChunk;                                       // [2][3][rows][kChunk]
    float *sA2 = reinterpret_cast<float *>(RU + 6 * rows * kChunk);          // [rows][kRowStride]
    float *sCarry = sA2 + rows * kRowStride;
    const float *rowA2 = sA2 + rloc * kRowStride;
    float *rowCarry = sCarry + rloc * kRowStride;

    const Tin *Bsrc[2] = {static_cast<const Tin *>(p.B) + b * N * L,
                          static_cast<const Tin *>(p.C) + b * N * L};
    const Tin *Usrc[3] = {static_cast<const Tin *>(p.u), static_cast<const Tin *>(p.delta),
                          static_cast<const Tin *>(p.z)};
    Tout *y_row = static_cast<Tout *>(p.y) + row * L;

    // A[d, n] log2(e) (0 for the padding states) and the state entering the
    // chunk: registers when a lane owns its row (W = 1; A re-read per chunk,
    // an L1 hit, above 16 states), per-row shared tables when W lanes share it.
    constexpr bool kRowInRegs = kW == 1;
    constexpr bool kA2InRegs = kRowInRegs && kNmax <= 16;
    const float *A_d = p.A + d * N;
    float A2[kA2InRegs ? kNmax : 1], carry[kRowInRegs ? kNmax : 1];
    if constexpr (kRowInRegs) {
#pragma unroll
        for (int n = 0; n < kNmax; ++n) {
            if constexpr (kA2InRegs) A2[n] = n < N ? A_d[n] * kLog2e : 0.f;
            carry[n] = (p.init_state != nullptr && n < N) ? p.init_state[row * N + n] : 0.f;
        }
    } else {
        for (int idx = tid; idx < rows * kNmax; idx += nthreads) {
            const int r = idx / kNmax, n = idx % kNmax;
            const int64_t dr = d0 + r < p.dim ? d0 + r : p.dim - 1;
            sA2[r * kRowStride + n] = n < N ? p.A[dr * N + n] * kLog2e : 0.f;
            sCarry[r * kRowStride + n] =
                (p.init_state != nullptr && n < N) ? p.init_state[(b * p.dim + dr) * N + n] : 0.f;
        }
        // (visible after the first __syncthreads of the chunk loop, or the one
        // before the last-state store)
    }
    const float Dd = p.D ? p.D[d] : 0.f;
    const float bias = p.delta_bias ? p.delta_bias[d] : 0.f;

    // Global row of block row r (mirrored past the end).
    auto grow = [&](int r) -> int64_t {
        const int64_t dr = d0 + r < p.dim ? d0 + r : p.dim - 1;
        return b * p.dim + dr;
    };
    // Position, in elements, of chunk step e within a row of RU.
    auto ru_pos = [&](int e) {
        const int s = e / kK, i = e % kK;
        return ((i / kUnit) * kW + s) * kUnit + (i % kUnit);
    };
    const int nstreams = has_z ? 3 : 2;
    auto chunk_async = [&](int64_t c0) { return vec && c0 + kChunk <= L; };
    // Queue the 16-byte copies of chunk c0 into RB and RU[buf].
    auto issue_copies = [&](int64_t c0, int buf) {
        constexpr int kBCUnits = 2 * kNmax * kUnitsPerRow;
        for (int u = tid; u < kBCUnits; u += nthreads) {
            const int j = u % kUnitsPerRow, rowid = u / kUnitsPerRow;
            const int t = rowid / kNmax, n = rowid % kNmax;
            if (n < N)
                cp_async16(RB + (rowid * kChunk + j * kUnit), Bsrc[t] + (int64_t)n * L + c0 + j * kUnit);
        }
        Tin *dst = RU + buf * 3 * rows * kChunk;
        const int uunits = nstreams * rows * kUnitsPerRow;
        for (int u = tid; u < uunits; u += nthreads) {
            const int j = u % kUnitsPerRow, sr = u / kUnitsPerRow;
            const int t = sr / rows, r = sr % rows;
            cp_async16(dst + (t * rows + r) * kChunk + ru_pos(j * kUnit),
                       Usrc[t] + grow(r) * L + c0 + j * kUnit);
        }
        cp_async_commit();
    };
    // B and C of chunk c0 into F as fp32: from RB, or element by element from
    // global memory (partial or unaligned chunk); padding states get zeros.
    auto fill_F = [&](int64_t c0, bool from_RB) {
        constexpr int kBCUnits = 2 * kNmax * kUnitsPerRow;
        for (int u = tid; u < kBCUnits; u += nthreads) {
            const int j = u % kUnitsPerRow, rowid = u / kUnitsPerRow;
            const int t = rowid / kNmax, n = rowid % kNmax;
            float v[kUnit];
            if (n >= N) {
#pragma unroll
                for (int m = 0; m < kUnit; ++m) v[m] = 0.f;
            } else if (from_RB) {
                const uint4 raw = *reinterpret_cast<const uint4 *>(RB + (rowid * kChunk + j * kUnit));
                const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                for (int m = 0; m < kUnit; ++m) v[m] = Io<Tin>::widen(w, m);
            } else {
                const Tin *src = Bsrc[t] + (int64_t)n * L;
#pragma unroll
                for (int m = 0; m < kUnit; ++m) {
                    const int64_t l = c0 + j * kUnit + m;
                    uint32_t bits = 0u;
                    if (l < L) bits = Io<Tin>::bits(src, l);
                    if constexpr (sizeof(Tin) == 2) bits <<= 16;
                    v[m] = __uint_as_float(bits);
                }
            }
#pragma unroll
            for (int m = 0; m < kUnit; m += 4) {
                const int e = j * kUnit + m;  // step within the chunk
                const int s = e / kK, q = (e % kK) / 4;
                F[(rowid * (kK / 4) + q) * kW + s] = make_float4(v[m], v[m + 1], v[m + 2], v[m + 3]);
            }
        }
    };
    // Streams of chunk c0 into RU[buf] element by element (partial or
    // unaligned chunk); steps past L read 0.
    auto fill_RU_scalar = [&](int64_t c0, int buf) {
        Tin *dst = RU + buf * 3 * rows * kChunk;
        const int elems = nstreams * rows * kChunk;
        for (int e = tid; e < elems; e += nthreads) {
            const int i = e % kChunk, sr = e / kChunk;
            const int t = sr / rows, r = sr % rows;
            const int64_t l = c0 + i;
            Tin v;
            if (l < L) v = Usrc[t][grow(r) * L + l];
            else v = Tin(0.f);
            dst[(t * rows + r) * kChunk + ru_pos(i)] = v;
        }
    };
    // This lane's K steps of stream t, as raw words.
    auto lane_words = [&](int buf, int t, uint32_t (&w)[kLaneWords]) {
        const Tin *src = RU + (buf * 3 + t) * rows * kChunk + rloc * kChunk;
#pragma unroll
        for (int g = 0; g < kLaneUnits; ++g) {
            const uint4 x = *reinterpret_cast<const uint4 *>(src + (g * kW + seg) * kUnit);
            w[4 * g] = x.x, w[4 * g + 1] = x.y, w[4 * g + 2] = x.z, w[4 * g + 3] = x.w;
        }
    };
    // B or C of state n for this lane's steps, as step pairs (X[2j], X[2j+1]).
    auto load_pairs = [&](int t, int n, float2 (&X)[kJ]) {
        const float4 *src = F + (t * kNmax + n) * (kK / 4) * kW + seg;
#pragma unroll
        for (int q = 0; q < kK / 4; ++q) {
            const float4 x = src[q * kW];
            X[2 * q] = make_float2(x.x, x.y);
            X[2 * q + 1] = make_float2(x.z, x.w);
        }
    };

    if (L > 0 && chunk_async(0)) issue_copies(0, 0);

    int buf = 0;
    for (int64_t c0 = 0; c0 < L; c0 += kChunk, buf ^= 1) {
        const bool async_here = chunk_async(c0);
        if (async_here) cp_async_wait_all();
        __syncthreads();  // this chunk's copies have landed; every warp is done with F
        fill_F(c0, async_here);
        if (!async_here) fill_RU_scalar(c0, buf);
        __syncthreads();  // F and RU[buf] hold this chunk; RB is free
        if (c0 + kChunk < L && chunk_async(c0 + kChunk)) issue_copies(c0 + kChunk, buf ^ 1);

        const int64_t l0 = c0 + (int64_t)seg * kK;
        // delta' and delta' u per step, as step pairs; y starts at D u (§3.3).
        float2 dlp[kJ], dup[kJ], y[kJ];
        {
            uint32_t wu[kLaneWords], wd[kLaneWords];
            lane_words(buf, 0, wu);
            lane_words(buf, 1, wd);
            float dl[kK];
#pragma unroll
            for (int i = 0; i < kK; ++i) dl[i] = delta_transform<kFast>(Io<Tin>::widen(wd, i) + bias, softplus);
            if (c0 + kChunk > L) {  // steps past L become the identity (a = 1, b = 0)
#pragma unroll
                for (int i = 0; i < kK; ++i)
                    if (l0 + i >= L) dl[i] = 0.f;
            }
#pragma unroll
            for (int j = 0; j < kJ; ++j) {
                const float u0 = Io<Tin>::widen(wu, 2 * j), u1 = Io<Tin>::widen(wu, 2 * j + 1);
                dlp[j] = make_float2(dl[2 * j], dl[2 * j + 1]);
                dup[j] = make_float2(dl[2 * j] * u0, dl[2 * j + 1] * u1);
                y[j] = make_float2(Dd * u0, Dd * u1);
            }
        }

        if constexpr (kW == 1) {
#pragma unroll
            for (int n = 0; n < kNmax; ++n) {
                float A2n;
                if constexpr (kA2InRegs) A2n = A2[n];
                else A2n = n < N ? __ldg(A_d + n) * kLog2e : 0.f;
                const float2 A2d = make_float2(A2n, A2n);
                float2 Bp[kJ], Cp[kJ];
                load_pairs(0, n, Bp);
                load_pairs(1, n, Cp);
                float h = carry[n];
#pragma unroll
                for (int j = 0; j < kJ; ++j) {
                    const float2 t = __fmul2_rn(dlp[j], A2d);
                    const float2 bb = __fmul2_rn(dup[j], Bp[j]);
                    float2 hp;
                    hp.x = fmaf(sfu_exp2(t.x), h, bb.x);
                    hp.y = fmaf(sfu_exp2(t.y), hp.x, bb.y);
                    h = hp.y;
                    y[j] = __ffma2_rn(Cp[j], hp, y[j]);
                }
                carry[n] = h;
            }
        } else {
#pragma unroll 1
            for (int n0 = 0; n0 < kNmax; n0 += kS) {
                float A2s[kS], cin[kS];
#pragma unroll
                for (int s = 0; s < kS; ++s) A2s[s] = rowA2[n0 + s], cin[s] = rowCarry[n0 + s];
                // Pass 1: this lane's steps from a zero state; keep a and delta' u B.
                float2 a[kS][kJ], bb[kS][kJ];
                float h[kS], P[kS];
#pragma unroll
                for (int s = 0; s < kS; ++s) {
                    float2 Bp[kJ];
                    load_pairs(0, n0 + s, Bp);
                    const float2 A2d = make_float2(A2s[s], A2s[s]);
                    float hs = 0.f;
                    float2 Pp = make_float2(1.f, 1.f);
#pragma unroll
                    for (int j = 0; j < kJ; ++j) {
                        const float2 t = __fmul2_rn(dlp[j], A2d);
                        a[s][j] = make_float2(sfu_exp2(t.x), sfu_exp2(t.y));
                        bb[s][j] = __fmul2_rn(dup[j], Bp[j]);
                        hs = fmaf(a[s][j].x, hs, bb[s][j].x);
                        hs = fmaf(a[s][j].y, hs, bb[s][j].y);
                        Pp = __fmul2_rn(Pp, a[s][j]);
                    }
                    h[s] = hs;
                    P[s] = Pp.x * Pp.y;
                }
                // Scan of (P, h) over the row's W lanes.
#pragma unroll
                for (int off = 1; off < kW; off <<= 1) {
                    if constexpr (kS == 2) scan_stage2<kW>(P[0], h[0], P[1], h[1], off);
                    else scan_stage<kW>(P[0], h[0], off);
                }
                // States after this lane's steps; the lane before's is this one's start.
                float hin[kS];
#pragma unroll
                for (int s = 0; s < kS; ++s) {
                    const float X = fmaf(P[s], cin[s], h[s]);
                    const float up = __shfl_up_sync(kFull, X, 1, kW);
                    hin[s] = seg == 0 ? cin[s] : up;
                    st_shared_f1_if(rowCarry + n0 + s, X, seg == kW - 1);
                }
                // Pass 2: the true states and y.
#pragma unroll
                for (int s = 0; s < kS; ++s) {
                    float2 Cp[kJ];
                    load_pairs(1, n0 + s, Cp);
                    float hs = hin[s];
#pragma unroll
                    for (int j = 0; j < kJ; ++j) {
                        float2 hp;
                        hp.x = fmaf(a[s][j].x, hs, bb[s][j].x);
                        hp.y = fmaf(a[s][j].y, hp.x, bb[s][j].y);
                        hs = hp.y;
                        y[j] = __ffma2_rn(Cp[j], hp, y[j]);
                    }
                }
            }
        }

        float yv[kK];
#pragma unroll
        for (int j = 0; j < kJ; ++j) yv[2 * j] = y[j].x, yv[2 * j + 1] = y[j].y;
        if (has_z) {
            uint32_t wz[kLaneWords];
            lane_words(buf, 2, wz);
#pragma unroll
            for (int i = 0; i < kK; ++i) yv[i] *= silu<kFast>(Io<Tin>::widen(wz, i));
        }
        if (row_ok) store_run<kK>(y_row, l0, L, vec, yv);
    }

    if (p.last_state != nullptr) {
        if constexpr (kRowInRegs) {
            if (row_ok) {
#pragma unroll
                for (int n = 0; n < kNmax; ++n)
                    if (n < N) p.last_state[row * N + n] = carry[n];
            }
        } else {
            __syncthreads();  // the row tables are written (also when L == 0)
            if (row_ok)
                for (int n = seg; n < N; n += kW) p.last_state[row * N + n] = rowCarry[n];
        }
    }
}

// ------------------------------------------------------------ direct kernel
// No scan: the G lanes of a row (G = 1, 2, 4 or 8) each own N/G of its states
// and run the plain sequential recurrence of §3.2 over every step, states in
// registers.  Used when there are enough rows to fill the GPU.  Steps are the
// outer loop and state pairs the inner one, so each step has independent
// packed updates per state pair (n, n+1)
//   t = delta' (A_n, A_n+1) log2e,  a = 2^t (two MUFU.EX2),
//   h = a h + delta' u (B_n, B_n+1),  acc += (C_n, C_n+1) h      (f32x2)
// with only h, A and a few per-step values live.
//
// Steps come in sub-chunks of S (8, or 16 when 4 or 8 lanes share a row).
// Lane g of a row computes delta' and delta' u for S/G of them; with G > 1
// the row's lanes all-gather them through a small per-warp shared slab, and
// after the state loop each lane writes its partial sums of y over its states
// for all S steps there and reads back the G partials of its own S/G steps,
// which it finishes (D u, silu(z)) and stores.
//
// B and C (shared by all rows of a batch entry) are staged per block for
// kDirectStage steps: cp.async copies the raw rows into RB ahead of use, and
// the block converts them to fp32 in F (both buffers doubled, so that the
// next stage converts while this one runs: see direct_double_buffer), where
// float4 number
// i (kNmax/2) + q holds (B[2q][i], B[2q+1][i], C[2q][i], C[2q+1][i]); the
// lanes that own the same states read the same address (broadcast).  A stage
// that lies wholly inside the sequence with aligned rows takes a path with no
// bounds checks; the last, partial stage (or unaligned rows) a checked one.
#ifndef SS_DIRECT_MIN_BLOCKS
#define SS_DIRECT_MIN_BLOCKS 2
#endif
constexpr int kDirectStage = 64;  // steps per shared-memory stage

// Steps per register sub-chunk: 16 when 4 or 8 lanes share a row (few states
// per lane, so the per-sub-chunk exchanges and their latency are amortised
// over more steps), 8 otherwise (more states per lane: register pressure).
__host__ __device__ constexpr int direct_sub(int g) { return g >= 4 ? 16 : 8; }
// Floats per row of the gather slab: delta' and delta' u of each step, plus
// 4 to spread the rows over the banks.
__host__ __device__ constexpr int gather_stride(int g) { return 2 * direct_sub(g) + 4; }
// Reduce slab: lane (r, g) writes its sub-chunk's partial sums of y at
// lane * stride, then reads the partials of its own steps from the lanes of
// its row, `vec` floats per access.  Stride and width are chosen so that both
// the writes and the reads of a warp hit distinct banks in each 128-byte
// phase (checked with a model of the 32 four-byte banks).
__host__ __device__ constexpr int reduce_stride(int g) {
    return g <= 1 ? 0 : g == 2 ? 12 : g == 4 ? 20 : 18;
}
__host__ __device__ constexpr int reduce_vec(int g) { return g == 8 ? 2 : 4; }

// B/C stages are double-buffered (one block barrier per stage; the next
// stage's conversion overlaps this one's recurrence) unless a lane holds 16
// states: there the second buffer's shared memory would cost blocks per SM
// (measured: 16 x 4096 x 8192 x 32 layer 6.94 ms double-buffered, 6.24 ms not).
__host__ __device__ constexpr bool direct_double_buffer(int nmax, int g) { return nmax / g != 16; }

// Bytes of F per (step, state pair): fp32 (B_n, B_n+1, C_n, C_n+1) for fp32
// inputs.  For bf16 inputs F is narrower, which cuts the shared-memory
// traffic of the B/C reads, the busiest part of that pipe, at the cost of
// integer widening when read:
//  - a lane with 4 states keeps both bf16 pairs as two 32-bit words (8 bytes),
//    widened by shifts (mamba-130m-shaped layer 221 -> 205 us);
//  - a lane with 8 or more states keeps B as fp32 and only C packed
//    (12 bytes), half the widening: there the integer pipe, not shared
//    memory, was the tighter limit (16 x 4096 x 8192 layers with 32 / 64
//    states 5.74 -> 5.39 / 10.60 -> 10.14 ms, the 100k-step genomic layer
//    2.46 -> 2.40 ms against both packed; 6.24 / 10.98 / 2.40 ms all fp32).
__host__ __device__ constexpr size_t direct_f_bytes(size_t in_size, int nmax, int g) {
    return in_size == 2 ? (nmax / g >= 8 ? 12 : 8) : 16;
}

// B/C stage buffers (F, RB raw), one or two of each, then the slabs.
__host__ __device__ constexpr size_t direct_smem_bytes(size_t in_size, int nmax, int g, int warps) {
    return (direct_double_buffer(nmax, g) ? 2 : 1) *
               (direct_f_bytes(in_size, nmax, g) * (size_t)(nmax / 2) * kDirectStage + 2 * in_size * (size_t)nmax * kDirectStage) +
           (g > 1 ? sizeof(float) * (size_t)warps * ((32 / g) * gather_stride(g) + 32 * reduce_stride(g)) : 0);
}

// The dt_proj form (kDt): delta of the block's rows is one tensor-core
// product per 64-step stage, delta[rows, steps] = W_dt[rows, :] x delta_r[:, steps]
// (bf16 operands, fp32 accumulation in tensor memory), read by each lane for
// its own steps.  Extra shared memory after the slabs (rpad: dt_rank rounded
// up to 16): the A operand (W_dt rows of the 128 TMEM lanes, K-major, rpad/8
// K halves of 128 x 16 bytes), three B operand buffers (delta_r of a stage
// transposed, rpad/8 K halves of 64 x 16 bytes each), two mbarriers and the
// TMEM address; plus 1 KB of alignment slack.
__host__ __device__ constexpr size_t direct_dt_extra_bytes(int rpad) {
    return 1024 + (size_t)rpad * 256 + 3 * (size_t)rpad * 128 + 64;
}
// Largest dt_rank of the dt_proj form.
constexpr int kMaxDtRank = 64;

// kW consecutive floats to / from shared memory as one access (kW in {1, 2, 4}).
template <int kW>
__device__ __forceinline__ void st_vec(float *p, const float *v) {
    if constexpr (kW == 4) *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    else if constexpr (kW == 2) *reinterpret_cast<float2 *>(p) = make_float2(v[0], v[1]);
    else p[0] = v[0];
}
template <int kW>
__device__ __forceinline__ void ld_vec(const float *p, float *v) {
    if constexpr (kW == 4) {
        const float4 x = *reinterpret_cast<const float4 *>(p);
        v[0] = x.x, v[1] = x.y, v[2] = x.z, v[3] = x.w;
    } else if constexpr (kW == 2) {
        const float2 x = *reinterpret_cast<const float2 *>(p);
        v[0] = x.x, v[1] = x.y;
    } else {
        v[0] = p[0];
    }
}

// Load `bytes` (4, 8, 16 or 32) from 16/8/4-byte aligned global memory into words.
template <int kBytes>
__device__ __forceinline__ void ld_words(const void *src, uint32_t *w) {
    if constexpr (kBytes >= 16) {
#pragma unroll
        for (int g = 0; g < kBytes / 16; ++g) {
            const uint4 x = __ldg(reinterpret_cast<const uint4 *>(src) + g);
            w[4 * g] = x.x, w[4 * g + 1] = x.y, w[4 * g + 2] = x.z, w[4 * g + 3] = x.w;
        }
    } else if constexpr (kBytes == 8) {
        const uint2 x = __ldg(reinterpret_cast<const uint2 *>(src));
        w[0] = x.x, w[1] = x.y;
    } else if constexpr (kBytes == 4) {
        w[0] = __ldg(reinterpret_cast<const unsigned int *>(src));
    } else {
        w[0] = __ldg(reinterpret_cast<const unsigned short *>(src));
    }
}

// Register budget: 128 per thread (two 256-thread blocks per SM) while a
// lane holds up to 16 states; lanes holding 32 or more states (wide states,
// few lanes per row) run better with up to 255 registers and fewer warps.
template <int kStatesPerLane>
struct DirectOccupancy {
    static constexpr int kMinBlocks = kStatesPerLane <= 16 ? SS_DIRECT_MIN_BLOCKS : 1;
};

#ifdef SS_DIRECT_MAXNREG
#define SS_DIRECT_BOUNDS(SPL) __maxnreg__(SS_DIRECT_MAXNREG)
#else
#define SS_DIRECT_BOUNDS(SPL) __launch_bounds__(256, DirectOccupancy<SPL>::kMinBlocks)
#endif

// kReset: the instance that reads p.reset (sequence starts inside the rows);
// the other one has no code for it.  kDt: the instance whose delta is the
// dt_proj product (p.delta_r, p.W_dt; 4 warps, bf16, 2 or 4 lanes per row).
// kCkpt: the instance that writes the checkpoints p.ckpt (the others have no
// code for them: the stores cost registers and time in the step loop).
template <typename Tin, typename Tout, int kNmax, int kG, bool kReset = false, bool kDt = false, bool kCkpt = false>
__global__ void SS_DIRECT_BOUNDS(kNmax / kG) ss_fwd_direct_kernel(const FwdParams p) {
    constexpr int kPairs = kNmax / 2;
    constexpr int kPL = kPairs / kG;                        // state pairs per lane
    static_assert(kG == 1 || kG == 2 || kG == 4 || kG == 8, "1, 2, 4 or 8 lanes per row");
    static_assert(kPL >= 1, "at least one state pair per lane");
    constexpr int kDirectSub = direct_sub(kG);              // steps per sub-chunk
    constexpr int kGatherStride = gather_stride(kG);
    constexpr int kOwn = kDirectSub / kG;                   // steps owned per lane per sub-chunk
    constexpr int kOwnBytes = kOwn * (int)sizeof(Tin);
    constexpr int kOwnWords = (kOwnBytes + 3) / 4;
    constexpr int kUnit = Io<Tin>::kUnit;
    constexpr int kStageUnits = kDirectStage / kUnit;       // 16-byte units per (tensor, n) row
    constexpr int kSubs = kDirectStage / kDirectSub;
    constexpr int kRowsPerWarp = 32 / kG;
    constexpr int kAccs = kPL >= 4 ? 2 : 1;                 // y accumulators per step
    constexpr bool kFast = sizeof(Tin) == 2;
    constexpr bool kA2InRegs = kNmax / kG <= 32;
    static_assert(!kDt || (sizeof(Tin) == 2 && (kG == 2 || kG == 4) && !kReset && direct_double_buffer(kNmax, kG)),
                  "dt_proj form: bf16, 2 or 4 lanes per row, double-buffered stages, no sequence starts");

    const int tid = threadIdx.x;
    const int nthreads = blockDim.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int g = lane % kG;                                // state group of this lane
    const int r = lane / kG;                                // row within the warp
    const int rows = nthreads / kG;
    const int N = p.dstate;
    const int64_t blocks_per_seg = p.batch * p.dtiles;
    const int64_t seg = blockIdx.x / blocks_per_seg;
    const int64_t bt = blockIdx.x % blocks_per_seg;
    const int64_t b = bt / p.dtiles;
    const int64_t d_raw = (bt % p.dtiles) * rows + tid / kG;
    const bool row_ok = d_raw < p.dim;
    const int64_t d = row_ok ? d_raw : p.dim - 1;
    const int64_t L = p.seqlen;  // row length (stride)
    const int64_t row = b * p.dim + d;
    const bool vec = p.vec != 0;
    const bool softplus = p.softplus != 0;
    const bool has_z = p.z != nullptr;
    const bool want_y = p.y != nullptr;
    static_assert(direct_sub(kG) % kCkptStride == 0, "checkpoints at sub-chunk steps");
    // This block's steps: [c_begin, Lend) (the whole row unless segmented).
    const int64_t c_begin = seg * p.seg_len;
    const int64_t Lend = c_begin + p.seg_len < L ? c_begin + p.seg_len : L;

    extern __shared__ float4 smem[];
    // Stage buffers, one or two of each: F [kDirectStage][kPairs] float4, RB [2][kNmax][kDirectStage] raw.
    constexpr bool kDB = direct_double_buffer(kNmax, kG);
    constexpr int kNB = kDB ? 2 : 1;
    constexpr bool kPack = direct_f_bytes(sizeof(Tin), kNmax, kG) == 8;      // F as packed bf16 pairs
    constexpr bool kHalf = direct_f_bytes(sizeof(Tin), kNmax, kG) == 12;     // B fp32, C packed
    constexpr int kFUnits = (int)(kDirectStage * kPairs * direct_f_bytes(sizeof(Tin), kNmax, kG) / 16);  // float4 units per F buffer
    float4 *const F0 = smem, *const F1 = smem + (kNB - 1) * kFUnits;
    Tin *const RB0 = reinterpret_cast<Tin *>(smem + kNB * kFUnits);
    Tin *const RB1 = RB0 + (kNB - 1) * 2 * kNmax * kDirectStage;
    float4 *F = F0;                                                     // the stage being computed
    constexpr int kRS = reduce_stride(kG), kRV = reduce_vec(kG);
    float *slab = reinterpret_cast<float *>(RB1 + 2 * kNmax * kDirectStage) +
                  warp * (kRowsPerWarp * kGatherStride + 32 * kRS);
    float *gat = slab + r * kGatherStride;                  // this row: 8 delta', 8 delta' u
    float *red = slab + kRowsPerWarp * kGatherStride;       // per lane: 8 partial sums of y

    const int64_t bc_bstride = p.bc_bstride ? p.bc_bstride : N * L;
    const Tin *Bsrc[2] = {static_cast<const Tin *>(p.B) + b * bc_bstride,
                          static_cast<const Tin *>(p.C) + b * bc_bstride};
    // This lane's first owned step of each stream (advanced per sub-chunk).
    const Tin *u_own = static_cast<const Tin *>(p.u) + row * L + c_begin + g * kOwn;
    const Tin *d_own = kDt ? nullptr : static_cast<const Tin *>(p.delta) + row * L + c_begin + g * kOwn;
    const Tin *z_own = has_z ? static_cast<const Tin *>(p.z) + row * L + c_begin + g * kOwn : nullptr;
    Tout *const y_row = static_cast<Tout *>(p.y) + row * L;
    Tout *y_own = y_row + c_begin + g * kOwn;

    const int q0 = g * kPL;                                 // this lane's first state pair
    // This row's checkpoints (null when none are asked for, or a mirrored row).
    float *const ckpt_row = (kCkpt && row_ok)
                                ? p.ckpt + row * ((L + kCkptStride - 1) / kCkptStride) * N : nullptr;
    // Vector stores of the checkpoints: whole groups of 4 states in the row
    // (N a multiple of 4) and a 16-byte-aligned buffer; a lane's pairs start on
    // an even pair when it holds 2 or more (else one 8-byte pair).
    const bool ckpt_vec = N % 4 == 0 && (reinterpret_cast<uintptr_t>(p.ckpt) & 15u) == 0 && (kPL % 2 == 0 || kPL == 1);
    const float *A_d = p.A + d * N;
    float2 A2[kA2InRegs ? kPL : 1], h[kPL];
#pragma unroll
    for (int qq = 0; qq < kPL; ++qq) {
        const int n = 2 * (q0 + qq);
        if constexpr (kA2InRegs)
            A2[qq] = make_float2(n < N ? A_d[n] * kLog2e : 0.f, n + 1 < N ? A_d[n + 1] * kLog2e : 0.f);
        h[qq] = make_float2(0.f, 0.f);
        if (p.init_state != nullptr && seg == 0) {  // the given state enters the first segment only
            if (n < N) h[qq].x = p.init_state[row * N + n];
            if (n + 1 < N) h[qq].y = p.init_state[row * N + n + 1];
        }
    }
    const float Dd = p.D ? p.D[d] : 0.f;
    const float bias = p.delta_bias ? p.delta_bias[d] : 0.f;
    const uint8_t *const reset_b = kReset ? p.reset + b * L : nullptr;  // this batch entry's starts
    bool seg_reset = false;  // a sequence starts inside this segment

    auto stage_fast = [&](int64_t c0) { return vec && c0 + kDirectStage <= Lend; };
    auto issue_copies = [&](int64_t c0, Tin *RB) {
        for (int u = tid; u < 2 * kNmax * kStageUnits; u += nthreads) {
            const int j = u % kStageUnits, rowid = u / kStageUnits;
            const int t = rowid / kNmax, n = rowid % kNmax;
            if (n < N)
                cp_async16(RB + (rowid * kDirectStage + j * kUnit), Bsrc[t] + (int64_t)n * L + c0 + j * kUnit);
        }
        cp_async_commit();
    };
    // RB (or global memory, element by element) -> Fs: job (q, step block of 8).
    auto fill_F = [&](int64_t c0, bool from_RB, const Tin *RB, float4 *Fs) {
        for (int jb = tid; jb < kPairs * (kDirectStage / 8); jb += nthreads) {
            const int q = jb % kPairs, i0 = (jb / kPairs) * 8;
            float v[4][8];
#pragma unroll
            for (int c = 0; c < 4; ++c) {  // c: B[2q], B[2q+1], C[2q], C[2q+1]
                const int t = c >> 1, n = 2 * q + (c & 1);
                if (n >= N) {
#pragma unroll
                    for (int m = 0; m < 8; ++m) v[c][m] = 0.f;
                } else if (from_RB) {
                    const Tin *src = RB + (t * kNmax + n) * kDirectStage + i0;
#pragma unroll
                    for (int gg = 0; gg < 8 / kUnit; ++gg) {
                        const uint4 raw = *reinterpret_cast<const uint4 *>(src + gg * kUnit);
                        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                        for (int m = 0; m < kUnit; ++m) v[c][gg * kUnit + m] = Io<Tin>::widen(w, m);
                    }
                } else {
                    const Tin *src = Bsrc[t] + (int64_t)n * L;
#pragma unroll
                    for (int m = 0; m < 8; ++m) {
                        const int64_t l = c0 + i0 + m;
                        uint32_t bits = 0u;
                        if (l < Lend) bits = Io<Tin>::bits(src, l);
                        if constexpr (sizeof(Tin) == 2) bits <<= 16;
                        v[c][m] = __uint_as_float(bits);
                    }
                }
            }
            if constexpr (kHalf) {
                float2 *FB = reinterpret_cast<float2 *>(Fs);
                uint32_t *FC = reinterpret_cast<uint32_t *>(FB + kDirectStage * kPairs);
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    FB[(i0 + m) * kPairs + q] = make_float2(v[0][m], v[1][m]);
                    FC[(i0 + m) * kPairs + q] = (__float_as_uint(v[2][m]) >> 16) | (__float_as_uint(v[3][m]) & 0xffff0000u);
                }
            } else if constexpr (kPack) {
                uint2 *Fp = reinterpret_cast<uint2 *>(Fs);
#pragma unroll
                for (int m = 0; m < 8; ++m)
                    Fp[(i0 + m) * kPairs + q] =
                        make_uint2((__float_as_uint(v[0][m]) >> 16) | (__float_as_uint(v[1][m]) & 0xffff0000u),
                                   (__float_as_uint(v[2][m]) >> 16) | (__float_as_uint(v[3][m]) & 0xffff0000u));
            } else {
#pragma unroll
                for (int m = 0; m < 8; ++m) Fs[(i0 + m) * kPairs + q] = make_float4(v[0][m], v[1][m], v[2][m], v[3][m]);
            }
        }
    };
    // This lane's kOwn steps of a stream starting `off` elements past `own`
    // (0 past the end of the sequence), as raw words.
    auto load_own_checked = [&](const Tin *own, int64_t s0, uint32_t (&w)[kOwnWords]) {
        if (kOwnBytes >= 4 && vec && s0 + kOwn <= Lend) {
            ld_words<kOwnBytes>(own, w);
        } else {
#pragma unroll
            for (int j = 0; j < kOwnWords; ++j) w[j] = 0u;
#pragma unroll
            for (int i = 0; i < kOwn; ++i) {
                if (s0 + i < Lend) {
                    const uint32_t bits = Io<Tin>::bits(own, i);
                    if constexpr (sizeof(Tin) == 2) w[i >> 1] |= bits << (16 * (i & 1));
                    else w[i] = bits;
                }
            }
        }
    };

    uint32_t wu[kOwnWords], wd[kOwnWords], wz[kOwnWords];
    // Start flags of this lane's owned steps of the coming sub-chunk (loaded
    // one sub-chunk ahead, like u, delta and z).
    uint8_t rb[kReset ? kOwn : 1];
    auto load_starts = [&](int64_t s0) {
        if constexpr (kReset) {
#pragma unroll
            for (int i = 0; i < kOwn; ++i) rb[i] = s0 + i < Lend ? reset_b[s0 + i] : (uint8_t)0;
        }
    };
    load_starts(c_begin + g * kOwn);
    load_own_checked(u_own, c_begin + g * kOwn, wu);
    if constexpr (!kDt) load_own_checked(d_own, c_begin + g * kOwn, wd);
    else
#pragma unroll
        for (int j = 0; j < kOwnWords; ++j) wd[j] = 0u;
    if (has_z) load_own_checked(z_own, c_begin + g * kOwn, wz);

    // dt_proj form: the operands in shared memory, the TMEM accumulator, and
    // the first stage's product.  Stage k's delta sits in TMEM columns
    // [64 (k & 1), 64 (k & 1) + 64), column e holding step e of the stage in
    // the lane of the thread whose row it is.  A tcgen05.ld reads the same
    // columns for every thread of a warp (its address is warp-uniform), so
    // each thread loads the sub-chunk's kDirectSub columns and keeps its own
    // kOwn of them.  The product of stage k + 1 is issued at the start of
    // stage k (by thread 0), its B operand built at the start of stage k - 1
    // from delta_r loaded one stage before that.
    uint8_t *dt_A = nullptr, *dt_B = nullptr;
    uint64_t *dt_full = nullptr;
    uint32_t dt_taddr = 0, dt_col = 0;
    const int dt_R = kDt ? p.dt_rank : 0, dt_rpad = (dt_R + 15) / 16 * 16;
    const int64_t dt_nst = (Lend - c_begin + kDirectStage - 1) / kDirectStage;  // stages of this block
    bool dt_ok = true;
    uint4 dt_raw[kDt ? kMaxDtRank * 8 / 128 : 1];  // this thread's 16-byte chunks of delta_r of a coming stage
    const Tin *dt_src = kDt ? static_cast<const Tin *>(p.delta_r) + b * (p.dtr_bstride ? p.dtr_bstride : dt_R * L)
                            : nullptr;
    auto dt_load_raw = [&](int64_t k) {  // delta_r[b, r, stage k]: chunks (r, 8 steps)
#pragma unroll
        for (int q = 0; q < kMaxDtRank * 8 / 128; ++q) {
            const int c = tid + 128 * q, rr = c / 8, j = c % 8;
            const int64_t l0 = c_begin + k * kDirectStage + 8 * j;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (rr < dt_R) {
                const Tin *src = dt_src + (int64_t)rr * L + l0;
                if (vec && l0 + 8 <= Lend) {
                    v = __ldg(reinterpret_cast<const uint4 *>(src));
                } else {
                    uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        if (l0 + i < Lend) w[i >> 1] |= Io<Tin>::bits(src, i) << (16 * (i & 1));
                    v = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            dt_raw[q] = v;
        }
    };
    auto dt_build = [&](int64_t k) {  // B operand of stage k from dt_raw (transposed: N = steps, K = rank)
        uint8_t *Bb = dt_B + (size_t)(k % 3) * dt_rpad * 128;
#pragma unroll
        for (int q = 0; q < kMaxDtRank * 8 / 128; ++q) {
            const int c = tid + 128 * q, rr = c / 8, j = c % 8;
            if (rr < dt_R) {
                const uint32_t w[4] = {dt_raw[q].x, dt_raw[q].y, dt_raw[q].z, dt_raw[q].w};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int n = 8 * j + i;  // step of the stage = column of the product
                    *reinterpret_cast<uint16_t *>(Bb + (rr / 8) * 1024 + n * 16 + (rr % 8) * 2) =
                        (uint16_t)(w[i >> 1] >> (16 * (i & 1)));
                }
            }
        }
    };
    auto dt_issue = [&](int64_t k) {  // D[(k & 1)] = A x B(k), K = dt_rpad in steps of 16
        const uint32_t a0 = tc_smem_addr(dt_A), b0 = tc_smem_addr(dt_B + (size_t)(k % 3) * dt_rpad * 128);
        for (int j = 0; j < dt_rpad / 16; ++j)
            tc::mma_bf16_acc(dt_taddr + (uint32_t)((k & 1) * kDirectStage), tc::sdesc(a0 + j * 4096, 2048, 128),
                             tc::sdesc(b0 + j * 2048, 1024, 128), tc::idesc_bf16(128, kDirectStage), j > 0);
        tc::commit(&dt_full[k & 1]);
    };
    if constexpr (kDt) {
        const size_t slab_end = reinterpret_cast<size_t>(reinterpret_cast<float *>(RB1 + 2 * kNmax * kDirectStage) +
                                                         (nthreads / 32) * (kRowsPerWarp * kGatherStride + 32 * kRS));
        dt_A = reinterpret_cast<uint8_t *>((slab_end + 1023) / 1024 * 1024);
        dt_B = dt_A + (size_t)dt_rpad * 256;
        dt_full = reinterpret_cast<uint64_t *>(dt_B + (size_t)3 * dt_rpad * 128);
        uint32_t *dt_slot = reinterpret_cast<uint32_t *>(dt_full + 2);
        for (int i = tid; i < 3 * dt_rpad * 128 / 16; i += nthreads)
            reinterpret_cast<uint4 *>(dt_B)[i] = make_uint4(0u, 0u, 0u, 0u);
        const int64_t d0 = (bt % p.dtiles) * rows;
        const unsigned short *W16 = static_cast<const unsigned short *>(p.W_dt);
        for (int i = tid; i < 128 * dt_rpad; i += nthreads) {  // lane m's row: W_dt of its channel
            const int m = i / dt_rpad, k = i % dt_rpad;
            const int64_t dm = d0 + m / kG < p.dim ? d0 + m / kG : p.dim - 1;
            *reinterpret_cast<uint16_t *>(dt_A + (k / 8) * 2048 + m * 16 + (k % 8) * 2) =
                k < dt_R ? W16[dm * dt_R + k] : (uint16_t)0;
        }
        if (tid == 0) {
            tc::mbar_init(&dt_full[0], 1), tc::mbar_init(&dt_full[1], 1);
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
        if (warp == 0) tc::alloc(dt_slot, 128);
        __syncthreads();  // B buffers zeroed before the builds write into them
        if (dt_nst > 0) dt_load_raw(0), dt_build(0);
        if (dt_nst > 1) dt_load_raw(1), dt_build(1);
        if (dt_nst > 2) dt_load_raw(2);
        tc::fence_async_smem();
        tc::fence_before();
        __syncthreads();
        tc::fence_after();
        dt_taddr = *dt_slot;
        if (tid == 0 && dt_nst > 0) dt_issue(0);
    }
    // Stage k's B/C sit in F[k & 1]; the raw copies of stage k + 1 are in
    // flight (into RB[(k + 1) & 1]) while stage k is computed.  The first
    // stage is converted here.
    if (!kDB) {
        if (c_begin < Lend && stage_fast(c_begin)) issue_copies(c_begin, RB0);
    } else if (c_begin < Lend) {
        const int64_t c1 = c_begin + kDirectStage;
        const bool f0 = stage_fast(c_begin), f1 = c1 < Lend && stage_fast(c1);
        if (f0) issue_copies(c_begin, RB0);
        if (f1) issue_copies(c1, RB1);
        if (f0) {
            if (f1) cp_async_wait_one();
            else cp_async_wait_all();
        }
        __syncthreads();  // every thread's copies of the first stage have landed
        fill_F(c_begin, f0, RB0, F0);
    }
    float dsum = 0.f;  // sum of this lane's delta' (segment record)

    // One sub-chunk of 8 steps from step l0; kChecked: guard the sequence end.
    auto sub_chunk = [&](auto checked, int m, int64_t l0) {
        constexpr bool kChecked = decltype(checked)::value;
        uint32_t cu[kOwnWords], cd[kOwnWords], cz[kOwnWords];
#pragma unroll
        for (int j = 0; j < kOwnWords; ++j) cu[j] = wu[j], cd[j] = wd[j], cz[j] = wz[j];
        const int64_t s_next = l0 + kDirectSub + g * kOwn;   // next owned step
        u_own += kDirectSub;
        if constexpr (!kDt) d_own += kDirectSub;
        if (has_z) z_own += kDirectSub;
        if (kOwnBytes >= 4 && !kChecked && m + 1 < kSubs) {  // next sub-chunk lies in this full stage
            ld_words<kOwnBytes>(u_own, wu);
            if constexpr (!kDt) ld_words<kOwnBytes>(d_own, wd);
            if (has_z) ld_words<kOwnBytes>(z_own, wz);
        } else if (l0 + kDirectSub < Lend) {
            load_own_checked(u_own, s_next, wu);
            if constexpr (!kDt) load_own_checked(d_own, s_next, wd);
            if (has_z) load_own_checked(z_own, s_next, wz);
        }
        // dt_proj form: this lane's delta of its own steps, from tensor memory.
        uint32_t dtv[kDt ? kOwn : 1];
        if constexpr (kDt) {
            static_assert(kOwn == 4 && (kDirectSub == 8 || kDirectSub == 16), "4 own steps of 8 or 16");
            uint32_t all[kDirectSub];
            tc::ld_sync(dt_col + (uint32_t)(m * kDirectSub), all);
#pragma unroll
            for (int i = 0; i < kOwn; ++i) dtv[i] = all[i];
#pragma unroll
            for (int gg = 1; gg < kG; ++gg)
                if (g == gg) {
#pragma unroll
                    for (int i = 0; i < kOwn; ++i) dtv[i] = all[gg * kOwn + i];
                }
        }
        // Bit i: a sequence starts at step l0 + i (the state entering it is
        // zero).  Each lane reads its owned steps; the row's lanes (and so the
        // warp, whose rows share the batch entry) end up with the same mask.
        uint32_t rmask = 0u;
        if constexpr (kReset) {
#pragma unroll
            for (int i = 0; i < kOwn; ++i)
                if (rb[i] != 0) rmask |= 1u << (g * kOwn + i);
            load_starts(s_next);
            if constexpr (kG > 1) {
#pragma unroll
                for (int off = 1; off < kG; off *= 2) rmask |= __shfl_xor_sync(0xffffffffu, rmask, off, kG);
            }
            seg_reset |= rmask != 0u;
        }
        // delta' and delta' u of the owned steps (past L: the identity step).
        float dl_own[kOwn], du_own[kOwn], uo[kOwn];
#pragma unroll
        for (int i = 0; i < kOwn; ++i) {
            uo[i] = Io<Tin>::widen(cu, i);
            const float dx = kDt ? __uint_as_float(dtv[kDt ? i : 0]) : Io<Tin>::widen(cd, i);
            dl_own[i] = delta_transform<kFast>(dx + bias, softplus);
            if constexpr (kChecked) {
                if (l0 + g * kOwn + i >= Lend) dl_own[i] = 0.f;
            }
            du_own[i] = dl_own[i] * uo[i];
            dsum += dl_own[i];
        }
        // All 8 steps' values of the row.
        float dl[kDirectSub], du[kDirectSub];
        if constexpr (kG == 1) {
#pragma unroll
            for (int i = 0; i < kDirectSub; ++i) dl[i] = dl_own[i], du[i] = du_own[i];
        } else {
#pragma unroll
            for (int i = 0; i < kOwn; ++i)
                gat[g * kOwn + i] = dl_own[i], gat[kDirectSub + g * kOwn + i] = du_own[i];
            __syncwarp();
#pragma unroll
            for (int q4 = 0; q4 < kDirectSub / 4; ++q4) {
                const float4 a4 = reinterpret_cast<const float4 *>(gat)[q4];
                const float4 b4 = reinterpret_cast<const float4 *>(gat + kDirectSub)[q4];
                dl[4 * q4] = a4.x, dl[4 * q4 + 1] = a4.y, dl[4 * q4 + 2] = a4.z, dl[4 * q4 + 3] = a4.w;
                du[4 * q4] = b4.x, du[4 * q4 + 1] = b4.y, du[4 * q4 + 2] = b4.z, du[4 * q4 + 3] = b4.w;
            }
        }
        float part[kDirectSub];
        const float4 *Fm = F + (m * kDirectSub) * kPairs + q0;
        const uint2 *Fm2 = reinterpret_cast<const uint2 *>(F) + (m * kDirectSub) * kPairs + q0;
        const float2 *FmB = reinterpret_cast<const float2 *>(F) + (m * kDirectSub) * kPairs + q0;
        const uint32_t *FmC = reinterpret_cast<const uint32_t *>(reinterpret_cast<const float2 *>(F) + kDirectStage * kPairs) +
                              (m * kDirectSub) * kPairs + q0;
        auto A2_of = [&](int qq) {
            if constexpr (kA2InRegs) return A2[qq];
            const int n = 2 * (q0 + qq);
            return make_float2(n < N ? __ldg(A_d + n) * kLog2e : 0.f, n + 1 < N ? __ldg(A_d + n + 1) * kLog2e : 0.f);
        };
        // The state loop; with_starts: a start in this sub-chunk (zero the
        // state entering it).  The mask is warp-uniform, so a sub-chunk
        // without one takes the plain loop.
        auto steps = [&](auto with_starts) {
            constexpr bool kStarts = decltype(with_starts)::value;
#pragma unroll
            for (int i = 0; i < kDirectSub; ++i) {
                if (kCkpt && i % kCkptStride == 0 && ckpt_row != nullptr && l0 + i < Lend) {
                    float *dst = ckpt_row + ((l0 + i) / kCkptStride) * N;
                    if (ckpt_vec) {  // this lane's states as 16- (or 8-) byte streaming stores
#pragma unroll
                        for (int qq = 0; qq < kPL; qq += 2) {
                            const int n = 2 * (q0 + qq);
                            if (n >= N) continue;
                            if (qq + 1 < kPL)
                                __stcs(reinterpret_cast<float4 *>(dst + n),
                                       make_float4(h[qq].x, h[qq].y, h[qq + 1].x, h[qq + 1].y));
                            else
                                __stcs(reinterpret_cast<float2 *>(dst + n), h[qq]);
                        }
                    } else {
#pragma unroll
                        for (int qq = 0; qq < kPL; ++qq) {
                            const int n = 2 * (q0 + qq);
                            if (n < N) dst[n] = h[qq].x;
                            if (n + 1 < N) dst[n + 1] = h[qq].y;
                        }
                    }
                }
                const float2 d2 = make_float2(dl[i], dl[i]), u2 = make_float2(du[i], du[i]);
                float2 acc[kAccs];
#pragma unroll
                for (int k = 0; k < kAccs; ++k) acc[k] = make_float2(0.f, 0.f);
#pragma unroll
                for (int qq = 0; qq < kPL; ++qq) {
                    float4 bc;  // (B_n, B_n+1, C_n, C_n+1) of this step and state pair
                    if constexpr (kHalf) {
                        const float2 bb = FmB[i * kPairs + qq];
                        const uint32_t cw = FmC[i * kPairs + qq];
                        bc = make_float4(bb.x, bb.y, __uint_as_float(cw << 16), __uint_as_float(cw & 0xffff0000u));
                    } else if constexpr (kPack) {
                        const uint2 w = Fm2[i * kPairs + qq];
                        bc = make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u),
                                         __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xffff0000u));
                    } else {
                        bc = Fm[i * kPairs + qq];
                    }
                    const float2 t = __fmul2_rn(d2, A2_of(qq));
                    const float2 a = make_float2(sfu_exp2(t.x), sfu_exp2(t.y));
                    if constexpr (kStarts) {
                        if ((rmask >> i) & 1u) h[qq] = make_float2(0.f, 0.f);
                    }
                    h[qq] = __ffma2_rn(a, h[qq], __fmul2_rn(u2, make_float2(bc.x, bc.y)));
                    acc[qq % kAccs] = __ffma2_rn(make_float2(bc.z, bc.w), h[qq], acc[qq % kAccs]);
                }
                if constexpr (kAccs == 2) acc[0] = __fadd2_rn(acc[0], acc[1]);
                part[i] = acc[0].x + acc[0].y;
            }
        };
        if constexpr (kReset) {
            if (rmask != 0u) steps(std::true_type{});
            else steps(std::false_type{});
        } else {
            steps(std::false_type{});
        }
        // Totals of the owned steps (none without y: the backward's segment
        // summary runs this kernel for its segment records only).
        if (!want_y) {
            y_own += kDirectSub;
            return;
        }
        float yv[kOwn];
        if constexpr (kG == 1) {
#pragma unroll
            for (int i = 0; i < kOwn; ++i) yv[i] = part[i];
        } else {
            static_assert(kOwn % kRV == 0 && kRS % kRV == 0, "reduce slab accesses stay aligned");
            float *mine = red + lane * kRS;
#pragma unroll
            for (int k = 0; k < kDirectSub; k += kRV) st_vec<kRV>(mine + k, part + k);
            __syncwarp();
#pragma unroll
            for (int i = 0; i < kOwn; ++i) yv[i] = 0.f;
#pragma unroll
            for (int gg = 0; gg < kG; ++gg) {
                const float *src = red + (r * kG + gg) * kRS + g * kOwn;
#pragma unroll
                for (int k = 0; k < kOwn; k += kRV) {
                    float v[kRV];
                    ld_vec<kRV>(src + k, v);
#pragma unroll
                    for (int j = 0; j < kRV; ++j) yv[k + j] += v[j];
                }
            }
        }
#pragma unroll
        for (int i = 0; i < kOwn; ++i) yv[i] = fmaf(Dd, uo[i], yv[i]);  // + D u (§3.3)
        if (has_z) {
#pragma unroll
            for (int i = 0; i < kOwn; ++i) yv[i] *= silu<kFast>(Io<Tin>::widen(cz, i));
        }
        if (row_ok) {
            if constexpr (kChecked) {
                store_run<kOwn>(y_row, l0 + g * kOwn, Lend, vec, yv);
            } else {
                store_run<kOwn>(y_own, 0, kOwn, true, yv);
            }
        }
        y_own += kDirectSub;
    };

    int stage = 0;
    for (int64_t c0 = c_begin; c0 < Lend; c0 += kDirectStage, ++stage) {
        const bool fast = stage_fast(c0);
        const int64_t cn = c0 + kDirectStage, cnn = cn + kDirectStage;
        if constexpr (kDB) {
            const bool odd = stage & 1;
            F = odd ? F1 : F0;
            if (cn < Lend && stage_fast(cn)) cp_async_wait_all();  // the next stage's copies (the only group in flight)
            if constexpr (kDt) tc::fence_before();  // last stage's TMEM reads before the next product
            __syncthreads();  // F of this stage is complete; the next stage's raw copies have landed; the
                              // other F (last stage's) and this stage's RB (converted before) are free
            if (cn < Lend) fill_F(cn, stage_fast(cn), odd ? RB0 : RB1, odd ? F0 : F1);
            if (cnn < Lend && stage_fast(cnn)) issue_copies(cnn, odd ? RB1 : RB0);
            if constexpr (kDt) {
                if (tid == 0 && stage + 1 < dt_nst) {
                    tc::fence_after();
                    dt_issue(stage + 1);  // its B operand was built and fenced before this barrier
                }
                if (stage + 2 < dt_nst) dt_build(stage + 2);
                if (stage + 3 < dt_nst) dt_load_raw(stage + 3);
                tc::fence_async_smem();
                // This stage's product (issued a stage ago) is complete before its reads.
                if (!tc::mbar_wait(&dt_full[stage & 1], (uint32_t)((stage >> 1) & 1))) dt_ok = false;
                __syncwarp();
                tc::fence_after();
                dt_col = dt_taddr + ((uint32_t)(32 * warp) << 16) + (uint32_t)((stage & 1) * kDirectStage);
            }
        } else {
            if (fast) cp_async_wait_all();
            __syncthreads();  // RB holds this stage; every warp is done with F
            fill_F(c0, fast, RB0, F0);
            __syncthreads();  // F holds this stage; RB is free
            if (cn < Lend && stage_fast(cn)) issue_copies(cn, RB0);
        }

        if (fast) {
#pragma unroll 1
            for (int m = 0; m < kSubs; ++m) sub_chunk(std::false_type{}, m, c0 + m * kDirectSub);
        } else {
            const int nsub =
                (int)((Lend - c0 < kDirectStage ? Lend - c0 : kDirectStage) + kDirectSub - 1) / kDirectSub;
#pragma unroll 1
            for (int m = 0; m < nsub; ++m) sub_chunk(std::true_type{}, m, c0 + m * kDirectSub);
        }
    }

    if constexpr (kDt) {  // every product was waited for; every TMEM read is done before the free
        tc::fence_before();
        __syncthreads();
        if (warp == 0) tc::dealloc(dt_taddr, 128);
        if (!dt_ok && lane == 0 && p.status) atomicExch(p.status, kDeviceTimeout);
    }
    if (p.nseg > 1) {  // segment record for the fix-up kernel
        const int64_t rec = seg * (p.batch * p.dim) + row;
        if constexpr (kG > 1) {
#pragma unroll
            for (int sdist = 1; sdist < kG; sdist *= 2) dsum += __shfl_xor_sync(0xffffffffu, dsum, sdist, kG);
        }
        if (row_ok) {
#pragma unroll
            for (int qq = 0; qq < kPL; ++qq) {
                const int n = 2 * (q0 + qq);
                if (n < N) p.ws_hend[rec * N + n] = h[qq].x;
                if (n + 1 < N) p.ws_hend[rec * N + n + 1] = h[qq].y;
            }
            if (g == 0) p.ws_dsum[rec] = (kReset && seg_reset) ? -1.f : dsum;
        }
    } else if (p.last_state != nullptr && row_ok) {
#pragma unroll
        for (int qq = 0; qq < kPL; ++qq) {
            const int n = 2 * (q0 + qq);
            if (n < N) p.last_state[row * N + n] = h[qq].x;
            if (n + 1 < N) p.last_state[row * N + n + 1] = h[qq].y;
        }
    }
}

// ------------------------------------------------------------ fix-up kernels
// After the direct kernel ran every sequence segment from a zero state, the
// true state entering segment s > 0 is the carry of segments 0..s-1:
//   h_in(s) = P(s-1) h_in(s-1) + h_end(s-1),   P(j)_n = 2^(A_n log2e sum_j delta'),
// and its share of y at step l of segment s is
//   (sum_n C[b,n,l] 2^(A_n log2e S_l) h_in(s)_n) silu(z_l),   S_l = delta' summed
// over the segment up to and including l (linearity of the recurrence in h).
// A segment holding a sequence start (p.reset) passes no state on (P = 0,
// recorded as a delta' sum of -1), and the carried state's share ends at its
// first start.
//
// Two kernels.  ss_fwd_carry_kernel folds the segments of one row in order
// (one warp per row, states over lanes) and overwrites the record h_end(j)
// with h_in(j + 1), so that segment s finds its incoming state in record
// s - 1; it writes last_state = h_in(nseg) when asked.
// ss_fwd_fixup_kernel then adds the share of y: one warp per (row, segment
// s > 0), the steps over lanes, kFixupSteps per lane per chunk (lane i takes
// steps c + 32 k + i, so each load is one coalesced run), S by warp scans,
// states looped with h_in and A_n log2e in shared memory.  A warp stops
// after the chunk in which every state's exponent A_n log2e S passed -127
// (from there ex2.ftz returns exactly 0, so the remaining shares are exactly
// zero, and steps past that point are not rewritten) or that held a start.
// With bf16 output y is rounded twice: once by the direct kernel (its
// zero-state value y0) and once here after the share is added in fp32, so
// the result differs from the exact sum by up to half a bf16 ulp of y0 plus
// half a bf16 ulp of the result (2^-9 |y0| + 2^-9 |y| at most), more than one
// rounding only where the share cancels much of y0.
// The dt_proj form (p.delta null) recomputes delta = W_dt delta_r for the
// steps it corrects, in fp32 from the exact bf16 products (the direct kernel
// sums the same products on the tensor cores, in its own order).
template <int kNmax>
__global__ void __launch_bounds__(256) ss_fwd_carry_kernel(const FwdParams p) {
    constexpr int kPer = kNmax > 32 ? 2 : 1;  // states per lane
    constexpr int kBatchJ = 4;                // segment records loaded ahead
    const int64_t rows_total = p.batch * p.dim;
    const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (row >= rows_total) return;  // whole warps leave together
    const int64_t d = row % p.dim;
    const int N = p.dstate;
    float A2[kPer], h[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        const int n = lane + 32 * k;
        A2[k] = n < N ? p.A[d * N + n] * kLog2e : 0.f;
        h[k] = 0.f;
    }
    for (int j0 = 0; j0 < p.nseg; j0 += kBatchJ) {
        float ds[kBatchJ], he[kBatchJ][kPer];
#pragma unroll
        for (int jj = 0; jj < kBatchJ; ++jj) {
            const int64_t rec = (int64_t)(j0 + jj) * rows_total + row;
            const bool ok = j0 + jj < p.nseg;
            ds[jj] = ok ? p.ws_dsum[rec] : 0.f;
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                const int n = lane + 32 * k;
                he[jj][k] = ok && n < N ? p.ws_hend[rec * N + n] : 0.f;
            }
        }
#pragma unroll
        for (int jj = 0; jj < kBatchJ; ++jj) {
            const int j = j0 + jj;
            if (j >= p.nseg) break;
            const int64_t rec = (int64_t)j * rows_total + row;
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                const int n = lane + 32 * k;
                h[k] = fmaf(ds[jj] < 0.f ? 0.f : sfu_exp2(A2[k] * ds[jj]), h[k], he[jj][k]);
                if (n < N && j + 1 < p.nseg) p.ws_hend[rec * N + n] = h[k];
            }
        }
    }
    if (p.last_state != nullptr) {
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const int n = lane + 32 * k;
            if (n < N) p.last_state[row * N + n] = h[k];
        }
    }
}

constexpr int kFixupWarps = 8;
constexpr int kMaxDstate = 64;  // the largest state size the library takes
constexpr int kFixupSteps = 4;  // steps per lane per chunk (128-step chunks)

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(kFixupWarps * 32) ss_fwd_fixup_kernel(const FwdParams p) {
    constexpr bool kFast = sizeof(Tin) == 2;
    constexpr int kK = kFixupSteps;
    __shared__ float sh_h[kFixupWarps][kMaxDstate], sh_A2[kFixupWarps][kMaxDstate];
    __shared__ float sh_W[kFixupWarps][kMaxDtRank];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t rows_total = p.batch * p.dim;
    const int64_t task = (int64_t)blockIdx.x * kFixupWarps + warp;  // (row, segment s >= 1)
    if (task >= rows_total * (p.nseg - 1)) return;                 // whole warps leave together
    const int64_t row = task % rows_total;
    const int s = 1 + (int)(task / rows_total);
    const int64_t b = row / p.dim, d = row % p.dim;
    const int N = p.dstate;
    const int64_t L = p.seqlen;
    const bool dt = p.delta == nullptr;
    const int R = p.dt_rank;

    float A2max = __int_as_float(0xff800000u);  // -inf
    const int64_t rec_in = ((int64_t)(s - 1) * rows_total + row) * N;
    for (int n = lane; n < N; n += 32) {
        const float a2 = p.A[d * N + n] * kLog2e;
        sh_A2[warp][n] = a2;
        sh_h[warp][n] = p.ws_hend[rec_in + n];
        A2max = fmaxf(A2max, a2);
    }
    if (dt)
        for (int r = lane; r < R; r += 32)
            sh_W[warp][r] = static_cast<float>(static_cast<const Tin *>(p.W_dt)[d * R + r]);
#pragma unroll
    for (int off = 16; off >= 1; off /= 2) A2max = fmaxf(A2max, __shfl_xor_sync(0xffffffffu, A2max, off));
    __syncwarp();

    const Tin *dl_row = dt ? nullptr : static_cast<const Tin *>(p.delta) + row * L;
    const Tin *dr_b = dt ? static_cast<const Tin *>(p.delta_r) + b * (p.dtr_bstride ? p.dtr_bstride : R * L) : nullptr;
    const Tin *z_row = p.z ? static_cast<const Tin *>(p.z) + row * L : nullptr;
    const Tin *C_b = static_cast<const Tin *>(p.C) + b * (p.bc_bstride ? p.bc_bstride : N * L);
    Tout *y_row = static_cast<Tout *>(p.y) + row * L;
    const float bias = p.delta_bias ? p.delta_bias[d] : 0.f;
    const bool softplus = p.softplus != 0;
    const uint8_t *const reset_b = p.reset ? p.reset + b * L : nullptr;
    const int64_t c_begin = (int64_t)s * p.seg_len;
    const int64_t c_end = c_begin + p.seg_len < L ? c_begin + p.seg_len : L;
    float *const ckpt_b = p.ckpt != nullptr ? p.ckpt + row * ((L + kCkptStride - 1) / kCkptStride) * N : nullptr;

    float S0 = 0.f;  // delta' summed over the chunks before this one
    for (int64_t c = c_begin; c < c_end; c += 32 * kK) {
        float S[kK];
        bool in[kK];
        unsigned starts = 0;  // nonzero if a step of this chunk starts a sequence
        int first_start = 32 * kK;
#pragma unroll
        for (int k = 0; k < kK; ++k) {
            const int64_t l = c + 32 * k + lane;
            in[k] = l < c_end;
            float x = 0.f;
            if (in[k]) {
                if (dt) {
                    for (int r = 0; r < R; ++r) x = fmaf(sh_W[warp][r], static_cast<float>(dr_b[(int64_t)r * L + l]), x);
                } else {
                    x = static_cast<float>(dl_row[l]);
                }
            }
            S[k] = in[k] ? delta_transform<kFast>(x + bias, softplus) : 0.f;
            const unsigned m = __ballot_sync(0xffffffffu, in[k] && reset_b != nullptr && reset_b[l] != 0);
            if (m != 0 && first_start == 32 * kK) first_start = 32 * k + __ffs(m) - 1;
            starts |= m;
        }
        float own[kK];  // this lane's delta' of each of its steps
#pragma unroll
        for (int k = 0; k < kK; ++k) own[k] = S[k];
        // inclusive scan of delta' over the chunk's steps, in step order
#pragma unroll
        for (int k = 0; k < kK; ++k) {
#pragma unroll
            for (int off = 1; off < 32; off *= 2) {
                const float t = __shfl_up_sync(0xffffffffu, S[k], off);
                if (lane >= off) S[k] += t;
            }
            S[k] += S0;
            S0 = __shfl_sync(0xffffffffu, S[k], 31);
        }
        bool live[kK];
        bool any = false;
#pragma unroll
        for (int k = 0; k < kK; ++k) {
            live[k] = in[k] && 32 * k + lane < first_start && !(A2max * S[k] < -127.f);
            any |= live[k];
        }
        if (any) {
            float corr[kK];
#pragma unroll
            for (int k = 0; k < kK; ++k) corr[k] = 0.f;
#pragma unroll 4
            for (int n = 0; n < N; ++n) {
                const float a2 = sh_A2[warp][n], hn = sh_h[warp][n];
#pragma unroll
                for (int k = 0; k < kK; ++k) {
                    if (live[k]) {
                        const float cv = static_cast<float>(C_b[(int64_t)n * L + c + 32 * k + lane]);
                        corr[k] = fmaf(cv * sfu_exp2(a2 * S[k]), hn, corr[k]);
                    }
                }
            }
#pragma unroll
            for (int k = 0; k < kK; ++k) {
                if (live[k]) {
                    const int64_t l = c + 32 * k + lane;
                    float v = corr[k];
                    if (z_row) v *= silu<kFast>(static_cast<float>(z_row[l]));
                    y_row[l] = static_cast<Tout>(static_cast<float>(y_row[l]) + v);
                }
            }
        }
        // Checkpoints (the state entering steps l = 8k, after step l - 1):
        // the carried share 2^(A log2e S_(l-1)) h_in, up to and including the
        // segment's first start (a start zeroes the state only after it).
        if (ckpt_b != nullptr) {
#pragma unroll
            for (int k = 0; k < kK; ++k) {
                const int64_t l = c + 32 * k + lane;
                const float Sx = S[k] - own[k];
                if (in[k] && l % kCkptStride == 0 && 32 * k + lane <= first_start && !(A2max * Sx < -127.f)) {
                    float *ck = ckpt_b + (l / kCkptStride) * N;
                    for (int n = 0; n < N; ++n) ck[n] = fmaf(sfu_exp2(sh_A2[warp][n] * Sx), sh_h[warp][n], ck[n]);
                }
            }
        }
        if (starts != 0 || A2max * S0 < -127.f) break;
    }
}

}  // namespace selscan
