// Selective-scan forward kernel for sm_100a.
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
// chunk of W*8 consecutive steps, 8 steps per lane.  For every state n a lane
// runs its 8 steps from a zero state, recording the decays a_i and inputs b_i,
// then the W lanes combine their (prod a, h) pairs with a shuffle scan under
// the associative operator (a1, h1) . (a2, h2) = (a2 a1, a2 h1 + h2) (the
// operator of "手把手用PyTorch实现Mamba的SSM层" §3.2), restricted to diagonal A.
// The scan gives each lane its true incoming state; a second pass over the
// recorded (a_i, b_i) then yields the states and y.  The chunk's outgoing
// state per n stays in registers (`carry`) for the next chunk.  With W = 1 the
// lane owns the whole row and runs the plain sequential recurrence.
//
// exp(delta' A) is computed as ex2(delta' * (A log2 e)) on the SFU.  Streams
// u, delta and z are prefetched one chunk ahead into registers; B and C rows
// are shared by all rows of a batch and read through L1 (the lanes of a warp
// that sit at the same steps read the same addresses).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace selscan {

constexpr int kItems = 8;  // consecutive steps per lane per chunk
constexpr size_t kMaxSmemBytes = 227 * 1024;  // opt-in dynamic shared memory per block (sm_100)
constexpr float kLog2e = 1.4426950408889634f;

struct FwdParams {
    const void *u, *delta, *B, *C, *z;
    const float *A, *D, *delta_bias;
    void *y;
    float *last_state;
    int64_t batch, dim, seqlen;
    int dstate;
    int softplus;     // 1: softplus, 0: exp
    int vec;          // 1: every row of u/delta/z/B/C/y starts 16-byte aligned
    int64_t dtiles;   // row tiles per batch entry
};

// ---------------------------------------------------------------- element I/O
template <typename T>
struct Io;

template <>
struct Io<float> {
    static constexpr int kWords = kItems;  // one 32-bit word per element
    __device__ __forceinline__ static void widen(const uint32_t (&w)[kWords], float (&f)[kItems]) {
#pragma unroll
        for (int i = 0; i < kItems; ++i) f[i] = __uint_as_float(w[i]);
    }
    __device__ __forceinline__ static uint32_t bits(const float *p, int64_t i) {
        return __float_as_uint(p[i]);
    }
    __device__ __forceinline__ static void place(uint32_t (&w)[kWords], int i, uint32_t v) { w[i] = v; }
};

template <>
struct Io<__nv_bfloat16> {
    static constexpr int kWords = kItems / 2;  // two bf16 per word, element 2j in the low half
    __device__ __forceinline__ static void widen(const uint32_t (&w)[kWords], float (&f)[kItems]) {
#pragma unroll
        for (int j = 0; j < kWords; ++j) {
            f[2 * j] = __uint_as_float(w[j] << 16);
            f[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
        }
    }
    __device__ __forceinline__ static uint32_t bits(const __nv_bfloat16 *p, int64_t i) {
        return reinterpret_cast<const unsigned short *>(p)[i];
    }
    __device__ __forceinline__ static void place(uint32_t (&w)[kWords], int i, uint32_t v) {
        w[i >> 1] |= v << (16 * (i & 1));
    }
};

// Load steps [l0, l0 + 8) of one row as raw words; steps at or past L read 0.
// kStream: the data is read once (u, delta, z), so keep it out of L1.
template <typename T, bool kStream>
__device__ __forceinline__ void load_run(uint32_t (&w)[Io<T>::kWords], const T *row, int64_t l0,
                                         int64_t L, bool vec) {
    constexpr int kWords = Io<T>::kWords;
    if (vec && l0 + kItems <= L) {
        const uint4 *p = reinterpret_cast<const uint4 *>(row + l0);
#pragma unroll
        for (int j = 0; j < kWords / 4; ++j) {
            const uint4 v = kStream ? __ldcs(p + j) : __ldg(p + j);
            w[4 * j + 0] = v.x;
            w[4 * j + 1] = v.y;
            w[4 * j + 2] = v.z;
            w[4 * j + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < kWords; ++j) w[j] = 0u;
#pragma unroll
        for (int i = 0; i < kItems; ++i)
            if (l0 + i < L) Io<T>::place(w, i, Io<T>::bits(row, l0 + i));
    }
}

__device__ __forceinline__ void store_run(float *row, int64_t l0, int64_t L, bool vec,
                                          const float (&v)[kItems]) {
    if (vec && l0 + kItems <= L) {
        float4 *p = reinterpret_cast<float4 *>(row + l0);
        __stcs(p, make_float4(v[0], v[1], v[2], v[3]));
        __stcs(p + 1, make_float4(v[4], v[5], v[6], v[7]));
    } else {
#pragma unroll
        for (int i = 0; i < kItems; ++i)
            if (l0 + i < L) row[l0 + i] = v[i];
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

__device__ __forceinline__ void store_run(__nv_bfloat16 *row, int64_t l0, int64_t L, bool vec,
                                          const float (&v)[kItems]) {
    if (vec && l0 + kItems <= L) {
        uint4 q;
        q.x = pack_bf16x2(v[0], v[1]);
        q.y = pack_bf16x2(v[2], v[3]);
        q.z = pack_bf16x2(v[4], v[5]);
        q.w = pack_bf16x2(v[6], v[7]);
        __stcs(reinterpret_cast<uint4 *>(row + l0), q);
    } else {
#pragma unroll
        for (int i = 0; i < kItems; ++i)
            if (l0 + i < L) row[l0 + i] = __float2bfloat16_rn(v[i]);
    }
}

// 2^x on the SFU (MUFU.EX2), flushing subnormal results to zero.
__device__ __forceinline__ float sfu_exp2(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// log2(x) on the SFU (MUFU.LG2).
__device__ __forceinline__ float sfu_log2(float x) {
    float r;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// 1/x on the SFU (MUFU.RCP).
__device__ __forceinline__ float sfu_rcp(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

constexpr float kLn2 = 0.6931471805599453f;

// delta' of §2.2: torch's softplus (beta 1, linear above 20) or exp.
// kFast (bf16 inputs, whose values carry 2^-9 relative rounding):
//   softplus(x) = ln2 * log2(1 + e), e = 2^(x log2 e), on the SFU; when
//   e < 1/32 the rounding of 1 + e would dominate, so log1p(e) is taken from
//   its series e - e^2/2 + e^3/3 - e^4/4 (relative error below e^4/5 < 2e-7).
//   Relative error of delta' stays below about 1e-5.
// Otherwise (fp32 inputs): libm-accurate log1pf(expf(x)) and expf(x).
template <bool kFast>
__device__ __forceinline__ float delta_transform(float x, bool softplus) {
    if constexpr (kFast) {
        const float e = sfu_exp2(x * kLog2e);
        if (!softplus) return e;
        const float series = e * fmaf(-e, fmaf(-e, fmaf(-e, 0.25f, 1.f / 3.f), 0.5f), 1.f);
        const float viaLog = sfu_log2(1.f + e) * kLn2;
        const float sp = e < 0.03125f ? series : viaLog;
        return x > 20.f ? x : sp;
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

// float2 <-> one 64-bit register pair, for packed (f32x2) PTX operands.
__device__ __forceinline__ unsigned long long as_u64(float2 v) {
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(v.x), "f"(v.y));
    return r;
}
__device__ __forceinline__ float2 as_f2(unsigned long long r) {
    float2 v;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
    return v;
}

// Scan stage for a state pair held as packed (P, h): shuffle both halves of
// P and h `off` lanes up, then (only where the partner exists, shfl.up's
// predicate) h = P hu + h and P = P Pu as two f32x2 instructions.
template <int kW>
__device__ __forceinline__ void scan_stage_x2(unsigned long long &P, unsigned long long &h, int off) {
    constexpr int kSeg = (32 - kW) << 8;
    asm("{\n\t.reg .pred p;\n\t.reg .b32 p0, p1, h0, h1, u0, u1, v0, v1;\n\t"
        ".reg .b64 pu, hu;\n\t"
        "mov.b64 {p0, p1}, %0;\n\t"
        "mov.b64 {h0, h1}, %1;\n\t"
        "shfl.sync.up.b32 u0|p, p0, %2, %3, -1;\n\t"
        "shfl.sync.up.b32 u1, p1, %2, %3, -1;\n\t"
        "shfl.sync.up.b32 v0, h0, %2, %3, -1;\n\t"
        "shfl.sync.up.b32 v1, h1, %2, %3, -1;\n\t"
        "mov.b64 pu, {u0, u1};\n\t"
        "mov.b64 hu, {v0, v1};\n\t"
        "@p fma.rn.f32x2 %1, %0, hu, %1;\n\t"
        "@p mul.rn.f32x2 %0, %0, pu;\n\t}"
        : "+l"(P), "+l"(h)
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

// ------------------------------------------------------------------- kernel
// States are processed in pairs (n, n+1) held in float2 registers, so the
// per-step arithmetic of two states is one packed sm_100 instruction
// (fma/mul .f32x2): exponent arguments, delta' u B, the state update and the
// output accumulation.  The two exps stay two MUFU.EX2.
//
// Shared memory of one block, for a chunk of Lc = 8 W steps and the state
// bucket kNmax (states n >= N are zero rows, so they add nothing):
//   F: float, B and C of the chunk in a pair-interleaved order: for state pair
//      p and lane slot s, float4 number ((t kPairs + p) 4 + g) W + s holds
//      (X[2p][i], X[2p+1][i], X[2p][i+1], X[2p+1][i+1]) for steps i = 8s + 2g
//      and i + 1 of the chunk, X = B (t = 0) or C (t = 1).  The W slots of a
//      row read consecutive float4s (no bank conflicts); rows that share a
//      slot read the same address (broadcast).
//   R: Tin, [2][kNmax][Lc], raw copy of the chunk in global order, filled by
//      cp.async one chunk ahead (16-byte path only).
//   With W > 1 lanes per row, two per-row tables of kNmax + 2 floats (the
//      padding spreads rows over banks): A[d, n] log2(e), and the state that
//      enters the next chunk.  (With W = 1 a lane owns its row and keeps both
//      in registers.)
__host__ __device__ constexpr int chunk_len(int w) { return w * kItems; }

__host__ __device__ constexpr size_t smem_bytes(size_t in_size, int nmax, int w, int warps) {
    return (2 * sizeof(float) + 2 * in_size) * (size_t)nmax * (size_t)chunk_len(w) +
           (w > 1 ? 2 * sizeof(float) * (size_t)(nmax + 2) * (size_t)(warps * (32 / w)) : 0);
}

// State bucket (compile-time state count) for a runtime state count.
__host__ __device__ constexpr int state_bucket(int n) {
    return n <= 4 ? 4 : n <= 8 ? 8 : n <= 16 ? 16 : n <= 32 ? 32 : 64;
}

#ifndef SS_PAIR_UNROLL
#define SS_PAIR_UNROLL 1
#endif
constexpr int kPairUnroll = SS_PAIR_UNROLL;  // unroll of the W > 1 state-pair loop
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

__device__ __forceinline__ float2 f2(float v) { return make_float2(v, v); }

template <typename Tin, typename Tout, int kNmax, int kW>
__global__ void __launch_bounds__(256, Occupancy<kNmax>::kMinBlocks) ss_fwd_kernel(const FwdParams p) {
    static_assert(kW >= 1 && kW <= 32 && (32 % kW) == 0, "lanes per row must divide 32");
    static_assert(kItems == 8, "the F layout assumes 8 steps per lane");
    constexpr int kRowsPerWarp = 32 / kW;
    constexpr int kChunk = chunk_len(kW);
    constexpr int kPairs = kNmax / 2;
    constexpr int kG = kItems / 2;                      // float4s per lane per (tensor, pair)
    constexpr int kPairRow = kG * kW;                   // float4s per (tensor, pair) of F
    constexpr int kUnit = 16 / (int)sizeof(Tin);        // elements per 16-byte unit
    constexpr int kUnitsPerRow = kChunk / kUnit;        // a power of two
    constexpr int kUnits = 2 * kNmax * kUnitsPerRow;    // 16-byte units of B and C per chunk
    constexpr int kPairUnits = kUnits / 2;              // (unit, state pair) fill jobs
    constexpr int kWords = Io<Tin>::kWords;
    constexpr bool kFast = sizeof(Tin) == 2;            // bf16 inputs: SFU transforms
    constexpr int kRowStride = kNmax + 2;               // per-row tables (W > 1)
    constexpr unsigned kFull = 0xffffffffu;

    extern __shared__ float4 smem[];
    float4 *F = smem;                                                  // [2][kPairs][kPairRow]
    Tin *R = reinterpret_cast<Tin *>(smem + 2 * kPairs * kPairRow);     // [2][kNmax][kChunk]
    float *sA2 = reinterpret_cast<float *>(R + 2 * kNmax * kChunk);     // [rows][kRowStride]

    const int tid = threadIdx.x;
    const int nthreads = blockDim.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int seg = lane % kW;  // this lane's slot among the row's W lanes
    const int N = p.dstate;
    const int64_t rows_per_block = (int64_t)(nthreads >> 5) * kRowsPerWarp;
    const int64_t b = blockIdx.x / p.dtiles;
    const int64_t tile = blockIdx.x % p.dtiles;
    const int64_t d_raw = tile * rows_per_block + warp * kRowsPerWarp + lane / kW;
    // Rows past the end mirror the last row (valid addresses) and store nothing;
    // they must still run so that every lane takes part in the shuffles.
    const bool row_ok = d_raw < p.dim;
    const int64_t d = row_ok ? d_raw : p.dim - 1;
    const int64_t L = p.seqlen;
    const int64_t row = b * p.dim + d;
    const bool vec = p.vec != 0;
    const bool softplus = p.softplus != 0;
    const bool has_z = p.z != nullptr;

    const Tin *u_row = static_cast<const Tin *>(p.u) + row * L;
    const Tin *d_row = static_cast<const Tin *>(p.delta) + row * L;
    const Tin *z_row = has_z ? static_cast<const Tin *>(p.z) + row * L : nullptr;
    const Tin *B_b = static_cast<const Tin *>(p.B) + b * N * L;
    const Tin *C_b = static_cast<const Tin *>(p.C) + b * N * L;
    Tout *y_row = static_cast<Tout *>(p.y) + row * L;

    // A[d, n] * log2(e) (0 for the padding states n >= N) and the state
    // entering the chunk.  W = 1: registers (A in registers for up to 16
    // states; more states re-read it, an L1 hit, once per chunk).  W > 1: the
    // per-row shared tables, read by all W lanes of the row.
    constexpr bool kRowInRegs = kW == 1;
    constexpr bool kA2InRegs = kRowInRegs && kNmax <= 16;
    const float *A_d = p.A + d * N;
    float2 A2[kA2InRegs ? kPairs : 1], carry[kRowInRegs ? kPairs : 1];
    const int rloc = warp * kRowsPerWarp + lane / kW;  // row within the block
    float *sCarry = sA2 + rows_per_block * kRowStride;
    const float *rowA2 = sA2 + rloc * kRowStride;
    float *rowCarry = sCarry + rloc * kRowStride;
    if constexpr (kRowInRegs) {
#pragma unroll
        for (int q = 0; q < kPairs; ++q) {
            if constexpr (kA2InRegs)
                A2[q] = make_float2(2 * q < N ? A_d[2 * q] * kLog2e : 0.f,
                                    2 * q + 1 < N ? A_d[2 * q + 1] * kLog2e : 0.f);
            carry[q] = make_float2(0.f, 0.f);
        }
    } else {
        const int64_t d0 = tile * rows_per_block;
        for (int idx = tid; idx < rows_per_block * kNmax; idx += nthreads) {
            const int r = idx / kNmax, n = idx % kNmax;
            const int64_t dr = d0 + r < p.dim ? d0 + r : p.dim - 1;
            sA2[r * kRowStride + n] = n < N ? p.A[dr * N + n] * kLog2e : 0.f;
            sCarry[r * kRowStride + n] = 0.f;
        }
        // (visible after the first __syncthreads of the chunk loop, or the one
        // before the last-state store)
    }
    const float Dd = p.D ? p.D[d] : 0.f;
    const float bias = p.delta_bias ? p.delta_bias[d] : 0.f;

    // The block's B and C for steps [c0, c0 + kChunk): 16-byte async copies
    // into R when the whole chunk is in range and rows are aligned.
    auto chunk_async = [&](int64_t c0) { return vec && c0 + kChunk <= L; };
    auto issue_copies = [&](int64_t c0) {
        for (int u = tid; u < kUnits; u += nthreads) {
            const int j = u % kUnitsPerRow, rowid = u / kUnitsPerRow;
            const int t = rowid / kNmax, n = rowid % kNmax;
            if (n < N)
                cp_async16(R + (rowid * kChunk + j * kUnit),
                           (t ? C_b : B_b) + (int64_t)n * L + c0 + j * kUnit);
        }
        cp_async_commit();
    };
    // One 16-byte unit (kUnit steps) of state n's row, as floats: from R, or
    // element by element from global memory (partial or unaligned chunk);
    // padding states read zeros.
    auto read_unit = [&](int64_t c0, bool from_R, int t, int n, int j, float (&v)[kUnit]) {
        if (n >= N) {
#pragma unroll
            for (int m = 0; m < kUnit; ++m) v[m] = 0.f;
        } else if (from_R) {
            const uint4 raw =
                *reinterpret_cast<const uint4 *>(R + ((t * kNmax + n) * kChunk + j * kUnit));
            const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
            for (int m = 0; m < kUnit; ++m) {
                if constexpr (sizeof(Tin) == 2)
                    v[m] = __uint_as_float((m & 1) ? (w[m >> 1] & 0xffff0000u) : (w[m >> 1] << 16));
                else
                    v[m] = __uint_as_float(w[m]);
            }
        } else {
            const Tin *src = (t ? C_b : B_b) + (int64_t)n * L;
#pragma unroll
            for (int m = 0; m < kUnit; ++m) {
                const int64_t l = c0 + j * kUnit + m;
                uint32_t bits = 0u;
                if (l < L) bits = Io<Tin>::bits(src, l);
                if constexpr (sizeof(Tin) == 2) bits <<= 16;
                v[m] = __uint_as_float(bits);
            }
        }
    };
    // R (or global memory) -> F in the pair-interleaved order.
    auto fill_F = [&](int64_t c0, bool from_R) {
        for (int u = tid; u < kPairUnits; u += nthreads) {
            const int j = u % kUnitsPerRow, pr = u / kUnitsPerRow;  // pr = t * kPairs + pair
            const int t = pr / kPairs, q = pr % kPairs;
            float v0[kUnit], v1[kUnit];
            read_unit(c0, from_R, t, 2 * q, j, v0);
            read_unit(c0, from_R, t, 2 * q + 1, j, v1);
#pragma unroll
            for (int m = 0; m < kUnit; m += 2) {
                const int e = j * kUnit + m;  // step within the chunk (even)
                const int sl = e / kItems, g = (e % kItems) / 2;
                F[(pr * kG + g) * kW + sl] = make_float4(v0[m], v1[m], v0[m + 1], v1[m + 1]);
            }
        }
    };

    uint32_t wu[kWords], wd[kWords], wz[kWords];
    {
        const int64_t l0 = (int64_t)seg * kItems;
        load_run<Tin, true>(wu, u_row, l0, L, vec);
        load_run<Tin, true>(wd, d_row, l0, L, vec);
        if (has_z) load_run<Tin, true>(wz, z_row, l0, L, vec);
    }
    if (L > 0 && chunk_async(0)) issue_copies(0);

    for (int64_t c0 = 0; c0 < L; c0 += kChunk) {
        const bool async_here = chunk_async(c0);
        if (async_here) cp_async_wait_all();
        __syncthreads();  // R holds this chunk; every warp is done with F
        fill_F(c0, async_here);
        __syncthreads();  // F holds this chunk; R is free
        const bool more = c0 + kChunk < L;
        if (more && chunk_async(c0 + kChunk)) issue_copies(c0 + kChunk);

        const int64_t l0 = c0 + (int64_t)seg * kItems;
        float uf[kItems], df[kItems];
        Io<Tin>::widen(wu, uf);
        Io<Tin>::widen(wd, df);
        uint32_t wzc[kWords];
#pragma unroll
        for (int j = 0; j < kWords; ++j) wzc[j] = wz[j];
        if (more) {  // prefetch the next chunk of this lane's steps
            load_run<Tin, true>(wu, u_row, l0 + kChunk, L, vec);
            load_run<Tin, true>(wd, d_row, l0 + kChunk, L, vec);
            if (has_z) load_run<Tin, true>(wz, z_row, l0 + kChunk, L, vec);
        }

        // delta' and delta' * u, duplicated into both halves of a float2 to
        // pair with two states; steps past L become the identity (a = 1, b = 0).
        float dl[kItems];
#pragma unroll
        for (int i = 0; i < kItems; ++i) dl[i] = delta_transform<kFast>(df[i] + bias, softplus);
        if (c0 + kChunk > L) {
#pragma unroll
            for (int i = 0; i < kItems; ++i)
                if (l0 + i >= L) dl[i] = 0.f;
        }
        float2 dl2[kItems], du2[kItems], y2[kItems];
#pragma unroll
        for (int i = 0; i < kItems; ++i) {
            dl2[i] = f2(dl[i]);
            du2[i] = f2(dl[i] * uf[i]);
            y2[i] = make_float2(Dd * uf[i], 0.f);  // skip term D u (§3.3)
        }

        const float4 *FB = F + seg, *FC = F + kPairs * kPairRow + seg;
        // B (or C) of state pair q for this lane's 8 steps: Xp[i] = (X[2q][i], X[2q+1][i]).
        auto load_pair = [&](const float4 *base, int q, float2 (&Xp)[kItems]) {
#pragma unroll
            for (int g = 0; g < kG; ++g) {
                const float4 x = base[(q * kG + g) * kW];
                Xp[2 * g] = make_float2(x.x, x.y);
                Xp[2 * g + 1] = make_float2(x.z, x.w);
            }
        };
        if constexpr (kW == 1) {
#pragma unroll
            for (int q = 0; q < kPairs; ++q) {
                float2 A2q;
                if constexpr (kA2InRegs) A2q = A2[q];
                else A2q = make_float2(2 * q < N ? __ldg(A_d + 2 * q) * kLog2e : 0.f,
                                       2 * q + 1 < N ? __ldg(A_d + 2 * q + 1) * kLog2e : 0.f);
                float2 Bp[kItems], Cp[kItems];
                load_pair(FB, q, Bp);
                load_pair(FC, q, Cp);
                float2 h = carry[q];
#pragma unroll
                for (int i = 0; i < kItems; ++i) {
                    const float2 t = __fmul2_rn(dl2[i], A2q);
                    const float2 a = make_float2(sfu_exp2(t.x), sfu_exp2(t.y));
                    h = __ffma2_rn(a, h, __fmul2_rn(du2[i], Bp[i]));
                    y2[i] = __ffma2_rn(Cp[i], h, y2[i]);
                }
                carry[q] = h;
            }
        } else {
#pragma unroll kPairUnroll
            for (int q = 0; q < kPairs; ++q) {
                const float2 A2q = *reinterpret_cast<const float2 *>(rowA2 + 2 * q);
                const float2 cin = *reinterpret_cast<const float2 *>(rowCarry + 2 * q);
                float2 Bp[kItems];
                load_pair(FB, q, Bp);
                // Pass 1: this lane's steps from a zero state; keep a and delta' u B.
                float2 a[kItems], bb[kItems];
                float2 h = make_float2(0.f, 0.f), P = make_float2(1.f, 1.f);
#pragma unroll
                for (int i = 0; i < kItems; ++i) {
                    const float2 t = __fmul2_rn(dl2[i], A2q);
                    a[i] = make_float2(sfu_exp2(t.x), sfu_exp2(t.y));
                    bb[i] = __fmul2_rn(du2[i], Bp[i]);
                    h = __ffma2_rn(a[i], h, bb[i]);
                    P = __fmul2_rn(P, a[i]);
                }
                // Scan of (P, h) over the row's W lanes.
                {
                    unsigned long long P64 = as_u64(P), h64 = as_u64(h);
#pragma unroll
                    for (int off = 1; off < kW; off <<= 1) scan_stage_x2<kW>(P64, h64, off);
                    P = as_f2(P64);
                    h = as_f2(h64);
                }
                // States after this lane's steps, given the chunk's incoming states.
                const float2 X = __ffma2_rn(P, cin, h);
                const float2 up = make_float2(__shfl_up_sync(kFull, X.x, 1, kW),
                                              __shfl_up_sync(kFull, X.y, 1, kW));
                const float2 hin0 = seg == 0 ? cin : up;
                st_shared_f2_if(rowCarry + 2 * q, X, seg == kW - 1);
                float2 hin = hin0;
                // Pass 2: the true states and y.
                float2 Cp[kItems];
                load_pair(FC, q, Cp);
#pragma unroll
                for (int i = 0; i < kItems; ++i) {
                    hin = __ffma2_rn(a[i], hin, bb[i]);
                    y2[i] = __ffma2_rn(Cp[i], hin, y2[i]);
                }
            }
        }

        float y[kItems];
#pragma unroll
        for (int i = 0; i < kItems; ++i) y[i] = y2[i].x + y2[i].y;
        if (has_z) {
            float zf[kItems];
            Io<Tin>::widen(wzc, zf);
#pragma unroll
            for (int i = 0; i < kItems; ++i) y[i] *= silu<kFast>(zf[i]);
        }
        if (row_ok) store_run(y_row, l0, L, vec, y);
    }

    if (p.last_state != nullptr) {
        if constexpr (kRowInRegs) {
            if (row_ok) {
#pragma unroll
                for (int q = 0; q < kPairs; ++q) {
                    if (2 * q < N) p.last_state[row * N + 2 * q] = carry[q].x;
                    if (2 * q + 1 < N) p.last_state[row * N + 2 * q + 1] = carry[q].y;
                }
            }
        } else {
            __syncthreads();  // the row tables are written (also when L == 0)
            if (row_ok)
                for (int n = seg; n < N; n += kW) p.last_state[row * N + n] = rowCarry[n];
        }
    }
}

}  // namespace selscan
