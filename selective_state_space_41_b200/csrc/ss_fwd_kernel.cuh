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

// delta' of §2.2: torch's softplus (beta 1, linear above 20) or exp.
__device__ __forceinline__ float delta_transform(float x, bool softplus) {
    if (softplus) return x > 20.f ? x : log1pf(expf(x));
    return expf(x);
}

// silu(z) = z * sigmoid(z) (§3.3).
__device__ __forceinline__ float silu(float z) { return z / (1.f + expf(-z)); }

// ------------------------------------------------------------------- kernel
// Up to 256 threads per block.  For up to 32 states the register budget is
// capped at 128 per thread (two 256-thread blocks per SM); 64 states keep
// their 64 carries in registers and take up to 255.
template <int kNmax>
struct Occupancy {
    static constexpr int kMinBlocks = kNmax <= 32 ? 2 : 1;
};

template <typename Tin, typename Tout, int kNmax, int kW>
__global__ void __launch_bounds__(256, Occupancy<kNmax>::kMinBlocks) ss_fwd_kernel(const FwdParams p) {
    static_assert(kW >= 1 && kW <= 32 && (32 % kW) == 0, "lanes per row must divide 32");
    constexpr int kRowsPerWarp = 32 / kW;
    constexpr int kChunk = kW * kItems;
    constexpr int kWords = Io<Tin>::kWords;
    constexpr unsigned kFull = 0xffffffffu;

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int seg = lane % kW;  // this lane's slot among the row's W lanes
    const int64_t rows_per_block = (int64_t)(blockDim.x >> 5) * kRowsPerWarp;
    const int64_t b = blockIdx.x / p.dtiles;
    const int64_t tile = blockIdx.x % p.dtiles;
    const int64_t d_raw = tile * rows_per_block + warp * kRowsPerWarp + lane / kW;
    // Rows past the end mirror the last row (valid addresses) and store nothing;
    // they must still run so that every lane takes part in the shuffles.
    const bool row_ok = d_raw < p.dim;
    const int64_t d = row_ok ? d_raw : p.dim - 1;
    const int N = p.dstate;
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

    // A[d, n] * log2(e), held in registers for up to 16 states; more states
    // re-read it (an L1 hit) once per chunk to leave room for the carries.
    constexpr bool kA2InRegs = kNmax <= 16;
    const float *A_d = p.A + d * N;
    float A2[kA2InRegs ? kNmax : 1], carry[kNmax];
#pragma unroll
    for (int n = 0; n < kNmax; ++n) {
        if constexpr (kA2InRegs) A2[n] = n < N ? A_d[n] * kLog2e : 0.f;
        carry[n] = 0.f;
    }
    const float Dd = p.D ? p.D[d] : 0.f;
    const float bias = p.delta_bias ? p.delta_bias[d] : 0.f;

    uint32_t wu[kWords], wd[kWords], wz[kWords];
    {
        const int64_t l0 = (int64_t)seg * kItems;
        load_run<Tin, true>(wu, u_row, l0, L, vec);
        load_run<Tin, true>(wd, d_row, l0, L, vec);
        if (has_z) load_run<Tin, true>(wz, z_row, l0, L, vec);
    }

    for (int64_t c0 = 0; c0 < L; c0 += kChunk) {
        const int64_t l0 = c0 + (int64_t)seg * kItems;
        float uf[kItems], df[kItems], zf[kItems];
        Io<Tin>::widen(wu, uf);
        Io<Tin>::widen(wd, df);
        if (has_z) Io<Tin>::widen(wz, zf);
        if (c0 + kChunk < L) {  // prefetch the next chunk
            load_run<Tin, true>(wu, u_row, l0 + kChunk, L, vec);
            load_run<Tin, true>(wd, d_row, l0 + kChunk, L, vec);
            if (has_z) load_run<Tin, true>(wz, z_row, l0 + kChunk, L, vec);
        }

        // delta' and delta' * u; steps past L become the identity (a = 1, b = 0).
        float dl[kItems], du[kItems], y[kItems];
#pragma unroll
        for (int i = 0; i < kItems; ++i) {
            const float v = delta_transform(df[i] + bias, softplus);
            dl[i] = (l0 + i < L) ? v : 0.f;
            du[i] = dl[i] * uf[i];
            y[i] = 0.f;
        }

#pragma unroll
        for (int n = 0; n < kNmax; ++n) {
            if (n < N) {
                float A2n;
                if constexpr (kA2InRegs) A2n = A2[n];
                else A2n = __ldg(A_d + n) * kLog2e;
                uint32_t wb[kWords], wc[kWords];
                load_run<Tin, false>(wb, B_b + (int64_t)n * L, l0, L, vec);
                load_run<Tin, false>(wc, C_b + (int64_t)n * L, l0, L, vec);
                float Bv[kItems], Cv[kItems];
                Io<Tin>::widen(wb, Bv);
                Io<Tin>::widen(wc, Cv);
                if constexpr (kW == 1) {
                    float h = carry[n];
#pragma unroll
                    for (int i = 0; i < kItems; ++i) {
                        const float a = sfu_exp2(dl[i] * A2n);
                        h = fmaf(a, h, du[i] * Bv[i]);
                        y[i] = fmaf(Cv[i], h, y[i]);
                    }
                    carry[n] = h;
                } else {
                    float a[kItems], bb[kItems];
                    float h = 0.f, P = 1.f;
#pragma unroll
                    for (int i = 0; i < kItems; ++i) {
                        a[i] = sfu_exp2(dl[i] * A2n);
                        bb[i] = du[i] * Bv[i];
                        h = fmaf(a[i], h, bb[i]);
                        P *= a[i];
                    }
                    // Inclusive scan of (P, h) over the row's W lanes.
#pragma unroll
                    for (int off = 1; off < kW; off <<= 1) {
                        const float Pu = __shfl_up_sync(kFull, P, off, kW);
                        const float hu = __shfl_up_sync(kFull, h, off, kW);
                        if (seg >= off) {
                            h = fmaf(P, hu, h);
                            P *= Pu;
                        }
                    }
                    // State after this lane's steps, given the chunk's incoming state.
                    const float X = fmaf(P, carry[n], h);
                    float hin = __shfl_up_sync(kFull, X, 1, kW);
                    if (seg == 0) hin = carry[n];
                    carry[n] = __shfl_sync(kFull, X, kW - 1, kW);
#pragma unroll
                    for (int i = 0; i < kItems; ++i) {
                        hin = fmaf(a[i], hin, bb[i]);
                        y[i] = fmaf(Cv[i], hin, y[i]);
                    }
                }
            }
        }

#pragma unroll
        for (int i = 0; i < kItems; ++i) {
            float v = fmaf(Dd, uf[i], y[i]);
            if (has_z) v *= silu(zf[i]);
            y[i] = v;
        }
        if (row_ok) store_run(y_row, l0, L, vec, y);
    }

    if (p.last_state != nullptr && row_ok) {
#pragma unroll
        for (int n = 0; n < kNmax; ++n)
            if (n < N && (n % kW) == seg) p.last_state[row * N + n] = carry[n];
    }
}

}  // namespace selscan
