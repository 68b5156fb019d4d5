// Backward of the selective-scan forward: gradients of sum(dy * y).
//
// The forward is the sequential recurrence of the selective_scan_ref
// walkthrough ("Mamba代码实战：手把手教你用PyTorch复现选择性扫描核心逻辑（附避坑指南）",
// §2.2-§3.3), which trains it through autograd; these kernels are its chain
// rule written out.  With g_l = dy_l silu(z_l) (dy_l without a gate), the
// state's adjoint runs backwards over the steps:
//   lam_ln = g_l C_nl + a_(l+1)n lam_(l+1)n,        a_ln = exp(delta'_l A_n),
// and per row (b, d):
//   dz_l = dy_l s_l silu'(z_l)  (s_l = sum_n C_nl h_ln + D u_l, the gate's input)
//   du_l = g_l D + delta'_l sum_n lam_ln B_nl
//   ddelta'_l = u_l sum_n lam_ln B_nl + sum_n lam_ln a_ln h_(l-1)n A_n
//   ddelta_l = ddelta'_l softplus'(x_l)  (sigmoid(x_l); 1 above 20; delta'_l in exp mode)
//   dA_n += lam_ln a_ln h_(l-1)n delta'_l;  dD += g_l u_l;  dbias += ddelta_l
//   dB_nl += lam_ln delta'_l u_l,  dC_nl += g_l h_ln   (summed over the rows d of batch b)
//
// Layout of the work (state split over kG lanes of a warp, 4 states per lane,
// as in the direct forward kernel):
//   phase A runs the forward over the row and stores the state at the start
//   of every 8-step sub-chunk (checkpoints);
//   phase B walks the stages and their sub-chunks backwards: it recomputes the
//   sub-chunk's decays and states from its checkpoint (kept in registers),
//   runs the adjoint over its 8 steps, sums the per-row terms over the kG
//   lanes and the dB/dC terms over the block's rows in shared memory, and
//   writes per-block partial sums of dB/dC, which a second kernel adds up in
//   a fixed order (with the per-row partials of dA, dD and dbias).
// With sequence starts (p.reset, the forward's (batch, L) mask: the state
// entering a start is zero), h_(l-1) has no part in h_l at a start l: both
// passes zero the state entering it, and the adjoint passes nothing from l to
// l-1 and has no h_(l-1) term there (ddelta', dA).
// From a given state (p.init_state, the forward of ss_fwd_state): phase A
// starts from it, and the adjoint carried past step 0, a_0 lam_0, is the
// gradient with respect to it (p.d_init_state).  With a gradient on the last
// state (p.dlast: the loss also has sum(dlast h_(L-1)), as when the state
// feeds the next piece of a sequence) the adjoint starts from dlast instead
// of zero past the end.
#pragma once

#include <type_traits>

#include "ss_fwd_kernel.cuh"

namespace selscan {

struct BwdParams {
    const void *u, *delta, *B, *C, *z, *dy;   // dy has the dtype of y
    const float *A, *D, *delta_bias;
    void *du, *ddelta, *dz;                   // dtype of u
    float *ckpt;                              // (rows, nsub, dstate) states at sub-chunk starts
    float *ws_dBC;                            // (dtiles, batch, 2, dstate, seqlen) block partials of dB, dC
    float *ws_dA;                             // (rows, dstate) per-row partials of dA
    float *ws_dD, *ws_dbias;                  // (rows) per-row partials
    int64_t batch, dim, seqlen;
    int dstate;
    int softplus;
    int vec;                                  // every row of B and C starts 16-byte aligned
    int vec_rows;                             // every row of u, delta, z and dy starts 16-byte aligned
    int64_t dtiles;                           // row tiles per batch entry
    int64_t nsub;                             // sub-chunks per row
    const uint8_t *reset;                     // (batch, seqlen) sequence starts, or null
    int reset_vec;                            // every 8-step group of reset is 8-byte aligned
    const float *init_state;                  // (batch, dim, dstate) state before step 0, or null (zero)
    const float *dlast;                       // (batch, dim, dstate) gradient wrt the last state, or null
    float *d_init_state;                      // (batch, dim, dstate) gradient wrt the state before step 0, or null
    // Sequence segments (nseg > 1): block (s, b, tile) runs steps
    // [s seg_len, (s + 1) seg_len) from seg_h[s - 1] (the true state entering
    // segment s, s >= 1) and with seg_dl[s] (the adjoint entering its last
    // step from the right, s <= nseg - 2) as its last-state gradient; the
    // per-row partials of dA, dD and dbias are kept per segment, at
    // (s rows_all + row), rows_all the rows of the whole batch.
    int64_t seg_len;
    int nseg;
    int64_t rows_all;
    const float *seg_h;                       // (nseg * seg_h_k, rows, dstate)
    // The entering state of segment s is seg_h[seg_h_k s - 1]: the forward
    // summary may cut each segment into seg_h_k pieces (more blocks).
    int seg_h_k = 1;
    const float *seg_dl;                      // (nseg, rows, dstate)
    // Nonzero: ckpt holds the forward's checkpoints (written by the forward
    // with checkpoints, ss_fwd_ckpt) and phase A is skipped.
    int ckpt_given;
};

constexpr int kBwdSub = 8;                    // steps per sub-chunk
constexpr int kBwdThreads = 128;              // threads per block (4 warps)
constexpr int kBwdStage = 64;                 // steps per B/C stage in shared memory
constexpr int kBwdGather = 3 * kBwdSub + 4;   // floats per row: delta', delta' u, g of 8 steps (+pad)
constexpr int kBwdReduce = 3 * kBwdSub + 4;   // floats per lane: s, sum lam B, sum lam a h A of 8 steps (+pad)

// Lanes per row for the backward: 4 states per lane (16 lanes for 64 states).
__host__ __device__ constexpr int bwd_lanes(int nmax) { return nmax / 4 < 1 ? 1 : nmax / 4; }

// The block's dB/dC terms of a sub-chunk: per (dB or dC, state n) a group of
// 8 steps x (rows + 2) floats, groups `bwd_group_stride` floats apart.  The
// padding puts the lanes of one store instruction (rows r, state groups g) on
// distinct banks, and keeps every row of rows 8-byte aligned for the float2
// reads of the row sums.
__host__ __device__ constexpr int bwd_group_stride(int rows, int g) {
    return kBwdSub * (rows + 2) + (g == 2 ? 4 : g >= 4 ? 2 : 0);
}

__host__ __device__ constexpr size_t bwd_smem_bytes(size_t in_size, int nmax, int warps) {
    const int g = bwd_lanes(nmax);
    const int rows = warps * 32 / g;
    return 4 * sizeof(float) * (size_t)(nmax / 2) * kBwdStage +        // F
           2 * in_size * (size_t)nmax * kBwdStage +                     // RB
           sizeof(float) * (size_t)warps * ((32 / g) * kBwdGather + 32 * kBwdReduce) +
           sizeof(float) * (size_t)2 * nmax * bwd_group_stride(rows, g);  // dB/dC terms of the block's rows
}

// sigmoid(x) = 1 / (1 + exp(-x)); kFast on the SFU.
template <bool kFast>
__device__ __forceinline__ float sigmoid_of(float x) {
    if constexpr (kFast) return sfu_rcp(1.f + sfu_exp2(-x * kLog2e));
    else return 1.f / (1.f + expf(-x));
}

// Three 128-thread blocks per SM (at most 168 registers a thread): with the
// 4-warp blocks of the mamba-130m-shaped layer (384 blocks) that is one wave
// on 148 SMs.  Measured there on an earlier form of the kernel: 1.35 ms
// against 1.77 ms at 255 registers (two blocks per SM); four blocks at 128
// registers (the dB/dC slab summed in two halves to fit) spill 260 bytes and
// take 1.68 ms against 1.01 ms from the forward's checkpoints.
#ifndef SS_BWD_MIN_BLOCKS
#define SS_BWD_MIN_BLOCKS 3
#endif

// Blocks of 128 threads (4 warps).  kReset: the instance that reads p.reset.
// kZ = false: the instance for a scan without the z gate, which leaves out the
// gate input s = sum_n C h (only dz needs it): its products in the
// recomputation and its sums over the row's lanes (genomic-shaped layer:
// 17.70 -> 16.49 ms from the forward's checkpoints, the same bits).
template <typename Tin, typename Tout, int kNmax, bool kReset = false, bool kZ = true>
__global__ void __launch_bounds__(128, SS_BWD_MIN_BLOCKS) ss_bwd_kernel(const BwdParams p) {
    constexpr int kG = bwd_lanes(kNmax);
    constexpr int kPairs = kNmax / 2;
    constexpr int kPL = kPairs / kG;                  // state pairs per lane (2)
    static_assert(kPL * kG == kPairs && kPL >= 1, "whole state pairs per lane");
    // Steps of a sub-chunk owned per lane (their per-row work: delta', the
    // gate, the outputs); with more lanes than steps (16 lanes for 64 states),
    // one lane in every kStride owns one step.
    constexpr int kOwn = kG <= kBwdSub ? kBwdSub / kG : 1;
    constexpr int kStride = kG <= kBwdSub ? 1 : kG / kBwdSub;
    constexpr int kUnit = Io<Tin>::kUnit;
    constexpr int kStageUnits = kBwdStage / kUnit;
    constexpr int kRowsPerWarp = 32 / kG;
    constexpr bool kFast = sizeof(Tin) == 2;
    constexpr int kInWords = (kOwn * (int)sizeof(Tin) + 3) / 4;
    constexpr int kDyWords = (kOwn * (int)sizeof(Tout) + 3) / 4;

    const int tid = threadIdx.x;
    constexpr int nthreads = kBwdThreads;             // the launch uses exactly this block size
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int g = lane % kG;
    const int r = lane / kG;
    constexpr int rows = nthreads / kG;               // rows of the block
    const int rib = tid / kG;                         // this lane's row within the block
    constexpr int RS = rows + 2;                      // floats per step in the block's dB/dC slab
    constexpr int GS = bwd_group_stride(rows, kG);    // floats per (dB or dC, state) group
    const int N = p.dstate;
    const int64_t blocks_per_seg = p.batch * p.dtiles;
    const int seg = (int)(blockIdx.x / blocks_per_seg);
    const int64_t b = (blockIdx.x % blocks_per_seg) / p.dtiles;
    const int64_t dtile = blockIdx.x % p.dtiles;
    const int64_t d_raw = dtile * rows + rib;
    const bool row_ok = d_raw < p.dim;
    const int64_t d = row_ok ? d_raw : p.dim - 1;     // mirrored rows contribute nothing (g = 0)
    const int64_t L = p.seqlen;                       // row length (stride)
    const int64_t row = b * p.dim + d;
    // This block's steps: [c_begin, Lend) (the whole row unless segmented).
    const int64_t c_begin = (int64_t)seg * p.seg_len;
    const int64_t Lend = c_begin + p.seg_len < L ? c_begin + p.seg_len : L;
    const int64_t rows_grp = p.batch * p.dim;         // rows of this launch
    const bool vec = p.vec != 0;
    const bool vrows = p.vec_rows != 0;
    const bool softplus = p.softplus != 0;
    const bool has_z = kZ && p.z != nullptr;

    extern __shared__ float4 smem[];
    float4 *F = smem;                                                   // [kBwdStage][kPairs]
    Tin *RB = reinterpret_cast<Tin *>(smem + kBwdStage * kPairs);        // [2][kNmax][kBwdStage]
    float *slab = reinterpret_cast<float *>(RB + 2 * kNmax * kBwdStage) +
                  warp * (kRowsPerWarp * kBwdGather + 32 * kBwdReduce);
    float *gat = slab + r * kBwdGather;                                 // this row: delta', delta' u, g
    float *red = slab + kRowsPerWarp * kBwdGather;                      // per lane: 3 x 8 partial sums
    float *dbc = reinterpret_cast<float *>(RB + 2 * kNmax * kBwdStage) +
                 (nthreads / 32) * (kRowsPerWarp * kBwdGather + 32 * kBwdReduce);  // [2][kNmax] groups of [8][RS]

    const Tin *Bsrc[2] = {static_cast<const Tin *>(p.B) + b * N * L,
                          static_cast<const Tin *>(p.C) + b * N * L};
    const Tin *u_row = static_cast<const Tin *>(p.u) + row * L;
    const Tin *d_row = static_cast<const Tin *>(p.delta) + row * L;
    const Tin *z_row = has_z ? static_cast<const Tin *>(p.z) + row * L : nullptr;
    const Tout *dy_row = static_cast<const Tout *>(p.dy) + row * L;
    Tin *du_row = static_cast<Tin *>(p.du) + row * L;
    Tin *dd_row = static_cast<Tin *>(p.ddelta) + row * L;
    Tin *dz_row = has_z ? static_cast<Tin *>(p.dz) + row * L : nullptr;
    float *ck_row = p.ckpt + row * p.nsub * N;

    const int q0 = g * kPL;
    const bool owner = g % kStride == 0;
    const int j0 = (g / kStride) * kOwn;              // first owned step within a sub-chunk
    const float *A_d = p.A + d * N;
    float2 A2[kPL], Aln[kPL];                          // A log2(e) and A
#pragma unroll
    for (int qq = 0; qq < kPL; ++qq) {
        const int n = 2 * (q0 + qq);
        Aln[qq] = make_float2(n < N ? A_d[n] : 0.f, n + 1 < N ? A_d[n + 1] : 0.f);
        A2[qq] = make_float2(Aln[qq].x * kLog2e, Aln[qq].y * kLog2e);
    }
    const float Dd = p.D ? p.D[d] : 0.f;
    const float bias = p.delta_bias ? p.delta_bias[d] : 0.f;

    // B/C of a stage: raw copies into RB by cp.async (issued one stage ahead),
    // converted into F (fp32 float4 per step and state pair) at the stage's start.
    auto stage_fast = [&](int64_t c0) { return vec && c0 >= c_begin && c0 + kBwdStage <= Lend; };
    auto issue_copies = [&](int64_t c0) {
        for (int u = tid; u < 2 * kNmax * kStageUnits; u += nthreads) {
            const int j = u % kStageUnits, rowid = u / kStageUnits;
            const int t = rowid / kNmax, n = rowid % kNmax;
            if (n < N)
                cp_async16(RB + (rowid * kBwdStage + j * kUnit), Bsrc[t] + (int64_t)n * L + c0 + j * kUnit);
        }
        cp_async_commit();
    };
    // Make F hold the stage from c0 (its copies were issued earlier when it is
    // fast), then start the copies of the stage from `next` (if any).
    auto load_stage = [&](int64_t c0, int64_t next) {
        const bool fast = stage_fast(c0);
        if (fast) cp_async_wait_all();
        __syncthreads();  // RB holds the stage; every warp is done with F
        for (int jb = tid; jb < kPairs * (kBwdStage / 8); jb += nthreads) {
            const int q = jb % kPairs, i0 = (jb / kPairs) * 8;
            float v[4][8];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int t = c >> 1, n = 2 * q + (c & 1);
                if (n >= N) {
#pragma unroll
                    for (int m = 0; m < 8; ++m) v[c][m] = 0.f;
                } else if (fast) {
                    const Tin *src = RB + (t * kNmax + n) * kBwdStage + i0;
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
#pragma unroll
            for (int m = 0; m < 8; ++m) F[(i0 + m) * kPairs + q] = make_float4(v[0][m], v[1][m], v[2][m], v[3][m]);
        }
        __syncthreads();  // F holds the stage; RB is free
        if (stage_fast(next)) issue_copies(next);
    };
    auto put = [&](Tin *dst, int64_t l, float v) {
        if (l < Lend) dst[l] = static_cast<Tin>(v);
    };

    // This lane's kOwn steps of a row stream from step `so` as raw words (0 past the end).
    auto load_own = [&](const auto *src, int64_t so, uint32_t *w) {
        using T = std::remove_cv_t<std::remove_pointer_t<decltype(src)>>;
        constexpr int kBytes = kOwn * (int)sizeof(T), kWords = (kBytes + 3) / 4;
        if (kBytes >= 4 && vrows && so + kOwn <= Lend) {
            ld_words<kBytes>(src + so, w);
        } else {
#pragma unroll
            for (int j = 0; j < kWords; ++j) w[j] = 0u;
#pragma unroll
            for (int i = 0; i < kOwn; ++i) {
                if (so + i < Lend) {
                    const uint32_t bits = Io<T>::bits(src, so + i);
                    if constexpr (sizeof(T) == 2) w[i >> 1] |= bits << (16 * (i & 1));
                    else w[i] = bits;
                }
            }
        }
    };

    // Start flags of the 8 steps from l0 (one byte each, as two words), read
    // one sub-chunk ahead; every lane of the block reads the same ones.
    const uint8_t *const reset_b = kReset ? p.reset + b * L : nullptr;
    auto load_flags = [&](int64_t l0, uint2 &w) {
        if constexpr (kReset) {
            if (p.reset_vec && l0 + kBwdSub <= Lend) {
                w = __ldg(reinterpret_cast<const uint2 *>(reset_b + l0));
            } else {
                w = make_uint2(0u, 0u);
#pragma unroll
                for (int i = 0; i < kBwdSub; ++i)
                    if (l0 + i < Lend && reset_b[l0 + i] != 0) (i < 4 ? w.x : w.y) |= 1u << (8 * (i & 3));
            }
        }
    };
    // Bit i: a sequence starts at step l0 + i.
    auto flag_bits = [&](uint2 w) {
        uint32_t mask = 0u;
#pragma unroll
        for (int i = 0; i < kBwdSub; ++i)
            if (((i < 4 ? w.x : w.y) >> (8 * (i & 3))) & 0xffu) mask |= 1u << i;
        return mask;
    };
    uint2 wfl = make_uint2(0u, 0u);  // flags of the next sub-chunk

    // ---------------------------------------------------------------- phase A
    float2 h[kPL];
#pragma unroll
    for (int qq = 0; qq < kPL; ++qq) {  // the state before step 0 (mirrored rows: the true row's)
        const int n = 2 * (q0 + qq);
        h[qq] = make_float2(0.f, 0.f);
        // the given state enters segment 0; segment s >= 1 starts from the true carry
        const float *h_src =
            seg == 0 ? p.init_state : p.seg_h + ((int64_t)p.seg_h_k * seg - 1) * rows_grp * N;
        if (h_src != nullptr) {
            if (n < N) h[qq].x = h_src[row * N + n];
            if (n + 1 < N) h[qq].y = h_src[row * N + n + 1];
        }
    }
    uint32_t wu[kInWords], wd[kInWords];  // raw owned inputs of the next sub-chunk
    // With the forward's checkpoints given (p.ckpt_given) there is no phase A.
    if (Lend > c_begin && !p.ckpt_given) {
        load_own(u_row, c_begin + j0, wu);
        load_own(d_row, c_begin + j0, wd);
        load_flags(c_begin, wfl);
        if (stage_fast(c_begin)) issue_copies(c_begin);
    }
    for (int64_t c0 = c_begin; c0 < Lend && !p.ckpt_given; c0 += kBwdStage) {
        load_stage(c0, c0 + kBwdStage < Lend ? c0 + kBwdStage : -1);
        const int nsub = (int)(((Lend - c0 < kBwdStage ? Lend - c0 : kBwdStage) + kBwdSub - 1) / kBwdSub);
#pragma unroll 1
        for (int m = 0; m < nsub; ++m) {
            const int64_t l0 = c0 + m * kBwdSub;
            const int64_t k = l0 / kBwdSub;
#pragma unroll
            for (int qq = 0; qq < kPL; ++qq) {  // (mirrored rows read the true row's checkpoints)
                const int n = 2 * (q0 + qq);
                if (row_ok && n < N) ck_row[k * N + n] = h[qq].x;
                if (row_ok && n + 1 < N) ck_row[k * N + n + 1] = h[qq].y;
            }
#pragma unroll
            for (int i = 0; i < kOwn; ++i) {
                const int64_t l = l0 + j0 + i;
                const float dl = l < Lend ? delta_transform<kFast>(Io<Tin>::widen(wd, i) + bias, softplus) : 0.f;
                if (owner) {
                    gat[j0 + i] = dl;
                    gat[kBwdSub + j0 + i] = dl * Io<Tin>::widen(wu, i);
                }
            }
            const uint32_t starts = kReset ? flag_bits(wfl) : 0u;
            if (l0 + kBwdSub < Lend) {
                load_own(u_row, l0 + kBwdSub + j0, wu);
                load_own(d_row, l0 + kBwdSub + j0, wd);
                load_flags(l0 + kBwdSub, wfl);
            }
            __syncwarp();
            float dl[kBwdSub], du[kBwdSub];
#pragma unroll
            for (int q4 = 0; q4 < kBwdSub / 4; ++q4) {
                const float4 x = reinterpret_cast<const float4 *>(gat)[q4];
                const float4 y = reinterpret_cast<const float4 *>(gat + kBwdSub)[q4];
                dl[4 * q4] = x.x, dl[4 * q4 + 1] = x.y, dl[4 * q4 + 2] = x.z, dl[4 * q4 + 3] = x.w;
                du[4 * q4] = y.x, du[4 * q4 + 1] = y.y, du[4 * q4 + 2] = y.z, du[4 * q4 + 3] = y.w;
            }
            __syncwarp();
            const float4 *Fm = F + (m * kBwdSub) * kPairs + q0;
#pragma unroll
            for (int i = 0; i < kBwdSub; ++i) {
                const float2 d2 = make_float2(dl[i], dl[i]), u2 = make_float2(du[i], du[i]);
#pragma unroll
                for (int qq = 0; qq < kPL; ++qq) {
                    const float4 bc = Fm[i * kPairs + qq];
                    const float2 t = __fmul2_rn(d2, A2[qq]);
                    const float2 a = make_float2(sfu_exp2(t.x), sfu_exp2(t.y));
                    if constexpr (kReset) {
                        if ((starts >> i) & 1u) h[qq] = make_float2(0.f, 0.f);
                    }
                    h[qq] = __ffma2_rn(a, h[qq], __fmul2_rn(u2, make_float2(bc.x, bc.y)));
                }
            }
        }
    }
    __syncthreads();  // every checkpoint is written (mirrored rows read other lanes' ones)

    // This thread's slots of the block's dB/dC sums: output o = (which * kNmax
    // + n) * 8 + i, the slab offset of its row group and the address of step
    // i of its (which, n) row in the block partials (to be indexed by l0).
    constexpr int kOut = 2 * kNmax * kBwdSub;
    constexpr int kOutPer = (kOut + nthreads - 1) / nthreads;
    int out_src[kOutPer], out_i[kOutPer];
    float *out_dst[kOutPer];
#pragma unroll
    for (int k = 0; k < kOutPer; ++k) {
        const int o = tid + k * nthreads;
        const int i = o % kBwdSub, grp = o / kBwdSub;  // grp = which * kNmax + n
        const int which = grp / kNmax, n = grp % kNmax;
        const bool ok = o < kOut && n < N;
        out_src[k] = ok ? grp * GS + i * RS : -1;
        out_i[k] = i;
        out_dst[k] = ok ? p.ws_dBC + (((dtile * p.batch + b) * 2 + which) * N + n) * L + i : nullptr;
    }

    // ---------------------------------------------------------------- phase B
    float2 carry[kPL], dA_acc[kPL];  // carry: a_(l+1) lam_(l+1); past the end, dlast (or zero)
#pragma unroll
    for (int qq = 0; qq < kPL; ++qq) {
        const int n = 2 * (q0 + qq);
        carry[qq] = make_float2(0.f, 0.f), dA_acc[qq] = make_float2(0.f, 0.f);
        // the last segment from the given last-state gradient, the others from
        // the adjoint entering from the right; mirrored rows carry nothing
        const float *c_src = seg == p.nseg - 1 ? p.dlast : p.seg_dl + ((int64_t)seg * rows_grp) * N;
        if (c_src != nullptr && row_ok) {
            if (n < N) carry[qq].x = c_src[row * N + n];
            if (n + 1 < N) carry[qq].y = c_src[row * N + n + 1];
        }
    }
    float dD_acc = 0.f, dbias_acc = 0.f;
    const int64_t nstages = (Lend - c_begin + kBwdStage - 1) / kBwdStage;
    // Prefetched for the next sub-chunk (backwards): its checkpoint and raw owned inputs.
    float2 h0n[kPL];
    uint32_t wz[kInWords], wdy[kDyWords];
    auto prefetch = [&](int64_t l0) {
        const int64_t k = l0 / kBwdSub;
#pragma unroll
        for (int qq = 0; qq < kPL; ++qq) {
            const int n = 2 * (q0 + qq);
            h0n[qq] = make_float2(n < N ? ck_row[k * N + n] : 0.f, n + 1 < N ? ck_row[k * N + n + 1] : 0.f);
        }
        load_own(u_row, l0 + j0, wu);
        load_own(d_row, l0 + j0, wd);
        if (has_z) load_own(z_row, l0 + j0, wz);
        load_own(dy_row, l0 + j0, wdy);
        load_flags(l0, wfl);
    };
    if (Lend > c_begin) prefetch(((Lend - 1) / kBwdSub) * kBwdSub);
    if (p.ckpt_given && nstages > 0) {  // no phase A: start the last stage's copies here
        const int64_t c_last = c_begin + (nstages - 1) * kBwdStage;
        if (stage_fast(c_last)) issue_copies(c_last);
    }
    for (int64_t st = nstages - 1; st >= 0; --st) {
        const int64_t c0 = c_begin + st * kBwdStage;
        if (st == nstages - 1 && !p.ckpt_given) {  // F still holds the last stage from phase A
            if (stage_fast(c0 - kBwdStage)) issue_copies(c0 - kBwdStage);
        } else {
            load_stage(c0, c0 - kBwdStage);
        }
        const int nsub = (int)(((Lend - c0 < kBwdStage ? Lend - c0 : kBwdStage) + kBwdSub - 1) / kBwdSub);
#pragma unroll 1
        for (int m = nsub - 1; m >= 0; --m) {
            const int64_t l0 = c0 + m * kBwdSub;
            // Owned steps: the per-row quantities, shared with the row's lanes.
            float o_u[kOwn], o_x[kOwn], o_dl[kOwn], o_z[kOwn], o_dy[kOwn], o_sg[kOwn], o_g[kOwn];
#pragma unroll
            for (int i = 0; i < kOwn; ++i) {
                const int64_t l = l0 + j0 + i;
                o_u[i] = Io<Tin>::widen(wu, i);
                o_x[i] = Io<Tin>::widen(wd, i) + bias;
                o_dl[i] = l < Lend ? delta_transform<kFast>(o_x[i], softplus) : 0.f;
                o_dy[i] = row_ok ? Io<Tout>::widen(wdy, i) : 0.f;
                o_z[i] = has_z ? Io<Tin>::widen(wz, i) : 0.f;
                o_sg[i] = has_z ? sigmoid_of<kFast>(o_z[i]) : 1.f;
                o_g[i] = has_z ? o_dy[i] * o_z[i] * o_sg[i] : o_dy[i];
                if (owner) {
                    gat[j0 + i] = o_dl[i];
                    gat[kBwdSub + j0 + i] = o_dl[i] * o_u[i];
                    gat[2 * kBwdSub + j0 + i] = o_g[i];
                }
            }
            float2 h0[kPL];
#pragma unroll
            for (int qq = 0; qq < kPL; ++qq) h0[qq] = h0n[qq];
            const uint32_t starts = kReset ? flag_bits(wfl) : 0u;
            if (l0 > c_begin) prefetch(l0 - kBwdSub);
            __syncwarp();
            float dl[kBwdSub], du[kBwdSub], gg[kBwdSub];
#pragma unroll
            for (int q4 = 0; q4 < kBwdSub / 4; ++q4) {
                const float4 x = reinterpret_cast<const float4 *>(gat)[q4];
                const float4 y = reinterpret_cast<const float4 *>(gat + kBwdSub)[q4];
                const float4 w = reinterpret_cast<const float4 *>(gat + 2 * kBwdSub)[q4];
                dl[4 * q4] = x.x, dl[4 * q4 + 1] = x.y, dl[4 * q4 + 2] = x.z, dl[4 * q4 + 3] = x.w;
                du[4 * q4] = y.x, du[4 * q4 + 1] = y.y, du[4 * q4 + 2] = y.z, du[4 * q4 + 3] = y.w;
                gg[4 * q4] = w.x, gg[4 * q4 + 1] = w.y, gg[4 * q4 + 2] = w.z, gg[4 * q4 + 3] = w.w;
            }

            // Recompute the sub-chunk's decays and states from its checkpoint.
            float2 a[kBwdSub][kPL], hs[kBwdSub][kPL];
            float sp[kBwdSub];
            const float4 *Fm = F + (m * kBwdSub) * kPairs + q0;
#pragma unroll
            for (int i = 0; i < kBwdSub; ++i) {
                const float2 d2 = make_float2(dl[i], dl[i]), u2 = make_float2(du[i], du[i]);
                float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                for (int qq = 0; qq < kPL; ++qq) {
                    const float4 bc = Fm[i * kPairs + qq];
                    const float2 t = __fmul2_rn(d2, A2[qq]);
                    a[i][qq] = make_float2(sfu_exp2(t.x), sfu_exp2(t.y));
                    float2 prev = i ? hs[i - 1][qq] : h0[qq];
                    if constexpr (kReset) {
                        if ((starts >> i) & 1u) prev = make_float2(0.f, 0.f);
                    }
                    hs[i][qq] = __ffma2_rn(a[i][qq], prev, __fmul2_rn(u2, make_float2(bc.x, bc.y)));
                    if constexpr (kZ) acc = __ffma2_rn(make_float2(bc.z, bc.w), hs[i][qq], acc);
                }
                sp[i] = acc.x + acc.y;
            }
            // The adjoint over the sub-chunk, last step first.
            // B/C of each step are read two steps ahead: the compiler cannot
            // move a shared-memory load above the dB/dC stores of the steps in
            // between, so without this every read would wait its full latency.
            float lb[kBwdSub], lha[kBwdSub];
            float4 bc_next[kPL], bc_next2[kPL];
#pragma unroll
            for (int qq = 0; qq < kPL; ++qq) bc_next[qq] = Fm[(kBwdSub - 1) * kPairs + qq];
#pragma unroll
            for (int qq = 0; qq < kPL; ++qq) bc_next2[qq] = Fm[(kBwdSub - 2) * kPairs + qq];
#pragma unroll
            for (int i = kBwdSub - 1; i >= 0; --i) {
                const float2 g2 = make_float2(gg[i], gg[i]), u2 = make_float2(du[i], du[i]);
                float2 sLB = make_float2(0.f, 0.f), sLHA = make_float2(0.f, 0.f);
                float4 bc_cur[kPL];
#pragma unroll
                for (int qq = 0; qq < kPL; ++qq) {
                    bc_cur[qq] = bc_next[qq];
                    bc_next[qq] = bc_next2[qq];
                    if (i > 1) bc_next2[qq] = Fm[(i - 2) * kPairs + qq];
                }
#pragma unroll
                for (int qq = 0; qq < kPL; ++qq) {
                    const float4 bc = bc_cur[qq];
                    const float2 lam = __ffma2_rn(g2, make_float2(bc.z, bc.w), carry[qq]);
                    const float2 dCp = __fmul2_rn(g2, hs[i][qq]);
                    const float2 dBp = __fmul2_rn(lam, u2);
                    float2 hp = i ? hs[i - 1][qq] : h0[qq];
                    float2 la = __fmul2_rn(lam, a[i][qq]);   // a lam: the carry to the step before
                    if constexpr (kReset) {
                        if ((starts >> i) & 1u) hp = make_float2(0.f, 0.f), la = make_float2(0.f, 0.f);
                    }
                    const float2 t = __fmul2_rn(la, hp);             // lam a h_prev
                    sLB = __ffma2_rn(lam, make_float2(bc.x, bc.y), sLB);
                    sLHA = __ffma2_rn(t, Aln[qq], sLHA);
                    dA_acc[qq] = __ffma2_rn(t, make_float2(dl[i], dl[i]), dA_acc[qq]);
                    carry[qq] = la;
                    const int n = 2 * (q0 + qq);
                    float *slot = dbc + i * RS + rib;
                    slot[n * GS] = dBp.x;
                    slot[(n + 1) * GS] = dBp.y;
                    slot[(kNmax + n) * GS] = dCp.x;
                    slot[(kNmax + n + 1) * GS] = dCp.y;
                }
                lb[i] = sLB.x + sLB.y;
                lha[i] = sLHA.x + sLHA.y;
            }
            // Per-row sums over the row's lanes: s (minus D u), sum lam B, sum lam a h A.
            float4 *mine = reinterpret_cast<float4 *>(red + lane * kBwdReduce);
#pragma unroll
            for (int q4 = 0; q4 < kBwdSub / 4; ++q4) {
                if constexpr (kZ) mine[q4] = make_float4(sp[4 * q4], sp[4 * q4 + 1], sp[4 * q4 + 2], sp[4 * q4 + 3]);
                mine[kBwdSub / 4 + q4] = make_float4(lb[4 * q4], lb[4 * q4 + 1], lb[4 * q4 + 2], lb[4 * q4 + 3]);
                mine[kBwdSub / 2 + q4] = make_float4(lha[4 * q4], lha[4 * q4 + 1], lha[4 * q4 + 2], lha[4 * q4 + 3]);
            }
            __syncwarp();
            // Sums over the row's lanes of this lane's owned steps (vector reads).
            constexpr int kRV = kOwn >= 4 ? 4 : kOwn;
            float sS[kOwn], sB[kOwn], sH[kOwn];
#pragma unroll
            for (int i = 0; i < kOwn; ++i) sS[i] = 0.f, sB[i] = 0.f, sH[i] = 0.f;
#pragma unroll
            for (int q = 0; q < kG; ++q) {
                const float *src = red + (r * kG + q) * kBwdReduce + j0;
#pragma unroll
                for (int i = 0; i < kOwn; i += kRV) {
                    float v0[kRV] = {}, v1[kRV], v2[kRV];
                    if constexpr (kZ) ld_vec<kRV>(src + i, v0);
                    ld_vec<kRV>(src + kBwdSub + i, v1);
                    ld_vec<kRV>(src + 2 * kBwdSub + i, v2);
#pragma unroll
                    for (int e = 0; e < kRV; ++e) sS[i + e] += v0[e], sB[i + e] += v1[e], sH[i + e] += v2[e];
                }
            }
#pragma unroll
            for (int i = 0; i < kOwn; ++i) {
                const int j = j0 + i;
                float s = sS[i];
                const float LB = sB[i], LHA = sH[i];
                const int64_t l = l0 + j;
                s = fmaf(Dd, o_u[i], s);
                const float ddl = fmaf(o_u[i], LB, LHA);
                const float dx = softplus ? (o_x[i] > 20.f ? ddl : ddl * sigmoid_of<kFast>(o_x[i])) : ddl * o_dl[i];
                if (owner && row_ok && l < Lend) {
                    put(du_row, l, fmaf(o_g[i], Dd, o_dl[i] * LB));
                    put(dd_row, l, dx);
                    if (has_z) put(dz_row, l, o_dy[i] * s * o_sg[i] * fmaf(o_z[i], 1.f - o_sg[i], 1.f));
                    dD_acc = fmaf(o_g[i], o_u[i], dD_acc);
                    dbias_acc += dx;
                }
            }
            // dB, dC of the sub-chunk summed over the block's rows (row pairs as float2);
            // this thread's output slots and their addresses are fixed (set up once).
            __syncthreads();
#pragma unroll
            for (int k = 0; k < kOutPer; ++k) {
                if (out_src[k] < 0) continue;
                const float2 *src = reinterpret_cast<const float2 *>(dbc + out_src[k]);
                float2 s2 = make_float2(0.f, 0.f);
                float2 t2 = make_float2(0.f, 0.f);  // two partial sums in flight
#pragma unroll
                for (int q = 0; q < rows / 2; q += 2) {
                    s2 = __fadd2_rn(s2, src[q]);
                    if (q + 1 < rows / 2) t2 = __fadd2_rn(t2, src[q + 1]);
                }
                s2 = __fadd2_rn(s2, t2);
                if (l0 + out_i[k] < Lend) out_dst[k][l0] = s2.x + s2.y;
            }
            __syncthreads();  // the slabs are free for the next sub-chunk
        }
    }

    // The adjoint carried past step 0 is the gradient wrt the state before it.
    if (p.d_init_state != nullptr && row_ok && seg == 0) {
#pragma unroll
        for (int qq = 0; qq < kPL; ++qq) {
            const int n = 2 * (q0 + qq);
            if (n < N) p.d_init_state[row * N + n] = carry[qq].x;
            if (n + 1 < N) p.d_init_state[row * N + n + 1] = carry[qq].y;
        }
    }
    // Per-row partials of dA, dD and dbias (per segment).
    const int64_t prow = (int64_t)seg * p.rows_all + row;
    if (row_ok) {
#pragma unroll
        for (int qq = 0; qq < kPL; ++qq) {
            const int n = 2 * (q0 + qq);
            if (n < N) p.ws_dA[prow * N + n] = dA_acc[qq].x;
            if (n + 1 < N) p.ws_dA[prow * N + n + 1] = dA_acc[qq].y;
        }
    }
    if constexpr (kG > 1) {
#pragma unroll
        for (int sdist = 1; sdist < kG; sdist *= 2) {
            dD_acc += __shfl_xor_sync(0xffffffffu, dD_acc, sdist, kG);
            dbias_acc += __shfl_xor_sync(0xffffffffu, dbias_acc, sdist, kG);
        }
    }
    if (row_ok && g == 0) {
        p.ws_dD[prow] = dD_acc;
        p.ws_dbias[prow] = dbias_acc;
    }
}

// ------------------------------------------------------ sequence segments
// For few rows and a long sequence the backward runs each row's sequence as
// nseg segments, as extra rows.  Segment s needs the true state entering it
// and the adjoint entering its last step from the right; both come from
// per-segment summaries, folded across the segments in order:
//  - forward: h_end(s), the state at the end of s from a zero state, and
//    P(s) = 2^(A log2e sum_s delta') (0 if s holds a sequence start), written
//    by the forward direct kernel in its segment mode without y; the fold
//    h_in(s) = P(s-1) h_in(s-1) + h_end(s-1) is the forward's carry kernel;
//  - backward: lam0(s), the adjoint carried past the first step of s when the
//    adjoint past its last step is zero (the recurrence lam_l = g_l C_l +
//    a_(l+1) lam_(l+1) does not involve the state); the fold
//    D(nseg-1) = dlast (or 0), D(s-1) = lam0(s) + P(s) D(s) gives segment
//    s's last-state gradient D(s).
// ss_bwd_seg_adjoint_kernel computes lam0(s) for s >= 1: one thread per
// (segment, row, group of up to 8 states), the steps backwards 8 at a time
// (vector loads when the rows are 16-byte aligned), exps on the SFU; it also
// records each segment's delta' sum (-1 with a start) for the fold, so the
// fold needs no forward pass when the forward's checkpoints are given.
template <typename Tin, typename Tout, int kNmax>
__global__ void __launch_bounds__(128, 3) ss_bwd_seg_adjoint_kernel(const BwdParams p, float *lam0, float *dsum) {
    constexpr bool kFast = sizeof(Tin) == 2;
    constexpr int kS = kNmax < 8 ? kNmax : 8;          // states per thread
    constexpr int kT = kNmax / kS;                      // threads per (segment, row)
    constexpr int kP = kS / 2 > 0 ? kS / 2 : 1;         // state pairs per thread
    constexpr int kWin = 8 * (int)sizeof(Tin) / 4;      // words of 8 steps of an input row
    constexpr int kWout = 8 * (int)sizeof(Tout) / 4;    // words of 8 steps of dy
    const int64_t rows = p.batch * p.dim;
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int q = (int)(t % kT);
    const int64_t rs = t / kT;
    if (rs >= rows * (p.nseg - 1)) return;
    const int64_t row = rs % rows;
    const int s = 1 + (int)(rs / rows);
    const int64_t b = row / p.dim, d = row % p.dim;
    const int N = p.dstate;
    const int64_t L = p.seqlen;
    const int64_t c_begin = (int64_t)s * p.seg_len;
    const int64_t Lend = c_begin + p.seg_len < L ? c_begin + p.seg_len : L;
    const bool softplus = p.softplus != 0;
    const bool has_z = p.z != nullptr;
    const float bias = p.delta_bias ? p.delta_bias[d] : 0.f;
    float2 A2[kP], carry[kP];
#pragma unroll
    for (int k = 0; k < kP; ++k) {
        const int n = q * kS + 2 * k;
        A2[k] = make_float2(n < N ? p.A[d * N + n] * kLog2e : 0.f, n + 1 < N ? p.A[d * N + n + 1] * kLog2e : 0.f);
        carry[k] = make_float2(0.f, 0.f);
    }
    const Tin *d_row = static_cast<const Tin *>(p.delta) + row * L;
    const Tin *z_row = has_z ? static_cast<const Tin *>(p.z) + row * L : nullptr;
    const Tout *dy_row = static_cast<const Tout *>(p.dy) + row * L;
    const Tin *C_b = static_cast<const Tin *>(p.C) + b * N * L;
    const uint8_t *reset_b = p.reset ? p.reset + b * L : nullptr;
    const bool vrows = p.vec_rows != 0, vbc = p.vec != 0;

    // The raw words of a group of 8 steps [l0, l0 + 8): delta, z, dy, this
    // thread's C rows, start flags (zero past the segment's end).  The group
    // before (in time) is loaded while this one is computed.
    struct Raw {
        uint32_t d[kWin], z[kWin], dy[kWout], c[2 * kP][kWin];
        uint32_t st;
    };
    auto load_row = [&](const auto *src, int64_t l0, bool vec_ok, uint32_t *w, auto words) {
        using T = std::remove_cv_t<std::remove_pointer_t<decltype(src)>>;
        constexpr int kW = decltype(words)::value;
        if (vec_ok && l0 + 8 <= Lend) {
            ld_words<8 * (int)sizeof(T)>(src + l0, w);
        } else {
#pragma unroll
            for (int k = 0; k < kW; ++k) w[k] = 0u;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (l0 + i < Lend) {
                    const uint32_t bits = Io<T>::bits(src, l0 + i);
                    if constexpr (sizeof(T) == 2) w[i >> 1] |= bits << (16 * (i & 1));
                    else w[i] = bits;
                }
            }
        }
    };
    auto load_group = [&](int64_t l0, Raw &r) {
        load_row(d_row, l0, vrows, r.d, std::integral_constant<int, kWin>{});
        if (has_z) load_row(z_row, l0, vrows, r.z, std::integral_constant<int, kWin>{});
        load_row(dy_row, l0, vrows, r.dy, std::integral_constant<int, kWout>{});
#pragma unroll
        for (int k = 0; k < 2 * kP; ++k) {
            const int n = q * kS + k;
            if (n < N) {
                load_row(C_b + (int64_t)n * L, l0, vbc, r.c[k], std::integral_constant<int, kWin>{});
            } else {
#pragma unroll
                for (int w = 0; w < kWin; ++w) r.c[k][w] = 0u;
            }
        }
        r.st = 0u;
        if (reset_b != nullptr) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (l0 + i < Lend && reset_b[l0 + i] != 0) r.st |= 1u << i;
        }
    };

    // Groups of 8 steps, the last one first (c_begin is a multiple of 64, so
    // every group starts on a multiple of 8).
    int64_t l0 = ((Lend - 1) / 8) * 8;
    Raw nxt;
    load_group(l0, nxt);
    float dl_sum = 0.f;      // delta' over the segment (its decay product's exponent)
    uint32_t any_start = 0u;  // a sequence start inside the segment
    for (; l0 >= c_begin; l0 -= 8) {
        const Raw cur = nxt;
        any_start |= cur.st;
        if (l0 - 8 >= c_begin) load_group(l0 - 8, nxt);
        float dl[8], g[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const bool in = l0 + i < Lend;
            const float x = Io<Tin>::widen(cur.d, i) + bias;
            const float dyv = Io<Tout>::widen(cur.dy, i);
            dl[i] = in ? delta_transform<kFast>(x, softplus) : 0.f;
            dl_sum += dl[i];
            if (has_z) {
                const float zv = Io<Tin>::widen(cur.z, i);
                g[i] = dyv * zv * sigmoid_of<kFast>(zv);
            } else {
                g[i] = dyv;
            }
        }
        // lam_l = g_l C_l + carry; carry = a_l lam_l (nothing past a start).
#pragma unroll
        for (int i = 7; i >= 0; --i) {
            const float2 d2 = make_float2(dl[i], dl[i]), g2 = make_float2(g[i], g[i]);
            const bool st = (cur.st >> i) & 1u;
#pragma unroll
            for (int k = 0; k < kP; ++k) {
                const float2 cv = make_float2(Io<Tin>::widen(cur.c[2 * k], i), Io<Tin>::widen(cur.c[2 * k + 1], i));
                const float2 lam = __ffma2_rn(g2, cv, carry[k]);
                const float2 tt = __fmul2_rn(d2, A2[k]);
                carry[k] = st ? make_float2(0.f, 0.f) : __fmul2_rn(make_float2(sfu_exp2(tt.x), sfu_exp2(tt.y)), lam);
            }
        }
    }
#pragma unroll
    for (int k = 0; k < kP; ++k) {
        const int n = q * kS + 2 * k;
        if (n < N) lam0[((int64_t)s * rows + row) * N + n] = carry[k].x;
        if (n + 1 < N) lam0[((int64_t)s * rows + row) * N + n + 1] = carry[k].y;
    }
    // the segment's record for the backward fold (-1: it passes nothing on)
    if (q == 0) dsum[(int64_t)s * rows + row] = any_start != 0u ? -1.f : dl_sum;
}

// The backward fold: D(nseg-1) = dlast (or 0); D(s-1) = lam0(s) + P(s) D(s),
// P(s) = 2^(A log2e dsum(s)), 0 where dsum(s) < 0 (a start in s).  One warp
// per row, states over lanes; D(s) written for s <= nseg - 2.
template <int kNmax>
__global__ void __launch_bounds__(256) ss_bwd_seg_fold_kernel(const BwdParams p, const float *lam0,
                                                              const float *dsum, float *D) {
    constexpr int kPer = kNmax > 32 ? 2 : 1;
    const int64_t rows = p.batch * p.dim;
    const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const int64_t d = row % p.dim;
    const int N = p.dstate;
    float A2[kPer], v[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        const int n = lane + 32 * k;
        A2[k] = n < N ? p.A[d * N + n] * kLog2e : 0.f;
        v[k] = n < N && p.dlast != nullptr ? p.dlast[row * N + n] : 0.f;
    }
    for (int s = p.nseg - 1; s >= 1; --s) {
        const float ds = dsum[(int64_t)s * rows + row];
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const int n = lane + 32 * k;
            if (n < N) {
                v[k] = fmaf(ds < 0.f ? 0.f : sfu_exp2(A2[k] * ds), v[k], lam0[((int64_t)s * rows + row) * N + n]);
                D[((int64_t)(s - 1) * rows + row) * N + n] = v[k];
            }
        }
    }
}

// dB, dC = the block partials summed over the row tiles, in tile order.  With
// whole float4 rows (N L a multiple of 4, 16-byte aligned buffers) a thread
// sums four consecutive outputs and keeps eight tiles' loads in flight (each
// output still adds its tiles in order, so the bits do not change; the plain
// form ran at 2 TB/s, waiting on one load at a time).
static __global__ void __launch_bounds__(256) ss_bwd_reduce_bc_kernel(const BwdParams p, float *dB, float *dC) {
    const int64_t per = (int64_t)p.dstate * p.seqlen;
    const int64_t total = p.batch * 2 * per;
    const bool vec4 = per % 4 == 0 && ((reinterpret_cast<uintptr_t>(p.ws_dBC) | reinterpret_cast<uintptr_t>(dB) |
                                        reinterpret_cast<uintptr_t>(dC)) & 15u) == 0;
    if (vec4) {  // four consecutive outputs per thread, eight tiles' loads in flight
        const int64_t per4 = per / 4, tstride = p.batch * 2 * per4;
        const float4 *src = reinterpret_cast<const float4 *>(p.ws_dBC);
        for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total / 4;
             e += (int64_t)gridDim.x * blockDim.x) {
            const int64_t b = e / (2 * per4), which = (e / per4) % 2, q = e % per4;
            const float4 *t0 = src + (b * 2 + which) * per4 + q;
            float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
            int64_t t = 0;
            for (; t + 8 <= p.dtiles; t += 8) {
                float4 v[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) v[k] = __ldcs(t0 + (t + k) * tstride);
#pragma unroll
                for (int k = 0; k < 8; ++k) s.x += v[k].x, s.y += v[k].y, s.z += v[k].z, s.w += v[k].w;
            }
            for (; t < p.dtiles; ++t) {
                const float4 v = __ldcs(t0 + t * tstride);
                s.x += v.x, s.y += v.y, s.z += v.z, s.w += v.w;
            }
            reinterpret_cast<float4 *>(which ? dC : dB)[b * per4 + q] = s;
        }
        return;
    }
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t b = e / (2 * per), which = (e / per) % 2, nl = e % per;
        float s = 0.f;
        for (int64_t t = 0; t < p.dtiles; ++t) s += p.ws_dBC[((t * p.batch + b) * 2 + which) * per + nl];
        (which ? dC : dB)[b * per + nl] = s;
    }
}

// dA, dD, dbias = the per-row partials summed over the segments and the
// batch, in (segment, batch) order.
static __global__ void __launch_bounds__(256) ss_bwd_reduce_rows_kernel(const BwdParams p, float *dA, float *dD,
                                                                  float *dbias) {
    const int64_t N = p.dstate;
    const int64_t total = p.dim * (N + 2);
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        if (e < p.dim * N) {
            float s = 0.f;
            for (int sg = 0; sg < p.nseg; ++sg)
                for (int64_t b = 0; b < p.batch; ++b) s += p.ws_dA[((int64_t)sg * p.rows_all + b * p.dim) * N + e];
            dA[e] = s;
        } else {
            const int64_t j = e - p.dim * N, d = j % p.dim;
            const bool is_bias = j >= p.dim;
            float *out = is_bias ? dbias : dD;
            if (out == nullptr) continue;
            const float *src = is_bias ? p.ws_dbias : p.ws_dD;
            float s = 0.f;
            for (int sg = 0; sg < p.nseg; ++sg)
                for (int64_t b = 0; b < p.batch; ++b) s += src[(int64_t)sg * p.rows_all + b * p.dim + d];
            out[d] = s;
        }
    }
}

}  // namespace selscan
