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
#pragma once

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
    int vec;                                  // every row of u/delta/z/dy/du/ddelta/dz starts 16-byte aligned
    int64_t dtiles;                           // row tiles per batch entry
    int64_t nsub;                             // sub-chunks per row
};

constexpr int kBwdSub = 8;                    // steps per sub-chunk
constexpr int kBwdStage = 64;                 // steps per B/C stage in shared memory
constexpr int kBwdGather = 3 * kBwdSub + 4;   // floats per row: delta', delta' u, g of 8 steps (+pad)
constexpr int kBwdReduce = 3 * kBwdSub + 1;   // floats per lane: s, sum lam B, sum lam a h A of 8 steps (+pad)

// Lanes per row for the backward: 4 states per lane.
__host__ __device__ constexpr int bwd_lanes(int nmax) { return nmax / 4 < 1 ? 1 : nmax / 4; }

__host__ __device__ constexpr size_t bwd_smem_bytes(size_t in_size, int nmax, int warps) {
    const int g = bwd_lanes(nmax);
    const int rows = warps * 32 / g;
    return 4 * sizeof(float) * (size_t)(nmax / 2) * kBwdStage +        // F
           2 * in_size * (size_t)nmax * kBwdStage +                     // RB
           sizeof(float) * (size_t)warps * ((32 / g) * kBwdGather + 32 * kBwdReduce) +
           sizeof(float) * (size_t)2 * kBwdSub * nmax * (rows + 2);     // dB/dC terms of the block's rows
}

// sigmoid(x) = 1 / (1 + exp(-x)); kFast on the SFU.
template <bool kFast>
__device__ __forceinline__ float sigmoid_of(float x) {
    if constexpr (kFast) return sfu_rcp(1.f + sfu_exp2(-x * kLog2e));
    else return 1.f / (1.f + expf(-x));
}

template <typename Tin, typename Tout, int kNmax>
__global__ void __launch_bounds__(256) ss_bwd_kernel(const BwdParams p) {
    constexpr int kG = bwd_lanes(kNmax);
    constexpr int kPairs = kNmax / 2;
    constexpr int kPL = kPairs / kG;                  // state pairs per lane (2)
    static_assert(kPL * kG == kPairs && kPL >= 1, "whole state pairs per lane");
    constexpr int kOwn = kBwdSub / kG;                // steps owned per lane per sub-chunk
    static_assert(kOwn >= 1, "at most 8 lanes per row");
    constexpr int kUnit = Io<Tin>::kUnit;
    constexpr int kStageUnits = kBwdStage / kUnit;
    constexpr int kRowsPerWarp = 32 / kG;
    constexpr bool kFast = sizeof(Tin) == 2;

    const int tid = threadIdx.x;
    const int nthreads = blockDim.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int g = lane % kG;
    const int r = lane / kG;
    const int rows = nthreads / kG;                   // rows of the block
    const int rib = tid / kG;                         // this lane's row within the block
    const int RS = rows + 2;                          // stride of the block's dB/dC slab
    const int N = p.dstate;
    const int64_t b = blockIdx.x / p.dtiles;
    const int64_t dtile = blockIdx.x % p.dtiles;
    const int64_t d_raw = dtile * rows + rib;
    const bool row_ok = d_raw < p.dim;
    const int64_t d = row_ok ? d_raw : p.dim - 1;     // mirrored rows contribute nothing (g = 0)
    const int64_t L = p.seqlen;
    const int64_t row = b * p.dim + d;
    const bool vec = p.vec != 0;
    const bool softplus = p.softplus != 0;
    const bool has_z = p.z != nullptr;

    extern __shared__ float4 smem[];
    float4 *F = smem;                                                   // [kBwdStage][kPairs]
    Tin *RB = reinterpret_cast<Tin *>(smem + kBwdStage * kPairs);        // [2][kNmax][kBwdStage]
    float *slab = reinterpret_cast<float *>(RB + 2 * kNmax * kBwdStage) +
                  warp * (kRowsPerWarp * kBwdGather + 32 * kBwdReduce);
    float *gat = slab + r * kBwdGather;                                 // this row: delta', delta' u, g
    float *red = slab + kRowsPerWarp * kBwdGather;                      // per lane: 3 x 8 partial sums
    float *dbc = reinterpret_cast<float *>(RB + 2 * kNmax * kBwdStage) +
                 (nthreads / 32) * (kRowsPerWarp * kBwdGather + 32 * kBwdReduce);  // [2][8][kNmax][RS]

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

    // B/C of the stage from c0 into F (fp32 float4 per step and state pair).
    auto load_stage = [&](int64_t c0) {
        const bool fast = vec && c0 + kBwdStage <= L;
        __syncthreads();  // every warp is done with F (and RB)
        if (fast) {
            for (int u = tid; u < 2 * kNmax * kStageUnits; u += nthreads) {
                const int j = u % kStageUnits, rowid = u / kStageUnits;
                const int t = rowid / kNmax, n = rowid % kNmax;
                if (n < N)
                    cp_async16(RB + (rowid * kBwdStage + j * kUnit), Bsrc[t] + (int64_t)n * L + c0 + j * kUnit);
            }
            cp_async_commit();
            cp_async_wait_all();
            __syncthreads();
        }
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
                        if (l < L) bits = Io<Tin>::bits(src, l);
                        if constexpr (sizeof(Tin) == 2) bits <<= 16;
                        v[c][m] = __uint_as_float(bits);
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < 8; ++m) F[(i0 + m) * kPairs + q] = make_float4(v[0][m], v[1][m], v[2][m], v[3][m]);
        }
        __syncthreads();  // F holds the stage
    };
    // One input element as float (0 past the end).
    auto in_at = [&](const Tin *src, int64_t l) -> float {
        if (l >= L) return 0.f;
        uint32_t bits = Io<Tin>::bits(src, l);
        if constexpr (sizeof(Tin) == 2) bits <<= 16;
        return __uint_as_float(bits);
    };
    auto dy_at = [&](int64_t l) -> float {
        if (l >= L) return 0.f;
        return static_cast<float>(dy_row[l]);
    };
    auto put = [&](Tin *dst, int64_t l, float v) {
        if (l < L) dst[l] = static_cast<Tin>(v);
    };

    // ---------------------------------------------------------------- phase A
    float2 h[kPL];
#pragma unroll
    for (int qq = 0; qq < kPL; ++qq) h[qq] = make_float2(0.f, 0.f);
    for (int64_t c0 = 0; c0 < L; c0 += kBwdStage) {
        load_stage(c0);
        const int nsub = (int)(((L - c0 < kBwdStage ? L - c0 : kBwdStage) + kBwdSub - 1) / kBwdSub);
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
                const int64_t l = l0 + g * kOwn + i;
                const float dl = l < L ? delta_transform<kFast>(in_at(d_row, l) + bias, softplus) : 0.f;
                gat[g * kOwn + i] = dl;
                gat[kBwdSub + g * kOwn + i] = dl * in_at(u_row, l);
            }
            __syncwarp();
            float dl[kBwdSub], du[kBwdSub];
#pragma unroll
            for (int i = 0; i < kBwdSub; ++i) dl[i] = gat[i], du[i] = gat[kBwdSub + i];
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
                    h[qq] = __ffma2_rn(a, h[qq], __fmul2_rn(u2, make_float2(bc.x, bc.y)));
                }
            }
        }
    }

    // ---------------------------------------------------------------- phase B
    float2 carry[kPL], dA_acc[kPL];
#pragma unroll
    for (int qq = 0; qq < kPL; ++qq) carry[qq] = make_float2(0.f, 0.f), dA_acc[qq] = make_float2(0.f, 0.f);
    float dD_acc = 0.f, dbias_acc = 0.f;
    const int64_t nstages = (L + kBwdStage - 1) / kBwdStage;
    for (int64_t st = nstages - 1; st >= 0; --st) {
        const int64_t c0 = st * kBwdStage;
        load_stage(c0);
        const int nsub = (int)(((L - c0 < kBwdStage ? L - c0 : kBwdStage) + kBwdSub - 1) / kBwdSub);
#pragma unroll 1
        for (int m = nsub - 1; m >= 0; --m) {
            const int64_t l0 = c0 + m * kBwdSub;
            const int64_t k = l0 / kBwdSub;
            // Owned steps: the per-row quantities, shared with the row's lanes.
            float o_u[kOwn], o_x[kOwn], o_dl[kOwn], o_z[kOwn], o_dy[kOwn], o_sg[kOwn];
#pragma unroll
            for (int i = 0; i < kOwn; ++i) {
                const int64_t l = l0 + g * kOwn + i;
                o_u[i] = in_at(u_row, l);
                o_x[i] = in_at(d_row, l) + bias;
                o_dl[i] = l < L ? delta_transform<kFast>(o_x[i], softplus) : 0.f;
                o_dy[i] = row_ok ? dy_at(l) : 0.f;
                o_z[i] = has_z ? in_at(z_row, l) : 0.f;
                o_sg[i] = has_z ? sigmoid_of<kFast>(o_z[i]) : 1.f;
                const float gl = has_z ? o_dy[i] * o_z[i] * o_sg[i] : o_dy[i];
                gat[g * kOwn + i] = o_dl[i];
                gat[kBwdSub + g * kOwn + i] = o_dl[i] * o_u[i];
                gat[2 * kBwdSub + g * kOwn + i] = gl;
            }
            __syncwarp();
            float dl[kBwdSub], du[kBwdSub], gg[kBwdSub];
#pragma unroll
            for (int i = 0; i < kBwdSub; ++i) dl[i] = gat[i], du[i] = gat[kBwdSub + i], gg[i] = gat[2 * kBwdSub + i];

            // Recompute the sub-chunk's decays and states from its checkpoint.
            float2 h0[kPL], a[kBwdSub][kPL], hs[kBwdSub][kPL];
#pragma unroll
            for (int qq = 0; qq < kPL; ++qq) {
                const int n = 2 * (q0 + qq);
                h0[qq] = make_float2(n < N ? ck_row[k * N + n] : 0.f, n + 1 < N ? ck_row[k * N + n + 1] : 0.f);
            }
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
                    hs[i][qq] = __ffma2_rn(a[i][qq], i ? hs[i - 1][qq] : h0[qq], __fmul2_rn(u2, make_float2(bc.x, bc.y)));
                    acc = __ffma2_rn(make_float2(bc.z, bc.w), hs[i][qq], acc);
                }
                sp[i] = acc.x + acc.y;
            }
            // The adjoint over the sub-chunk, last step first.
            float lb[kBwdSub], lha[kBwdSub];
#pragma unroll
            for (int i = kBwdSub - 1; i >= 0; --i) {
                const float2 g2 = make_float2(gg[i], gg[i]), u2 = make_float2(du[i], du[i]);
                float2 sLB = make_float2(0.f, 0.f), sLHA = make_float2(0.f, 0.f);
#pragma unroll
                for (int qq = 0; qq < kPL; ++qq) {
                    const float4 bc = Fm[i * kPairs + qq];
                    const float2 lam = __ffma2_rn(g2, make_float2(bc.z, bc.w), carry[qq]);
                    const float2 dCp = __fmul2_rn(g2, hs[i][qq]);
                    const float2 dBp = __fmul2_rn(lam, u2);
                    const float2 hp = i ? hs[i - 1][qq] : h0[qq];
                    const float2 t = __fmul2_rn(__fmul2_rn(lam, a[i][qq]), hp);  // lam a h_prev
                    sLB = __ffma2_rn(lam, make_float2(bc.x, bc.y), sLB);
                    sLHA = __ffma2_rn(t, Aln[qq], sLHA);
                    dA_acc[qq] = __ffma2_rn(t, make_float2(dl[i], dl[i]), dA_acc[qq]);
                    carry[qq] = __fmul2_rn(a[i][qq], lam);
                    const int n = 2 * (q0 + qq);
                    dbc[((0 * kBwdSub + i) * kNmax + n) * RS + rib] = dBp.x;
                    dbc[((0 * kBwdSub + i) * kNmax + n + 1) * RS + rib] = dBp.y;
                    dbc[((1 * kBwdSub + i) * kNmax + n) * RS + rib] = dCp.x;
                    dbc[((1 * kBwdSub + i) * kNmax + n + 1) * RS + rib] = dCp.y;
                }
                lb[i] = sLB.x + sLB.y;
                lha[i] = sLHA.x + sLHA.y;
            }
            // Per-row sums over the row's lanes: s (minus D u), sum lam B, sum lam a h A.
            float *mine = red + lane * kBwdReduce;
#pragma unroll
            for (int i = 0; i < kBwdSub; ++i) mine[i] = sp[i], mine[kBwdSub + i] = lb[i], mine[2 * kBwdSub + i] = lha[i];
            __syncwarp();
#pragma unroll
            for (int i = 0; i < kOwn; ++i) {
                const int j = g * kOwn + i;
                float s = 0.f, LB = 0.f, LHA = 0.f;
#pragma unroll
                for (int q = 0; q < kG; ++q) {
                    const float *src = red + (r * kG + q) * kBwdReduce;
                    s += src[j], LB += src[kBwdSub + j], LHA += src[2 * kBwdSub + j];
                }
                const int64_t l = l0 + j;
                const float gl = gg[j];
                s = fmaf(Dd, o_u[i], s);
                const float ddl = fmaf(o_u[i], LB, LHA);
                const float dx = softplus ? (o_x[i] > 20.f ? ddl : ddl * sigmoid_of<kFast>(o_x[i])) : ddl * o_dl[i];
                if (row_ok && l < L) {
                    put(du_row, l, fmaf(gl, Dd, o_dl[i] * LB));
                    put(dd_row, l, dx);
                    if (has_z) put(dz_row, l, o_dy[i] * s * o_sg[i] * fmaf(o_z[i], 1.f - o_sg[i], 1.f));
                    dD_acc = fmaf(gl, o_u[i], dD_acc);
                    dbias_acc += dx;
                }
            }
            // dB, dC of the sub-chunk summed over the block's rows.
            __syncthreads();
            const int nout = 2 * kBwdSub * kNmax;
            for (int o = tid; o < nout; o += nthreads) {
                const int n = o % kNmax, i = (o / kNmax) % kBwdSub, which = o / (kNmax * kBwdSub);
                const float *src = dbc + o * RS;
                float s = 0.f;
                for (int q = 0; q < rows; ++q) s += src[q];
                const int64_t l = l0 + i;
                if (n < N && l < L)
                    p.ws_dBC[(((dtile * p.batch + b) * 2 + which) * N + n) * L + l] = s;
            }
            __syncthreads();  // the slabs are free for the next sub-chunk
        }
    }

    // Per-row partials of dA, dD and dbias.
    if (row_ok) {
#pragma unroll
        for (int qq = 0; qq < kPL; ++qq) {
            const int n = 2 * (q0 + qq);
            if (n < N) p.ws_dA[row * N + n] = dA_acc[qq].x;
            if (n + 1 < N) p.ws_dA[row * N + n + 1] = dA_acc[qq].y;
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
        p.ws_dD[row] = dD_acc;
        p.ws_dbias[row] = dbias_acc;
    }
}

// dB, dC = the block partials summed over the row tiles, in tile order.
static __global__ void __launch_bounds__(256) ss_bwd_reduce_bc_kernel(const BwdParams p, float *dB, float *dC) {
    const int64_t per = (int64_t)p.dstate * p.seqlen;
    const int64_t total = p.batch * 2 * per;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t b = e / (2 * per), which = (e / per) % 2, nl = e % per;
        float s = 0.f;
        for (int64_t t = 0; t < p.dtiles; ++t) s += p.ws_dBC[((t * p.batch + b) * 2 + which) * per + nl];
        (which ? dC : dB)[b * per + nl] = s;
    }
}

// dA, dD, dbias = the per-row partials summed over the batch, in batch order.
static __global__ void __launch_bounds__(256) ss_bwd_reduce_rows_kernel(const BwdParams p, float *dA, float *dD,
                                                                  float *dbias) {
    const int64_t N = p.dstate;
    const int64_t total = p.dim * (N + 2);
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        if (e < p.dim * N) {
            float s = 0.f;
            for (int64_t b = 0; b < p.batch; ++b) s += p.ws_dA[b * p.dim * N + e];
            dA[e] = s;
        } else {
            const int64_t j = e - p.dim * N, d = j % p.dim;
            const bool is_bias = j >= p.dim;
            float *out = is_bias ? dbias : dD;
            if (out == nullptr) continue;
            const float *src = is_bias ? p.ws_dbias : p.ws_dD;
            float s = 0.f;
            for (int64_t b = 0; b < p.batch; ++b) s += src[b * p.dim + d];
            out[d] = s;
        }
    }
}

}  // namespace selscan
