// The direct kernel with B and C delivered through tensor memory (sm_100a).
//
// Same arithmetic and work mapping as ss_fwd_direct_kernel (G lanes of a row
// each own N/G of its states and run the plain sequential recurrence of the
// selective_scan_ref walkthrough, "Mamba代码实战" §3.2), for bf16 inputs.
// What changes is how a lane gets B[b, n, l] and C[b, n, l] for its states:
//
//   B and C are shared by every row (channel) of a batch entry.  The block
//   stages their raw bf16 rows (cp.async), lays them out as the B operand X
//   (K = 16 rows x N columns, K-major, no swizzle) of one tcgen05 MMA per
//   block of steps, and multiplies by a fixed 0/1 selection matrix E
//   (128 x 16, E[m][k] = 1 iff k = m mod G):
//       D[m][c] = sum_k E[m][k] X[k][c] = X[m mod G][c].
//   Row k < G of X holds, column by column, the values lane group k needs
//   (for each step: B of its states, then C of its states), so TMEM lane m
//   (thread m) receives exactly its own B/C values, widened to fp32 by the
//   tensor core.  The products are 1 x bf16 and the other terms 0 x bf16, so
//   D is exact.  (A non-finite B or C value turns its whole step's column
//   block non-finite through the 0 x inf terms.)  Each thread reads its values
//   with tcgen05.ld: no shared-memory reads and no integer widening of B/C.
//
// Pipeline.  Steps come in 64-step stages.  At the start of stage s the four
// warps meet (a block barrier), build X of stage s + 1 from its raw rows
// (which landed during stage s - 1), start the raw copies of stage s + 2, and
// meet again (X complete before an MMA reads it).  TMEM holds kNBuf buffers, each one block of a quarter sub-chunk
// (kBuf steps x 2 x states-per-lane columns), filled in turn: full[b]
// (tcgen05.commit) says buffer b holds its next block.  A warp waits on full
// before its first load from a buffer and, once its last load from it has
// landed, counts itself out on a shared-memory counter; the fourth warp to do
// so issues the MMA of the block kNBuf further on into that buffer.  There is
// no producer warp and no warp waits on another except through full (the
// MMAs run up to kNBuf - 1 blocks ahead of the slowest warp) and the stage
// barrier.  Each 16-column load is issued one chunk ahead of its use.
//
// Every wait on full is bounded (about a second of clock cycles).  On
// time-out the warps leave the stage loop together at the next stage barrier,
// the block records SS_DEVICE_TIMEOUT in p.status, waits (bounded) for the
// MMAs it issued, frees its tensor memory and returns.
#pragma once

#include "ss_fwd_kernel.cuh"
#include "ss_tcgen05.cuh"

namespace selscan {



// Geometry of the TMEM-fed kernel for a state bucket and a state split G.
template <int kNmax, int kG>
struct TmemGeom {
    static constexpr int kS = kNmax / kG;                    // states per lane
    static constexpr int kPL = kS / 2;                       // state pairs per lane
    static constexpr int kVals = 2 * kS;                     // TMEM columns per step (B, then C)
    static constexpr int kSub = direct_sub(kG);              // steps per sub-chunk
    static constexpr int kNBuf = 4;                          // TMEM buffers
    static constexpr int kBuf = kSub / kNBuf;                // steps per TMEM buffer (a quarter sub-chunk)
    static constexpr int kBufCols = kBuf * kVals;            // MMA N
    static constexpr int kCols = kNBuf * kBufCols;           // TMEM columns allocated
    static constexpr int kWarps = 4;                         // 128 threads = 128 TMEM lanes
    static constexpr int kThreads = 32 * kWarps;
    static constexpr int kRowsPerWarp = 32 / kG;
    static constexpr int kRows = kWarps * kRowsPerWarp;      // channels per block
    static constexpr int kBlocksPerStage = kDirectStage / kBuf;
    static constexpr int kRBStride = kDirectStage + 8;       // raw row stride (elements): rows spread over banks
    // gather slab: per row and step (delta', delta', delta' u, delta' u), rows
    // padded by 16 bytes to spread them over the banks; then the reduce slab
    static constexpr int kGatherStride = 4 * kSub + 4;
    // shared memory, byte offsets
    static constexpr size_t kOffE = 0;                                        // E, first K half: 128 x 16 B
    static constexpr size_t kXBytes = (size_t)kDirectStage * kVals * 16;      // X of one stage
    static constexpr size_t kOffX = 2048;                                     // two stage buffers
    static constexpr size_t kOffZ = kOffX + 2 * kXBytes;                      // zeros: second K halves
    static constexpr size_t kOffRB = kOffZ + 2048;                            // raw B/C, two stages
    static constexpr size_t kRBBytes = 2 * (size_t)kNmax * kRBStride * 2;
    static constexpr size_t kOffSlab = kOffRB + 2 * kRBBytes;
    static constexpr size_t kSlabFloats = (size_t)kRowsPerWarp * kGatherStride + 32 * reduce_stride(kG);
    static constexpr size_t kOffBar = kOffSlab + (size_t)kWarps * kSlabFloats * 4;
    // full[kNBuf] (8 B each), release counters and issue counters (4 B each), TMEM address, abort flag
    static constexpr size_t kBytes = kOffBar + 8 * kNBuf + 8 * kNBuf + 16;
    static_assert(kCols == 32 || kCols == 64 || kCols == 128, "TMEM allocation: a power of 2, at most 128");
    static_assert(kBufCols % 16 == 0 && kBufCols >= 16 && kBufCols <= 256, "MMA N for M = 128");
    static_assert(kG <= 8, "lane groups fit the first K half of X");
    static_assert(kBlocksPerStage >= kNBuf, "an MMA runs at most one stage ahead");
};

__host__ __device__ constexpr bool tmem_supported(int nmax, int g) {
    // 2, 4 or 8 lanes per row; 2 to 8 states per lane; all buffers within
    // 128 TMEM columns; MMA N of each buffer (a quarter sub-chunk of
    // columns) a multiple of 16
    return g >= 2 && g <= 8 && nmax / g >= 2 && nmax / g <= 8 && nmax / g * 2 * direct_sub(g) <= 128 &&
           (nmax / g * 2 * direct_sub(g) / 4) % 16 == 0;
}

// Dynamic shared memory of one block (at least 48 KB, so that at most four
// blocks share an SM and their TMEM allocations always fit its 512 columns).
template <int kNmax, int kG>
__host__ __device__ constexpr size_t tmem_smem_bytes() {
    return TmemGeom<kNmax, kG>::kBytes > 48 * 1024 ? TmemGeom<kNmax, kG>::kBytes : 48 * 1024;
}

// Shared-memory atomic add (relaxed).  It orders nothing but itself: a warp
// counts itself out of a buffer only after its tensor-memory loads from it
// have completed (tcgen05.wait::ld), and the MMA that overwrites the buffer
// is issued after the fourth count returns, so the loads precede the write;
// X is made visible to the MMAs by the stage barriers, not by this counter.
__device__ __forceinline__ uint32_t atom_add_relaxed(uint32_t *p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.relaxed.cta.shared::cta.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(smem_addr(p)), "r"(v)
                 : "memory");
    return old;
}

template <typename Tout, int kNmax, int kG>
__global__ void __launch_bounds__(TmemGeom<kNmax, kG>::kThreads, 3) ss_fwd_tmem_kernel(const FwdParams p) {
    using Tin = __nv_bfloat16;
    using Geo = TmemGeom<kNmax, kG>;
    constexpr int kS = Geo::kS, kPL = Geo::kPL, kVals = Geo::kVals, kSub = Geo::kSub;
    constexpr int kBufCols = Geo::kBufCols, kWarps = Geo::kWarps, kNBuf = Geo::kNBuf;
    constexpr int kBPS = Geo::kBlocksPerStage;
    constexpr int kOwn = kSub / kG;                       // steps owned per lane per sub-chunk
    constexpr int kOwnBytes = kOwn * 2;
    constexpr int kOwnWords = (kOwnBytes + 3) / 4;
    constexpr int kGatherStride = Geo::kGatherStride;
    constexpr int kRS = reduce_stride(kG), kRV = reduce_vec(kG);
    constexpr int kAccs = kPL >= 4 ? 2 : 1;
    constexpr int kLd = 16 / kVals;                       // steps per 16-column load (chunk)
    constexpr int kChunks = kSub * kVals / 16;            // chunks per sub-chunk
    constexpr int kCPB = kBufCols / 16;                   // chunks per buffer
    constexpr int kSubsPerStage = kDirectStage / kSub;
    constexpr size_t kRBElems = Geo::kRBBytes / sizeof(Tin);  // raw B/C of one stage
    constexpr uint32_t kIdesc = tc::idesc_bf16(128, kBufCols);
    static_assert(kVals <= 16 && 16 % kVals == 0, "whole steps per 16-column load");

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint16_t *const E = reinterpret_cast<uint16_t *>(smem_raw + Geo::kOffE);
    uint8_t *const X0 = smem_raw + Geo::kOffX;
    uint8_t *const Z = smem_raw + Geo::kOffZ;
    Tin *const RB0 = reinterpret_cast<Tin *>(smem_raw + Geo::kOffRB);
    uint64_t *const full = reinterpret_cast<uint64_t *>(smem_raw + Geo::kOffBar);
    uint32_t *const released = reinterpret_cast<uint32_t *>(full + kNBuf);   // per buffer: warps counted out
    uint32_t *const issued = released + kNBuf;                               // per buffer: MMAs issued
    uint32_t *const tslot = issued + kNBuf;

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int g = lane % kG;
    const int r = lane / kG;
    const int N = p.dstate;
    const int64_t L = p.seqlen;
    const int64_t blocks_per_seg = p.batch * p.dtiles;
    const int64_t seg = blockIdx.x / blocks_per_seg;
    const int64_t bt = blockIdx.x % blocks_per_seg;
    const int64_t b = bt / p.dtiles;
    const int64_t c_begin = seg * p.seg_len;
    const int64_t Lend = c_begin + p.seg_len < L ? c_begin + p.seg_len : L;
    const int64_t len = Lend - c_begin;
    const int64_t nsub = (len + kSub - 1) / kSub;
    const int64_t nstages = (len + kDirectStage - 1) / kDirectStage;
    const int64_t nblocks = kNBuf * nsub;
    const bool vec = p.vec != 0;
    const Tin *Bsrc[2] = {static_cast<const Tin *>(p.B) + b * N * L, static_cast<const Tin *>(p.C) + b * N * L};

    // ---- set-up: E, zeroed X buffers and Z, barriers, counters, TMEM
    for (int i = tid; i < 128 * 8; i += kWarps * 32) {
        const int m = i / 8, k = i % 8;
        E[i] = k == m % kG ? (uint16_t)0x3F80u : (uint16_t)0;  // bf16 1.0 / 0.0
    }
    {
        uint4 *zx = reinterpret_cast<uint4 *>(X0);
        const int n16 = (int)((2 * Geo::kXBytes + 2048) / 16);  // both X buffers and Z (contiguous)
        for (int i = tid; i < n16; i += kWarps * 32) zx[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    if (tid == 0) {
        for (int i = 0; i < kNBuf; ++i) tc::mbar_init(&full[i], 1), released[i] = 0u, issued[i] = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) tc::alloc(tslot, Geo::kCols);

    // Raw B/C rows of the stage from c0 into RB (16-byte cp.async when the
    // stage is whole and aligned, element loads with zero fill otherwise);
    // one commit group per stage.
    auto stage_in = [&](int64_t c0, Tin *RB) {
        if (vec && c0 + kDirectStage <= Lend) {
            constexpr int kChunks16 = kDirectStage / 8;  // 16-byte chunks per row
            for (int u = tid; u < 2 * kNmax * kChunks16; u += kWarps * 32) {
                const int t = u / (kNmax * kChunks16), n = (u / kChunks16) % kNmax, j = u % kChunks16;
                if (n < N) cp_async16(RB + (t * kNmax + n) * Geo::kRBStride + j * 8, Bsrc[t] + (int64_t)n * L + c0 + j * 8);
            }
        } else {
            for (int u = tid; u < 2 * kNmax * kDirectStage; u += kWarps * 32) {
                const int t = u / (kNmax * kDirectStage), n = (u / kDirectStage) % kNmax, e = u % kDirectStage;
                if (n < N) {
                    const int64_t l = c0 + e;
                    reinterpret_cast<unsigned short *>(RB)[(t * kNmax + n) * Geo::kRBStride + e] =
                        l < Lend ? reinterpret_cast<const unsigned short *>(Bsrc[t])[(int64_t)n * L + l]
                                 : (unsigned short)0;
                }
            }
        }
        cp_async_commit();
    };
    // X of stage s from its raw rows: column e * kVals + j (step e, value j),
    // row k (bytes 2k, 2k + 1) = value j of lane group k: B (j < kS) or C of
    // state k * kS + j % kS; past the sequence end or N, zero.  Bytes past
    // 2 kG stay zero.
    auto build_X = [&](int64_t s) {
        const unsigned short *rb16 = reinterpret_cast<const unsigned short *>(RB0 + (s & 1) * kRBElems);
        uint8_t *X = X0 + (s & 1) * Geo::kXBytes;
        for (int col = tid; col < kDirectStage * kVals; col += kWarps * 32) {
            const int e = col / kVals, j = col % kVals, t = j / kS, jj = j % kS;
            const bool in = c_begin + s * kDirectStage + e < Lend;
            uint32_t w[(kG + 1) / 2];
#pragma unroll
            for (int q = 0; q < (kG + 1) / 2; ++q) w[q] = 0u;
#pragma unroll
            for (int k = 0; k < kG; ++k) {
                const int n = k * kS + jj;
                const uint32_t v = (n < N && in) ? rb16[(t * kNmax + n) * Geo::kRBStride + e] : 0u;
                w[k / 2] |= v << (16 * (k & 1));
            }
            uint8_t *dst = X + (size_t)col * 16;
            if constexpr (kG >= 8) *reinterpret_cast<uint4 *>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
            else if constexpr (kG >= 4) *reinterpret_cast<uint2 *>(dst) = make_uint2(w[0], w[1]);
            else *reinterpret_cast<uint32_t *>(dst) = w[0];
        }
        tc::fence_async_smem();  // X is read by the tensor core (async proxy)
    };

    if (nstages > 0) stage_in(c_begin, RB0);
    if (nstages > 1) stage_in(c_begin + kDirectStage, RB0 + kRBElems);
    tc::fence_async_smem();
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t taddr = *tslot;
    const uint32_t e_addr = smem_addr(E), z_addr = smem_addr(Z);
    const uint64_t descE = tc::sdesc(e_addr, z_addr - e_addr, 128);
    // The MMA of block j (buffer j % kNBuf) from X of its stage.
    auto issue_mma = [&](int64_t j) {
        const int64_t st = j / kBPS;
        const uint32_t xa = smem_addr(X0 + (st & 1) * Geo::kXBytes + (size_t)(j % kBPS) * kBufCols * 16);
        const int buf = (int)(j % kNBuf);
        tc::mma_bf16(taddr + (uint32_t)(buf * kBufCols), descE, tc::sdesc(xa, z_addr - xa, 128), kIdesc);
        tc::commit(&full[buf]);
        issued[buf] += 1u;
    };
    if (nstages > 0) {
        if (nstages > 1) cp_async_wait_one();
        else cp_async_wait_all();
        __syncthreads();  // stage 0's raw rows have landed
        build_X(0);
        __syncthreads();
        if (tid == 0) {
            tc::fence_after();
            for (int64_t j = 0; j < kNBuf && j < nblocks; ++j) issue_mma(j);
        }
    }

    // ---- compute
    const int64_t d_raw = (bt % p.dtiles) * Geo::kRows + tid / kG;
    const bool row_ok = d_raw < p.dim;
    const int64_t d = row_ok ? d_raw : p.dim - 1;
    const int64_t row = b * p.dim + d;
    const bool softplus = p.softplus != 0;
    const bool has_z = p.z != nullptr;
    float *slab = reinterpret_cast<float *>(smem_raw + Geo::kOffSlab) + warp * Geo::kSlabFloats;
    float4 *const gat4 = reinterpret_cast<float4 *>(slab + r * kGatherStride);
    float *red = slab + Geo::kRowsPerWarp * kGatherStride;
    const Tin *u_own = static_cast<const Tin *>(p.u) + row * L + c_begin + g * kOwn;
    const Tin *d_own = static_cast<const Tin *>(p.delta) + row * L + c_begin + g * kOwn;
    const Tin *z_own = has_z ? static_cast<const Tin *>(p.z) + row * L + c_begin + g * kOwn : nullptr;
    Tout *const y_row = static_cast<Tout *>(p.y) + row * L;
    Tout *y_own = y_row + c_begin + g * kOwn;
    const uint32_t t_lane = taddr + ((uint32_t)(32 * warp) << 16);

    const int q0 = g * kPL;
    const float *A_d = p.A + d * N;
    float2 A2[kPL], h[kPL];
#pragma unroll
    for (int qq = 0; qq < kPL; ++qq) {
        const int n = 2 * (q0 + qq);
        A2[qq] = make_float2(n < N ? A_d[n] * kLog2e : 0.f, n + 1 < N ? A_d[n + 1] * kLog2e : 0.f);
        h[qq] = make_float2(0.f, 0.f);
        if (p.init_state != nullptr && seg == 0) {
            if (n < N) h[qq].x = p.init_state[row * N + n];
            if (n + 1 < N) h[qq].y = p.init_state[row * N + n + 1];
        }
    }
    const float Dd = p.D ? p.D[d] : 0.f;
    const float bias = p.delta_bias ? p.delta_bias[d] : 0.f;

    auto load_own_checked = [&](const Tin *own, int64_t s0, uint32_t (&w)[kOwnWords]) {
        if (kOwnBytes >= 4 && vec && s0 + kOwn <= Lend) {
            ld_words<kOwnBytes>(own, w);
        } else {
#pragma unroll
            for (int jw = 0; jw < kOwnWords; ++jw) w[jw] = 0u;
#pragma unroll
            for (int i = 0; i < kOwn; ++i)
                if (s0 + i < Lend) w[i >> 1] |= Io<Tin>::bits(own, i) << (16 * (i & 1));
        }
    };
    uint32_t wu[kOwnWords], wd[kOwnWords], wz[kOwnWords];
    load_own_checked(u_own, c_begin + g * kOwn, wu);
    load_own_checked(d_own, c_begin + g * kOwn, wd);
    if (has_z) load_own_checked(z_own, c_begin + g * kOwn, wz);
    float dsum = 0.f;
    bool ok = true;

    // One sub-chunk (kSub steps from l0; global index m).
    auto sub_chunk = [&](int64_t m) {
        const int64_t l0 = c_begin + m * kSub;
        const bool checked = !(vec && l0 + kSub <= Lend);
        uint32_t cu[kOwnWords], cd[kOwnWords], cz[kOwnWords];
#pragma unroll
        for (int jw = 0; jw < kOwnWords; ++jw) cu[jw] = wu[jw], cd[jw] = wd[jw], cz[jw] = wz[jw];
        const int64_t s_next = l0 + kSub + g * kOwn;
        u_own += kSub, d_own += kSub;
        if (has_z) z_own += kSub;
        if (l0 + kSub < Lend) {  // this lane's steps of the next sub-chunk, one sub-chunk ahead
            load_own_checked(u_own, s_next, wu);
            load_own_checked(d_own, s_next, wd);
            if (has_z) load_own_checked(z_own, s_next, wz);
        }
        // delta' and delta' u of the owned steps (past the end: the identity step)
        float dl_own[kOwn], du_own[kOwn], uo[kOwn];
#pragma unroll
        for (int i = 0; i < kOwn; ++i) {
            uo[i] = Io<Tin>::widen(cu, i);
            dl_own[i] = delta_transform<true>(Io<Tin>::widen(cd, i) + bias, softplus);
            if (checked && l0 + g * kOwn + i >= Lend) dl_own[i] = 0.f;
            du_own[i] = dl_own[i] * uo[i];
            dsum += dl_own[i];
        }
        // Every lane of the row needs delta' and delta' u of all kSub steps,
        // as the pairs (delta', delta') and (delta' u, delta' u) of the packed
        // products: each lane stores its own steps' quadruples, then reads one
        // quadruple per step in the state loop.
#pragma unroll
        for (int i = 0; i < kOwn; ++i) gat4[g * kOwn + i] = make_float4(dl_own[i], dl_own[i], du_own[i], du_own[i]);
        __syncwarp();
        // The state loop over the sub-chunk's TMEM buffers: 16-column chunks,
        // each loaded one chunk ahead (registers v[c & 1]).
        float part[kSub];
        uint32_t v[2][16];
        const uint32_t parity = (uint32_t)(m & 1);
        if (!tc::mbar_wait(&full[0], parity)) ok = false;
        __syncwarp();
        tc::fence_after();
        tc::ld16(t_lane, v[0]);
        tc::ld16_wait(v[0]);
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
            if (c + 1 < kChunks) {
                if ((c + 1) % kCPB == 0) {  // first chunk of the next buffer
                    if (!tc::mbar_wait(&full[(c + 1) / kCPB], parity)) ok = false;
                    __syncwarp();
                    tc::fence_after();
                }
                tc::ld16(t_lane + (uint32_t)((c + 1) * 16), v[(c + 1) & 1]);
            }
#pragma unroll
            for (int ii = 0; ii < kLd; ++ii) {
                const int i = c * kLd + ii;  // step within the sub-chunk
                const uint32_t *bc = &v[c & 1][ii * kVals];
                const float4 q4 = gat4[i];
                const float2 d2 = make_float2(q4.x, q4.y), u2 = make_float2(q4.z, q4.w);
                float2 acc[kAccs];
#pragma unroll
                for (int k = 0; k < kAccs; ++k) acc[k] = make_float2(0.f, 0.f);
#pragma unroll
                for (int qq = 0; qq < kPL; ++qq) {
                    const float2 Bp = make_float2(__uint_as_float(bc[2 * qq]), __uint_as_float(bc[2 * qq + 1]));
                    const float2 Cp = make_float2(__uint_as_float(bc[kS + 2 * qq]), __uint_as_float(bc[kS + 2 * qq + 1]));
                    const float2 t = __fmul2_rn(d2, A2[qq]);
                    const float2 a = make_float2(sfu_exp2(t.x), sfu_exp2(t.y));
                    h[qq] = __ffma2_rn(a, h[qq], __fmul2_rn(u2, Bp));
                    acc[qq % kAccs] = __ffma2_rn(Cp, h[qq], acc[qq % kAccs]);
                }
                if constexpr (kAccs == 2) acc[0] = __fadd2_rn(acc[0], acc[1]);
                part[i] = acc[0].x + acc[0].y;
            }
            if ((c + 1) % kCPB == 0) {
                // The last chunk of buffer bb has landed and been used: count
                // this warp out; the fourth warp issues the block kNBuf on.
                const int bb = c / kCPB;
                tc::fence_before();
                __syncwarp();
                if (lane == 0) {
                    const uint32_t old = atom_add_relaxed(&released[bb], 1u);
                    const int64_t jn = m * kNBuf + bb + kNBuf;
                    if (old % kWarps == kWarps - 1 && jn < nblocks) {
                        tc::fence_after();
                        issue_mma(jn);
                    }
                }
            }
            if (c + 1 < kChunks) tc::ld16_wait(v[(c + 1) & 1]);
        }
        // Totals of the owned steps.
        float yv[kOwn];
        {
            static_assert(kOwn % kRV == 0 && kRS % kRV == 0, "reduce slab accesses stay aligned");
            float *mine = red + lane * kRS;
#pragma unroll
            for (int k = 0; k < kSub; k += kRV) st_vec<kRV>(mine + k, part + k);
            __syncwarp();
#pragma unroll
            for (int i = 0; i < kOwn; ++i) yv[i] = 0.f;
#pragma unroll
            for (int gg = 0; gg < kG; ++gg) {
                const float *src = red + (r * kG + gg) * kRS + g * kOwn;
#pragma unroll
                for (int k = 0; k < kOwn; k += kRV) {
                    float vv[kRV];
                    ld_vec<kRV>(src + k, vv);
#pragma unroll
                    for (int jv = 0; jv < kRV; ++jv) yv[k + jv] += vv[jv];
                }
            }
        }
#pragma unroll
        for (int i = 0; i < kOwn; ++i) yv[i] = fmaf(Dd, uo[i], yv[i]);  // + D u (§3.3)
        if (has_z) {
#pragma unroll
            for (int i = 0; i < kOwn; ++i) yv[i] *= silu<true>(Io<Tin>::widen(cz, i));
        }
        if (row_ok) {
            if (checked) store_run<kOwn>(y_row, l0 + g * kOwn, Lend, vec, yv);
            else store_run<kOwn>(y_own, 0, kOwn, true, yv);
        }
        y_own += kSub;
        __syncwarp();  // the slabs are rewritten by the next sub-chunk
    };

    bool aborted = false;
    for (int64_t s = 0; s < nstages; ++s) {
        if (s + 1 < nstages) {
            cp_async_wait_all();  // stage s + 1's raw rows (the only group in flight)
            // Every thread's copies have landed; every warp has finished stage
            // s - 1, so X and the raw buffer of stage s - 1 are free.  A warp
            // whose wait ran out makes all of them leave here together.
            if (__syncthreads_or(!ok)) {
                aborted = true;
                break;
            }
            build_X(s + 1);
            if (s + 2 < nstages) stage_in(c_begin + (s + 2) * kDirectStage, RB0 + (s & 1) * kRBElems);
            __syncthreads();  // X of stage s + 1 is complete before any MMA reading it is issued
        }
        const int64_t m_end = (s + 1) * kSubsPerStage < nsub ? (s + 1) * kSubsPerStage : nsub;
#pragma unroll 1
        for (int64_t m = s * kSubsPerStage; m < m_end; ++m) sub_chunk(m);
    }
    if (__syncthreads_or(!ok)) aborted = true;

    if (!aborted) {
        if (p.nseg > 1) {  // segment record for the fix-up kernel
            const int64_t rec = seg * (p.batch * p.dim) + row;
#pragma unroll
            for (int sd = 1; sd < kG; sd *= 2) dsum += __shfl_xor_sync(0xffffffffu, dsum, sd, kG);
            if (row_ok) {
#pragma unroll
                for (int qq = 0; qq < kPL; ++qq) {
                    const int n = 2 * (q0 + qq);
                    if (n < N) p.ws_hend[rec * N + n] = h[qq].x;
                    if (n + 1 < N) p.ws_hend[rec * N + n + 1] = h[qq].y;
                }
                if (g == 0) p.ws_dsum[rec] = dsum;
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

    // ---- tear-down: every MMA issued has completed (normally all were
    // already waited for) and every TMEM read is done before the free.
    cp_async_wait_all();
    if (tid == 0) {
        bool drained = true;
        for (int bb = 0; bb < kNBuf; ++bb) {
            const uint32_t n = issued[bb];
            if (n > 0 && !tc::mbar_wait(&full[bb], (n - 1) & 1u)) drained = false;
        }
        if ((aborted || !drained) && p.status) atomicExch(p.status, kDeviceTimeout);
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    if (warp == 0) tc::dealloc(taddr, Geo::kCols);
}

}  // namespace selscan
