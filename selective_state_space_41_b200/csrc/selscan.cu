// libselscan: C ABI of the selective scan -- forward, host-buffer forms,
// decoding step and backward (declarations and the meaning of every argument
// are in include/selscan.h).
//
// Host side: validates the descriptor and pointers before touching CUDA,
// picks a launch shape, and dispatches to the kernel instance for the dtype
// pair, the state-size bucket (4/8/16/32/64) and the lanes-per-row count.

#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <cstddef>
#include <cstdint>

#include <mutex>

#include "selscan.h"
#include "ss_bwd_launch.h"
#include "ss_step_kernel.cuh"
#include "ss_launch.h"

// The device status word: a kernel whose bounded wait ran out writes a
// nonzero code here (read and cleared by ss_device_status).
static __device__ int g_ss_device_status;

namespace {

using selscan::FwdParams;

constexpr int kMaxState = 64;
constexpr int kMaxDevices = 64;

// Device address of g_ss_device_status on the current device (looked up once
// per device), or null when the runtime cannot give it (then the kernels
// record nothing).
int *device_status_ptr() {
    static std::mutex mu;
    static int *addr[kMaxDevices];
    static bool tried[kMaxDevices];
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!tried[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_ss_device_status) == cudaSuccess) addr[dev] = static_cast<int *>(p);
        else (void)cudaGetLastError();
        tried[dev] = true;
    }
    return addr[dev];
}

// TMEM-fed direct kernel (split_states = 2): bf16 inputs, a state split and
// bucket it is built for.
bool tmem_ok(const ss_desc *desc, int lanes) {
    return desc->in_dtype == SS_BF16 && selscan::tmem_supported(selscan::state_bucket((int)desc->dstate), lanes);
}
size_t tmem_smem(int nmax, int lanes) {
    switch (nmax * 16 + lanes) {
        case 8 * 16 + 2: return selscan::tmem_smem_bytes<8, 2>();
        case 8 * 16 + 4: return selscan::tmem_smem_bytes<8, 4>();
        case 16 * 16 + 2: return selscan::tmem_smem_bytes<16, 2>();
        case 16 * 16 + 4: return selscan::tmem_smem_bytes<16, 4>();
        case 16 * 16 + 8: return selscan::tmem_smem_bytes<16, 8>();
        case 32 * 16 + 8: return selscan::tmem_smem_bytes<32, 8>();
        default: return 0;
    }
}

size_t dtype_size(ss_dtype t) { return t == SS_BF16 ? 2 : 4; }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// a * b without signed overflow; false if it would exceed INT64_MAX / 8.
bool mul_ok(int64_t a, int64_t b, int64_t *out) {
    if (a == 0 || b == 0) {
        *out = 0;
        return true;
    }
    if (a > (INT64_MAX / 8) / b) return false;
    *out = a * b;
    return true;
}

struct Sizes {
    int64_t rows, elems, bc_elems;  // B*D, B*D*L, B*N*L
};

ss_status check_desc(const ss_desc *desc, Sizes *s) {
    if (!desc) return SS_ERR_NULL_POINTER;
    if (desc->batch < 0 || desc->dim < 0 || desc->seqlen < 0) return SS_ERR_BAD_SHAPE;
    if (desc->dstate < 1 || desc->dstate > kMaxState) return SS_ERR_UNSUPPORTED_DSTATE;
    const bool in_ok = desc->in_dtype == SS_F32 || desc->in_dtype == SS_BF16;
    const bool out_ok = desc->out_dtype == desc->in_dtype ||
                        (desc->in_dtype == SS_BF16 && desc->out_dtype == SS_F32);
    if (!in_ok || !out_ok) return SS_ERR_UNSUPPORTED_DTYPE;
    int64_t t;
    if (!mul_ok(desc->batch, desc->dim, &s->rows)) return SS_ERR_BAD_SHAPE;
    if (!mul_ok(s->rows, desc->seqlen, &s->elems)) return SS_ERR_BAD_SHAPE;
    if (!mul_ok(desc->batch, desc->dstate, &t) || !mul_ok(t, desc->seqlen, &s->bc_elems))
        return SS_ERR_BAD_SHAPE;
    if (!mul_ok(s->rows, desc->dstate, &t)) return SS_ERR_BAD_SHAPE;
    return SS_OK;
}

int sm_count() {
    static std::atomic<int> cache[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    int v = cache[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
        v = 148;
    cache[dev].store(v, std::memory_order_relaxed);
    return v;
}

// Dynamic shared memory of one block: B and C of one chunk for the state
// bucket as fp32, plus a raw copy in the input dtype (see the kernel).
size_t smem_for(const ss_desc *desc, int lanes, int split, int warps) {
    const int nmax = selscan::state_bucket((int)desc->dstate);
    if (split == 2) return tmem_smem(nmax, lanes);
    if (lanes == 1 || split) return selscan::direct_smem_bytes(dtype_size(desc->in_dtype), nmax, lanes, warps);
    return selscan::smem_bytes(dtype_size(desc->in_dtype), nmax, lanes, warps);
}

// A resolved launch: kernel shape plus sequence segmentation.
struct Plan {
    int lanes, split, warps;
    int nseg;        // 1: no segmentation
    int64_t seg_len;
};

constexpr int64_t kMinSegSteps = 2048;  // segments shorter than this are not worth a fix-up

size_t workspace_for(const ss_desc *desc, int64_t rows, const Plan &pl) {
    if (pl.nseg <= 1) return 0;
    return (size_t)pl.nseg * (size_t)rows * (size_t)(desc->dstate + 1) * sizeof(float);
}

// Segment length for nseg segments: a multiple of the direct kernel's stage
// (so segment starts keep 16-byte alignment); returns the segment count it gives.
int segment(const ss_desc *desc, int nseg, int64_t *seg_len) {
    const int64_t L = desc->seqlen;
    if (L <= 0 || nseg <= 1) {
        *seg_len = L;
        return 1;
    }
    int64_t len = (L + nseg - 1) / nseg;
    len = (len + selscan::kDirectStage - 1) / selscan::kDirectStage * selscan::kDirectStage;
    *seg_len = len;
    return (int)((L + len - 1) / len);
}

// Launch shape.  The direct kernel (lanes split a row's states, no scan) has
// the least work per state update, so it is used whenever the rows alone
// can give each SM sub-partition (4 per SM) enough warps: the smallest split
// G in {1, 2, 4} (at most half the state bucket) with at least 4 warps per
// sub-partition (with 64 states, 32 states per lane once that gives 2 warps:
// 16 states per lane there measured 3x slower), or G = 4 down to 1.5 warps.
// 32 states take 2 lanes of 16 rather than one of 32, whose 254 registers
// leave 2 warps per sub-partition (16 x 4096 x 8192 x 32 layer: 6.0 against
// 7.2 ms).  With fewer rows and a long sequence,
// and a workspace, the sequence is cut into segments of at least
// kMinSegSteps steps that the direct kernel runs as extra rows (2-way state
// split, about 7 warps per sub-partition) and the fix-up kernel joins.
// Otherwise the steps are split across lanes (scan kernel): the smallest W
// giving 3 warps per sub-partition, no more lanes than the sequence can feed,
// and a block within half of an SM's shared memory.  direct_only (sequence
// starts given, which only the direct kernel reads): the direct kernel with
// the widest state split instead of the scan kernel.
Plan heuristic(const ss_desc *desc, int64_t rows, int sms, size_t workspace_bytes,
               bool direct_only = false) {
    Plan pl{1, 0, 4, 1, desc->seqlen};
    if (rows <= 0 || desc->seqlen <= 0) return pl;
    const int64_t slots = (int64_t)sms * 4 * 32;  // lanes per "one warp per sub-partition"
    const int bucket = selscan::state_bucket((int)desc->dstate);
    const int gmax = bucket / 2 >= 4 ? 4 : 2;
    int g = 1;
    while (g < gmax && rows * g < 4 * slots) g *= 2;
    if (bucket >= 64 && rows * (bucket / 32) >= 2 * slots) g = bucket / 32;
    if (rows * g >= 2 * slots || rows * gmax * 2 >= 3 * slots) {
        pl.lanes = g;
        pl.split = g > 1 ? 1 : 0;
        return pl;
    }
    const int gs = bucket / 2 >= 2 ? 2 : 1;  // segmented: 2-way state split
    int64_t want = (7 * slots) / (rows * gs);
    if (want > desc->seqlen / kMinSegSteps) want = desc->seqlen / kMinSegSteps;
    if (want >= 2) {
        Plan sp{gs, gs > 1 ? 1 : 0, 4, 1, 0};
        sp.nseg = segment(desc, (int)want, &sp.seg_len);
        if (sp.nseg >= 2 && workspace_for(desc, rows, sp) <= workspace_bytes) return sp;
    }
    if (direct_only) {
        pl.lanes = gmax;
        pl.split = 1;
        return pl;
    }
    int w = 2;
    while (w < 32 && rows * w < 3 * slots) w *= 2;
    while (w > 2 && (int64_t)selscan::chunk_len(w) / 2 >= desc->seqlen) w /= 2;
    while (w > 2 && smem_for(desc, w, 0, 8) > selscan::kMaxSmemBytes / 2) w /= 2;
    pl.lanes = w;
    pl.split = 0;
    pl.warps = 8;
    return pl;
}

// The caller's launch config (zeros: the heuristic's choices) resolved into a
// plan; SS_ERR_BAD_CONFIG for unsupported values.
ss_status resolve(const ss_desc *desc, int64_t rows, const ss_launch_config *cfg,
                  size_t workspace_bytes, Plan *out, bool direct_only = false) {
    Plan pl = heuristic(desc, rows, sm_count(), workspace_bytes, direct_only);
    if (cfg) {
        const int lanes = cfg->lanes_per_row, warps = cfg->warps_per_block, split = cfg->split_states;
        if (lanes != 0 && (lanes < 1 || lanes > 32 || (lanes & (lanes - 1)) != 0)) return SS_ERR_BAD_CONFIG;
        if (split != 0 && split != 1 && split != 2) return SS_ERR_BAD_CONFIG;
        if (warps != 0 && warps != 1 && warps != 2 && warps != 4 && warps != 8) return SS_ERR_BAD_CONFIG;
        if (cfg->segments < 0) return SS_ERR_BAD_CONFIG;
        if (lanes != 0) {
            pl.lanes = lanes;
            pl.split = split;
            if (cfg->segments == 0) pl.nseg = 1, pl.seg_len = desc->seqlen;
        }
        if (warps != 0) pl.warps = warps;
        if (cfg->segments == 1) {
            pl.nseg = 1;
            pl.seg_len = desc->seqlen;
        } else if (cfg->segments > 1) {
            pl.nseg = segment(desc, cfg->segments, &pl.seg_len);
        }
    }
    const bool direct = pl.lanes == 1 || pl.split;
    if (cfg && cfg->segments > 1 && !direct) return SS_ERR_BAD_CONFIG;  // segments need the direct kernel
    // The direct kernel splits the state pairs of the state bucket over 1, 2, 4 or 8 lanes.
    if (direct && (pl.lanes > 8 || selscan::state_bucket((int)desc->dstate) / 2 < pl.lanes))
        return SS_ERR_BAD_CONFIG;
    if (pl.nseg > 1 && !direct) return SS_ERR_BAD_CONFIG;  // segments run in the direct kernel
    if (direct_only && !direct) return SS_ERR_BAD_CONFIG;  // sequence starts: direct kernel only
    if (pl.split == 2) {  // TMEM-fed: bf16, a supported split, 4 compute warps, no sequence starts
        if (!tmem_ok(desc, pl.lanes) || direct_only) return SS_ERR_BAD_CONFIG;
        if (cfg && cfg->warps_per_block != 0 && cfg->warps_per_block != 4) return SS_ERR_BAD_CONFIG;
        pl.warps = 4;
    }
    if (pl.nseg < 1) pl.nseg = 1;
    if (pl.nseg == 1) pl.seg_len = desc->seqlen;
    *out = pl;
    return SS_OK;
}

// The launcher for the state bucket that holds n (4, 8, 16, 32 or 64).
#define SS_PICK_BUCKET(PREFIX)                                                 \
    cudaError_t (*fn)(int, int, dim3, dim3, size_t, cudaStream_t, const FwdParams &) = \
        n <= 4 ? selscan::PREFIX##_n4                                     \
        : n <= 8 ? selscan::PREFIX##_n8                                   \
        : n <= 16 ? selscan::PREFIX##_n16                                 \
        : n <= 32 ? selscan::PREFIX##_n32                                 \
                  : selscan::PREFIX##_n64;                                \
    return fn(lanes, split, grid, block, smem, s, p);

cudaError_t launch_f32_f32(int n, int lanes, int split, dim3 grid, dim3 block, size_t smem,
                           cudaStream_t s, const FwdParams &p) {
    SS_PICK_BUCKET(launch_f32_f32)
}
cudaError_t launch_bf16_bf16(int n, int lanes, int split, dim3 grid, dim3 block, size_t smem,
                             cudaStream_t s, const FwdParams &p) {
    SS_PICK_BUCKET(launch_bf16_bf16)
}
cudaError_t launch_bf16_f32(int n, int lanes, int split, dim3 grid, dim3 block, size_t smem,
                            cudaStream_t s, const FwdParams &p) {
    SS_PICK_BUCKET(launch_bf16_f32)
}

// The fix-up after a segmented direct kernel: the carry fold (one warp per
// row), then the correction of y (one warp per (row, segment >= 1)).
cudaError_t launch_fixup(const ss_desc *desc, int64_t rows, int nseg, cudaStream_t s, const FwdParams &p) {
    const int nmax = selscan::state_bucket((int)desc->dstate);
    const dim3 fold_grid((unsigned)((rows + 7) / 8));
    if (nmax > 32)
        selscan::ss_fwd_carry_kernel<64><<<fold_grid, 256, 0, s>>>(p);
    else
        selscan::ss_fwd_carry_kernel<32><<<fold_grid, 256, 0, s>>>(p);
    const int64_t tasks = rows * (nseg - 1);
    const dim3 grid((unsigned)((tasks + selscan::kFixupWarps - 1) / selscan::kFixupWarps));
    const dim3 block(selscan::kFixupWarps * 32);
    if (desc->in_dtype == SS_F32)
        selscan::ss_fwd_fixup_kernel<float, float><<<grid, block, 0, s>>>(p);
    else if (desc->out_dtype == SS_BF16)
        selscan::ss_fwd_fixup_kernel<__nv_bfloat16, __nv_bfloat16><<<grid, block, 0, s>>>(p);
    else
        selscan::ss_fwd_fixup_kernel<__nv_bfloat16, float><<<grid, block, 0, s>>>(p);
    return cudaGetLastError();
}

// The dt_proj form (delta_r given): bf16, the direct kernel with 4 warps and
// 2 or 4 lanes per row (double-buffered stages); the heuristic's state split
// and segments when they fit, else 4 (or 2) lanes and one pass.
bool dt_plan(const ss_desc *desc, Plan *pl) {
    const int bucket = selscan::state_bucket((int)desc->dstate);
    auto fits = [&](int g) { return g <= bucket / 2 && selscan::direct_double_buffer(bucket, g); };
    if (!((pl->split == 1 || pl->lanes == 1) && (pl->lanes == 2 || pl->lanes == 4) && fits(pl->lanes))) {
        pl->lanes = fits(4) ? 4 : fits(2) ? 2 : 0;
        pl->nseg = 1;
        pl->seg_len = desc->seqlen;
    }
    pl->split = 1;
    pl->warps = 4;
    return pl->lanes != 0;
}

ss_status fwd_impl(const ss_desc *desc, const void *u, const void *delta, const float *A,
                   const void *B, const void *C, const float *D, const void *z,
                   const float *delta_bias, int delta_softplus, const float *initial_state,
                   const uint8_t *reset, void *y, float *last_state, const ss_launch_config *cfg,
                   void *workspace, size_t workspace_bytes, ss_stream_t stream,
                   const void *delta_r = nullptr, const void *W_dt = nullptr, int dt_rank = 0,
                   float *ckpt = nullptr, int64_t bc_bstride = 0, int64_t dtr_bstride = 0) {
    Sizes sz;
    ss_status st = check_desc(desc, &sz);
    if (st != SS_OK) return st;
    if (!workspace) workspace_bytes = 0;
    const bool dt = dt_rank != 0;  // the dt_proj form (ss_fwd_dtproj)
    if (dt && desc->in_dtype != SS_BF16) return SS_ERR_UNSUPPORTED_DTYPE;
    if (dt && (dt_rank < 1 || dt_rank > selscan::kMaxDtRank)) return SS_ERR_BAD_SHAPE;
    Plan pl;
    // sequence starts and checkpoints are read / written by the direct kernel only
    st = resolve(desc, sz.rows, cfg, workspace_bytes, &pl, reset != nullptr || ckpt != nullptr);
    if (st != SS_OK) return st;
    if (dt && !dt_plan(desc, &pl)) return SS_ERR_BAD_CONFIG;
    if (ckpt != nullptr && (pl.split == 2 || dt)) return SS_ERR_BAD_CONFIG;  // the shared-memory direct kernel
    if (ckpt != nullptr && !aligned(ckpt, 4)) return SS_ERR_MISALIGNED;
    if (sz.rows == 0) return SS_OK;  // no rows: nothing to read or write
    const bool need_seq = desc->seqlen > 0;
    if (!A) return SS_ERR_NULL_POINTER;
    if (need_seq && (!u || (!dt && !delta) || (dt && (!delta_r || !W_dt)) || !B || !C || !y))
        return SS_ERR_NULL_POINTER;
    if (!need_seq && !last_state) return SS_OK;  // nothing to write
    if (!need_seq) pl.nseg = 1, pl.seg_len = 0;
    if (initial_state && !aligned(initial_state, 4)) return SS_ERR_MISALIGNED;

    const size_t ein = dtype_size(desc->in_dtype), eout = dtype_size(desc->out_dtype);
    const void *in_ptrs[] = {u, delta, B, C, z, delta_r, W_dt};
    for (const void *q : in_ptrs)
        if (q && !aligned(q, ein)) return SS_ERR_MISALIGNED;
    if ((y && !aligned(y, eout)) || !aligned(A, 4) || (D && !aligned(D, 4)) ||
        (delta_bias && !aligned(delta_bias, 4)) || (last_state && !aligned(last_state, 4)))
        return SS_ERR_MISALIGNED;
    const size_t ws_need = workspace_for(desc, sz.rows, pl);
    if (ws_need > workspace_bytes) return SS_ERR_WORKSPACE;
    if (ws_need && !aligned(workspace, 16)) return SS_ERR_MISALIGNED;

    // 16-byte vector path: every row of every streamed tensor starts aligned.
    bool vec = (desc->seqlen * (int64_t)ein) % 16 == 0 && (desc->seqlen * (int64_t)eout) % 16 == 0;
    for (const void *q : {u, delta, B, C, z, delta_r})
        if (q && !aligned(q, 16)) vec = false;
    if (y && !aligned(y, 16)) vec = false;

    size_t smem = smem_for(desc, pl.lanes, pl.split, pl.warps);
    if (dt) {  // + the dt_proj operands; at least 47 KB so that at most 4 blocks (4 x 128 TMEM columns) share an SM
        smem += selscan::direct_dt_extra_bytes((dt_rank + 15) / 16 * 16);
        if (smem < 47 * 1024) smem = 47 * 1024;
    }
    if (smem > selscan::kMaxSmemBytes) return SS_ERR_BAD_CONFIG;
    const int64_t rows_per_block = (int64_t)pl.warps * (32 / pl.lanes);  // compute warps
    const int64_t dtiles = (desc->dim + rows_per_block - 1) / rows_per_block;
    const int64_t blocks = dtiles * desc->batch * pl.nseg;
    if (blocks > INT_MAX || sz.rows * pl.nseg > INT_MAX) return SS_ERR_BAD_SHAPE;

    FwdParams p;
    p.u = u;
    p.delta = delta;
    p.B = B;
    p.C = C;
    p.z = z;
    p.A = A;
    p.D = D;
    p.delta_bias = delta_bias;
    p.y = y;
    p.last_state = last_state;
    p.init_state = initial_state;
    p.reset = reset;
    p.batch = desc->batch;
    p.dim = desc->dim;
    p.seqlen = desc->seqlen;
    p.dstate = (int)desc->dstate;
    p.softplus = delta_softplus ? 1 : 0;
    p.vec = vec ? 1 : 0;
    p.dtiles = dtiles;
    p.seg_len = pl.seg_len;
    p.nseg = pl.nseg;
    p.ws_hend = pl.nseg > 1 ? static_cast<float *>(workspace) : nullptr;
    p.ws_dsum = pl.nseg > 1 ? p.ws_hend + (size_t)pl.nseg * sz.rows * desc->dstate : nullptr;
    p.status = (pl.split == 2 || dt) ? device_status_ptr() : nullptr;
    p.delta_r = delta_r;
    p.W_dt = W_dt;
    p.dt_rank = dt_rank;
    p.ckpt = ckpt;
    p.bc_bstride = bc_bstride;
    p.dtr_bstride = dtr_bstride;

    const dim3 grid((unsigned)blocks), block((unsigned)(pl.warps * 32));
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int n = p.dstate, lanes = pl.lanes, split = pl.split;
    cudaError_t err;
    if (desc->in_dtype == SS_F32)
        err = launch_f32_f32(n, lanes, split, grid, block, smem, s, p);
    else if (desc->out_dtype == SS_BF16)
        err = launch_bf16_bf16(n, lanes, split, grid, block, smem, s, p);
    else
        err = launch_bf16_f32(n, lanes, split, grid, block, smem, s, p);
    if (err == cudaSuccess && pl.nseg > 1) err = launch_fixup(desc, sz.rows, pl.nseg, s, p);
    return err == cudaSuccess ? SS_OK : SS_ERR_CUDA;
}

// ---------------------------------------------------------------- backward
constexpr int kBwdWarps = selscan::kBwdThreads / 32;

// The backward runs the batch in groups of `group` entries, one launch of
// the adjoint kernel (and of the dB/dC sum) per group, so that the
// checkpoints and the dB/dC block partials, which grow with B*D*L*N, are
// held for one group at a time: the workspace of a group stays within
// kBwdGroupBytes (whole batch entries, at least one; groups of equal size up
// to the last).  The per-row partials of dA, dD and ddelta_bias are kept for
// every row and summed once at the end, in batch order, so the grouping
// changes no result bit.
constexpr size_t kBwdGroupBytes = (size_t)7 << 30;

struct BwdLayout {
    int lanes, rows;        // lanes per row, rows per block
    int64_t dtiles, nsub;
    int64_t group;          // batch entries per launch
    int nseg;               // sequence segments (1: none)
    int64_t seg_len;
    int fsum_k;             // forward-summary segments per segment (1, 2 or 4)
    size_t off_ckpt, off_dbc, off_dA, off_dD, off_dbias;                  // workspace byte offsets
    size_t off_hend, off_dsum, off_lam0, off_D, total;                    // segment records (nseg > 1)
};

// Sequence segments of the backward: when one batch group's blocks cannot
// give every SM three (the genomic shape: 4 x 1024 rows, 128 blocks of 32
// rows), the sequence is cut into segments of at least kMinSegSteps steps (a
// multiple of 64) so that about six blocks per SM run, each segment of each
// row from the true state entering it and the true adjoint entering its end
// (see ss_bwd_kernel.cuh).
int bwd_segments(const ss_desc *desc, int64_t blocks, int64_t *seg_len) {
    const int64_t sms = sm_count();
    *seg_len = desc->seqlen;
    if (blocks <= 0 || blocks >= 3 * sms || desc->seqlen < 2 * kMinSegSteps) return 1;
    int64_t want = (6 * sms + blocks - 1) / blocks;
    if (want > desc->seqlen / kMinSegSteps) want = desc->seqlen / kMinSegSteps;
    if (want < 2) return 1;
    return segment(desc, (int)want, seg_len);
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// ckpt_given: the forward's checkpoints come from the caller (ss_bwd_ckpt),
// so the workspace holds none; the plan is the same.
BwdLayout bwd_layout(const ss_desc *desc, const Sizes &sz, bool ckpt_given = false) {
    BwdLayout lo{};
    const int nmax = selscan::state_bucket((int)desc->dstate);
    lo.lanes = selscan::bwd_lanes(nmax);
    lo.rows = kBwdWarps * 32 / lo.lanes;
    lo.dtiles = (desc->dim + lo.rows - 1) / lo.rows;
    lo.nsub = (desc->seqlen + selscan::kBwdSub - 1) / selscan::kBwdSub;
    const size_t N = (size_t)desc->dstate, rows = (size_t)sz.rows, L = (size_t)desc->seqlen;
    // bytes one batch entry adds to the checkpoints and the block partials
    const size_t per_entry = (size_t)desc->dim * (size_t)lo.nsub * N * 4 + (size_t)lo.dtiles * 2 * N * L * 4;
    int64_t group = desc->batch;
    if (per_entry > 0 && desc->batch > 0) {
        const int64_t fit = (int64_t)(kBwdGroupBytes / per_entry);
        const int64_t cap = fit < 1 ? 1 : fit;
        const int64_t ngroups = (desc->batch + cap - 1) / cap;
        group = (desc->batch + ngroups - 1) / ngroups;
    }
    lo.group = group;
    lo.nseg = bwd_segments(desc, lo.dtiles * group, &lo.seg_len);
    // The forward summary (run only without the forward's checkpoints) is the
    // direct kernel with 64-row blocks, half the adjoint kernel's row tiles:
    // over the adjoint's segments it would fill under one wave of the GPU
    // (the genomic layer: 448 blocks), so it cuts each segment into four (or
    // two) pieces where they stay whole 64-step stages (genomic layer's plain
    // backward 22.75 ms uncut, 22.39 in halves, 22.17 in quarters).
    lo.fsum_k = 1;
    if (lo.nseg > 1 && !ckpt_given) lo.fsum_k = lo.seg_len % 256 == 0 ? 4 : lo.seg_len % 128 == 0 ? 2 : 1;
    const size_t grows = (size_t)group * (size_t)desc->dim, S = (size_t)lo.nseg;
    lo.off_ckpt = 0;
    lo.off_dbc = align256(lo.off_ckpt + (ckpt_given ? 0 : grows * (size_t)lo.nsub * N * 4));
    lo.off_dA = align256(lo.off_dbc + (size_t)lo.dtiles * (size_t)group * 2 * N * L * 4);
    lo.off_dD = align256(lo.off_dA + S * rows * N * 4);
    lo.off_dbias = align256(lo.off_dD + S * rows * 4);
    lo.off_hend = align256(lo.off_dbias + S * rows * 4);
    const size_t seg_rec = lo.nseg > 1 ? S * grows : 0;  // (segment, row) records of one group
    const size_t fsum_rec = seg_rec * (size_t)lo.fsum_k;  // the forward summary's records
    lo.off_dsum = align256(lo.off_hend + fsum_rec * N * 4);
    lo.off_lam0 = align256(lo.off_dsum + fsum_rec * 4);
    lo.off_D = align256(lo.off_lam0 + seg_rec * N * 4);
    lo.total = align256(lo.off_D + seg_rec * N * 4);
    return lo;
}

template <typename Tin, typename Tout>
cudaError_t launch_step(int T, dim3 grid, cudaStream_t s, const selscan::StepParams &p) {
    switch (T) {
        case 2: selscan::ss_step_kernel<Tin, Tout, 2><<<grid, 256, 0, s>>>(p); break;
        case 4: selscan::ss_step_kernel<Tin, Tout, 4><<<grid, 256, 0, s>>>(p); break;
        case 8: selscan::ss_step_kernel<Tin, Tout, 8><<<grid, 256, 0, s>>>(p); break;
        case 16: selscan::ss_step_kernel<Tin, Tout, 16><<<grid, 256, 0, s>>>(p); break;
        default: selscan::ss_step_kernel<Tin, Tout, 32><<<grid, 256, 0, s>>>(p); break;
    }
    return cudaGetLastError();
}

#define SS_PICK_BWD(PREFIX)                                                                  \
    n <= 4 ? selscan::PREFIX##_n4 : n <= 8 ? selscan::PREFIX##_n8 : n <= 16 ? selscan::PREFIX##_n16 \
    : n <= 32 ? selscan::PREFIX##_n32 : selscan::PREFIX##_n64

}  // namespace

extern "C" {

ss_status ss_fwd(const ss_desc *desc, const void *u, const void *delta, const float *A,
                 const void *B, const void *C, const float *D, const void *z,
                 const float *delta_bias, int delta_softplus, void *y, float *last_state,
                 ss_stream_t stream) {
    return fwd_impl(desc, u, delta, A, B, C, D, z, delta_bias, delta_softplus, nullptr, nullptr, y,
                    last_state, nullptr, nullptr, 0, stream);
}

ss_status ss_fwd_ws(const ss_desc *desc, const void *u, const void *delta, const float *A,
                    const void *B, const void *C, const float *D, const void *z,
                    const float *delta_bias, int delta_softplus, void *y, float *last_state,
                    void *workspace, size_t workspace_bytes, ss_stream_t stream) {
    return fwd_impl(desc, u, delta, A, B, C, D, z, delta_bias, delta_softplus, nullptr, nullptr, y,
                    last_state, nullptr, workspace, workspace_bytes, stream);
}

ss_status ss_fwd_with_config(const ss_desc *desc, const void *u, const void *delta,
                             const float *A, const void *B, const void *C, const float *D,
                             const void *z, const float *delta_bias, int delta_softplus,
                             void *y, float *last_state, const ss_launch_config *config,
                             void *workspace, size_t workspace_bytes, ss_stream_t stream) {
    if (!config) return SS_ERR_NULL_POINTER;
    return fwd_impl(desc, u, delta, A, B, C, D, z, delta_bias, delta_softplus, nullptr, nullptr, y,
                    last_state, config, workspace, workspace_bytes, stream);
}

ss_status ss_fwd_state(const ss_desc *desc, const void *u, const void *delta, const float *A,
                       const void *B, const void *C, const float *D, const void *z,
                       const float *delta_bias, int delta_softplus, const float *initial_state,
                       void *y, float *last_state, const ss_launch_config *config, void *workspace,
                       size_t workspace_bytes, ss_stream_t stream) {
    return fwd_impl(desc, u, delta, A, B, C, D, z, delta_bias, delta_softplus, initial_state, nullptr,
                    y, last_state, config, workspace, workspace_bytes, stream);
}

ss_status ss_fwd_dtproj(const ss_desc *desc, int dt_rank, const void *u, const void *delta_r,
                        const void *W_dt, const float *A, const void *B, const void *C, const float *D,
                        const void *z, const float *delta_bias, int delta_softplus, void *y,
                        float *last_state, void *workspace, size_t workspace_bytes, ss_stream_t stream) {
    if (dt_rank == 0) return SS_ERR_BAD_SHAPE;
    return fwd_impl(desc, u, nullptr, A, B, C, D, z, delta_bias, delta_softplus, nullptr, nullptr, y, last_state,
                    nullptr, workspace, workspace_bytes, stream, delta_r, W_dt, dt_rank);
}

ss_status ss_fwd_xdbl(const ss_desc *desc, int dt_rank, const void *u, const void *x_dbl, const void *W_dt,
                      const float *A, const float *D, const void *z, const float *delta_bias, int delta_softplus,
                      void *y, float *last_state, void *workspace, size_t workspace_bytes, ss_stream_t stream) {
    Sizes sz;
    const ss_status st = check_desc(desc, &sz);
    if (st != SS_OK) return st;
    if (dt_rank < 1 || dt_rank > selscan::kMaxDtRank) return SS_ERR_BAD_SHAPE;
    if (desc->in_dtype != SS_BF16) return SS_ERR_UNSUPPORTED_DTYPE;
    if (!x_dbl && sz.rows > 0 && desc->seqlen > 0) return SS_ERR_NULL_POINTER;
    // delta_r, B and C are the row ranges [0, R), [R, R + N), [R + N, R + 2N)
    // of each batch entry's (R + 2N, L) block.
    const int64_t L = desc->seqlen, N = desc->dstate, feats = dt_rank + 2 * N;
    const size_t e = dtype_size(desc->in_dtype);
    const char *xb = static_cast<const char *>(x_dbl);
    const void *B = xb ? xb + (size_t)dt_rank * (size_t)L * e : nullptr;
    const void *C = xb ? xb + (size_t)(dt_rank + N) * (size_t)L * e : nullptr;
    return fwd_impl(desc, u, nullptr, A, B, C, D, z, delta_bias, delta_softplus, nullptr, nullptr, y, last_state,
                    nullptr, workspace, workspace_bytes, stream, x_dbl, W_dt, dt_rank, nullptr, feats * L, feats * L);
}

ss_status ss_fwd_ckpt(const ss_desc *desc, const void *u, const void *delta, const float *A, const void *B,
                      const void *C, const float *D, const void *z, const float *delta_bias, int delta_softplus,
                      const float *initial_state, const uint8_t *reset, void *y, float *last_state, float *ckpt,
                      void *workspace, size_t workspace_bytes, ss_stream_t stream) {
    if (!ckpt && desc && desc->batch > 0 && desc->dim > 0 && desc->seqlen > 0) return SS_ERR_NULL_POINTER;
    return fwd_impl(desc, u, delta, A, B, C, D, z, delta_bias, delta_softplus, initial_state, reset, y, last_state,
                    nullptr, workspace, workspace_bytes, stream, nullptr, nullptr, 0, ckpt);
}

ss_status ss_fwd_reset(const ss_desc *desc, const void *u, const void *delta, const float *A,
                       const void *B, const void *C, const float *D, const void *z,
                       const float *delta_bias, int delta_softplus, const uint8_t *reset,
                       const float *initial_state, void *y, float *last_state,
                       const ss_launch_config *config, void *workspace, size_t workspace_bytes,
                       ss_stream_t stream) {
    if (!reset && desc && desc->batch > 0 && desc->dim > 0 && desc->seqlen > 0) return SS_ERR_NULL_POINTER;
    return fwd_impl(desc, u, delta, A, B, C, D, z, delta_bias, delta_softplus, initial_state, reset, y,
                    last_state, config, workspace, workspace_bytes, stream);
}

ss_status ss_fwd_heuristic(const ss_desc *desc, size_t workspace_bytes, ss_launch_config *config) {
    Sizes sz;
    ss_status st = check_desc(desc, &sz);
    if (st != SS_OK) return st;
    if (!config) return SS_ERR_NULL_POINTER;
    const Plan pl = heuristic(desc, sz.rows, sm_count(), workspace_bytes);
    config->lanes_per_row = pl.lanes;
    config->split_states = pl.split;
    config->warps_per_block = pl.warps;
    config->segments = pl.nseg;
    return SS_OK;
}

size_t ss_fwd_workspace_bytes(const ss_desc *desc, const ss_launch_config *config) {
    Sizes sz;
    if (check_desc(desc, &sz) != SS_OK) return 0;
    Plan pl;
    if (resolve(desc, sz.rows, config, SIZE_MAX, &pl) != SS_OK) return 0;
    return workspace_for(desc, sz.rows, pl);
}

ss_status ss_fwd_hostio(const ss_desc *desc, const void *h_u, const void *h_delta,
                        const float *h_A, const void *h_B, const void *h_C, const float *h_D,
                        const void *h_z, const float *h_delta_bias, int delta_softplus,
                        void *h_y, float *h_last_state, void *d_u, void *d_delta, float *d_A,
                        void *d_B, void *d_C, float *d_D, void *d_z, float *d_delta_bias,
                        void *d_y, float *d_last_state, void *d_workspace, size_t workspace_bytes,
                        ss_stream_t stream) {
    Sizes sz;
    ss_status st = check_desc(desc, &sz);
    if (st != SS_OK) return st;
    if (sz.rows == 0) return SS_OK;
    // Optional operands: host and device buffers present together or not at all.
    if ((!h_D) != (!d_D) || (!h_z) != (!d_z) || (!h_delta_bias) != (!d_delta_bias) ||
        (!h_last_state) != (!d_last_state))
        return SS_ERR_NULL_POINTER;
    if (!h_A || !d_A) return SS_ERR_NULL_POINTER;
    if (desc->seqlen > 0 && (!h_u || !h_delta || !h_B || !h_C || !h_y || !d_u || !d_delta ||
                             !d_B || !d_C || !d_y))
        return SS_ERR_NULL_POINTER;

    const size_t ein = dtype_size(desc->in_dtype), eout = dtype_size(desc->out_dtype);
    const size_t n_seq = (size_t)sz.elems * ein, n_bc = (size_t)sz.bc_elems * ein;
    const size_t n_A = (size_t)desc->dim * desc->dstate * 4, n_vec = (size_t)desc->dim * 4;
    const size_t n_y = (size_t)sz.elems * eout, n_last = (size_t)sz.rows * desc->dstate * 4;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const cudaMemcpyKind h2d = cudaMemcpyHostToDevice, d2h = cudaMemcpyDeviceToHost;

    struct Copy {
        void *dst;
        const void *src;
        size_t bytes;
    } in_copies[] = {{d_u, h_u, n_seq},  {d_delta, h_delta, n_seq}, {d_A, h_A, n_A},
                     {d_B, h_B, n_bc},   {d_C, h_C, n_bc},          {d_D, h_D, n_vec},
                     {d_z, h_z, n_seq},  {d_delta_bias, h_delta_bias, n_vec}};
    for (const Copy &c : in_copies)
        if (c.dst && c.bytes && cudaMemcpyAsync(c.dst, c.src, c.bytes, h2d, s) != cudaSuccess)
            return SS_ERR_CUDA;
    st = fwd_impl(desc, d_u, d_delta, d_A, d_B, d_C, d_D, d_z, d_delta_bias, delta_softplus, nullptr,
                  nullptr, d_y, d_last_state, nullptr, d_workspace, workspace_bytes, stream);
    if (st != SS_OK) return st;
    if (n_y && cudaMemcpyAsync(h_y, d_y, n_y, d2h, s) != cudaSuccess) return SS_ERR_CUDA;
    if (d_last_state && cudaMemcpyAsync(h_last_state, d_last_state, n_last, d2h, s) != cudaSuccess)
        return SS_ERR_CUDA;
    return SS_OK;
}

ss_status ss_fwd_hostio_streams(const ss_desc *desc, const void *h_u, const void *h_delta,
                                const float *h_A, const void *h_B, const void *h_C, const float *h_D,
                                const void *h_z, const float *h_delta_bias, int delta_softplus,
                                void *h_y, float *h_last_state, void *d_u, void *d_delta, float *d_A,
                                void *d_B, void *d_C, float *d_D, void *d_z, float *d_delta_bias,
                                void *d_y, float *d_last_state, void *d_workspace,
                                size_t workspace_bytes, const ss_stream_t *streams, int nstreams,
                                int chunks) {
    Sizes sz;
    ss_status st = check_desc(desc, &sz);
    if (st != SS_OK) return st;
    if (!streams || nstreams < 1 || nstreams > 16 || chunks < 0) return SS_ERR_BAD_CONFIG;
    if (sz.rows == 0) return SS_OK;
    if ((!h_D) != (!d_D) || (!h_z) != (!d_z) || (!h_delta_bias) != (!d_delta_bias) ||
        (!h_last_state) != (!d_last_state))
        return SS_ERR_NULL_POINTER;
    if (!h_A || !d_A) return SS_ERR_NULL_POINTER;
    if (desc->seqlen > 0 && (!h_u || !h_delta || !h_B || !h_C || !h_y || !d_u || !d_delta ||
                             !d_B || !d_C || !d_y))
        return SS_ERR_NULL_POINTER;

    const int64_t Bt = desc->batch, Dm = desc->dim, L = desc->seqlen, N = desc->dstate;
    const size_t ein = dtype_size(desc->in_dtype), eout = dtype_size(desc->out_dtype);
    const cudaMemcpyKind h2d = cudaMemcpyHostToDevice, d2h = cudaMemcpyDeviceToHost;
    int nch = chunks > 0 ? chunks : (int)(Bt < 2 * nstreams ? Bt : 2 * nstreams);
    if (nch > Bt) nch = (int)Bt;
    cudaStream_t s0 = reinterpret_cast<cudaStream_t>(streams[0]);

    // Order this call after everything queued on any of the streams, copy the
    // per-channel operands on the first stream, and let every stream wait for them.
    cudaEvent_t ev[16] = {};
    auto cleanup = [&]() {
        for (int k = 0; k < nstreams; ++k)
            if (ev[k]) cudaEventDestroy(ev[k]);
    };
    for (int k = 0; k < nstreams; ++k)
        if (cudaEventCreateWithFlags(&ev[k], cudaEventDisableTiming) != cudaSuccess) return cleanup(), SS_ERR_CUDA;
    for (int k = 1; k < nstreams; ++k) {
        cudaStream_t sk = reinterpret_cast<cudaStream_t>(streams[k]);
        if (cudaEventRecord(ev[k], sk) != cudaSuccess || cudaStreamWaitEvent(s0, ev[k], 0) != cudaSuccess)
            return cleanup(), SS_ERR_CUDA;
    }
    const size_t n_A = (size_t)Dm * N * 4, n_vec = (size_t)Dm * 4;
    if (cudaMemcpyAsync(d_A, h_A, n_A, h2d, s0) != cudaSuccess ||
        (d_D && cudaMemcpyAsync(d_D, h_D, n_vec, h2d, s0) != cudaSuccess) ||
        (d_delta_bias && cudaMemcpyAsync(d_delta_bias, h_delta_bias, n_vec, h2d, s0) != cudaSuccess) ||
        cudaEventRecord(ev[0], s0) != cudaSuccess)
        return cleanup(), SS_ERR_CUDA;
    for (int k = 1; k < nstreams; ++k)
        if (cudaStreamWaitEvent(reinterpret_cast<cudaStream_t>(streams[k]), ev[0], 0) != cudaSuccess)
            return cleanup(), SS_ERR_CUDA;

    // Each chunk of batch entries: its inputs in, its forward, its outputs out,
    // all on one stream (chunk c on stream c mod nstreams, with that stream's
    // share of the workspace), so copies of one chunk overlap the work of others.
    const size_t ws_share = nstreams > 0 ? (workspace_bytes / (size_t)nstreams) / 256 * 256 : 0;
    for (int c = 0; c < nch; ++c) {
        const int64_t b0 = Bt * c / nch, b1 = Bt * (c + 1) / nch, bc = b1 - b0;
        if (bc <= 0) continue;
        const int k = c % nstreams;
        cudaStream_t sk = reinterpret_cast<cudaStream_t>(streams[k]);
        const size_t seq0 = (size_t)(b0 * Dm * L), nseq = (size_t)(bc * Dm * L);
        const size_t bc0 = (size_t)(b0 * N * L), nbc = (size_t)(bc * N * L);
        const size_t st0 = (size_t)(b0 * Dm * N), nst = (size_t)(bc * Dm * N);
        auto off = [](const void *p, size_t e) -> void * {
            return p ? const_cast<char *>(static_cast<const char *>(p)) + e : nullptr;
        };
        struct Copy {
            void *dst;
            const void *src;
            size_t bytes;
        } in_copies[] = {{off(d_u, seq0 * ein), off(h_u, seq0 * ein), nseq * ein},
                         {off(d_delta, seq0 * ein), off(h_delta, seq0 * ein), nseq * ein},
                         {off(d_z, seq0 * ein), off(h_z, seq0 * ein), nseq * ein},
                         {off(d_B, bc0 * ein), off(h_B, bc0 * ein), nbc * ein},
                         {off(d_C, bc0 * ein), off(h_C, bc0 * ein), nbc * ein}};
        for (const Copy &cp : in_copies)
            if (cp.dst && cp.bytes && cudaMemcpyAsync(cp.dst, cp.src, cp.bytes, h2d, sk) != cudaSuccess)
                return cleanup(), SS_ERR_CUDA;
        ss_desc dc = *desc;
        dc.batch = bc;
        st = fwd_impl(&dc, off(d_u, seq0 * ein), off(d_delta, seq0 * ein), d_A, off(d_B, bc0 * ein),
                      off(d_C, bc0 * ein), d_D, off(d_z, seq0 * ein), d_delta_bias, delta_softplus, nullptr,
                      nullptr, off(d_y, seq0 * eout), static_cast<float *>(off(d_last_state, st0 * 4)), nullptr,
                      d_workspace ? off(d_workspace, (size_t)k * ws_share) : nullptr,
                      d_workspace ? ws_share : 0, reinterpret_cast<ss_stream_t>(sk));
        if (st != SS_OK) return cleanup(), st;
        if (nseq && cudaMemcpyAsync(off(h_y, seq0 * eout), off(d_y, seq0 * eout), nseq * eout, d2h, sk) !=
                        cudaSuccess)
            return cleanup(), SS_ERR_CUDA;
        if (d_last_state && cudaMemcpyAsync(off(h_last_state, st0 * 4), off(d_last_state, st0 * 4), nst * 4,
                                            d2h, sk) != cudaSuccess)
            return cleanup(), SS_ERR_CUDA;
    }
    cleanup();  // (events are released once their waits are done)
    return SS_OK;
}

size_t ss_bwd_workspace_bytes(const ss_desc *desc) {
    Sizes sz;
    if (check_desc(desc, &sz) != SS_OK) return 0;
    return bwd_layout(desc, sz).total;
}

ss_status ss_bwd_heuristic(const ss_desc *desc, int64_t *batch_group, int *segments) {
    Sizes sz;
    const ss_status st = check_desc(desc, &sz);
    if (st != SS_OK) return st;
    if (!batch_group || !segments) return SS_ERR_NULL_POINTER;
    const BwdLayout lo = bwd_layout(desc, sz);
    *batch_group = lo.group;
    *segments = lo.nseg;
    return SS_OK;
}

}  // extern "C"

namespace {

// The per-segment summaries and their folds for one batch group (q: the
// group's backward parameters): the forward direct kernel in segment mode
// without y (end states and delta' sums), the forward carry fold (true
// entering states), the adjoint summaries and the backward fold (true
// last-state gradients), into the workspace's segment records.
template <typename Tin, typename Tout>
cudaError_t launch_seg_adjoint(int nmax, dim3 grid, cudaStream_t s, const selscan::BwdParams &q, float *lam0,
                               float *dsum) {
    switch (nmax) {
        case 4: selscan::ss_bwd_seg_adjoint_kernel<Tin, Tout, 4><<<grid, 128, 0, s>>>(q, lam0, dsum); break;
        case 8: selscan::ss_bwd_seg_adjoint_kernel<Tin, Tout, 8><<<grid, 128, 0, s>>>(q, lam0, dsum); break;
        case 16: selscan::ss_bwd_seg_adjoint_kernel<Tin, Tout, 16><<<grid, 128, 0, s>>>(q, lam0, dsum); break;
        case 32: selscan::ss_bwd_seg_adjoint_kernel<Tin, Tout, 32><<<grid, 128, 0, s>>>(q, lam0, dsum); break;
        default: selscan::ss_bwd_seg_adjoint_kernel<Tin, Tout, 64><<<grid, 128, 0, s>>>(q, lam0, dsum); break;
    }
    return cudaGetLastError();
}

ss_status bwd_segment_summaries(const ss_desc *desc, const BwdLayout &lo, const selscan::BwdParams &q, char *ws,
                                cudaStream_t s) {
    const int nmax = selscan::state_bucket(q.dstate), n = nmax;
    const int64_t grows = q.batch * q.dim;
    const size_t ein = dtype_size(desc->in_dtype);
    float *hend = reinterpret_cast<float *>(ws + lo.off_hend);
    float *dsum = reinterpret_cast<float *>(ws + lo.off_dsum);
    float *lam0 = reinterpret_cast<float *>(ws + lo.off_lam0);
    float *D = reinterpret_cast<float *>(ws + lo.off_D);

    // Forward summaries (only when the adjoint kernel runs its own phase A:
    // the forward's checkpoints already hold the true states): the direct
    // kernel with 2 lanes per row (1 below 4 states), segment mode, no y, no
    // gate or skip (they do not touch the state).
    cudaError_t err;
    const dim3 fold_grid((unsigned)((grows + 7) / 8));
    if (!q.ckpt_given) {
        FwdParams f{};
        f.u = q.u, f.delta = q.delta, f.B = q.B, f.C = q.C, f.z = nullptr;
        f.A = q.A, f.D = nullptr, f.delta_bias = q.delta_bias;
        f.y = nullptr, f.last_state = nullptr, f.init_state = q.init_state, f.reset = q.reset;
        f.batch = q.batch, f.dim = q.dim, f.seqlen = q.seqlen, f.dstate = q.dstate, f.softplus = q.softplus;
        bool vec = (q.seqlen * (int64_t)ein) % 16 == 0;
        for (const void *ptr : {q.u, q.delta, q.B, q.C})
            if (ptr && !aligned(ptr, 16)) vec = false;
        f.vec = vec ? 1 : 0;
        const int lanes = nmax / 2 >= 2 ? 2 : 1, warps = 4;
        const int64_t rows_per_block = (int64_t)warps * (32 / lanes);
        f.dtiles = (q.dim + rows_per_block - 1) / rows_per_block;
        f.seg_len = q.seg_len / lo.fsum_k, f.nseg = q.nseg * lo.fsum_k;
        f.ws_hend = hend, f.ws_dsum = dsum;
        f.status = nullptr, f.delta_r = nullptr, f.W_dt = nullptr, f.dt_rank = 0;
        const size_t smem = selscan::direct_smem_bytes(ein, nmax, lanes, warps);
        const dim3 grid((unsigned)(f.dtiles * q.batch * f.nseg)), block((unsigned)(warps * 32));
        const int split = lanes > 1 ? 1 : 0;
        if (desc->in_dtype == SS_F32) err = launch_f32_f32(n, lanes, split, grid, block, smem, s, f);
        else if (desc->out_dtype == SS_BF16) err = launch_bf16_bf16(n, lanes, split, grid, block, smem, s, f);
        else err = launch_bf16_f32(n, lanes, split, grid, block, smem, s, f);
        if (err != cudaSuccess) return SS_ERR_CUDA;
        if (nmax > 32) selscan::ss_fwd_carry_kernel<64><<<fold_grid, 256, 0, s>>>(f);
        else selscan::ss_fwd_carry_kernel<32><<<fold_grid, 256, 0, s>>>(f);
        if (cudaGetLastError() != cudaSuccess) return SS_ERR_CUDA;
    }

    // Adjoint summaries of segments 1.., then the backward fold.
    const int per = nmax < 8 ? 1 : nmax / 8;  // threads per (segment, row)
    const int64_t threads = grows * (q.nseg - 1) * per;
    const dim3 agrid((unsigned)((threads + 127) / 128));
    if (desc->in_dtype == SS_F32) err = launch_seg_adjoint<float, float>(nmax, agrid, s, q, lam0, dsum);
    else if (desc->out_dtype == SS_BF16)
        err = launch_seg_adjoint<__nv_bfloat16, __nv_bfloat16>(nmax, agrid, s, q, lam0, dsum);
    else err = launch_seg_adjoint<__nv_bfloat16, float>(nmax, agrid, s, q, lam0, dsum);
    if (err != cudaSuccess) return SS_ERR_CUDA;
    if (nmax > 32) selscan::ss_bwd_seg_fold_kernel<64><<<fold_grid, 256, 0, s>>>(q, lam0, dsum, D);
    else selscan::ss_bwd_seg_fold_kernel<32><<<fold_grid, 256, 0, s>>>(q, lam0, dsum, D);
    return cudaGetLastError() == cudaSuccess ? SS_OK : SS_ERR_CUDA;
}

ss_status bwd_impl(const ss_desc *desc, const void *u, const void *delta, const float *A, const void *B,
                   const void *C, const float *D, const void *z, const float *delta_bias,
                   int delta_softplus, const uint8_t *reset, const float *init_state,
                   const float *dlast, const void *dy, void *du, void *ddelta, float *dA, float *dB,
                   float *dC, float *dD, void *dz, float *ddelta_bias, float *d_init_state,
                   void *workspace, size_t workspace_bytes, ss_stream_t stream,
                   const float *fwd_ckpt = nullptr) {
    Sizes sz;
    ss_status st = check_desc(desc, &sz);
    if (st != SS_OK) return st;
    if (!A || !dA) return SS_ERR_NULL_POINTER;
    const bool work = sz.rows > 0 && desc->seqlen > 0;
    if (work && (!u || !delta || !B || !C || !dy || !du || !ddelta || !dB || !dC)) return SS_ERR_NULL_POINTER;
    if ((D && !dD) || (z && !dz) || (delta_bias && !ddelta_bias)) return SS_ERR_NULL_POINTER;
    const size_t ein = dtype_size(desc->in_dtype), eout = dtype_size(desc->out_dtype);
    const void *in_ptrs[] = {u, delta, B, C, z, du, ddelta, dz};
    for (const void *q : in_ptrs)
        if (q && !aligned(q, ein)) return SS_ERR_MISALIGNED;
    const void *f_ptrs[] = {A, D, delta_bias, dA, dB, dC, dD, ddelta_bias, init_state, dlast, d_init_state, fwd_ckpt};
    for (const void *q : f_ptrs)
        if (q && !aligned(q, 4)) return SS_ERR_MISALIGNED;
    if (dy && !aligned(dy, eout)) return SS_ERR_MISALIGNED;
    const BwdLayout lo = bwd_layout(desc, sz, fwd_ckpt != nullptr);
    if (!workspace || workspace_bytes < lo.total) return SS_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return SS_ERR_MISALIGNED;
    const int64_t blocks = lo.dtiles * lo.group * lo.nseg;
    if (blocks > INT_MAX || sz.rows * lo.nseg * 8 > INT_MAX) return SS_ERR_BAD_SHAPE;

    char *ws = static_cast<char *>(workspace);
    selscan::BwdParams p;
    p.u = u, p.delta = delta, p.B = B, p.C = C, p.z = z, p.dy = dy;
    p.A = A, p.D = D, p.delta_bias = delta_bias;
    p.du = du, p.ddelta = ddelta, p.dz = dz;
    p.ckpt = reinterpret_cast<float *>(ws + lo.off_ckpt);
    p.ws_dBC = reinterpret_cast<float *>(ws + lo.off_dbc);
    p.ws_dA = reinterpret_cast<float *>(ws + lo.off_dA);
    p.ws_dD = reinterpret_cast<float *>(ws + lo.off_dD);
    p.ws_dbias = reinterpret_cast<float *>(ws + lo.off_dbias);
    p.batch = desc->batch, p.dim = desc->dim, p.seqlen = desc->seqlen;
    p.dstate = (int)desc->dstate;
    p.softplus = delta_softplus ? 1 : 0;
    p.vec = (desc->seqlen * (int64_t)ein) % 16 == 0 && (!B || aligned(B, 16)) && (!C || aligned(C, 16));
    p.vec_rows = (desc->seqlen * (int64_t)ein) % 16 == 0 && (desc->seqlen * (int64_t)eout) % 16 == 0 &&
                 (!u || aligned(u, 16)) && (!delta || aligned(delta, 16)) && (!z || aligned(z, 16)) &&
                 (!dy || aligned(dy, 16));
    p.dtiles = lo.dtiles;
    p.nsub = lo.nsub;
    p.reset = reset;
    p.reset_vec = reset && desc->seqlen % selscan::kBwdSub == 0 && aligned(reset, selscan::kBwdSub);
    p.init_state = init_state;
    p.dlast = dlast;
    p.d_init_state = d_init_state;
    p.seg_len = lo.nseg > 1 ? lo.seg_len : desc->seqlen;
    p.nseg = lo.nseg;
    p.rows_all = sz.rows;
    p.seg_h = nullptr;
    p.seg_dl = nullptr;
    p.ckpt_given = fwd_ckpt != nullptr ? 1 : 0;
    if (fwd_ckpt != nullptr) p.ckpt = const_cast<float *>(fwd_ckpt);  // read only in that mode

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int nmax = selscan::state_bucket(p.dstate), n = nmax;
    if (sz.rows > 0) {
        const size_t smem = selscan::bwd_smem_bytes(ein, nmax, kBwdWarps);
        cudaError_t (*fn)(dim3, dim3, size_t, cudaStream_t, const selscan::BwdParams &) =
            desc->in_dtype == SS_F32 ? (SS_PICK_BWD(bwd_f32_f32))
            : desc->out_dtype == SS_BF16 ? (SS_PICK_BWD(bwd_bf16_bf16))
                                         : (SS_PICK_BWD(bwd_bf16_f32));
        // One launch per batch group: every pointer indexed by batch entry
        // starts at the group's first entry; checkpoints and block partials
        // are reused, the per-row partials go to the group's rows.
        const int64_t DL = desc->dim * desc->seqlen, NL = desc->dstate * desc->seqlen;
        const int64_t DN = desc->dim * desc->dstate;
        for (int64_t b0 = 0; b0 < desc->batch; b0 += lo.group) {
            const int64_t gb = desc->batch - b0 < lo.group ? desc->batch - b0 : lo.group;
            selscan::BwdParams q = p;
            auto adv = [](const void *ptr, int64_t elems, size_t es) -> const void * {
                return ptr ? static_cast<const char *>(ptr) + elems * (int64_t)es : nullptr;
            };
            auto advm = [](void *ptr, int64_t elems, size_t es) -> void * {
                return ptr ? static_cast<char *>(ptr) + elems * (int64_t)es : nullptr;
            };
            q.batch = gb;
            q.u = adv(u, b0 * DL, ein), q.delta = adv(delta, b0 * DL, ein), q.z = adv(z, b0 * DL, ein);
            q.dy = adv(dy, b0 * DL, eout);
            q.B = adv(B, b0 * NL, ein), q.C = adv(C, b0 * NL, ein);
            q.du = advm(du, b0 * DL, ein), q.ddelta = advm(ddelta, b0 * DL, ein), q.dz = advm(dz, b0 * DL, ein);
            q.ws_dA = p.ws_dA + b0 * DN;
            q.ws_dD = p.ws_dD + b0 * desc->dim;
            q.ws_dbias = p.ws_dbias + b0 * desc->dim;
            q.reset = reset ? reset + b0 * desc->seqlen : nullptr;
            q.init_state = init_state ? init_state + b0 * DN : nullptr;
            q.dlast = dlast ? dlast + b0 * DN : nullptr;
            q.d_init_state = d_init_state ? d_init_state + b0 * DN : nullptr;
            if (fwd_ckpt != nullptr) q.ckpt = p.ckpt + b0 * desc->dim * lo.nsub * desc->dstate;
            if (lo.nseg > 1 && desc->seqlen > 0) {
                const ss_status ss = bwd_segment_summaries(desc, lo, q, ws, s);
                if (ss != SS_OK) return ss;
                q.seg_h = reinterpret_cast<const float *>(ws + lo.off_hend);
                q.seg_h_k = lo.fsum_k;
                q.seg_dl = reinterpret_cast<const float *>(ws + lo.off_D);
            }
            if (fn(dim3((unsigned)(lo.dtiles * gb * lo.nseg)), dim3(kBwdWarps * 32), smem, s, q) != cudaSuccess)
                return SS_ERR_CUDA;
            const int64_t bc = gb * 2 * NL;
            if (bc > 0) {  // one thread per four outputs when the kernel can read float4 rows
                const bool v4 = NL % 4 == 0 && aligned(q.ws_dBC, 16) && aligned(dB + b0 * NL, 16) &&
                                aligned(dC + b0 * NL, 16);
                const int64_t nb = ((v4 ? bc / 4 : bc) + 255) / 256;
                selscan::ss_bwd_reduce_bc_kernel<<<(unsigned)(nb < 4 * 148 * 8 ? nb : 4 * 148 * 8), 256, 0, s>>>(
                    q, dB + b0 * NL, dC + b0 * NL);
                if (cudaGetLastError() != cudaSuccess) return SS_ERR_CUDA;
            }
        }
    }
    const int64_t rr = desc->dim * (desc->dstate + 2);
    if (rr > 0) {
        const int64_t gb = (rr + 255) / 256;
        selscan::ss_bwd_reduce_rows_kernel<<<(unsigned)(gb < 4 * 148 ? gb : 4 * 148), 256, 0, s>>>(p, dA, dD,
                                                                                                 ddelta_bias);
        if (cudaGetLastError() != cudaSuccess) return SS_ERR_CUDA;
    }
    return SS_OK;
}

}  // namespace

extern "C" {

ss_status ss_bwd(const ss_desc *desc, const void *u, const void *delta, const float *A, const void *B,
                 const void *C, const float *D, const void *z, const float *delta_bias,
                 int delta_softplus, const void *dy, void *du, void *ddelta, float *dA, float *dB,
                 float *dC, float *dD, void *dz, float *ddelta_bias, void *workspace,
                 size_t workspace_bytes, ss_stream_t stream) {
    return bwd_impl(desc, u, delta, A, B, C, D, z, delta_bias, delta_softplus, nullptr, nullptr, nullptr, dy,
                    du, ddelta, dA, dB, dC, dD, dz, ddelta_bias, nullptr, workspace, workspace_bytes, stream);
}

ss_status ss_bwd_reset(const ss_desc *desc, const void *u, const void *delta, const float *A,
                       const void *B, const void *C, const float *D, const void *z,
                       const float *delta_bias, int delta_softplus, const uint8_t *reset,
                       const void *dy, void *du, void *ddelta, float *dA, float *dB, float *dC,
                       float *dD, void *dz, float *ddelta_bias, void *workspace,
                       size_t workspace_bytes, ss_stream_t stream) {
    if (!reset && desc && desc->batch > 0 && desc->dim > 0 && desc->seqlen > 0) return SS_ERR_NULL_POINTER;
    return bwd_impl(desc, u, delta, A, B, C, D, z, delta_bias, delta_softplus, reset, nullptr, nullptr, dy,
                    du, ddelta, dA, dB, dC, dD, dz, ddelta_bias, nullptr, workspace, workspace_bytes, stream);
}

ss_status ss_bwd_ckpt(const ss_desc *desc, const void *u, const void *delta, const float *A, const void *B,
                      const void *C, const float *D, const void *z, const float *delta_bias, int delta_softplus,
                      const uint8_t *reset, const float *ckpt, const float *d_last_state, const void *dy, void *du,
                      void *ddelta, float *dA, float *dB, float *dC, float *dD, void *dz, float *ddelta_bias,
                      float *d_initial_state, void *workspace, size_t workspace_bytes, ss_stream_t stream) {
    if (!ckpt && desc && desc->batch > 0 && desc->dim > 0 && desc->seqlen > 0) return SS_ERR_NULL_POINTER;
    return bwd_impl(desc, u, delta, A, B, C, D, z, delta_bias, delta_softplus, reset, nullptr, d_last_state, dy, du,
                    ddelta, dA, dB, dC, dD, dz, ddelta_bias, d_initial_state, workspace, workspace_bytes, stream,
                    ckpt);
}

size_t ss_bwd_ckpt_workspace_bytes(const ss_desc *desc) {
    Sizes sz;
    if (check_desc(desc, &sz) != SS_OK) return 0;
    return bwd_layout(desc, sz, true).total;
}

ss_status ss_bwd_state(const ss_desc *desc, const void *u, const void *delta, const float *A,
                       const void *B, const void *C, const float *D, const void *z,
                       const float *delta_bias, int delta_softplus, const uint8_t *reset,
                       const float *initial_state, const float *d_last_state, const void *dy, void *du,
                       void *ddelta, float *dA, float *dB, float *dC, float *dD, void *dz,
                       float *ddelta_bias, float *d_initial_state, void *workspace,
                       size_t workspace_bytes, ss_stream_t stream) {
    return bwd_impl(desc, u, delta, A, B, C, D, z, delta_bias, delta_softplus, reset, initial_state,
                    d_last_state, dy, du, ddelta, dA, dB, dC, dD, dz, ddelta_bias, d_initial_state, workspace,
                    workspace_bytes, stream);
}

ss_status ss_step(const ss_desc *desc, const void *u, const void *delta, const float *A, const void *B,
                  const void *C, const float *D, const void *z, const float *delta_bias,
                  int delta_softplus, float *state, void *y, ss_stream_t stream) {
    Sizes sz;
    ss_status st = check_desc(desc, &sz);
    if (st != SS_OK) return st;
    if (desc->seqlen != 1) return SS_ERR_BAD_SHAPE;
    if (sz.rows == 0) return SS_OK;
    if (!u || !delta || !A || !B || !C || !state || !y) return SS_ERR_NULL_POINTER;
    const size_t ein = dtype_size(desc->in_dtype), eout = dtype_size(desc->out_dtype);
    const void *in_ptrs[] = {u, delta, B, C, z};
    for (const void *q : in_ptrs)
        if (q && !aligned(q, ein)) return SS_ERR_MISALIGNED;
    if (!aligned(y, eout) || !aligned(A, 4) || !aligned(state, 4) || (D && !aligned(D, 4)) ||
        (delta_bias && !aligned(delta_bias, 4)))
        return SS_ERR_MISALIGNED;
    const int T = selscan::state_bucket((int)desc->dstate) / 2;  // threads per row: one per state pair
    const int64_t blocks = (sz.rows * T + 255) / 256;
    if (blocks > INT_MAX) return SS_ERR_BAD_SHAPE;
    selscan::StepParams p;
    p.u = u, p.delta = delta, p.B = B, p.C = C, p.z = z;
    p.A = A, p.D = D, p.delta_bias = delta_bias;
    p.state = state, p.y = y;
    p.batch = desc->batch, p.dim = desc->dim;
    p.dstate = (int)desc->dstate;
    p.softplus = delta_softplus ? 1 : 0;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const dim3 grid((unsigned)blocks);
    cudaError_t err;
    if (desc->in_dtype == SS_F32)
        err = launch_step<float, float>(T, grid, s, p);
    else if (desc->out_dtype == SS_BF16)
        err = launch_step<__nv_bfloat16, __nv_bfloat16>(T, grid, s, p);
    else
        err = launch_step<__nv_bfloat16, float>(T, grid, s, p);
    return err == cudaSuccess ? SS_OK : SS_ERR_CUDA;
}

const char *ss_status_string(ss_status status) {
    switch (status) {
        case SS_OK: return "ok";
        case SS_ERR_NULL_POINTER: return "a required pointer is NULL";
        case SS_ERR_BAD_SHAPE: return "a size is negative or too large";
        case SS_ERR_UNSUPPORTED_DTYPE: return "unsupported dtype pair";
        case SS_ERR_UNSUPPORTED_DSTATE: return "dstate must be in 1..64";
        case SS_ERR_MISALIGNED: return "a pointer is not aligned to its element size";
        case SS_ERR_CUDA: return "CUDA runtime error";
        case SS_ERR_BAD_CONFIG: return "unsupported launch shape";
        case SS_ERR_WORKSPACE: return "workspace missing or too small";
        case SS_ERR_SCRATCH_LIMIT: return "needs more scratch than the no-alloc entry's static array";
    }
    return "unknown status";
}

int ss_version(void) { return SS_VERSION; }

ss_status ss_device_status(int *code) {
    if (!code) return SS_ERR_NULL_POINTER;
    *code = 0;
    if (!device_status_ptr()) return SS_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_ss_device_status, sizeof(int)) != cudaSuccess) return SS_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_ss_device_status, &zero, sizeof(int)) != cudaSuccess) return SS_ERR_CUDA;
    }
    *code = v;
    return SS_OK;
}

}  // extern "C"
