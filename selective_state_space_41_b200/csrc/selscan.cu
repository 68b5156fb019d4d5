// libselscan: C ABI of the selective-scan forward (declarations and the
// meaning of every argument are in include/selscan.h).
//
// Host side: validates the descriptor and pointers before touching CUDA,
// picks a launch shape, and dispatches to the kernel instance for the dtype
// pair, the state-size bucket (4/8/16/32/64) and the lanes-per-row count.

#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <cstdint>

#include "selscan.h"
#include "ss_launch.h"

namespace {

using selscan::FwdParams;

constexpr int kMaxState = 64;
constexpr int kMaxDevices = 64;

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
    if (lanes == 1 || split) return selscan::direct_smem_bytes(dtype_size(desc->in_dtype), nmax, lanes, warps);
    return selscan::smem_bytes(dtype_size(desc->in_dtype), nmax, lanes, warps);
}

// Launch shape.  The direct kernel (lanes split a row's states, no scan) has
// the least work per state update, so it is used whenever the rows alone
// can give each SM sub-partition (4 per SM) enough warps: the smallest split
// G in {1, 2, 4} (at most half the state bucket) with at least 4 warps per
// sub-partition (with 32 or 64 states, 32 states per lane once that gives 2
// warps), or G = 4 down to 1.5 warps.  With fewer rows the steps are
// split instead (scan kernel): the smallest W giving 3 warps per
// sub-partition, no more lanes than the sequence can feed, and a block
// within half of an SM's shared memory.
void heuristic(const ss_desc *desc, int64_t rows, int sms, int *lanes, int *split, int *warps) {
    const int64_t slots = (int64_t)sms * 4 * 32;  // lanes per "one warp per sub-partition"
    const int bucket = selscan::state_bucket((int)desc->dstate);
    const int gmax = bucket / 2 >= 4 ? 4 : 2;
    int g = 1;
    while (g < gmax && rows * g < 4 * slots) g *= 2;
    // Wide states: 32 states per lane (uncapped registers) once the rows alone
    // give two warps per sub-partition.
    if (bucket >= 32 && rows * (bucket / 32) >= 2 * slots) g = bucket / 32;
    if (rows * g >= 2 * slots || rows * gmax * 2 >= 3 * slots) {
        *lanes = g;
        *split = g > 1 ? 1 : 0;
        *warps = 4;
        return;
    }
    int w = 2;
    while (w < 32 && rows * w < 3 * slots) w *= 2;
    while (w > 2 && (int64_t)selscan::chunk_len(w) / 2 >= desc->seqlen) w /= 2;
    while (w > 2 && smem_for(desc, w, 0, 8) > selscan::kMaxSmemBytes / 2) w /= 2;
    *lanes = w;
    *split = 0;
    *warps = 8;
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

ss_status fwd_impl(const ss_desc *desc, const void *u, const void *delta, const float *A,
                   const void *B, const void *C, const float *D, const void *z,
                   const float *delta_bias, int delta_softplus, void *y, float *last_state,
                   int lanes, int split, int warps, ss_stream_t stream) {
    Sizes sz;
    ss_status st = check_desc(desc, &sz);
    if (st != SS_OK) return st;
    if (lanes != 0 && (lanes < 1 || lanes > 32 || (lanes & (lanes - 1)) != 0))
        return SS_ERR_BAD_CONFIG;
    if (split != 0 && split != 1) return SS_ERR_BAD_CONFIG;
    if (warps != 0 && warps != 1 && warps != 2 && warps != 4 && warps != 8)
        return SS_ERR_BAD_CONFIG;
    if (sz.rows == 0) return SS_OK;  // no rows: nothing to read or write
    const bool need_seq = desc->seqlen > 0;
    if (!A) return SS_ERR_NULL_POINTER;
    if (need_seq && (!u || !delta || !B || !C || !y)) return SS_ERR_NULL_POINTER;
    if (!need_seq && !last_state) return SS_OK;  // nothing to write

    const size_t ein = dtype_size(desc->in_dtype), eout = dtype_size(desc->out_dtype);
    const void *in_ptrs[] = {u, delta, B, C, z};
    for (const void *q : in_ptrs)
        if (q && !aligned(q, ein)) return SS_ERR_MISALIGNED;
    if ((y && !aligned(y, eout)) || !aligned(A, 4) || (D && !aligned(D, 4)) ||
        (delta_bias && !aligned(delta_bias, 4)) || (last_state && !aligned(last_state, 4)))
        return SS_ERR_MISALIGNED;

    // 16-byte vector path: every row of every streamed tensor starts aligned.
    bool vec = (desc->seqlen * (int64_t)ein) % 16 == 0 && (desc->seqlen * (int64_t)eout) % 16 == 0;
    for (const void *q : in_ptrs)
        if (q && !aligned(q, 16)) vec = false;
    if (y && !aligned(y, 16)) vec = false;

    int sms = sm_count();
    int h_lanes, h_split, h_warps;
    heuristic(desc, sz.rows, sms, &h_lanes, &h_split, &h_warps);
    if (lanes == 0) {
        lanes = h_lanes;
        split = h_split;
    }
    if (warps == 0) warps = h_warps;
    // The direct kernel splits the state pairs of the state bucket over 1, 2, 4 or 8 lanes.
    if ((lanes == 1 || split) &&
        (lanes > 8 || selscan::state_bucket((int)desc->dstate) / 2 < lanes))
        return SS_ERR_BAD_CONFIG;

    const size_t smem = smem_for(desc, lanes, split, warps);
    if (smem > selscan::kMaxSmemBytes) return SS_ERR_BAD_CONFIG;
    const int64_t rows_per_block = (int64_t)warps * (32 / lanes);
    const int64_t dtiles = (desc->dim + rows_per_block - 1) / rows_per_block;
    const int64_t blocks = dtiles * desc->batch;
    if (blocks > INT_MAX) return SS_ERR_BAD_SHAPE;

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
    p.batch = desc->batch;
    p.dim = desc->dim;
    p.seqlen = desc->seqlen;
    p.dstate = (int)desc->dstate;
    p.softplus = delta_softplus ? 1 : 0;
    p.vec = vec ? 1 : 0;
    p.dtiles = dtiles;

    const dim3 grid((unsigned)blocks), block((unsigned)(warps * 32));
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int n = p.dstate;
    cudaError_t err;
    if (desc->in_dtype == SS_F32)
        err = launch_f32_f32(n, lanes, split, grid, block, smem, s, p);
    else if (desc->out_dtype == SS_BF16)
        err = launch_bf16_bf16(n, lanes, split, grid, block, smem, s, p);
    else
        err = launch_bf16_f32(n, lanes, split, grid, block, smem, s, p);
    return err == cudaSuccess ? SS_OK : SS_ERR_CUDA;
}

}  // namespace

extern "C" {

ss_status ss_fwd(const ss_desc *desc, const void *u, const void *delta, const float *A,
                 const void *B, const void *C, const float *D, const void *z,
                 const float *delta_bias, int delta_softplus, void *y, float *last_state,
                 ss_stream_t stream) {
    return fwd_impl(desc, u, delta, A, B, C, D, z, delta_bias, delta_softplus, y, last_state, 0, 0, 0,
                    stream);
}

ss_status ss_fwd_with_config(const ss_desc *desc, const void *u, const void *delta,
                             const float *A, const void *B, const void *C, const float *D,
                             const void *z, const float *delta_bias, int delta_softplus,
                             void *y, float *last_state, int lanes_per_row, int split_states,
                             int warps_per_block, ss_stream_t stream) {
    return fwd_impl(desc, u, delta, A, B, C, D, z, delta_bias, delta_softplus, y, last_state,
                    lanes_per_row, split_states, warps_per_block, stream);
}

ss_status ss_fwd_heuristic(const ss_desc *desc, int *lanes_per_row, int *split_states,
                           int *warps_per_block) {
    Sizes sz;
    ss_status st = check_desc(desc, &sz);
    if (st != SS_OK) return st;
    if (!lanes_per_row || !split_states || !warps_per_block) return SS_ERR_NULL_POINTER;
    heuristic(desc, sz.rows, sm_count(), lanes_per_row, split_states, warps_per_block);
    return SS_OK;
}

ss_status ss_fwd_hostio(const ss_desc *desc, const void *h_u, const void *h_delta,
                        const float *h_A, const void *h_B, const void *h_C, const float *h_D,
                        const void *h_z, const float *h_delta_bias, int delta_softplus,
                        void *h_y, float *h_last_state, void *d_u, void *d_delta, float *d_A,
                        void *d_B, void *d_C, float *d_D, void *d_z, float *d_delta_bias,
                        void *d_y, float *d_last_state, ss_stream_t stream) {
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
    st = fwd_impl(desc, d_u, d_delta, d_A, d_B, d_C, d_D, d_z, d_delta_bias, delta_softplus, d_y,
                  d_last_state, 0, 0, 0, stream);
    if (st != SS_OK) return st;
    if (n_y && cudaMemcpyAsync(h_y, d_y, n_y, d2h, s) != cudaSuccess) return SS_ERR_CUDA;
    if (d_last_state && cudaMemcpyAsync(h_last_state, d_last_state, n_last, d2h, s) != cudaSuccess)
        return SS_ERR_CUDA;
    return SS_OK;
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
    }
    return "unknown status";
}

int ss_version(void) { return SS_VERSION; }

}  // extern "C"
