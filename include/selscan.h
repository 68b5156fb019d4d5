/*
 * libselscan -- the selective scan of Mamba on NVIDIA B200 (sm_100a), C ABI:
 * the forward (from a zero or a given state, optionally with sequence starts
 * inside the rows), one-step decoding, and the backward (gradients of every
 * input, with or without sequence starts).
 *
 * The operation is the selective scan of Mamba as the selective_scan_ref
 * walkthrough defines it ("Mamba代码实战：手把手教你用PyTorch复现选择性扫描核心逻辑
 * （附避坑指南）"), for every batch b, channel d, step l and state n:
 *
 *   delta'[b,d,l] = softplus(delta[b,d,l] + delta_bias[d])   (delta_softplus != 0)
 *                 = exp(delta[b,d,l] + delta_bias[d])        (delta_softplus == 0)
 *                                                             -- §2.2 delta的预处理
 *   h[b,d,n] <- exp(delta' * A[d,n]) * h[b,d,n] + delta' * B[b,n,l] * u[b,d,l],
 *                                           h starting at 0   -- §3.1, §3.2
 *   y[b,d,l] = sum_n C[b,n,l] * h[b,d,n] + D[d] * u[b,d,l]    -- §3.2, §3.3
 *   y[b,d,l] *= z[b,d,l] * sigmoid(z[b,d,l])  when z is given  -- §3.3
 *   last_state[b,d,n] = h[b,d,n] after step L-1               -- §6 完整实现与测试
 *
 * softplus is torch's default (linear above 20).  The sum over n pairs the
 * state with C[b,n,l], as the mamba-minimal page writes it ("Mamba-minimal
 * 项目解析", 关键技术点 §1).  The argument list mirrors the page's
 * selective_scan_ref(u, delta, A, B, C, D, delta_bias, delta_softplus,
 * return_last_state) plus the z gate, the output buffers and a stream.
 *
 * Layout (row-major, innermost index contiguous, no padding or strides):
 *   u, delta, z, y : (batch, dim, seqlen)      -- §2.1 初始化参数
 *   A              : (dim, dstate)   float32
 *   B, C           : (batch, dstate, seqlen)
 *   D, delta_bias  : (dim)           float32
 *   last_state     : (batch, dim, dstate) float32
 * u, delta, B, C and z share `in_dtype`; y has `out_dtype`.
 *
 * Ownership: every pointer is caller-owned; the library allocates nothing,
 * keeps no state between calls and may be called from several threads.  Some
 * launch shapes need a device workspace, which the caller provides
 * (ss_fwd_ws, ss_fwd_workspace_bytes), or which ss_fwd_noalloc takes from a
 * fixed static device array (the one piece of state: its cached address).
 *
 * Errors: arguments are validated on the host before anything is launched;
 * a rejected call returns a status other than SS_OK and touches no memory.
 * Execution is asynchronous on `stream`; a launch failure returns
 * SS_ERR_CUDA, and faults during execution surface at the caller's next
 * synchronisation with that stream.
 */
#ifndef SELSCAN_H
#define SELSCAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SS_VERSION 100 /* 1.0.0 */

typedef enum {
    SS_OK = 0,
    SS_ERR_NULL_POINTER = 1,       /* a required pointer is NULL */
    SS_ERR_BAD_SHAPE = 2,          /* a size is negative or too large */
    SS_ERR_UNSUPPORTED_DTYPE = 3,  /* dtype pair not in {f32->f32, bf16->bf16, bf16->f32} */
    SS_ERR_UNSUPPORTED_DSTATE = 4, /* dstate outside 1..64 */
    SS_ERR_MISALIGNED = 5,         /* a pointer is not aligned to its element size */
    SS_ERR_CUDA = 6,               /* the CUDA runtime reported an error */
    SS_ERR_BAD_CONFIG = 7,         /* ss_fwd_with_config: unsupported launch shape */
    SS_ERR_WORKSPACE = 8,          /* the launch shape needs a larger workspace */
    SS_ERR_SCRATCH_LIMIT = 9       /* ss_fwd_noalloc: needs more than SS_NOALLOC_SCRATCH_BYTES */
} ss_status;

typedef enum { SS_F32 = 0, SS_BF16 = 1 } ss_dtype;

/* A CUDA stream handle; the same object as cudaStream_t / CUstream.  NULL is
 * the legacy default stream. */
typedef struct CUstream_st *ss_stream_t;

typedef struct {
    int64_t batch;     /* B >= 0 */
    int64_t dim;       /* D >= 0 (channels) */
    int64_t seqlen;    /* L >= 0 (steps) */
    int64_t dstate;    /* N in 1..64 (states per channel) */
    ss_dtype in_dtype;  /* u, delta, B, C, z */
    ss_dtype out_dtype; /* y: in_dtype, or SS_F32 for bf16 inputs */
} ss_desc;

/*
 * Selective-scan forward on the device.
 *   u, delta      device, (B, D, L) in_dtype, required
 *   A             device, (D, N) float32, required (the caller applies
 *                 A = -exp(A_log) if that is its parameterisation)
 *   B, C          device, (B, N, L) in_dtype, required
 *   D             device, (D,) float32, or NULL for no skip term
 *   z             device, (B, D, L) in_dtype, or NULL for no gate
 *   delta_bias    device, (D,) float32, or NULL for no bias
 *   delta_softplus  non-zero: softplus; zero: exp
 *   y             device, (B, D, L) out_dtype, required (may not alias inputs)
 *   last_state    device, (B, D, N) float32, or NULL (= return_last_state off)
 *   stream        the stream the work is queued on
 * Every pointer must be aligned to its element size.  Sizes with B*D == 0 or
 * L == 0 are valid: with L == 0 the last state (if asked for) is all zeros
 * (the initial state, for ss_fwd_state).
 * Arithmetic: float32 throughout (state, products and sums), whatever the
 * input dtype; results are bitwise reproducible run to run for a given
 * device, shape and pointer alignment.
 */
ss_status ss_fwd(const ss_desc *desc, const void *u, const void *delta, const float *A,
                 const void *B, const void *C, const float *D, const void *z,
                 const float *delta_bias, int delta_softplus, void *y, float *last_state,
                 ss_stream_t stream);

/*
 * Launch shape.  lanes_per_row in {1,2,4,8,16,32} is how many lanes of a warp
 * share one (b, d) row:
 *   split_states = 0: the lanes split the row's steps (each takes 8 steps per
 *     chunk up to 4 lanes, 16 from 8 lanes) and combine their states with a
 *     scan over the lanes;
 *   split_states = 1: the lanes (1, 2, 4 or 8, at most half the state bucket
 *     4/8/16/32/64 that holds dstate) split the row's states and each runs
 *     every step;
 *   split_states = 2: as 1, with B and C reaching the lanes through tensor
 *     memory (a tcgen05 MMA with a 0/1 selection matrix broadcasts each
 *     lane's B/C values into its TMEM lane).  bf16 inputs; 2 lanes holding
 *     4 or 8 states each, or 4 or 8 lanes holding 2 or 4 states each; no
 *     sequence starts; warps_per_block 0 or 4;
 *   one lane: the row's sequential recurrence in one lane, either way.
 * warps_per_block in {1,2,4,8}.
 * segments (states split or one lane only): 1 runs each row's whole sequence
 *   in one pass; k > 1 cuts it into about k segments (a multiple of 64 steps
 *   long) that run in parallel from a zero state, then a second kernel adds
 *   the state carried into each segment to its outputs (exactly: it stops
 *   once every state's decay of the carried state has underflowed to 0).  A
 *   segmented launch needs ss_fwd_workspace_bytes() of device workspace.
 * Zeros take the heuristic's choice for that field.
 */
typedef struct {
    int lanes_per_row;
    int split_states;
    int warps_per_block;
    int segments;
} ss_launch_config;

/*
 * As ss_fwd, with a device workspace the library may use for a faster launch
 * shape (sequence segments for long sequences with few rows).  workspace:
 * caller-owned device memory, 16-byte aligned, of workspace_bytes bytes
 * (NULL/0: none, then this is ss_fwd); its contents are scratch, overwritten,
 * and must not be shared by calls that overlap on the GPU.
 */
ss_status ss_fwd_ws(const ss_desc *desc, const void *u, const void *delta, const float *A,
                    const void *B, const void *C, const float *D, const void *z,
                    const float *delta_bias, int delta_softplus, void *y, float *last_state,
                    void *workspace, size_t workspace_bytes, ss_stream_t stream);

/*
 * Bytes of workspace the launch shape `config` (NULL: the heuristic's shape
 * when a workspace is available) uses for `desc`; 0 if it uses none or the
 * descriptor or config is invalid.
 */
size_t ss_fwd_workspace_bytes(const ss_desc *desc, const ss_launch_config *config);

/*
 * As ss_fwd_ws, with the launch shape chosen by the caller (for autotuning
 * and tests).  Results agree for every shape up to float32 rounding order
 * (and, for segmented bf16 outputs, one extra rounding of y in the steps the
 * carried state still reaches).  Returns SS_ERR_BAD_CONFIG for unsupported
 * values or a block needing more than 227 KB of shared memory, and
 * SS_ERR_WORKSPACE when the shape needs more workspace than given.
 */
ss_status ss_fwd_with_config(const ss_desc *desc, const void *u, const void *delta,
                             const float *A, const void *B, const void *C, const float *D,
                             const void *z, const float *delta_bias, int delta_softplus,
                             void *y, float *last_state, const ss_launch_config *config,
                             void *workspace, size_t workspace_bytes, ss_stream_t stream);

/*
 * As ss_fwd_with_config (config NULL: the heuristic's shape, as ss_fwd_ws),
 * starting from a given state instead of zero.  The walkthrough's state
 * always starts at zero (§3.2); this extension lets a sequence run in pieces,
 * each piece starting from the last state of the one before, down to single
 * steps (L = 1) for recurrent decoding:
 *   initial_state  device, (B, D, N) float32: the state before step 0, or
 *                  NULL for zero.  It may be the same buffer as last_state
 *                  (the state is then updated in place); it may not overlap
 *                  any other argument.
 * Other arguments and errors as ss_fwd_with_config.
 */
ss_status ss_fwd_state(const ss_desc *desc, const void *u, const void *delta, const float *A,
                       const void *B, const void *C, const float *D, const void *z,
                       const float *delta_bias, int delta_softplus, const float *initial_state,
                       void *y, float *last_state, const ss_launch_config *config, void *workspace,
                       size_t workspace_bytes, ss_stream_t stream);

/*
 * As ss_fwd_state, for rows that hold several sequences one after another
 * (packed or concatenated sequences, or a long sequence whose state is reset
 * at chosen steps): the state is reset at each sequence start, so nothing of
 * one sequence leaks into the next (the boundary reset of "Mamba实战：如何用
 * 选择性状态空间模型提升你的长序列处理效率（附代码）" §2, and its periodic reset
 * of very long sequences in §5).
 *   reset   device, (B, L) bytes, required when B*D*L > 0 (SS_ERR_NULL_POINTER
 *           otherwise); reset[b*L + l] != 0 means a new sequence starts at
 *           step l of every row of batch entry b: the state entering step l
 *           is zero, so h_l = delta'_l B_l u_l there, whatever came before
 *           (a reset at l = 0 overrides initial_state).  Read only.
 * The rows run in the direct kernel (the states split over the lanes; with a
 * workspace, in sequence segments as ss_fwd_ws, a segment that holds a start
 * passing no state on): a config asking for the scan kernel
 * (split_states = 0 with lanes_per_row > 1) returns SS_ERR_BAD_CONFIG.
 * Other arguments and errors as ss_fwd_state.
 */
ss_status ss_fwd_reset(const ss_desc *desc, const void *u, const void *delta, const float *A,
                       const void *B, const void *C, const float *D, const void *z,
                       const float *delta_bias, int delta_softplus, const uint8_t *reset,
                       const float *initial_state, void *y, float *last_state,
                       const ss_launch_config *config, void *workspace, size_t workspace_bytes,
                       ss_stream_t stream);

/*
 * The launch shape ss_fwd_ws would use for `desc` with `workspace_bytes` of
 * workspace (0: as ss_fwd).  Returns SS_OK, or the status ss_fwd would return
 * for a bad descriptor.
 */
ss_status ss_fwd_heuristic(const ss_desc *desc, size_t workspace_bytes, ss_launch_config *config);

/*
 * Host-buffer form: copies the inputs from host memory into caller-owned
 * device staging buffers, runs ss_fwd_ws, and copies y (and last_state) back to
 * host memory, all queued on `stream` (one cudaMemcpyAsync per buffer).  The
 * host buffers should be page-locked for the copies to be asynchronous; the
 * caller synchronises `stream` before reading the results.
 *   h_*  host pointers with the shapes and dtypes of ss_fwd (h_D, h_z,
 *        h_delta_bias, h_last_state may be NULL exactly when the matching
 *        device buffer is NULL)
 *   d_*  device buffers of the same sizes, used as ss_fwd's arguments
 *   d_workspace, workspace_bytes  as for ss_fwd_ws (NULL/0: none)
 */
ss_status ss_fwd_hostio(const ss_desc *desc, const void *h_u, const void *h_delta,
                        const float *h_A, const void *h_B, const void *h_C, const float *h_D,
                        const void *h_z, const float *h_delta_bias, int delta_softplus,
                        void *h_y, float *h_last_state, void *d_u, void *d_delta, float *d_A,
                        void *d_B, void *d_C, float *d_D, void *d_z, float *d_delta_bias,
                        void *d_y, float *d_last_state, void *d_workspace, size_t workspace_bytes,
                        ss_stream_t stream);

/*
 * The forward with delta produced inside the scan by the dt_proj map of the
 * mamba-minimal block (Mamba-minimal项目解析, 核心组件解析 §5 ssm: x_dbl = x_proj(x)
 * splits into delta (dt_rank features), B and C, and delta =
 * softplus(dt_proj(delta))): delta[b, d, l] = sum_r W_dt[d, r] delta_r[b, r, l],
 * then the scan of ss_fwd_ws with delta_bias as dt_proj's bias.  The product
 * runs on the tensor cores (tcgen05, bf16 operands, fp32 accumulation in
 * tensor memory) one 64-step stage ahead of the scan, so delta never goes
 * through device memory.
 *   dt_rank   1..64 (the features of delta_r)
 *   delta_r   device, (B, dt_rank, L) bf16, l contiguous (the layout of B and C)
 *   W_dt      device, (D, dt_rank) bf16 (dt_proj's weight)
 * desc->in_dtype must be SS_BF16 (SS_ERR_UNSUPPORTED_DTYPE otherwise); the
 * launch is the direct kernel with 2 or 4 lanes per row (the heuristic's
 * when it is one of those); no sequence starts and no initial state.  Other
 * arguments, workspace and errors as ss_fwd_ws; SS_ERR_BAD_SHAPE for a
 * dt_rank outside 1..64.
 */
ss_status ss_fwd_dtproj(const ss_desc *desc, int dt_rank, const void *u, const void *delta_r,
                        const void *W_dt, const float *A, const void *B, const void *C, const float *D,
                        const void *z, const float *delta_bias, int delta_softplus, void *y,
                        float *last_state, void *workspace, size_t workspace_bytes, ss_stream_t stream);

/*
 * ss_fwd_dtproj reading the x_proj output as it is (Mamba-minimal项目解析,
 * 核心组件解析 §5 ssm: x_dbl = x_proj(x), split into delta (dt_rank
 * features), B and C): delta_r, B and C are the row ranges [0, R),
 * [R, R + N) and [R + N, R + 2N) of each batch entry of one tensor, so the
 * split makes no copies.
 *   x_dbl   device, (B, dt_rank + 2 N, L) bf16, l contiguous (the layout of B
 *           and C of ss_fwd, with dt_rank + 2 N feature rows per batch entry)
 * Every other argument, the launch, workspace and errors as ss_fwd_dtproj
 * (B and C come from x_dbl); results equal ss_fwd_dtproj's on the three
 * ranges copied out, bit for bit.
 */
ss_status ss_fwd_xdbl(const ss_desc *desc, int dt_rank, const void *u, const void *x_dbl, const void *W_dt,
                      const float *A, const float *D, const void *z, const float *delta_bias, int delta_softplus,
                      void *y, float *last_state, void *workspace, size_t workspace_bytes, ss_stream_t stream);

/*
 * Bytes of the device scratch array built into the library for
 * ss_fwd_noalloc (8 MiB per device; a 4 x 1024-channel, 16-state layer over
 * 100000 steps needs 4,456,448 bytes = 4.25 MiB in its default launch shape).
 */
#define SS_NOALLOC_SCRATCH_BYTES (8u << 20)

/*
 * As ss_fwd_ws given all the workspace its launch shape can use (same launch
 * shape, bitwise the same results), but with the workspace taken from a
 * static device array of SS_NOALLOC_SCRATCH_BYTES bytes inside the library,
 * so the caller passes none and nothing is allocated.  This entry has no
 * counterpart in the method's description; it exists for callers that may
 * not allocate device memory when they call (a fixed memory budget, a host
 * framework that owns all allocation, or a path where the device-wide
 * synchronisation of cudaMalloc / cudaFree is not acceptable).
 *   - Returns SS_ERR_SCRATCH_LIMIT, launching nothing, when that launch shape
 *     needs more than SS_NOALLOC_SCRATCH_BYTES (ss_fwd_workspace_bytes(desc,
 *     NULL) says how much it needs); other errors as ss_fwd_ws.
 *   - The first call on each device (the device current at the call) looks
 *     up the array's device address with cudaGetSymbolAddress and caches it;
 *     make that first call before any stream capture on that device.  The
 *     cached address belongs to that device context: after cudaDeviceReset
 *     on the device it is stale, so do not call ss_fwd_noalloc on that
 *     device again in the same process.
 *   - All calls on one device share the one array: calls whose work overlaps
 *     on the GPU (other streams, other host threads) race on it and give
 *     wrong results.  Calls queued in order on one stream are safe.
 *   - The array needs no initialisation: each call writes every scratch word
 *     it reads before reading it.
 */
ss_status ss_fwd_noalloc(const ss_desc *desc, const void *u, const void *delta, const float *A,
                         const void *B, const void *C, const float *D, const void *z,
                         const float *delta_bias, int delta_softplus, void *y, float *last_state,
                         ss_stream_t stream);

/*
 * One step of recurrent decoding with the state updated in place: the same
 * arithmetic as ss_fwd_state with L = 1 and initial_state == last_state, by a
 * kernel made for it (one thread per row and state pair; the work is one read
 * and one write of the state).  desc->seqlen must be 1 (SS_ERR_BAD_SHAPE
 * otherwise).
 *   u, delta, z    device, (B, D) in_dtype (z NULL: no gate)
 *   B, C           device, (B, N) in_dtype
 *   A, D, delta_bias  as ss_fwd
 *   state          device, (B, D, N) float32: the state before the step on
 *                  entry, after it on return
 *   y              device, (B, D) out_dtype
 */
ss_status ss_step(const ss_desc *desc, const void *u, const void *delta, const float *A, const void *B,
                  const void *C, const float *D, const void *z, const float *delta_bias,
                  int delta_softplus, float *state, void *y, ss_stream_t stream);

/*
 * Backward of ss_fwd (state starting at zero): the gradients of sum(dy * y)
 * with respect to every input.  The walkthrough trains the forward through
 * autograd (§6); this is its chain rule written out (an adjoint state run
 * backwards over the steps from checkpoints of the forward state).
 *   dy                 device, (B, D, L) out_dtype: the gradient of y
 *   du, ddelta, dz     device, (B, D, L) in_dtype; dz required exactly when z is given
 *   dA                 device, (D, N) float32
 *   dB, dC             device, (B, N, L) float32
 *   dD, ddelta_bias    device, (D,) float32, required exactly when D / delta_bias are given
 *   workspace          device, 256-byte aligned, ss_bwd_workspace_bytes(desc)
 *                      bytes (forward-state checkpoints every 8 steps and
 *                      partial sums); scratch, not shared by overlapping calls
 * Other arguments as ss_fwd (N in 1..64).  Sums over rows (dA, dB, dC, dD,
 * ddelta_bias) are taken in a fixed order: results are bitwise reproducible.
 */
ss_status ss_bwd(const ss_desc *desc, const void *u, const void *delta, const float *A, const void *B,
                 const void *C, const float *D, const void *z, const float *delta_bias,
                 int delta_softplus, const void *dy, void *du, void *ddelta, float *dA, float *dB,
                 float *dC, float *dD, void *dz, float *ddelta_bias, void *workspace,
                 size_t workspace_bytes, ss_stream_t stream);

/*
 * ss_bwd for a forward run with sequence starts (ss_fwd_reset): the same
 * gradients, with `reset` the forward's (B, L) byte mask (required when
 * B*D*L > 0, SS_ERR_NULL_POINTER otherwise).  At a start l the state h_(l-1)
 * has no part in h_l, so no adjoint passes from step l to l-1 and the
 * h_(l-1) terms of ddelta and dA vanish there.  Workspace as ss_bwd
 * (ss_bwd_workspace_bytes); other arguments and errors as ss_bwd.
 */
ss_status ss_bwd_reset(const ss_desc *desc, const void *u, const void *delta, const float *A,
                       const void *B, const void *C, const float *D, const void *z,
                       const float *delta_bias, int delta_softplus, const uint8_t *reset,
                       const void *dy, void *du, void *ddelta, float *dA, float *dB, float *dC,
                       float *dD, void *dz, float *ddelta_bias, void *workspace,
                       size_t workspace_bytes, ss_stream_t stream);

/*
 * The backward of the forward from a given state (ss_fwd_state, or
 * ss_fwd_reset with sequence starts), for training a long sequence piece by
 * piece: each piece runs from the last state of the piece before, and the
 * gradient flows back through those states.  The loss is sum(dy * y) plus,
 * when d_last_state is given, sum(d_last_state * h_(L-1)) (the last state
 * feeding the next piece).  The pages train the forward through autograd
 * (Mamba代码实战 §6) and give no initial-state interface; this is the chain rule
 * of the §3.2 loop started from h_(-1) = initial_state:
 *   reset           device (B, L) bytes, or NULL: as ss_bwd_reset
 *   initial_state   device (B, D, N) float32, or NULL (zero)
 *   d_last_state    device (B, D, N) float32, or NULL (zero): the gradient
 *                   with respect to the state after step L-1
 *   d_initial_state device (B, D, N) float32 output, or NULL (not written):
 *                   the gradient with respect to the state before step 0,
 *                   a_0 * lam_0 (zero where a sequence starts at step 0;
 *                   d_last_state when L = 0)
 * Other arguments, workspace (ss_bwd_workspace_bytes) and errors as ss_bwd.
 * A piece's d_initial_state passed as the previous piece's d_last_state
 * gives, piece by piece, the gradients of the whole sequence.
 */
ss_status ss_bwd_state(const ss_desc *desc, const void *u, const void *delta, const float *A,
                       const void *B, const void *C, const float *D, const void *z,
                       const float *delta_bias, int delta_softplus, const uint8_t *reset,
                       const float *initial_state, const float *d_last_state, const void *dy, void *du,
                       void *ddelta, float *dA, float *dB, float *dC, float *dD, void *dz,
                       float *ddelta_bias, float *d_initial_state, void *workspace,
                       size_t workspace_bytes, ss_stream_t stream);

/*
 * The forward that also writes the checkpoints its backward needs (for
 * training: the backward, ss_bwd_ckpt, then skips its own forward pass over
 * the sequence, about one exp per state update fewer).  Arguments as
 * ss_fwd_reset (initial_state and reset may be NULL), launch shape from the
 * heuristic given the workspace, plus:
 *   ckpt    device, (B, D, ceil(L/8), N) float32 output: the state entering
 *           every step l = 8k, i.e. after step l-1 (before a sequence start
 *           at l zeroes it; the initial state at k = 0).  With sequence
 *           segments the fix-up completes the checkpoints of segments >= 1.
 * The checkpoints come from the direct kernel: where the heuristic would pick
 * the scan kernel (few rows, no workspace) the direct kernel's widest state
 * split runs instead.  y and last_state are bitwise those of ss_fwd_reset in
 * the same launch shape.  SS_ERR_NULL_POINTER when ckpt is NULL and there is
 * work; other errors as ss_fwd_reset.
 */
ss_status ss_fwd_ckpt(const ss_desc *desc, const void *u, const void *delta, const float *A, const void *B,
                      const void *C, const float *D, const void *z, const float *delta_bias, int delta_softplus,
                      const float *initial_state, const uint8_t *reset, void *y, float *last_state, float *ckpt,
                      void *workspace, size_t workspace_bytes, ss_stream_t stream);

/*
 * ss_bwd_state from the forward's checkpoints (ss_fwd_ckpt of the same
 * inputs, initial state and starts) instead of its own checkpointing pass.
 *   ckpt          device, (B, D, ceil(L/8), N) float32, read only
 *   d_last_state, d_initial_state, reset: as ss_bwd_state (the initial state
 *                 itself is in the checkpoints)
 *   workspace     ss_bwd_ckpt_workspace_bytes(desc) bytes (no checkpoint
 *                 region; ss_bwd_workspace_bytes is enough too)
 * The gradients equal ss_bwd_state's bit for bit when neither the forward
 * nor the backward cuts the sequence into segments (the checkpoints are then
 * the values the backward's own pass computes); with segments they differ
 * only in the fp32 rounding of the segment carries.  SS_ERR_NULL_POINTER when
 * ckpt is NULL and there is work.
 */
ss_status ss_bwd_ckpt(const ss_desc *desc, const void *u, const void *delta, const float *A, const void *B,
                      const void *C, const float *D, const void *z, const float *delta_bias, int delta_softplus,
                      const uint8_t *reset, const float *ckpt, const float *d_last_state, const void *dy, void *du,
                      void *ddelta, float *dA, float *dB, float *dC, float *dD, void *dz, float *ddelta_bias,
                      float *d_initial_state, void *workspace, size_t workspace_bytes, ss_stream_t stream);

/* Bytes of workspace ss_bwd_ckpt needs for `desc` (0 for an invalid descriptor). */
size_t ss_bwd_ckpt_workspace_bytes(const ss_desc *desc);

/* Bytes of workspace ss_bwd, ss_bwd_reset and ss_bwd_state need for `desc` (0 for an invalid descriptor). */
size_t ss_bwd_workspace_bytes(const ss_desc *desc);

/*
 * The launch plan of the backward for `desc` (host only, no CUDA call but
 * the device's SM count):
 *   batch_group  host out: batch entries per launch.  The batch runs in
 *                groups whose forward-state checkpoints and dB/dC block
 *                partials fit 7 GiB, so the workspace stays bounded for
 *                large layers; results do not depend on the grouping.
 *   segments     host out: sequence segments per row (1: none).  When one
 *                group's blocks cannot give each SM three, a long sequence
 *                (at least 4096 steps) is cut into segments of at least 2048
 *                steps, each run as extra rows from the true state entering
 *                it and the true adjoint leaving it, which two summary passes
 *                (a forward over each segment from a zero state, an adjoint
 *                pass over each segment from a zero end) and their folds
 *                across the segments provide.
 * Errors as ss_bwd's descriptor checks; SS_ERR_NULL_POINTER for a NULL out.
 */
ss_status ss_bwd_heuristic(const ss_desc *desc, int64_t *batch_group, int *segments);

/*
 * As ss_fwd_hostio, pipelined over `nstreams` caller-owned streams (1..16):
 * the batch is cut into `chunks` ranges of batch entries (0: min(batch,
 * 2 * nstreams)); range c has its inputs copied in, its forward run and its
 * outputs copied out on stream c mod nstreams, so the copies of one range
 * overlap the copies in the other direction and the kernels of others.  A,
 * D and delta_bias are copied once on streams[0], which the other streams
 * wait for; the call first orders itself after all work already queued on
 * any of the streams.  The workspace is split evenly over the streams (each
 * range runs the launch shape its share allows).  The caller synchronises
 * every stream before reading the results.  Returns SS_ERR_BAD_CONFIG for
 * a bad stream count or chunk count; other errors as ss_fwd_hostio.
 */
ss_status ss_fwd_hostio_streams(const ss_desc *desc, const void *h_u, const void *h_delta,
                                const float *h_A, const void *h_B, const void *h_C, const float *h_D,
                                const void *h_z, const float *h_delta_bias, int delta_softplus,
                                void *h_y, float *h_last_state, void *d_u, void *d_delta, float *d_A,
                                void *d_B, void *d_C, float *d_D, void *d_z, float *d_delta_bias,
                                void *d_y, float *d_last_state, void *d_workspace,
                                size_t workspace_bytes, const ss_stream_t *streams, int nstreams,
                                int chunks);

/* Static description of a status code (never NULL). */
const char *ss_status_string(ss_status status);

/* SS_VERSION of the built library. */
int ss_version(void);

/*
 * The current device's status word, then cleared (no counterpart on the
 * pages).  A kernel that waits on other warps of its block (the
 * tensor-memory-fed forward, split_states = 2) bounds every wait to about a
 * second; if one runs out it records SS_DEVICE_TIMEOUT here, stops, frees
 * its tensor memory and returns, so the context stays usable.  *code = 0
 * when nothing was recorded.  Synchronous (copies from the device);
 * SS_ERR_CUDA when the word cannot be read.
 */
#define SS_DEVICE_TIMEOUT 1
ss_status ss_device_status(int *code);

#ifdef __cplusplus
}
#endif

#endif /* SELSCAN_H */
