"""Python binding of libselscan (argument marshalling only).

Every function here maps torch tensors to the pointers, sizes and stream of
the C entry points of ``include/selscan.h`` and calls them; the computation
runs in the library's CUDA kernels.  PyTorch supplies device memory and the
current stream.  There is no fallback: if ``libselscan.so`` is missing or
fails to load, every call raises.

The Python names match the C entry points (``ss_fwd``, ``ss_fwd_ws``,
``ss_fwd_workspace_bytes``, ``ss_fwd_with_config``, ``ss_fwd_state``,
``ss_fwd_reset``, ``ss_fwd_heuristic``, ``ss_fwd_hostio``, ``ss_fwd_hostio_streams``,
``ss_fwd_noalloc``, ``ss_fwd_dtproj``, ``ss_step``, ``ss_bwd``, ``ss_bwd_reset``, ``ss_bwd_state``, ``ss_bwd_workspace_bytes``,
``ss_bwd_heuristic``, ``ss_fwd_ckpt``, ``ss_bwd_ckpt``, ``ss_bwd_ckpt_workspace_bytes``,
``ss_status_string``, ``ss_version``, ``ss_device_status``); ``ss_fwd`` dispatches to the
workspace, config, initial-state and sequence-start forms by keyword, ``ss_fwd_hostio`` to
the pipelined form when given streams.  ``selective_scan_fwd`` and
``selective_scan_bwd`` are the allocate-and-call convenience forms, with the
argument order of the walkthrough's selective_scan_ref
("Mamba代码实战：手把手教你用PyTorch复现选择性扫描核心逻辑（附避坑指南）", §6).
"""
import ctypes
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libselscan.so")

SS_F32, SS_BF16 = 0, 1
_DTYPE_CODE = {torch.float32: SS_F32, torch.bfloat16: SS_BF16}
STATUS_NAMES = {0: "SS_OK", 1: "SS_ERR_NULL_POINTER", 2: "SS_ERR_BAD_SHAPE",
                3: "SS_ERR_UNSUPPORTED_DTYPE", 4: "SS_ERR_UNSUPPORTED_DSTATE",
                5: "SS_ERR_MISALIGNED", 6: "SS_ERR_CUDA", 7: "SS_ERR_BAD_CONFIG",
                8: "SS_ERR_WORKSPACE", 9: "SS_ERR_SCRATCH_LIMIT"}

# SS_NOALLOC_SCRATCH_BYTES: the static scratch array behind ss_fwd_noalloc.
NOALLOC_SCRATCH_BYTES = 8 << 20

# Names the header declares; the ABI test checks each is exported.
EXPORTS = ("ss_fwd", "ss_fwd_ws", "ss_fwd_workspace_bytes", "ss_fwd_with_config", "ss_fwd_state",
           "ss_fwd_reset", "ss_fwd_heuristic", "ss_fwd_hostio", "ss_fwd_hostio_streams", "ss_fwd_noalloc",
           "ss_step", "ss_bwd", "ss_bwd_reset", "ss_bwd_state", "ss_bwd_workspace_bytes", "ss_status_string",
           "ss_version", "ss_device_status", "ss_fwd_dtproj", "ss_bwd_heuristic", "ss_fwd_ckpt", "ss_bwd_ckpt",
           "ss_bwd_ckpt_workspace_bytes", "ss_fwd_xdbl")


class SelscanError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({ss_status_string(status)})")


class Desc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("dim", ctypes.c_int64), ("seqlen", ctypes.c_int64),
                ("dstate", ctypes.c_int64), ("in_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int)]


class LaunchConfig(ctypes.Structure):
    """ss_launch_config: zeros take the heuristic's choice."""
    _fields_ = [("lanes_per_row", ctypes.c_int), ("split_states", ctypes.c_int),
                ("warps_per_block", ctypes.c_int), ("segments", ctypes.c_int)]


_lib = None


def lib():
    """The loaded ``libselscan.so`` (raises if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libselscan.so not built ({LIB_PATH}); run "
                               "`python -m selective_state_space_41_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I = ctypes.c_void_p, ctypes.c_int
        DP = ctypes.POINTER(Desc)
        L.ss_fwd.restype = I
        L.ss_fwd.argtypes = [DP, P, P, P, P, P, P, P, P, I, P, P, P]
        SZ = ctypes.c_size_t
        CP = ctypes.POINTER(LaunchConfig)
        L.ss_fwd_ws.restype = I
        L.ss_fwd_ws.argtypes = [DP, P, P, P, P, P, P, P, P, I, P, P, P, SZ, P]
        L.ss_fwd_workspace_bytes.restype = SZ
        L.ss_fwd_workspace_bytes.argtypes = [DP, CP]
        L.ss_fwd_with_config.restype = I
        L.ss_fwd_with_config.argtypes = [DP, P, P, P, P, P, P, P, P, I, P, P, CP, P, SZ, P]
        L.ss_fwd_state.restype = I
        L.ss_fwd_state.argtypes = [DP, P, P, P, P, P, P, P, P, I, P, P, P, CP, P, SZ, P]
        L.ss_fwd_reset.restype = I
        L.ss_fwd_reset.argtypes = [DP, P, P, P, P, P, P, P, P, I, P, P, P, P, CP, P, SZ, P]
        L.ss_fwd_heuristic.restype = I
        L.ss_fwd_heuristic.argtypes = [DP, SZ, CP]
        L.ss_fwd_hostio.restype = I
        L.ss_fwd_hostio.argtypes = [DP] + [P] * 8 + [I] + [P] * 12 + [P, SZ, P]
        L.ss_fwd_dtproj.restype = I
        L.ss_fwd_dtproj.argtypes = [DP, I] + [P] * 9 + [I, P, P, P, SZ, P]
        L.ss_fwd_xdbl.restype = I
        L.ss_fwd_xdbl.argtypes = [DP, I] + [P] * 7 + [I, P, P, P, SZ, P]
        L.ss_fwd_noalloc.restype = I
        L.ss_fwd_noalloc.argtypes = [DP, P, P, P, P, P, P, P, P, I, P, P, P]
        L.ss_fwd_hostio_streams.restype = I
        L.ss_fwd_hostio_streams.argtypes = [DP] + [P] * 8 + [I] + [P] * 12 + [P, SZ, P, I, I]
        L.ss_step.restype = I
        L.ss_step.argtypes = [DP] + [P] * 8 + [I, P, P, P]
        L.ss_bwd.restype = I
        L.ss_bwd.argtypes = [DP] + [P] * 8 + [I] + [P] * 9 + [P, SZ, P]
        L.ss_bwd_reset.restype = I
        L.ss_bwd_reset.argtypes = [DP] + [P] * 8 + [I] + [P] * 10 + [P, SZ, P]
        L.ss_bwd_state.restype = I
        L.ss_bwd_state.argtypes = [DP] + [P] * 8 + [I] + [P] * 13 + [P, SZ, P]
        L.ss_bwd_workspace_bytes.restype = SZ
        L.ss_bwd_workspace_bytes.argtypes = [DP]
        L.ss_fwd_ckpt.restype = I
        L.ss_fwd_ckpt.argtypes = [DP] + [P] * 8 + [I] + [P] * 5 + [P, SZ, P]
        L.ss_bwd_ckpt.restype = I
        L.ss_bwd_ckpt.argtypes = [DP] + [P] * 8 + [I] + [P] * 13 + [P, SZ, P]
        L.ss_bwd_ckpt_workspace_bytes.restype = SZ
        L.ss_bwd_ckpt_workspace_bytes.argtypes = [DP]
        L.ss_bwd_heuristic.restype = I
        L.ss_bwd_heuristic.argtypes = [DP, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(I)]
        L.ss_status_string.restype = ctypes.c_char_p
        L.ss_status_string.argtypes = [I]
        L.ss_version.restype = I
        L.ss_version.argtypes = []
        L.ss_device_status.restype = I
        L.ss_device_status.argtypes = [ctypes.POINTER(I)]
        _lib = L
    return _lib


def ss_status_string(status: int) -> str:
    return lib().ss_status_string(int(status)).decode()


def ss_version() -> int:
    return int(lib().ss_version())


# SS_DEVICE_TIMEOUT: a kernel's bounded wait on other warps of its block ran out.
SS_DEVICE_TIMEOUT = 1


def ss_device_status() -> int:
    """The current device's status word (0: nothing recorded), then cleared."""
    code = ctypes.c_int(0)
    _check(lib().ss_device_status(ctypes.byref(code)), "ss_device_status")
    return int(code.value)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def make_desc(batch, dim, seqlen, dstate, in_dtype, out_dtype=None) -> Desc:
    """A descriptor from sizes and torch dtypes (or SS_F32 / SS_BF16 codes)."""
    code = lambda t: _DTYPE_CODE[t] if isinstance(t, torch.dtype) else int(t)  # noqa: E731
    return Desc(int(batch), int(dim), int(seqlen), int(dstate), code(in_dtype),
                code(out_dtype if out_dtype is not None else in_dtype))


def _contig(t):
    """The C ABI takes dense row-major tensors; make them so (as the
    walkthrough's §4.1 does before its kernel call)."""
    return None if t is None else (t if t.is_contiguous() else t.contiguous())


def _check(status, where):
    if status != 0:
        raise SelscanError(status, where)


def _config(lanes_per_row, split_states, warps_per_block, segments):
    """split_states: False/0 (lanes split steps), True/1 (lanes split states),
    2 (lanes split states, B/C through tensor memory)."""
    if lanes_per_row is None and warps_per_block is None and segments is None:
        return None
    return LaunchConfig(int(lanes_per_row or 0), int(split_states or 0), int(warps_per_block or 0),
                        int(segments or 0))


def ss_fwd(u, delta, A, B, C, y, D=None, z=None, delta_bias=None, delta_softplus=False,
           last_state=None, stream=None, workspace=None, lanes_per_row=None, warps_per_block=None,
           split_states=False, segments=None, initial_state=None, reset=None):
    """Queue the forward on ``stream`` (default: the current stream).

    u, delta, z, y: (batch, dim, L); A: (dim, N) float32; B, C: (batch, N, L);
    D, delta_bias: (dim,) float32; last_state, initial_state: (batch, dim, N)
    float32.  ``workspace`` (a CUDA tensor, e.g. uint8 of
    ss_fwd_workspace_bytes()) selects ``ss_fwd_ws``; ``lanes_per_row`` /
    ``split_states`` / ``warps_per_block`` / ``segments`` select
    ``ss_fwd_with_config``; ``initial_state`` selects ``ss_fwd_state``;
    ``reset`` ((batch, L) uint8 or bool, nonzero where a new sequence starts)
    selects ``ss_fwd_reset``.  Raises SelscanError on a rejected call.
    """
    u, delta, A, B, C, D, z, delta_bias = map(_contig, (u, delta, A, B, C, D, z, delta_bias))
    if not (y.is_contiguous() and (last_state is None or last_state.is_contiguous())):
        raise ValueError("outputs must be contiguous")
    batch, dim, L = u.shape
    N = A.shape[-1]
    desc = make_desc(batch, dim, L, N, u.dtype, y.dtype)
    args = (ctypes.byref(desc), _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
            _ptr(delta_bias), 1 if delta_softplus else 0, _ptr(y), _ptr(last_state))
    ws = _ptr(workspace)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    s = _stream_handle(stream, u.device)
    cfg = _config(lanes_per_row, split_states, warps_per_block, segments)
    if initial_state is not None and not initial_state.is_contiguous():
        raise ValueError("initial_state must be contiguous")
    if reset is not None:
        if reset.dtype == torch.bool:
            reset = reset.view(torch.uint8)
        if reset.dtype != torch.uint8 or tuple(reset.shape) != (batch, L) or not reset.is_contiguous():
            raise ValueError("reset must be a contiguous (batch, L) uint8 or bool tensor")
        reset_args = args[:10] + (_ptr(reset), _ptr(initial_state)) + args[10:]
        _check(lib().ss_fwd_reset(*reset_args, ctypes.byref(cfg) if cfg is not None else None, ws,
                                  ws_bytes, s), "ss_fwd_reset")
    elif initial_state is not None:
        if not initial_state.is_contiguous():
            raise ValueError("initial_state must be contiguous")
        state_args = args[:10] + (_ptr(initial_state),) + args[10:]
        _check(lib().ss_fwd_state(*state_args, ctypes.byref(cfg) if cfg is not None else None, ws,
                                  ws_bytes, s), "ss_fwd_state")
    elif cfg is not None:
        _check(lib().ss_fwd_with_config(*args, ctypes.byref(cfg), ws, ws_bytes, s),
               "ss_fwd_with_config")
    elif workspace is not None:
        _check(lib().ss_fwd_ws(*args, ws, ws_bytes, s), "ss_fwd_ws")
    else:
        _check(lib().ss_fwd(*args, s), "ss_fwd")


def ss_fwd_dtproj(u, delta_r, W_dt, A, B, C, y, D=None, z=None, delta_bias=None, delta_softplus=True,
                  last_state=None, stream=None, workspace=None):
    """Queue the forward with delta = W_dt delta_r computed inside the scan
    (the dt_proj map).  delta_r: (batch, dt_rank, L) bf16; W_dt: (dim, dt_rank)
    bf16; other tensors as ``ss_fwd``."""
    u, delta_r, W_dt, A, B, C, D, z, delta_bias = map(_contig, (u, delta_r, W_dt, A, B, C, D, z, delta_bias))
    if not (y.is_contiguous() and (last_state is None or last_state.is_contiguous())):
        raise ValueError("outputs must be contiguous")
    batch, dim, L = u.shape
    R = W_dt.shape[-1]
    if tuple(delta_r.shape) != (batch, R, L) or tuple(W_dt.shape) != (dim, R):
        raise ValueError("delta_r must be (batch, dt_rank, L) and W_dt (dim, dt_rank)")
    desc = make_desc(batch, dim, L, A.shape[-1], u.dtype, y.dtype)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().ss_fwd_dtproj(ctypes.byref(desc), int(R), _ptr(u), _ptr(delta_r), _ptr(W_dt), _ptr(A), _ptr(B),
                               _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias), 1 if delta_softplus else 0, _ptr(y),
                               _ptr(last_state), _ptr(workspace), ws_bytes, _stream_handle(stream, u.device)),
           "ss_fwd_dtproj")


def ss_fwd_xdbl(u, x_dbl, W_dt, A, y, D=None, z=None, delta_bias=None, delta_softplus=True, last_state=None,
                stream=None, workspace=None):
    """Queue ss_fwd_dtproj with delta_r, B and C read from the x_proj output
    ``x_dbl`` ((batch, dt_rank + 2 N, L) bf16: feature rows [0, R) delta_r,
    [R, R + N) B, [R + N, R + 2N) C; no copies); W_dt: (dim, dt_rank) bf16,
    N = A.shape[1]; other tensors as ``ss_fwd``."""
    u, x_dbl, W_dt, A, D, z, delta_bias = map(_contig, (u, x_dbl, W_dt, A, D, z, delta_bias))
    if not (y.is_contiguous() and (last_state is None or last_state.is_contiguous())):
        raise ValueError("outputs must be contiguous")
    batch, dim, L = u.shape
    N, R = A.shape[-1], W_dt.shape[-1]
    if tuple(x_dbl.shape) != (batch, R + 2 * N, L) or tuple(W_dt.shape) != (dim, R):
        raise ValueError("x_dbl must be (batch, dt_rank + 2 N, L) and W_dt (dim, dt_rank)")
    desc = make_desc(batch, dim, L, N, u.dtype, y.dtype)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().ss_fwd_xdbl(ctypes.byref(desc), int(R), _ptr(u), _ptr(x_dbl), _ptr(W_dt), _ptr(A), _ptr(D),
                             _ptr(z), _ptr(delta_bias), 1 if delta_softplus else 0, _ptr(y), _ptr(last_state),
                             _ptr(workspace), ws_bytes, _stream_handle(stream, u.device)),
           "ss_fwd_xdbl")


def ss_fwd_noalloc(u, delta, A, B, C, y, D=None, z=None, delta_bias=None, delta_softplus=False,
                   last_state=None, stream=None):
    """Queue the forward with the library's static scratch array as the
    workspace (no device memory is allocated).  Same tensors as ``ss_fwd``;
    raises SelscanError (SS_ERR_SCRATCH_LIMIT) when the launch shape needs
    more than NOALLOC_SCRATCH_BYTES.  Calls that overlap on the GPU share the
    array and race."""
    u, delta, A, B, C, D, z, delta_bias = map(_contig, (u, delta, A, B, C, D, z, delta_bias))
    if not (y.is_contiguous() and (last_state is None or last_state.is_contiguous())):
        raise ValueError("outputs must be contiguous")
    batch, dim, L = u.shape
    desc = make_desc(batch, dim, L, A.shape[-1], u.dtype, y.dtype)
    _check(lib().ss_fwd_noalloc(ctypes.byref(desc), _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C),
                                _ptr(D), _ptr(z), _ptr(delta_bias), 1 if delta_softplus else 0,
                                _ptr(y), _ptr(last_state), _stream_handle(stream, u.device)),
           "ss_fwd_noalloc")


def ss_step(u, delta, A, B, C, state, y, D=None, z=None, delta_bias=None, delta_softplus=False,
            stream=None):
    """One decoding step, the state updated in place.  u, delta, z, y: (batch,
    dim); B, C: (batch, N); state: (batch, dim, N) float32."""
    u, delta, A, B, C, D, z, delta_bias = map(_contig, (u, delta, A, B, C, D, z, delta_bias))
    if not (state.is_contiguous() and y.is_contiguous()):
        raise ValueError("state and y must be contiguous")
    batch, dim = u.shape[0], u.shape[1]
    desc = make_desc(batch, dim, 1, A.shape[-1], u.dtype, y.dtype)
    _check(lib().ss_step(ctypes.byref(desc), _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                         _ptr(z), _ptr(delta_bias), 1 if delta_softplus else 0, _ptr(state), _ptr(y),
                         _stream_handle(stream, u.device)), "ss_step")


def ss_bwd_workspace_bytes(batch, dim, seqlen, dstate, in_dtype=torch.bfloat16, out_dtype=None) -> int:
    desc = make_desc(batch, dim, seqlen, dstate, in_dtype, out_dtype)
    return int(lib().ss_bwd_workspace_bytes(ctypes.byref(desc)))


def ss_bwd_heuristic(batch, dim, seqlen, dstate, in_dtype=torch.bfloat16, out_dtype=None) -> dict:
    """The backward's launch plan: batch entries per launch and sequence segments."""
    desc = make_desc(batch, dim, seqlen, dstate, in_dtype, out_dtype)
    group, segs = ctypes.c_int64(0), ctypes.c_int(0)
    _check(lib().ss_bwd_heuristic(ctypes.byref(desc), ctypes.byref(group), ctypes.byref(segs)), "ss_bwd_heuristic")
    return {"batch_group": int(group.value), "segments": int(segs.value)}


def ss_bwd(u, delta, A, B, C, dy, grads, D=None, z=None, delta_bias=None, delta_softplus=False,
           workspace=None, stream=None, reset=None, initial_state=None, d_last_state=None):
    """Queue the backward: ``grads`` maps du, ddelta, dA, dB, dC and (when the
    operand is given) dD, dz, ddelta_bias to output tensors (du, ddelta, dz in
    u's dtype; the others float32), and optionally dinitial_state ((batch,
    dim, N) float32).  ``workspace``: a CUDA tensor of at least
    ss_bwd_workspace_bytes() bytes (allocated here when None).  ``reset``: the
    forward's (batch, L) mask of sequence starts (selects ``ss_bwd_reset``).
    ``initial_state`` / ``d_last_state`` ((batch, dim, N) float32) or a
    dinitial_state output select ``ss_bwd_state``."""
    u, delta, A, B, C, dy, D, z, delta_bias = map(_contig, (u, delta, A, B, C, dy, D, z, delta_bias))
    batch, dim, L = u.shape
    N = A.shape[-1]
    desc = make_desc(batch, dim, L, N, u.dtype, dy.dtype)
    if workspace is None:
        n = ss_bwd_workspace_bytes(batch, dim, L, N, u.dtype, dy.dtype)
        workspace = torch.empty(max(n, 1), dtype=torch.uint8, device=u.device)
    g = lambda k: _ptr(grads.get(k))  # noqa: E731
    head = (ctypes.byref(desc), _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
            _ptr(delta_bias), 1 if delta_softplus else 0)
    tail = (_ptr(dy), g("du"), g("ddelta"), g("dA"), g("dB"), g("dC"), g("dD"), g("dz"), g("ddelta_bias"),
            _ptr(workspace), workspace.numel() * workspace.element_size(), _stream_handle(stream, u.device))
    if reset is not None:
        if reset.dtype == torch.bool:
            reset = reset.view(torch.uint8)
        if reset.dtype != torch.uint8 or tuple(reset.shape) != (batch, L) or not reset.is_contiguous():
            raise ValueError("reset must be a contiguous (batch, L) uint8 or bool tensor")
    for t in (initial_state, d_last_state, grads.get("dinitial_state")):
        if t is not None and not (t.is_contiguous() and tuple(t.shape) == (batch, dim, N) and t.dtype == torch.float32):
            raise ValueError("states must be contiguous (batch, dim, N) float32 tensors")
    if initial_state is not None or d_last_state is not None or grads.get("dinitial_state") is not None:
        _check(lib().ss_bwd_state(*head, _ptr(reset), _ptr(initial_state), _ptr(d_last_state), *tail[:9],
                                  g("dinitial_state"), *tail[9:]), "ss_bwd_state")
    elif reset is not None:
        _check(lib().ss_bwd_reset(*head, _ptr(reset), *tail), "ss_bwd_reset")
    else:
        _check(lib().ss_bwd(*head, *tail), "ss_bwd")


def ckpt_shape(batch, dim, seqlen, dstate):
    """Shape of the forward's checkpoints: (batch, dim, ceil(seqlen / 8), dstate)."""
    return (batch, dim, (seqlen + 7) // 8, dstate)


def ss_fwd_ckpt(u, delta, A, B, C, y, ckpt, D=None, z=None, delta_bias=None, delta_softplus=False,
                last_state=None, initial_state=None, reset=None, stream=None, workspace=None):
    """Queue the forward that also writes the backward's checkpoints into
    ``ckpt`` (float32, ckpt_shape(...)); other arguments as ``ss_fwd``
    (``workspace``: a CUDA tensor enabling sequence segments, or None)."""
    u, delta, A, B, C, D, z, delta_bias = map(_contig, (u, delta, A, B, C, D, z, delta_bias))
    batch, dim, L = u.shape
    N = A.shape[-1]
    if tuple(ckpt.shape) != ckpt_shape(batch, dim, L, N) or ckpt.dtype != torch.float32 or not ckpt.is_contiguous():
        raise ValueError("ckpt must be a contiguous float32 tensor of ckpt_shape(batch, dim, L, N)")
    if reset is not None and reset.dtype == torch.bool:
        reset = reset.view(torch.uint8)
    desc = make_desc(batch, dim, L, N, u.dtype, y.dtype)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().ss_fwd_ckpt(ctypes.byref(desc), _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                             _ptr(delta_bias), 1 if delta_softplus else 0, _ptr(initial_state), _ptr(reset), _ptr(y),
                             _ptr(last_state), _ptr(ckpt), _ptr(workspace), ws_bytes,
                             _stream_handle(stream, u.device)), "ss_fwd_ckpt")


def ss_bwd_ckpt_workspace_bytes(batch, dim, seqlen, dstate, in_dtype=torch.bfloat16, out_dtype=None) -> int:
    desc = make_desc(batch, dim, seqlen, dstate, in_dtype, out_dtype)
    return int(lib().ss_bwd_ckpt_workspace_bytes(ctypes.byref(desc)))


def ss_bwd_ckpt(u, delta, A, B, C, dy, ckpt, grads, D=None, z=None, delta_bias=None, delta_softplus=False,
                reset=None, d_last_state=None, workspace=None, stream=None):
    """Queue the backward from the forward's checkpoints (``ss_fwd_ckpt``):
    ``grads`` as ``ss_bwd`` (with an optional dinitial_state output)."""
    u, delta, A, B, C, dy, D, z, delta_bias = map(_contig, (u, delta, A, B, C, dy, D, z, delta_bias))
    batch, dim, L = u.shape
    N = A.shape[-1]
    if tuple(ckpt.shape) != ckpt_shape(batch, dim, L, N) or ckpt.dtype != torch.float32 or not ckpt.is_contiguous():
        raise ValueError("ckpt must be a contiguous float32 tensor of ckpt_shape(batch, dim, L, N)")
    if reset is not None and reset.dtype == torch.bool:
        reset = reset.view(torch.uint8)
    desc = make_desc(batch, dim, L, N, u.dtype, dy.dtype)
    if workspace is None:
        n = ss_bwd_ckpt_workspace_bytes(batch, dim, L, N, u.dtype, dy.dtype)
        workspace = torch.empty(max(n, 1), dtype=torch.uint8, device=u.device)
    g = lambda k: _ptr(grads.get(k))  # noqa: E731
    _check(lib().ss_bwd_ckpt(ctypes.byref(desc), _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                             _ptr(delta_bias), 1 if delta_softplus else 0, _ptr(reset), _ptr(ckpt),
                             _ptr(d_last_state), _ptr(dy), g("du"), g("ddelta"), g("dA"), g("dB"), g("dC"), g("dD"),
                             g("dz"), g("ddelta_bias"), g("dinitial_state"), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream_handle(stream, u.device)),
           "ss_bwd_ckpt")


def _grad_outputs(u, A, D, z, delta_bias, with_initial_state):
    """Output tensors of the backward: du, ddelta, dz in u's dtype; dA, dB,
    dC, dD, ddelta_bias (and dinitial_state) float32; None for absent operands."""
    batch, dim, L = u.shape
    N = A.shape[-1]
    dev, f32 = u.device, torch.float32
    grads = {"du": torch.empty_like(u), "ddelta": torch.empty_like(u),
             "dA": torch.empty((dim, N), dtype=f32, device=dev),
             "dB": torch.empty((batch, N, L), dtype=f32, device=dev),
             "dC": torch.empty((batch, N, L), dtype=f32, device=dev),
             "dD": torch.empty(dim, dtype=f32, device=dev) if D is not None else None,
             "dz": torch.empty_like(u) if z is not None else None,
             "ddelta_bias": torch.empty(dim, dtype=f32, device=dev) if delta_bias is not None else None}
    if with_initial_state:
        grads["dinitial_state"] = torch.empty((batch, dim, N), dtype=f32, device=dev)
    return grads


def selective_scan_bwd(u, delta, A, B, C, dy, D=None, z=None, delta_bias=None, delta_softplus=False,
                       stream=None, reset=None, initial_state=None, d_last_state=None, ckpt=None):
    """Gradients of sum(dy * y) (+ sum(d_last_state * last state)) as a dict
    (see ss_bwd); allocates the outputs; dinitial_state when an initial
    state or a last-state gradient is given."""
    grads = _grad_outputs(u, A, D, z, delta_bias, initial_state is not None or d_last_state is not None)
    if ckpt is not None:  # from the forward's checkpoints (ss_fwd_ckpt); they hold the initial state
        ss_bwd_ckpt(u, delta, A, B, C, dy, ckpt, grads, D=D, z=z, delta_bias=delta_bias,
                    delta_softplus=delta_softplus, reset=reset, d_last_state=d_last_state, stream=stream)
        return grads
    ss_bwd(u, delta, A, B, C, dy, grads, D=D, z=z, delta_bias=delta_bias,
           delta_softplus=delta_softplus, stream=stream, reset=reset, initial_state=initial_state,
           d_last_state=d_last_state)
    return grads


def ss_fwd_workspace_bytes(batch, dim, seqlen, dstate, in_dtype=torch.bfloat16, out_dtype=None,
                           lanes_per_row=None, split_states=False, warps_per_block=None,
                           segments=None) -> int:
    """Workspace bytes of the heuristic's shape (or the given one)."""
    desc = make_desc(batch, dim, seqlen, dstate, in_dtype, out_dtype)
    cfg = _config(lanes_per_row, split_states, warps_per_block, segments)
    return int(lib().ss_fwd_workspace_bytes(ctypes.byref(desc),
                                            ctypes.byref(cfg) if cfg is not None else None))


def workspace_for(batch, dim, seqlen, dstate, in_dtype, out_dtype=None, device="cuda", **config):
    """A uint8 CUDA tensor large enough for the launch shape, or None if it needs none."""
    n = ss_fwd_workspace_bytes(batch, dim, seqlen, dstate, in_dtype, out_dtype, **config)
    return torch.empty(n, dtype=torch.uint8, device=device) if n else None


def ss_fwd_heuristic(batch, dim, seqlen, dstate, in_dtype=torch.bfloat16, out_dtype=None,
                     workspace_bytes=0):
    """The launch shape the library picks, as a dict."""
    desc = make_desc(batch, dim, seqlen, dstate, in_dtype, out_dtype)
    cfg = LaunchConfig()
    _check(lib().ss_fwd_heuristic(ctypes.byref(desc), int(workspace_bytes), ctypes.byref(cfg)),
           "ss_fwd_heuristic")
    return {"lanes_per_row": cfg.lanes_per_row, "split_states": int(cfg.split_states),
            "warps_per_block": cfg.warps_per_block, "segments": cfg.segments}


def ss_fwd_hostio(host: dict, dev: dict, delta_softplus=False, stream=None, workspace=None,
                  streams=None, chunks=0):
    """Host-buffer form: ``host`` and ``dev`` map u, delta, A, B, C, D, z,
    delta_bias, y, last_state to host (ideally pinned) and device tensors of
    the same shapes (optional entries None in both).  Queues copies in, the
    forward, and copies of y / last_state out on ``stream``; with ``streams``
    (a list of CUDA streams) the work is pipelined over them by batch ranges
    (``ss_fwd_hostio_streams``) and the caller synchronises every stream."""
    g = lambda m, k: m.get(k)  # noqa: E731
    batch, dim, L = host["u"].shape
    N = host["A"].shape[-1]
    desc = make_desc(batch, dim, L, N, host["u"].dtype, host["y"].dtype)
    names_in = ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")
    h_in = [_ptr(g(host, k)) for k in names_in]
    d_all = [_ptr(g(dev, k)) for k in names_in + ("y", "last_state")]
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    if streams:
        handles = (ctypes.c_void_p * len(streams))(*[st.cuda_stream for st in streams])
        _check(lib().ss_fwd_hostio_streams(ctypes.byref(desc), *h_in, 1 if delta_softplus else 0,
                                           _ptr(host["y"]), _ptr(g(host, "last_state")), *d_all,
                                           _ptr(workspace), ws_bytes, handles, len(streams), int(chunks)),
               "ss_fwd_hostio_streams")
        return
    s = _stream_handle(stream, dev["u"].device)
    _check(lib().ss_fwd_hostio(ctypes.byref(desc), *h_in, 1 if delta_softplus else 0,
                               _ptr(host["y"]), _ptr(g(host, "last_state")), *d_all,
                               _ptr(workspace), ws_bytes, s),
           "ss_fwd_hostio")


def selective_scan_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=False,
                       return_last_state=False, out_dtype=None, stream=None, initial_state=None,
                       reset=None):
    """y (and the last state) of the selective scan, computed by libselscan.

    Same arguments as the walkthrough's selective_scan_ref, plus the z gate
    and an optional float32 (batch, dim, N) state before step 0 and (batch, L)
    mask of sequence starts (the state entering a start is zero).  Inputs must
    be CUDA tensors; y is allocated in ``out_dtype`` (default: u's dtype),
    last_state in float32.
    """
    if not u.is_cuda:
        raise ValueError("selective_scan_fwd runs on CUDA tensors only")
    batch, dim, L = u.shape
    N = A.shape[-1]
    y = torch.empty((batch, dim, L), dtype=out_dtype or u.dtype, device=u.device)
    last = (torch.empty((batch, dim, N), dtype=torch.float32, device=u.device)
            if return_last_state else None)
    ws = workspace_for(batch, dim, L, N, u.dtype, y.dtype, device=u.device)
    ss_fwd(u, delta, A, B, C, y, D=D, z=z, delta_bias=delta_bias, delta_softplus=delta_softplus,
           last_state=last, stream=stream, workspace=ws, initial_state=initial_state, reset=reset)
    return (y, last) if return_last_state else y


class SelectiveScanFn(torch.autograd.Function):
    """The scan as a torch autograd Function: the forward is ``ss_fwd_ckpt``
    (keeping the backward's checkpoints for the saved context), the backward
    ``ss_bwd_ckpt`` (all gradients, no second forward pass).  When no input
    needs a gradient the forward is plain ``ss_fwd`` and nothing is saved.
    Optional: a float32 (batch, dim, N) state before step 0 (differentiable),
    a (batch, L) mask of sequence starts, and the last state as a second
    output (differentiable: a loss on it, as when it feeds the next piece of
    a sequence, reaches every input).  Gradients come back in the dtypes of
    their inputs (dB, dC are summed in fp32 and then cast for bf16 B, C)."""

    @staticmethod
    def forward(ctx, u, delta, A, B, C, D, z, delta_bias, initial_state, reset, delta_softplus, return_last_state):
        u, delta, A, B, C, D, z, delta_bias, initial_state, reset = map(
            _contig, (u, delta, A, B, C, D, z, delta_bias, initial_state, reset))
        batch, dim, L = u.shape
        N = A.shape[-1]
        y = torch.empty_like(u)
        last = torch.empty((batch, dim, N), dtype=torch.float32, device=u.device) if return_last_state else None
        ws = workspace_for(batch, dim, L, N, u.dtype, y.dtype, device=u.device)
        kw = dict(D=D, z=z, delta_bias=delta_bias, delta_softplus=delta_softplus, last_state=last,
                  initial_state=initial_state, reset=reset, workspace=ws)
        if not any(ctx.needs_input_grad):
            ss_fwd(u, delta, A, B, C, y, **kw)
            return (y, last) if return_last_state else y
        ck = torch.empty(ckpt_shape(batch, dim, L, N), dtype=torch.float32, device=u.device)
        ss_fwd_ckpt(u, delta, A, B, C, y, ck, **kw)
        ctx.save_for_backward(u, delta, A, B, C, D, z, delta_bias, reset, ck)
        ctx.delta_softplus = bool(delta_softplus)
        ctx.has_h0 = initial_state is not None
        ctx.return_last_state = bool(return_last_state)
        return (y, last) if return_last_state else y

    @staticmethod
    @torch.autograd.function.once_differentiable
    def backward(ctx, dy, dlast=None):
        u, delta, A, B, C, D, z, delta_bias, reset, ck = ctx.saved_tensors
        g = _grad_outputs(u, A, D, z, delta_bias, ctx.has_h0 and ctx.needs_input_grad[8])
        ss_bwd_ckpt(u, delta, A, B, C, dy.contiguous(), ck, g, D=D, z=z, delta_bias=delta_bias,
                    delta_softplus=ctx.delta_softplus, reset=reset,
                    d_last_state=dlast.contiguous() if dlast is not None else None)
        return (g["du"], g["ddelta"], g["dA"], g["dB"].to(B.dtype), g["dC"].to(C.dtype), g["dD"], g["dz"],
                g["ddelta_bias"], g.get("dinitial_state"), None, None, None)


def selective_scan_fn(u, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=False,
                      initial_state=None, reset=None, return_last_state=False):
    """y (and, with return_last_state, the float32 last state) of the
    selective scan (argument order of the walkthrough's selective_scan_ref,
    plus an optional initial state and mask of sequence starts),
    differentiable through torch autograd; see SelectiveScanFn."""
    if reset is not None and reset.dtype == torch.bool:
        reset = reset.view(torch.uint8)
    return SelectiveScanFn.apply(u, delta, A, B, C, D, z, delta_bias, initial_state, reset, delta_softplus,
                                 return_last_state)
