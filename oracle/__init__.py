"""fp64 CPU oracle for the selective-scan forward and its gradients (TEST
INFRASTRUCTURE).

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg may import this package.  The product path (the CUDA library and
its Python binding) never does, and shares no code with it.

``selective_scan`` widens every input exactly to float64 (bf16 and fp32 values
are exactly representable) and runs the sequential loop of ``ss_oracle.c``.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_libs = {}


def _load(path=None):
    """The oracle library at ``path`` (default: the built ``liboracle.so``)."""
    if path is None:
        path = _build.build()
    if path not in _libs:
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        lib.ss_oracle_fwd.restype = ctypes.c_int
        lib.ss_oracle_fwd.argtypes = [i64, i64, i64, i64, P, P, P, P, P, P, P, P,
                                      ctypes.c_int, P, P, ctypes.c_int]
        lib.ss_oracle_fwd_reset.restype = ctypes.c_int
        lib.ss_oracle_fwd_reset.argtypes = [i64, i64, i64, i64] + [P] * 8 + [ctypes.c_int] + [P] * 4 + \
            [ctypes.c_int]
        lib.ss_oracle_fwd_init.restype = ctypes.c_int
        lib.ss_oracle_fwd_init.argtypes = [i64, i64, i64, i64, P, P, P, P, P, P, P, P,
                                           ctypes.c_int, P, P, P, ctypes.c_int]
        if hasattr(lib, "ss_oracle_bwd"):  # (a planted-mistake build of the forward alone has none)
            lib.ss_oracle_bwd_full.restype = ctypes.c_int
            lib.ss_oracle_bwd_full.argtypes = [i64, i64, i64, i64] + [P] * 8 + [ctypes.c_int] + \
                [P] * 18 + [ctypes.c_int]
            lib.ss_oracle_bwd_reset.restype = ctypes.c_int
            lib.ss_oracle_bwd_reset.argtypes = [i64, i64, i64, i64] + [P] * 8 + [ctypes.c_int] + \
                [P] * 10 + [ctypes.c_int]
            lib.ss_oracle_bwd.restype = ctypes.c_int
            lib.ss_oracle_bwd.argtypes = [i64, i64, i64, i64] + [P] * 8 + [ctypes.c_int] + [P] * 9 + \
                [ctypes.c_int]
        lib.ss_oracle_threads.restype = ctypes.c_int
        lib.ss_oracle_threads.argtypes = []
        _libs[path] = lib
    return _libs[path]


def max_threads() -> int:
    """Threads the oracle's OpenMP loop uses when asked for "all"."""
    return int(_load().ss_oracle_threads())


def _f64(x):
    """Exact widening to a C-contiguous float64 numpy array (None stays None)."""
    if x is None:
        return None
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().to("cpu", torch.float64).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def selective_scan(u, delta, A, B, C, D=None, z=None, delta_bias=None,
                   delta_softplus=False, return_last_state=False, nthreads=0, lib=None,
                   initial_state=None, reset=None):
    """y[b,d,l] (and the state after the last step) in float64.

    Shapes: u, delta, z (batch, dim, L); A (dim, N); B, C (batch, N, L);
    D, delta_bias (dim,); initial_state (batch, dim, N), the state before
    step 0 (zero when None); reset (batch, L), nonzero where a new sequence
    starts (the state entering that step is zero).  Returns y, or (y, last_state (batch, dim, N)).
    ``lib`` selects another build of the oracle library by path (the pin tests
    use it to show that planted mistakes are caught).
    """
    u, delta, A, B, C =(_f64(t) for t in (u, delta, A, B, C))
    D, z, delta_bias = _f64(D), _f64(z), _f64(delta_bias)
    batch, dim, L = u.shape
    N = A.shape[1]
    if delta.shape != u.shape:
        raise ValueError("u and delta must have the same shape")
    if A.shape != (dim, N) or B.shape != (batch, N, L) or C.shape != (batch, N, L):
        raise ValueError("bad A/B/C shape")
    if z is not None and z.shape != u.shape:
        raise ValueError("bad z shape")
    for v in (D, delta_bias):
        if v is not None and v.shape != (dim,):
            raise ValueError("bad D/delta_bias shape")
    h0 = _f64(initial_state)
    if h0 is not None and h0.shape != (batch, dim, N):
        raise ValueError("bad initial_state shape")
    rs = None
    if reset is not None:
        rs = np.ascontiguousarray(np.asarray(reset) != 0, dtype=np.uint8)
        if rs.shape != (batch, L):
            raise ValueError("bad reset shape")
    y = np.zeros((batch, dim, L), dtype=np.float64)
    last = np.zeros((batch, dim, N), dtype=np.float64) if return_last_state else None
    if rs is not None:
        rc = _load(lib).ss_oracle_fwd_reset(batch, dim, L, N, _ptr(u), _ptr(delta), _ptr(A), _ptr(B),
                                            _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
                                            1 if delta_softplus else 0, _ptr(rs), _ptr(h0), _ptr(y),
                                            _ptr(last), int(nthreads))
    elif h0 is None:
        rc = _load(lib).ss_oracle_fwd(batch, dim, L, N, _ptr(u), _ptr(delta), _ptr(A), _ptr(B),
                                      _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
                                      1 if delta_softplus else 0, _ptr(y), _ptr(last), int(nthreads))
    else:
        rc = _load(lib).ss_oracle_fwd_init(batch, dim, L, N, _ptr(u), _ptr(delta), _ptr(A), _ptr(B),
                                           _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
                                           1 if delta_softplus else 0, _ptr(h0), _ptr(y), _ptr(last),
                                           int(nthreads))
    if rc != 0:
        raise RuntimeError("oracle rejected its arguments")
    return (y, last) if return_last_state else y


def delta_from_projection(delta_r, W_dt):
    """delta[b, d, l] = sum_r W_dt[d, r] delta_r[b, r, l]: the dt_proj linear
    map of the mamba-minimal block ("Mamba-minimal项目解析", 核心组件解析 §5,
    ``ssm``: x_dbl = x_proj(x), split into delta (dt_rank features), B, C;
    delta = softplus(dt_proj(delta))), without its bias (the scan adds the
    bias as delta_bias before the softplus).  delta_r (batch, dt_rank, L),
    W_dt (dim, dt_rank); widened exactly to float64, one float64 matmul."""
    r, w = _f64(delta_r), _f64(W_dt)
    if r.ndim != 3 or w.ndim != 2 or r.shape[1] != w.shape[1]:
        raise ValueError("delta_r (batch, dt_rank, L) and W_dt (dim, dt_rank)")
    return np.ascontiguousarray(np.matmul(w[None, :, :], r))


def selective_scan_dtproj(u, delta_r, W_dt, A, B, C, D=None, z=None, delta_bias=None,
                          delta_softplus=True, return_last_state=False, nthreads=0):
    """The forward with delta produced by the dt_proj map from its low-rank
    input: ``selective_scan(u, W_dt delta_r, ...)`` (see delta_from_projection)."""
    return selective_scan(u, delta_from_projection(delta_r, W_dt), A, B, C, D=D, z=z, delta_bias=delta_bias,
                          delta_softplus=delta_softplus, return_last_state=return_last_state,
                          nthreads=nthreads)


def selective_scan_bwd(u, delta, A, B, C, dy, D=None, z=None, delta_bias=None,
                       delta_softplus=False, nthreads=0, lib=None, reset=None, initial_state=None,
                       dlast_state=None, magnitudes=False):
    """Gradients of sum(dy * y) (plus sum(dlast_state * last state) when
    ``dlast_state`` (batch, dim, N) is given) for the forward of
    ``selective_scan`` (``reset`` and ``initial_state`` as there), in
    float64, as a dict: du, ddelta, dz (batch, dim, L); dA (dim, N); dB, dC
    (batch, N, L); dD, ddelta_bias (dim,); dinitial_state (batch, dim, N) when
    an initial state is given.  The entries of absent optional operands are
    None.
    ``magnitudes``: also ``mag_<name>`` for each gradient that is a sum over
    rows or steps (dA, dB, dC, dD, ddelta_bias): the sum of the absolute
    values of its terms, the state and the adjoint in each taken at the
    magnitudes of their recursions (see ss_oracle_bwd.c), which scales the
    tolerance of a finite-precision sum element by element."""
    u, delta, A, B, C, dy = (_f64(t) for t in (u, delta, A, B, C, dy))
    D, z, delta_bias = _f64(D), _f64(z), _f64(delta_bias)
    batch, dim, L = u.shape
    N = A.shape[1]
    if delta.shape != u.shape or dy.shape != u.shape:
        raise ValueError("u, delta and dy must have the same shape")
    if A.shape != (dim, N) or B.shape != (batch, N, L) or C.shape != (batch, N, L):
        raise ValueError("bad A/B/C shape")
    g = {"du": np.zeros_like(u), "ddelta": np.zeros_like(u), "dA": np.zeros((dim, N)),
         "dB": np.zeros((batch, N, L)), "dC": np.zeros((batch, N, L)),
         "dD": np.zeros(dim) if D is not None else None,
         "dz": np.zeros_like(u) if z is not None else None,
         "ddelta_bias": np.zeros(dim) if delta_bias is not None else None}
    rs = None
    if reset is not None:
        rs = np.ascontiguousarray(np.asarray(reset) != 0, dtype=np.uint8)
        if rs.shape != (batch, L):
            raise ValueError("bad reset shape")
    h0 = _f64(initial_state)
    if h0 is not None and h0.shape != (batch, dim, N):
        raise ValueError("bad initial_state shape")
    dlast = _f64(dlast_state)
    if dlast is not None and dlast.shape != (batch, dim, N):
        raise ValueError("bad dlast_state shape")
    if h0 is None and dlast is None and not magnitudes:
        rc = _load(lib).ss_oracle_bwd_reset(batch, dim, L, N, _ptr(u), _ptr(delta), _ptr(A), _ptr(B),
                                            _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
                                            1 if delta_softplus else 0, _ptr(rs), _ptr(dy), _ptr(g["du"]),
                                            _ptr(g["ddelta"]), _ptr(g["dA"]), _ptr(g["dB"]), _ptr(g["dC"]),
                                            _ptr(g["dD"]), _ptr(g["dz"]), _ptr(g["ddelta_bias"]),
                                            int(nthreads))
    else:
        if h0 is not None:
            g["dinitial_state"] = np.zeros((batch, dim, N))
        m = {}
        if magnitudes:
            m = {"mag_dA": np.zeros((dim, N)), "mag_dB": np.zeros((batch, N, L)),
                 "mag_dC": np.zeros((batch, N, L)),
                 "mag_dD": np.zeros(dim) if D is not None else None,
                 "mag_ddelta_bias": np.zeros(dim) if delta_bias is not None else None}
        rc = _load(lib).ss_oracle_bwd_full(
            batch, dim, L, N, _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
            _ptr(delta_bias), 1 if delta_softplus else 0, _ptr(rs), _ptr(h0), _ptr(dlast), _ptr(dy),
            _ptr(g["du"]),
            _ptr(g["ddelta"]), _ptr(g["dA"]), _ptr(g["dB"]), _ptr(g["dC"]), _ptr(g["dD"]), _ptr(g["dz"]),
            _ptr(g["ddelta_bias"]), _ptr(g.get("dinitial_state")), _ptr(m.get("mag_dA")),
            _ptr(m.get("mag_dB")), _ptr(m.get("mag_dC")), _ptr(m.get("mag_dD")),
            _ptr(m.get("mag_ddelta_bias")), int(nthreads))
        g.update(m)
    if rc != 0:
        raise RuntimeError("oracle rejected its arguments")
    return g


def selective_scan_rows(inputs, rows, nthreads=0):
    """Oracle outputs for selected (b, d) rows of a problem held as host tensors.

    ``inputs`` maps the names u, delta, A, B, C, D, z, delta_bias,
    delta_softplus, return_last_state; ``rows`` is a list of (b, d).  Each row
    is run as its own batch-1, dim-1 problem (rows are independent).
    Returns (y_rows (R, L), last_rows (R, N) or None).
    """
    ys, lasts = [], []
    for (b, d) in rows:
        sl = lambda t: None if t is None else t[b:b + 1, d:d + 1]  # noqa: E731
        pd = lambda t: None if t is None else t[d:d + 1]  # noqa: E731
        out = selective_scan(sl(inputs["u"]), sl(inputs["delta"]), inputs["A"][d:d + 1],
                             inputs["B"][b:b + 1], inputs["C"][b:b + 1], pd(inputs.get("D")),
                             sl(inputs.get("z")), pd(inputs.get("delta_bias")),
                             inputs["delta_softplus"], True, nthreads)
        ys.append(out[0][0, 0])
        lasts.append(out[1][0, 0])
    return np.stack(ys), np.stack(lasts)
