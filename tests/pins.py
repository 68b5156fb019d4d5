"""Pins for the fp64 oracle: checks against facts that do not come from the
oracle itself.  Each ``pin_*`` takes ``scan`` (a callable with the oracle's
``selective_scan`` signature) and raises AssertionError when it disagrees.

The definition pinned is the selective-scan forward of the walkthrough page
"Mamba代码实战：手把手教你用PyTorch复现选择性扫描核心逻辑（附避坑指南）"
(§2.2 delta transform, §3.1 discretisation, §3.2 the sequential state loop,
§3.3 skip and gate, §6 last state), with y summed against C[b, n, l] as the
mamba-minimal page ("Mamba-minimal项目解析", 关键技术点 §1) writes it.

Independent references used here: the hand-worked golden example, the closed
form of a constant-coefficient recurrence (geometric series), a brute-force
unrolled sum written as products of decays, scipy.signal.lfilter for the
time-invariant case, torch's softplus/silu for the scalar transforms, and
structural invariants (causality, linearity, separability over states,
last state consistent with y).
"""
import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rel_err(got, want):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    return float(np.max(np.abs(got - want) / (1.0 + np.abs(want)))) if want.size else 0.0


def _assert_close(got, want, tol, what):
    e = _rel_err(got, want)
    assert e <= tol, f"{what}: max |err|/(1+|want|) = {e:.3e} > {tol:.1e}"


def _softplus_ref(x):
    return F.softplus(torch.as_tensor(x, dtype=torch.float64)).numpy()


def _silu_ref(x):
    return F.silu(torch.as_tensor(x, dtype=torch.float64)).numpy()


def _rand(rng, *shape):
    return rng.standard_normal(shape)


# --------------------------------------------------------------------------
def pin_hand_worked(scan):
    """The golden example of tests/golden/hand_worked.json, both delta modes,
    with and without the gate."""
    g = json.load(open(os.path.join(GOLDEN, "hand_worked.json")))
    inp, exp_ = g["inputs"], g["expected"]
    ln2 = math.log(2.0)
    u = np.array(inp["u"])
    A = np.array(inp["A"])
    B = np.array(inp["B_times_ln2"]) / ln2
    C = np.array(inp["C"])
    D = np.array(inp["D"])
    z = np.array(inp["z"])
    tol = g["tolerance_rel"]
    modes = [(np.full(u.shape, math.log(ln2)), False), (np.array(inp["delta_softplus_mode"]), True)]
    for delta, sp in modes:
        y, last = scan(u, delta, A, B, C, D=D, delta_softplus=sp, return_last_state=True)
        _assert_close(y, exp_["y"], tol, f"hand-worked y (softplus={sp})")
        _assert_close(last, exp_["last_state"], tol, f"hand-worked last state (softplus={sp})")
        yg = scan(u, delta, A, B, C, D=D, z=z, delta_softplus=sp)
        _assert_close(yg, exp_["y_gated"], tol, f"hand-worked gated y (softplus={sp})")


def pin_delta_transform(scan):
    """delta' exposed directly: with N=1, A=0 (dA=1), B=C=u=1 the output is
    the running sum of delta', so y[0] = delta'[0] and y[t]-y[t-1] = delta'[t].
    Compared with torch's softplus (threshold 20) and exp."""
    raw = np.array([-30.0, -5.0, -0.7, 0.0, 0.3, 4.0, 19.9, 20.0, 20.5, 25.0])
    bias = np.array([0.25])
    L = raw.size
    one = np.ones((1, 1, L))
    for sp in (True, False):
        r = raw if sp else np.clip(raw, -30, 5)
        y = scan(one, r.reshape(1, 1, L), np.zeros((1, 1)), one, one, delta_bias=bias,
                 delta_softplus=sp)
        d_got = np.diff(np.concatenate([[0.0], y[0, 0]]))
        d_want = _softplus_ref(r + bias[0]) if sp else np.exp(r + bias[0])
        _assert_close(d_got, d_want, 1e-13, f"delta transform (softplus={sp})")


def pin_closed_form(scan):
    """Constant delta, A, B, u over l: each state is a geometric series,
    h_t = beta (1 - a^t) / (1 - a) with a = exp(delta' A_n), beta = delta' B_n u.
    C varies over l, D and a delta bias are present."""
    rng = np.random.default_rng(11)
    Bt, Dm, L, N = 2, 3, 40, 5
    raw = rng.uniform(-1.5, 0.5, size=(Bt, Dm))
    bias = rng.uniform(-0.3, 0.3, size=Dm)
    uc = rng.standard_normal((Bt, Dm))
    A = -0.1 * (np.arange(1, N + 1)[None, :] * rng.uniform(0.5, 1.5, size=(Dm, 1)))
    Bc = rng.standard_normal((Bt, N))
    C = rng.standard_normal((Bt, N, L))
    Dv = rng.standard_normal(Dm)
    delta = np.repeat(raw[:, :, None], L, axis=2)
    u = np.repeat(uc[:, :, None], L, axis=2)
    Bm = np.repeat(Bc[:, :, None], L, axis=2)
    for sp in (True, False):
        y, last = scan(u, delta, A, Bm, C, D=Dv, delta_bias=bias, delta_softplus=sp,
                       return_last_state=True)
        x = raw + bias[None, :]
        dl = _softplus_ref(x) if sp else np.exp(x)
        t = np.arange(1, L + 1)
        want = np.empty((Bt, Dm, L))
        want_last = np.empty((Bt, Dm, N))
        for b in range(Bt):
            for d in range(Dm):
                a = np.exp(dl[b, d] * A[d])                       # (N,)
                beta = dl[b, d] * Bc[b] * uc[b, d]                  # (N,)
                h = beta[:, None] * (1 - a[:, None] ** t[None, :]) / (1 - a[:, None])  # (N, L)
                want[b, d] = (C[b] * h).sum(0) + Dv[d] * uc[b, d]
                want_last[b, d] = h[:, -1]
        _assert_close(y, want, 1e-11, f"closed form y (softplus={sp})")
        _assert_close(last, want_last, 1e-11, f"closed form last state (softplus={sp})")


def brute_force(u, delta, A, B, C, D, z, bias, sp):
    """Unrolled-sum reference (pure Python loops, tiny sizes only):
    h[t, n] = sum_{s <= t} (prod_{s < r <= t} a[r, n]) * delta'[s] B[n, s] u[s]."""
    Bt, Dm, L = u.shape
    N = A.shape[1]
    x = delta + (bias[None, :, None] if bias is not None else 0.0)
    dl = _softplus_ref(x) if sp else np.exp(x)
    y = np.zeros((Bt, Dm, L))
    last = np.zeros((Bt, Dm, N))
    for b in range(Bt):
        for d in range(Dm):
            for t in range(L):
                acc = 0.0
                for n in range(N):
                    h = 0.0
                    for s in range(t + 1):
                        decay = 1.0
                        for r in range(s + 1, t + 1):
                            decay *= math.exp(dl[b, d, r] * A[d, n])
                        h += decay * dl[b, d, s] * B[b, n, s] * u[b, d, s]
                    acc += C[b, n, t] * h
                    if t == L - 1:
                        last[b, d, n] = h
                if D is not None:
                    acc += D[d] * u[b, d, t]
                y[b, d, t] = acc
    if z is not None:
        y = y * _silu_ref(z)
    return y, last


def pin_brute_force(scan):
    """Random tiny problems (non-square shapes so a transposed index shows)
    against the unrolled sum, every optional operand on and off."""
    rng = np.random.default_rng(7)
    Bt, Dm, L, N = 2, 3, 7, 4
    for case in range(4):
        u = _rand(rng, Bt, Dm, L)
        delta = _rand(rng, Bt, Dm, L)
        A = -rng.uniform(0.2, 2.0, size=(Dm, N))
        Bm = _rand(rng, Bt, N, L)
        C = _rand(rng, Bt, N, L)
        D = _rand(rng, Dm) if case % 2 == 0 else None
        z = _rand(rng, Bt, Dm, L) if case in (1, 2) else None
        bias = _rand(rng, Dm) * 0.5 if case >= 2 else None
        sp = case != 3
        y, last = scan(u, delta, A, Bm, C, D=D, z=z, delta_bias=bias, delta_softplus=sp,
                       return_last_state=True)
        yw, lw = brute_force(u, delta, A, Bm, C, D, z, bias, sp)
        _assert_close(y, yw, 1e-12, f"brute force y (case {case})")
        _assert_close(last, lw, 1e-12, f"brute force last state (case {case})")


def pin_lfilter(scan):
    """Time-invariant case (delta and B constant over l, u varying): each state
    is a first-order IIR filter of u, h = lfilter([delta' B_n], [1, -a_n], u)."""
    from scipy.signal import lfilter
    rng = np.random.default_rng(5)
    Bt, Dm, L, N = 2, 2, 300, 6
    raw = rng.uniform(-2.0, 1.0, size=(Bt, Dm))
    A = -np.arange(1, N + 1, dtype=np.float64)[None, :].repeat(Dm, 0) * 0.05
    Bc = rng.standard_normal((Bt, N))
    u = rng.standard_normal((Bt, Dm, L))
    C = rng.standard_normal((Bt, N, L))
    Dv = rng.standard_normal(Dm)
    delta = np.repeat(raw[:, :, None], L, axis=2)
    Bm = np.repeat(Bc[:, :, None], L, axis=2)
    y, last = scan(u, delta, A, Bm, C, D=Dv, delta_softplus=True, return_last_state=True)
    dl = _softplus_ref(raw)
    want = np.zeros((Bt, Dm, L))
    want_last = np.zeros((Bt, Dm, N))
    for b in range(Bt):
        for d in range(Dm):
            for n in range(N):
                a = math.exp(dl[b, d] * A[d, n])
                h = lfilter([dl[b, d] * Bc[b, n]], [1.0, -a], u[b, d])
                want[b, d] += C[b, n] * h
                want_last[b, d, n] = h[-1]
            want[b, d] += Dv[d] * u[b, d]
    _assert_close(y, want, 1e-11, "lfilter y")
    _assert_close(last, want_last, 1e-11, "lfilter last state")


def pin_delta_to_zero(scan):
    """delta' -> 0 exactly (raw delta = -1e4: softplus and exp both give 0 in
    float64): no state moves, so y = D*u exactly, times silu(z) when gated."""
    rng = np.random.default_rng(3)
    Bt, Dm, L, N = 2, 3, 9, 4
    u = _rand(rng, Bt, Dm, L)
    delta = np.full((Bt, Dm, L), -1e4)
    A = -rng.uniform(0.5, 2, size=(Dm, N))
    Bm, C = _rand(rng, Bt, N, L), _rand(rng, Bt, N, L)
    Dv = _rand(rng, Dm)
    z = _rand(rng, Bt, Dm, L)
    for sp in (True, False):
        y, last = scan(u, delta, A, Bm, C, D=Dv, delta_softplus=sp, return_last_state=True)
        assert np.array_equal(y, Dv[None, :, None] * u), "delta->0 must give y = D*u exactly"
        assert np.all(last == 0.0), "delta->0 must leave the state at zero"
        yg = scan(u, delta, A, Bm, C, D=Dv, z=z, delta_softplus=sp)
        _assert_close(yg, Dv[None, :, None] * u * _silu_ref(z), 1e-15, "delta->0 gated")


def pin_causality(scan):
    """Changing any input at step t leaves y[:t] bitwise unchanged and does
    change y[t]."""
    rng = np.random.default_rng(9)
    Bt, Dm, L, N = 1, 2, 12, 3
    base = dict(u=_rand(rng, Bt, Dm, L), delta=_rand(rng, Bt, Dm, L),
                A=-rng.uniform(0.2, 1.5, (Dm, N)), B=_rand(rng, Bt, N, L),
                C=_rand(rng, Bt, N, L), z=_rand(rng, Bt, Dm, L))
    D = _rand(rng, Dm)
    y0 = scan(base["u"], base["delta"], base["A"], base["B"], base["C"], D=D, z=base["z"],
              delta_softplus=True)
    t = 5
    for key in ("u", "delta", "B", "C", "z"):
        p = {k: v.copy() for k, v in base.items()}
        p[key][..., t] += 0.75
        y1 = scan(p["u"], p["delta"], p["A"], p["B"], p["C"], D=D, z=p["z"], delta_softplus=True)
        assert np.array_equal(y0[..., :t], y1[..., :t]), f"perturbing {key} at t changed y before t"
        assert np.all(y0[..., t] != y1[..., t]), f"perturbing {key} at t left y[t] unchanged"


def pin_linearity(scan):
    """With delta, B, C, z fixed, y is linear in u: y(a u1 + u2) = a y(u1) + y(u2)."""
    rng = np.random.default_rng(4)
    Bt, Dm, L, N = 2, 3, 20, 4
    delta, z = _rand(rng, Bt, Dm, L), _rand(rng, Bt, Dm, L)
    A = -rng.uniform(0.2, 1.5, (Dm, N))
    Bm, C, D = _rand(rng, Bt, N, L), _rand(rng, Bt, N, L), _rand(rng, Dm)
    u1, u2 = _rand(rng, Bt, Dm, L), _rand(rng, Bt, Dm, L)
    alpha = -1.7
    f = lambda u: scan(u, delta, A, Bm, C, D=D, z=z, delta_softplus=True)  # noqa: E731
    _assert_close(f(alpha * u1 + u2), alpha * f(u1) + f(u2), 1e-12, "linearity in u")


def pin_state_separability(scan):
    """States do not interact: y - D u over N states equals the sum of the
    single-state runs (each with its own column of A, B, C)."""
    rng = np.random.default_rng(8)
    Bt, Dm, L, N = 2, 2, 15, 5
    u, delta = _rand(rng, Bt, Dm, L), _rand(rng, Bt, Dm, L)
    A = -rng.uniform(0.2, 1.5, (Dm, N))
    Bm, C, D = _rand(rng, Bt, N, L), _rand(rng, Bt, N, L), _rand(rng, Dm)
    full = scan(u, delta, A, Bm, C, D=D, delta_softplus=True) - D[None, :, None] * u
    parts = sum(scan(u, delta, A[:, n:n + 1], Bm[:, n:n + 1], C[:, n:n + 1], delta_softplus=True)
                for n in range(N))
    _assert_close(full, parts, 1e-12, "separability over states")


def pin_last_state(scan):
    """The last state of the prefix [0, t] is the state that produced y[t]:
    y[t] (no D, no gate) = sum_n C[n, t] * last_state(prefix t+1)[n], for every t;
    and an empty sequence leaves the zero state."""
    rng = np.random.default_rng(6)
    Bt, Dm, L, N = 1, 2, 10, 3
    u, delta = _rand(rng, Bt, Dm, L), _rand(rng, Bt, Dm, L)
    A = -rng.uniform(0.2, 1.5, (Dm, N))
    Bm, C = _rand(rng, Bt, N, L), _rand(rng, Bt, N, L)
    y = scan(u, delta, A, Bm, C, delta_softplus=True)
    for t in range(L):
        _, last = scan(u[..., :t + 1], delta[..., :t + 1], A, Bm[..., :t + 1], C[..., :t + 1],
                       delta_softplus=True, return_last_state=True)
        want = np.einsum("bn,bdn->bd", C[:, :, t], last)
        _assert_close(y[..., t], want, 1e-13, f"last state vs y at t={t}")
    _, last0 = scan(u[..., :0], delta[..., :0], A, Bm[..., :0], C[..., :0],
                    delta_softplus=True, return_last_state=True)
    assert np.all(last0 == 0.0), "empty sequence must leave the zero state"


# ---- initial state (extension: the walkthrough's state always starts at 0;
# a given state before step 0 lets a sequence run in pieces).

def pin_initial_state_closed_form(scan):
    """Constant delta, A, B, u from a given state h0: each state is
    h_t = a^t h0 + beta (1 - a^t) / (1 - a) (t = 1..L steps taken)."""
    rng = np.random.default_rng(23)
    Bt, Dm, L, N = 2, 3, 30, 4
    raw = rng.uniform(-1.5, 0.5, size=(Bt, Dm))
    uc = rng.standard_normal((Bt, Dm))
    A = -0.15 * (np.arange(1, N + 1)[None, :] * rng.uniform(0.5, 1.5, size=(Dm, 1)))
    Bc = rng.standard_normal((Bt, N))
    C = rng.standard_normal((Bt, N, L))
    Dv = rng.standard_normal(Dm)
    h0 = rng.standard_normal((Bt, Dm, N)) * 3.0
    delta = np.repeat(raw[:, :, None], L, axis=2)
    u = np.repeat(uc[:, :, None], L, axis=2)
    Bm = np.repeat(Bc[:, :, None], L, axis=2)
    y, last = scan(u, delta, A, Bm, C, D=Dv, delta_softplus=True, return_last_state=True,
                   initial_state=h0)
    dl = _softplus_ref(raw)
    t = np.arange(1, L + 1)
    want = np.empty((Bt, Dm, L))
    want_last = np.empty((Bt, Dm, N))
    for b in range(Bt):
        for d in range(Dm):
            a = np.exp(dl[b, d] * A[d])
            beta = dl[b, d] * Bc[b] * uc[b, d]
            at = a[:, None] ** t[None, :]
            h = at * h0[b, d][:, None] + beta[:, None] * (1 - at) / (1 - a[:, None])
            want[b, d] = (C[b] * h).sum(0) + Dv[d] * uc[b, d]
            want_last[b, d] = h[:, -1]
    _assert_close(y, want, 1e-11, "closed form from h0: y")
    _assert_close(last, want_last, 1e-11, "closed form from h0: last state")


def pin_initial_state_brute_force(scan):
    """Tiny random problems from a given state against the unrolled sum plus
    the decayed initial state, prod_{r <= t} a[r, n] * h0[n]."""
    rng = np.random.default_rng(29)
    Bt, Dm, L, N = 2, 3, 6, 4
    u = _rand(rng, Bt, Dm, L)
    delta = _rand(rng, Bt, Dm, L)
    A = -rng.uniform(0.2, 2.0, size=(Dm, N))
    Bm = _rand(rng, Bt, N, L)
    C = _rand(rng, Bt, N, L)
    h0 = _rand(rng, Bt, Dm, N)
    z = _rand(rng, Bt, Dm, L)
    y, last = scan(u, delta, A, Bm, C, z=z, delta_softplus=True, return_last_state=True,
                   initial_state=h0)
    y0, last0 = brute_force(u, delta, A, Bm, C, None, None, None, True)
    dl = _softplus_ref(delta)
    for b in range(Bt):
        for d in range(Dm):
            for n in range(N):
                decay = 1.0
                for t in range(L):
                    decay *= math.exp(dl[b, d, t] * A[d, n])
                    y0[b, d, t] += C[b, n, t] * decay * h0[b, d, n]
                last0[b, d, n] += decay * h0[b, d, n]
    _assert_close(y, y0 * _silu_ref(z), 1e-12, "brute force from h0: y")
    _assert_close(last, last0, 1e-12, "brute force from h0: last state")


def pin_initial_state_continuity(scan):
    """Running steps [0, k) and then [k, L) from the state the first piece
    left equals running [0, L) in one piece, y and last state."""
    rng = np.random.default_rng(31)
    Bt, Dm, L, N = 2, 3, 50, 5
    u = _rand(rng, Bt, Dm, L)
    delta = _rand(rng, Bt, Dm, L)
    A = -rng.uniform(0.05, 1.0, size=(Dm, N))
    Bm = _rand(rng, Bt, N, L)
    C = _rand(rng, Bt, N, L)
    Dv = _rand(rng, Dm)
    z = _rand(rng, Bt, Dm, L)
    bias = _rand(rng, Dm) * 0.3
    kw = dict(D=Dv, delta_bias=bias, delta_softplus=True, return_last_state=True)
    y, last = scan(u, delta, A, Bm, C, z=z, **kw)
    for k in (1, 17, 49):
        y1, h1 = scan(u[..., :k], delta[..., :k], A, Bm[..., :k], C[..., :k], z=z[..., :k], **kw)
        y2, h2 = scan(u[..., k:], delta[..., k:], A, Bm[..., k:], C[..., k:], z=z[..., k:],
                      initial_state=h1, **kw)
        _assert_close(np.concatenate([y1, y2], axis=-1), y, 1e-13, f"pieces at {k}: y")
        _assert_close(h2, last, 1e-13, f"pieces at {k}: last state")


# ---- sequence starts (extension: the boundary reset of "Mamba实战：如何用选择性
# 状态空间模型提升你的长序列处理效率（附代码）" §2; the state entering a start is zero).

def pin_reset_hand_worked(scan):
    """The golden example of tests/golden/hand_worked.json with a sequence
    start at step 1 and at step 2 (values derived by hand there), both delta
    modes; a start at step 0 changes nothing."""
    g = json.load(open(os.path.join(GOLDEN, "hand_worked.json")))
    inp, exp_ = g["inputs"], g["expected"]
    ln2 = math.log(2.0)
    u = np.array(inp["u"])
    A = np.array(inp["A"])
    B = np.array(inp["B_times_ln2"]) / ln2
    C = np.array(inp["C"])
    D = np.array(inp["D"])
    tol = g["tolerance_rel"]
    L = u.shape[-1]
    for delta, sp in [(np.full(u.shape, math.log(ln2)), False), (np.array(inp["delta_softplus_mode"]), True)]:
        for at, key in ((1, "start_at_1"), (2, "start_at_2"), (0, None)):
            reset = np.zeros((u.shape[0], L), dtype=np.uint8)
            reset[:, at] = 1
            y, last = scan(u, delta, A, B, C, D=D, delta_softplus=sp, return_last_state=True, reset=reset)
            want = g["expected_reset"][key] if key else exp_
            _assert_close(y, want["y"], tol, f"hand-worked start at {at} y (softplus={sp})")
            _assert_close(last, want["last_state"], tol, f"hand-worked start at {at} last state (softplus={sp})")


def pin_reset_pieces(scan):
    """Rows holding several sequences: with starts marked, y over each piece
    and the last state equal independent runs of the pieces (each from the
    zero state, the first one from the given initial state unless a start
    sits at step 0), batch entry by batch entry."""
    rng = np.random.default_rng(37)
    Bt, Dm, L, N = 2, 3, 40, 4
    u = _rand(rng, Bt, Dm, L)
    delta = _rand(rng, Bt, Dm, L)
    A = -rng.uniform(0.05, 1.0, size=(Dm, N))
    Bm = _rand(rng, Bt, N, L)
    C = _rand(rng, Bt, N, L)
    Dv = _rand(rng, Dm)
    z = _rand(rng, Bt, Dm, L)
    bias = _rand(rng, Dm) * 0.3
    h0 = _rand(rng, Bt, Dm, N)
    starts = {0: [7, 8, 23], 1: [0, 15, 39]}
    reset = np.zeros((Bt, L), dtype=np.uint8)
    for b, ls in starts.items():
        reset[b, ls] = 1
    kw = dict(D=Dv, delta_bias=bias, delta_softplus=True, return_last_state=True)
    y, last = scan(u, delta, A, Bm, C, z=z, initial_state=h0, reset=reset, **kw)
    for b, ls in starts.items():
        cuts = [0] + [l for l in ls if l > 0] + [L]
        for k in range(len(cuts) - 1):
            lo, hi = cuts[k], cuts[k + 1]
            first_from_h0 = lo == 0 and 0 not in ls
            yp, hp = scan(u[b:b + 1, :, lo:hi], delta[b:b + 1, :, lo:hi], A, Bm[b:b + 1, :, lo:hi],
                          C[b:b + 1, :, lo:hi], z=z[b:b + 1, :, lo:hi],
                          initial_state=h0[b:b + 1] if first_from_h0 else None, **kw)
            _assert_close(y[b:b + 1, :, lo:hi], yp, 1e-15, f"batch {b} piece [{lo}, {hi}): y")
        _assert_close(last[b:b + 1], hp, 1e-15, f"batch {b}: last state")


def pin_reset_every_step(scan):
    """A start at every step leaves no memory: y_l = (sum_n C[n,l] delta'_l
    B[n,l] u_l + D u_l) silu(z_l), and the last state is delta'_L B[:,L] u_L."""
    rng = np.random.default_rng(41)
    Bt, Dm, L, N = 2, 3, 12, 5
    u = _rand(rng, Bt, Dm, L)
    delta = _rand(rng, Bt, Dm, L)
    A = -rng.uniform(0.05, 1.0, size=(Dm, N))
    Bm = _rand(rng, Bt, N, L)
    C = _rand(rng, Bt, N, L)
    Dv = _rand(rng, Dm)
    z = _rand(rng, Bt, Dm, L)
    h0 = _rand(rng, Bt, Dm, N)
    y, last = scan(u, delta, A, Bm, C, D=Dv, z=z, delta_softplus=True, return_last_state=True,
                   initial_state=h0, reset=np.ones((Bt, L), dtype=np.uint8))
    dl = _softplus_ref(delta)
    h = dl[:, :, None, :] * Bm[:, None, :, :] * u[:, :, None, :]       # (b, d, n, l)
    want = ((C[:, None, :, :] * h).sum(2) + Dv[None, :, None] * u) * _silu_ref(z)
    _assert_close(y, want, 1e-13, "start at every step: y")
    _assert_close(last, h[..., -1], 1e-13, "start at every step: last state")


def pin_reset_none(scan):
    """An all-zero start mask is no mask; a single start changes y from that
    step on and not before it."""
    rng = np.random.default_rng(43)
    Bt, Dm, L, N = 2, 2, 20, 3
    u = _rand(rng, Bt, Dm, L)
    delta = _rand(rng, Bt, Dm, L)
    A = -rng.uniform(0.05, 1.0, size=(Dm, N))
    Bm = _rand(rng, Bt, N, L)
    C = _rand(rng, Bt, N, L)
    y = scan(u, delta, A, Bm, C, delta_softplus=True)
    y0 = scan(u, delta, A, Bm, C, delta_softplus=True, reset=np.zeros((Bt, L), dtype=np.uint8))
    assert np.array_equal(y, y0), "all-zero start mask must be no mask"
    one = np.zeros((Bt, L), dtype=np.uint8)
    one[1, 9] = 1
    y1 = scan(u, delta, A, Bm, C, delta_softplus=True, reset=one)
    assert np.array_equal(y1[0], y[0]) and np.array_equal(y1[1, :, :9], y[1, :, :9]), \
        "a start must not change other batch entries or earlier steps"
    assert np.all(y1[1, :, 9] != y[1, :, 9]), "a start must change its own step"


ALL_PINS = [pin_hand_worked, pin_delta_transform, pin_closed_form, pin_brute_force,
            pin_lfilter, pin_delta_to_zero, pin_causality, pin_linearity,
            pin_state_separability, pin_last_state, pin_initial_state_closed_form,
            pin_initial_state_brute_force, pin_initial_state_continuity, pin_reset_hand_worked, pin_reset_pieces,
            pin_reset_every_step, pin_reset_none]
