"""Pins for the fp64 backward oracle (gradients of sum(dy * y)).

Each ``pin_*`` takes ``grad`` (a callable with the signature of
``oracle.selective_scan_bwd``) and ``scan`` (the forward oracle, pinned on its
own in ``pins.py``) and raises AssertionError on a disagreement.  The
reference for every gradient is a central finite difference of the forward:
(F(x + eps v) - F(x - eps v)) / (2 eps) with F = sum(dy * y), which involves
no gradient formula at all.
"""
import numpy as np

NAMES = [("u", "du"), ("delta", "ddelta"), ("A", "dA"), ("B", "dB"), ("C", "dC"), ("D", "dD"),
         ("z", "dz"), ("delta_bias", "ddelta_bias")]


def _problem(rng, Bt, Dm, L, N, with_D=True, with_z=True, with_bias=True, bias_shift=0.0):
    p = {"u": rng.standard_normal((Bt, Dm, L)), "delta": rng.standard_normal((Bt, Dm, L)),
         "A": -rng.uniform(0.2, 2.0, size=(Dm, N)), "B": rng.standard_normal((Bt, N, L)),
         "C": rng.standard_normal((Bt, N, L)),
         "D": rng.standard_normal(Dm) if with_D else None,
         "z": rng.standard_normal((Bt, Dm, L)) if with_z else None,
         "delta_bias": (rng.standard_normal(Dm) * 0.3 + bias_shift) if with_bias else None}
    return p


def _F(scan, p, dy, sp):
    y = scan(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
             delta_bias=p["delta_bias"], delta_softplus=sp)
    return float((np.asarray(y) * dy).sum())


def _grads(grad, p, dy, sp):
    return grad(p["u"], p["delta"], p["A"], p["B"], p["C"], dy, D=p["D"], z=p["z"],
                delta_bias=p["delta_bias"], delta_softplus=sp)


def _fd_dir(scan, p, dy, sp, name, v, eps=1e-6):
    hi = dict(p, **{name: p[name] + eps * v})
    lo = dict(p, **{name: p[name] - eps * v})
    return (_F(scan, hi, dy, sp) - _F(scan, lo, dy, sp)) / (2 * eps)


def pin_bwd_directional(grad, scan):
    """<gradient, v> against the central difference along a random v, for
    every input, softplus and exp modes, every optional operand on and off."""
    rng = np.random.default_rng(41)
    for case, (sp, wD, wz, wb) in enumerate([(True, True, True, True), (False, True, False, True),
                                             (True, False, True, False), (False, False, False, False)]):
        p = _problem(rng, 2, 3, 9, 4, wD, wz, wb)
        dy = rng.standard_normal((2, 3, 9))
        g = _grads(grad, p, dy, sp)
        for name, gname in NAMES:
            if p[name] is None:
                assert g[gname] is None, f"{gname} given for an absent operand"
                continue
            v = rng.standard_normal(p[name].shape)
            fd = _fd_dir(scan, p, dy, sp, name, v)
            an = float((g[gname] * v).sum())
            assert abs(fd - an) <= 1e-7 * (1.0 + abs(fd)), \
                f"case {case} d/d{name}: analytic {an!r} vs finite difference {fd!r}"


def pin_bwd_every_element(grad, scan):
    """Every element of every gradient of a tiny problem against its own
    central difference (unit directions)."""
    rng = np.random.default_rng(43)
    p = _problem(rng, 2, 2, 5, 3)
    dy = rng.standard_normal((2, 2, 5))
    for sp in (True, False):
        g = _grads(grad, p, dy, sp)
        for name, gname in NAMES:
            arr = p[name]
            for idx in np.ndindex(arr.shape):
                v = np.zeros_like(arr)
                v[idx] = 1.0
                fd = _fd_dir(scan, p, dy, sp, name, v)
                an = float(g[gname][idx])
                assert abs(fd - an) <= 1e-7 * (1.0 + abs(fd)), \
                    f"{gname}{idx} (softplus={sp}): analytic {an!r} vs finite difference {fd!r}"


def pin_bwd_softplus_linear_region(grad, scan):
    """delta + bias above torch's softplus threshold (20), where softplus is
    the identity and its derivative is 1."""
    rng = np.random.default_rng(47)
    p = _problem(rng, 1, 2, 6, 3, bias_shift=25.0)
    p["A"] = p["A"] * 0.01  # keep exp(delta' A) away from underflow
    dy = rng.standard_normal((1, 2, 6))
    g = _grads(grad, p, dy, True)
    for name, gname in [("delta", "ddelta"), ("delta_bias", "ddelta_bias")]:
        v = rng.standard_normal(p[name].shape)
        fd = _fd_dir(scan, p, dy, True, name, v)
        an = float((g[gname] * v).sum())
        assert abs(fd - an) <= 1e-7 * (1.0 + abs(fd)), f"d/d{name} above the threshold: {an!r} vs {fd!r}"


def pin_bwd_sequence_starts(grad, scan):
    """With sequence starts (the state entering a start is zero), every
    gradient against central differences of the forward with the same starts:
    directions for every input of a mid-sized problem, and every element of a
    tiny one (starts at step 0, inside, on consecutive steps and at the end)."""
    rng = np.random.default_rng(53)
    cases = [((2, 3, 12, 4), {0: [4, 5, 11], 1: [0, 7]}), ((2, 2, 6, 3), {0: [2], 1: [0, 3, 4]})]
    for k, ((Bt, Dm, L, N), starts) in enumerate(cases):
        p = _problem(rng, Bt, Dm, L, N)
        dy = rng.standard_normal((Bt, Dm, L))
        reset = np.zeros((Bt, L), dtype=np.uint8)
        for b, ls in starts.items():
            reset[b, ls] = 1

        def F(q):
            y = scan(q["u"], q["delta"], q["A"], q["B"], q["C"], D=q["D"], z=q["z"],
                     delta_bias=q["delta_bias"], delta_softplus=True, reset=reset)
            return float((np.asarray(y) * dy).sum())

        g = grad(p["u"], p["delta"], p["A"], p["B"], p["C"], dy, D=p["D"], z=p["z"],
                 delta_bias=p["delta_bias"], delta_softplus=True, reset=reset)
        for name, gname in NAMES:
            dirs = ([rng.standard_normal(p[name].shape)] if k == 0 else
                    [np.eye(p[name].size)[i].reshape(p[name].shape) for i in range(p[name].size)])
            for v in dirs:
                eps = 1e-6
                fd = (F(dict(p, **{name: p[name] + eps * v})) - F(dict(p, **{name: p[name] - eps * v}))) / (2 * eps)
                an = float((g[gname] * v).sum())
                assert abs(fd - an) <= 1e-7 * (1.0 + abs(fd)), \
                    f"starts case {k} d/d{name}: analytic {an!r} vs finite difference {fd!r}"


def pin_bwd_initial_state(grad, scan):
    """From a given state before step 0: the gradient with respect to that
    state, and every other gradient, against central differences of the
    forward from the same state; every element of a tiny problem, directions
    for a mid-sized one, with and without sequence starts (a start at step 0
    cuts the given state off: its gradient is zero there)."""
    rng = np.random.default_rng(59)
    cases = [((2, 3, 10, 4), None), ((2, 2, 5, 3), None), ((2, 2, 6, 3), {0: [0, 3], 1: [2]})]
    for k, ((Bt, Dm, L, N), starts) in enumerate(cases):
        p = _problem(rng, Bt, Dm, L, N)
        p["h0"] = rng.standard_normal((Bt, Dm, N))
        dy = rng.standard_normal((Bt, Dm, L))
        reset = None
        if starts is not None:
            reset = np.zeros((Bt, L), dtype=np.uint8)
            for b, ls in starts.items():
                reset[b, ls] = 1

        def F(q):
            y = scan(q["u"], q["delta"], q["A"], q["B"], q["C"], D=q["D"], z=q["z"],
                     delta_bias=q["delta_bias"], delta_softplus=True, initial_state=q["h0"], reset=reset)
            return float((np.asarray(y) * dy).sum())

        g = grad(p["u"], p["delta"], p["A"], p["B"], p["C"], dy, D=p["D"], z=p["z"],
                 delta_bias=p["delta_bias"], delta_softplus=True, reset=reset, initial_state=p["h0"])
        for name, gname in NAMES + [("h0", "dinitial_state")]:
            dirs = ([rng.standard_normal(p[name].shape)] if k == 0 else
                    [np.eye(p[name].size)[i].reshape(p[name].shape) for i in range(p[name].size)])
            for v in dirs:
                eps = 1e-6
                fd = (F(dict(p, **{name: p[name] + eps * v})) - F(dict(p, **{name: p[name] - eps * v}))) / (2 * eps)
                an = float((g[gname] * v).sum())
                assert abs(fd - an) <= 1e-7 * (1.0 + abs(fd)), \
                    f"initial-state case {k} d/d{name}: analytic {an!r} vs finite difference {fd!r}"
        if starts is not None:
            assert not g["dinitial_state"][0].any(), "a start at step 0 must cut the given state off"


def pin_bwd_term_magnitudes(grad, scan):
    """The sums of |terms| that scale the tolerance of the summed gradients,
    each term taken with the state and the adjoint replaced by the
    magnitudes of their own recursions: with one row and one step (no
    initial state) neither has a recursion, so every sum over rows and steps
    has one term and equals the gradient's absolute value, except
    ddelta_bias, whose one step still sums over the states (|g C_n B_n u|
    sigmoid(x) summed over n); in general each is at least |gradient|; the
    sums over channels of dB and dC are the single-channel problems' sums
    added up (each channel adds its own terms); and where the adjoint
    cancels (two steps, lam_0 = g_0 C_0 + a_1 g_1 C_1 close to zero) the
    dB term is the closed form (|g_0 C_0| + a_1 |g_1 C_1|) |d_0 u_0|, far
    above |dB|."""
    rng = np.random.default_rng(61)
    p = _problem(rng, 1, 1, 1, 3)
    dy = rng.standard_normal((1, 1, 1))
    g = grad(p["u"], p["delta"], p["A"], p["B"], p["C"], dy, D=p["D"], z=p["z"],
             delta_bias=p["delta_bias"], delta_softplus=True, magnitudes=True)
    for k in ("dA", "dB", "dC", "dD"):  # (the products are associated differently: to rounding)
        assert np.allclose(g["mag_" + k], np.abs(g[k]), rtol=1e-14, atol=0), f"one term: mag_{k} != |{k}|"
    x = p["delta"][0, 0, 0] + p["delta_bias"][0]
    sig = lambda v: 1.0 / (1.0 + np.exp(-v))  # noqa: E731
    gg = dy[0, 0, 0] * p["z"][0, 0, 0] * sig(p["z"][0, 0, 0])
    want = sum(abs(gg * p["C"][0, n, 0] * p["B"][0, n, 0] * p["u"][0, 0, 0]) for n in range(3)) * sig(x)
    assert np.isclose(g["mag_ddelta_bias"][0], want, rtol=1e-12, atol=0), "one step: mag_ddelta_bias"
    p = _problem(rng, 2, 4, 9, 3)
    dy = rng.standard_normal((2, 4, 9))
    g = grad(p["u"], p["delta"], p["A"], p["B"], p["C"], dy, D=p["D"], z=p["z"],
             delta_bias=p["delta_bias"], delta_softplus=True, magnitudes=True)
    for k in ("dA", "dB", "dC", "dD", "ddelta_bias"):
        assert (g["mag_" + k] >= np.abs(g[k]) * (1 - 1e-12)).all(), f"mag_{k} below |{k}|"
    for k in ("dB", "dC"):
        acc = np.zeros_like(g[k])
        for d in range(4):
            q = {n: (None if v is None else (v[:, d:d + 1] if v.ndim == 3 and v.shape[1] == 4 and n not in ("B", "C")
                                             else v[d:d + 1] if n in ("A", "D", "delta_bias") else v))
                 for n, v in p.items()}
            gd = grad(q["u"], q["delta"], q["A"], q["B"], q["C"], dy[:, d:d + 1], D=q["D"], z=q["z"],
                      delta_bias=q["delta_bias"], delta_softplus=True, magnitudes=True)
            acc += gd["mag_" + k]
        assert np.allclose(g["mag_" + k], acc, rtol=1e-12, atol=0), f"mag_{k} != sum over channels"
    # cancelling adjoint: one channel, one state, two steps, no gate or skip
    u = np.array([[[0.7, -1.3]]]); delta = np.array([[[0.4, -0.2]]]); A = np.array([[-0.9]])
    B = np.array([[[1.1, 0.6]]]); C1 = 0.8
    sp = lambda v: np.log1p(np.exp(v))  # noqa: E731
    a1 = np.exp(sp(delta[0, 0, 1]) * A[0, 0])
    dy = np.array([[[1.0, 0.5]]])
    C0 = -a1 * dy[0, 0, 1] * C1 / dy[0, 0, 0] * (1 + 1e-6)   # g_0 C_0 = -a_1 g_1 C_1 (1 + 1e-6)
    C = np.array([[[C0, C1]]])
    g = grad(u, delta, A, B, C, dy, delta_softplus=True, magnitudes=True)
    want = (abs(dy[0, 0, 0] * C0) + a1 * abs(dy[0, 0, 1] * C1)) * abs(sp(delta[0, 0, 0]) * u[0, 0, 0])
    assert np.isclose(g["mag_dB"][0, 0, 0], want, rtol=1e-12, atol=0), "cancelling adjoint: mag_dB"
    assert g["mag_dB"][0, 0, 0] > 1e5 * abs(g["dB"][0, 0, 0]), "cancelling adjoint: mag_dB must stay large"


def pin_bwd_last_state_gradient(grad, scan):
    """A gradient on the last state (the loss sum(dy * y) + sum(dlast * h_L),
    as when the state feeds the next piece of a sequence): every gradient,
    with and without an initial state and starts, against central differences
    of that loss; and a piece's gradient wrt its initial state fed back as the
    previous piece's dlast reproduces the whole sequence's gradients."""
    rng = np.random.default_rng(67)
    for k, (Bt, Dm, L, N, with_h0, starts) in enumerate([(2, 2, 7, 3, False, None), (2, 2, 6, 3, True, {0: [2], 1: [0]})]):
        p = _problem(rng, Bt, Dm, L, N)
        p["h0"] = rng.standard_normal((Bt, Dm, N)) if with_h0 else None
        dy = rng.standard_normal((Bt, Dm, L))
        dlast = rng.standard_normal((Bt, Dm, N))
        reset = None
        if starts is not None:
            reset = np.zeros((Bt, L), dtype=np.uint8)
            for b, ls in starts.items():
                reset[b, ls] = 1

        def F(q):
            y, last = scan(q["u"], q["delta"], q["A"], q["B"], q["C"], D=q["D"], z=q["z"], delta_bias=q["delta_bias"],
                           delta_softplus=True, initial_state=q["h0"], reset=reset, return_last_state=True)
            return float((np.asarray(y) * dy).sum() + (np.asarray(last) * dlast).sum())

        g = grad(p["u"], p["delta"], p["A"], p["B"], p["C"], dy, D=p["D"], z=p["z"], delta_bias=p["delta_bias"],
                 delta_softplus=True, reset=reset, initial_state=p["h0"], dlast_state=dlast)
        names = NAMES + ([("h0", "dinitial_state")] if with_h0 else [])
        for name, gname in names:
            for i in range(p[name].size):
                v = np.eye(p[name].size)[i].reshape(p[name].shape)
                eps = 1e-6
                fd = (F(dict(p, **{name: p[name] + eps * v})) - F(dict(p, **{name: p[name] - eps * v}))) / (2 * eps)
                an = float((g[gname] * v).sum())
                assert abs(fd - an) <= 1e-7 * (1.0 + abs(fd)), \
                    f"dlast case {k} d/d{name}: analytic {an!r} vs finite difference {fd!r}"
    # two pieces: [0, 5) then [5, 11), the second starting from the first's last state
    p = _problem(rng, 2, 3, 11, 4)
    dy = rng.standard_normal((2, 3, 11))
    whole = grad(p["u"], p["delta"], p["A"], p["B"], p["C"], dy, D=p["D"], z=p["z"], delta_bias=p["delta_bias"],
                 delta_softplus=True)
    cut = 5
    sl = lambda t, a, b: t[..., a:b]  # noqa: E731
    _, h1 = scan(sl(p["u"], 0, cut), sl(p["delta"], 0, cut), p["A"], sl(p["B"], 0, cut), sl(p["C"], 0, cut), D=p["D"],
                 z=sl(p["z"], 0, cut), delta_bias=p["delta_bias"], delta_softplus=True, return_last_state=True)
    g2 = grad(sl(p["u"], cut, 11), sl(p["delta"], cut, 11), p["A"], sl(p["B"], cut, 11), sl(p["C"], cut, 11),
              sl(dy, cut, 11), D=p["D"], z=sl(p["z"], cut, 11), delta_bias=p["delta_bias"], delta_softplus=True,
              initial_state=h1)
    g1 = grad(sl(p["u"], 0, cut), sl(p["delta"], 0, cut), p["A"], sl(p["B"], 0, cut), sl(p["C"], 0, cut),
              sl(dy, 0, cut), D=p["D"], z=sl(p["z"], 0, cut), delta_bias=p["delta_bias"], delta_softplus=True,
              dlast_state=g2["dinitial_state"])
    for k in ("du", "ddelta", "dz", "dB", "dC"):
        assert np.allclose(np.concatenate([g1[k], g2[k]], axis=-1), whole[k], rtol=1e-12, atol=1e-13), f"pieces: {k}"
    for k in ("dA", "dD", "ddelta_bias"):
        assert np.allclose(g1[k] + g2[k], whole[k], rtol=1e-12, atol=1e-13), f"pieces: {k}"


ALL_PINS = [pin_bwd_directional, pin_bwd_every_element, pin_bwd_softplus_linear_region,
            pin_bwd_sequence_starts, pin_bwd_initial_state, pin_bwd_term_magnitudes,
            pin_bwd_last_state_gradient]
