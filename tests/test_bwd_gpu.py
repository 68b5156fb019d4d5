"""Backward (ss_bwd) through the C ABI against the fp64 backward oracle,
which finite differences of the pinned forward oracle pin.

Tolerances (the pages state none for gradients; derived from the arithmetic):
  per-element gradients du, ddelta, dz:  |err| <= tol (1 + |ref|), tol 1e-4
    for fp32 inputs, 2e-2 for bf16 (outputs rounded to bf16, 2^-9, plus the
    SFU forms of exp, softplus and sigmoid);
  sums over rows and steps dA, dB, dC, dD, ddelta_bias, element by element:
    |err| <= tol (S + 1e-6 max S), S = the sum of the absolute values of that
    element's terms (from the oracle), tol 1e-4 for fp32 inputs, 1e-3 for
    bf16: each term carries a relative error of the order of the fp32 and
    SFU rounding of its factors, and the fp32 sum adds rounding of the order
    of eps times the partial sums, both bounded by a multiple of S.  The state
    and the adjoint inside a term are sums built by their recursions, whose
    terms can cancel, so S takes them at the magnitudes of those recursions
    (the sums of their own terms' absolute values).  The floor 1e-6 max S only
    matters for elements whose terms all vanish.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import to_dev
from selective_state_space_41_b200 import gen, selscan, workloads as W

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DY_STREAM = 9
ELEM = {"du", "ddelta", "dz"}
TOL_ELEM = {torch.float32: 1e-4, torch.bfloat16: 2e-2}
TOL_SUM = {torch.float32: 1e-4, torch.bfloat16: 1e-3}


def check_summed(k, g, want, mag, tol, what):
    """Element by element: |g - want| <= tol (mag + 1e-6 max mag)."""
    bound = tol * (mag + 1e-6 * float(np.max(mag)))
    err = np.abs(g - want)
    worst = int(np.argmax(err - bound))
    assert (err <= bound).all(), (f"{what}: {k} element {np.unravel_index(worst, err.shape)}: |err| "
                                  f"{err.flat[worst]:.3e} > {bound.flat[worst]:.3e} "
                                  f"(ref {want.flat[worst]:.4e}, sum |terms| {mag.flat[worst]:.3e})")


def _case(batch, dim, L, N, dtype, seed, out_dtype=None, **kw):
    w = W.custom("bwd", batch, dim, L, N, dtype, seed, **kw)
    inp = W.make_inputs(w)
    inp["dy"] = gen.fill((batch, dim, L), out_dtype or dtype, seed, DY_STREAM)
    return inp


def _check(inp, dtype, what, reset=None):
    d = to_dev(inp)
    got = selscan.selective_scan_bwd(d["u"], d["delta"], d["A"], d["B"], d["C"], d["dy"], D=d.get("D"),
                                     z=d.get("z"), delta_bias=d.get("delta_bias"),
                                     delta_softplus=inp["delta_softplus"],
                                     reset=None if reset is None else torch.as_tensor(reset).cuda())
    torch.cuda.synchronize()
    ref = oracle.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["dy"],
                                    D=inp.get("D"), z=inp.get("z"), delta_bias=inp.get("delta_bias"),
                                    delta_softplus=inp["delta_softplus"], reset=reset, magnitudes=True)
    for k, want in ref.items():
        if k.startswith("mag_"):
            continue
        if want is None:
            assert got[k] is None
            continue
        g = got[k].detach().to("cpu", torch.float64).numpy()
        assert np.isfinite(g).all(), f"{what}: {k} not finite"
        if want.size == 0:
            continue
        if k in ELEM:
            e = float(np.max(np.abs(g - want) / (1.0 + np.abs(want))))
            assert e <= TOL_ELEM[dtype], f"{what}: {k} max |err|/(1+|ref|) = {e:.3e}"
        else:
            check_summed(k, g, want, ref["mag_" + k], TOL_SUM[dtype], what)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("N", [4, 8, 9, 16, 32, 33, 64])
def test_bwd_state_sizes(dtype, N):
    """Every state bucket, ragged length (partial stage and sub-chunk) and
    channels (mirrored rows in the last tile), every operand present."""
    _check(_case(2, 45, 203, N, dtype, seed=N + 100, has_z=True, return_last_state=False), dtype, f"N={N}")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("has_z,D_kind,bias_kind,softplus",
                         [(False, "none", "none", True), (True, "ones", "zeros", False),
                          (False, "normal", "uniform_dt", True), (True, "none", "normal", False)])
def test_bwd_optional_operands(dtype, has_z, D_kind, bias_kind, softplus):
    inp = _case(3, 33, 130, 16, dtype, seed=7, has_z=has_z, D_kind=D_kind, bias_kind=bias_kind,
                delta_softplus=softplus)
    _check(inp, dtype, f"z={has_z} D={D_kind} bias={bias_kind} softplus={softplus}")


def test_bwd_bf16_in_f32_dy():
    _check(_case(2, 40, 150, 16, torch.bfloat16, seed=11, out_dtype=torch.float32, has_z=True),
           torch.bfloat16, "bf16 in, f32 dy")


@pytest.mark.parametrize("L", [1, 7, 8, 64, 65])
def test_bwd_short_sequences(L):
    _check(_case(2, 20, L, 16, torch.float32, seed=L, has_z=True), torch.float32, f"L={L}")


def test_bwd_mamba130m_one_batch():
    """One batch entry of the mamba-130m-shaped layer (1536 channels x 2048 steps)."""
    w = W.with_shape(W.WORKLOADS[W.MAMBA130M], batch=1)
    inp = W.make_inputs(w)
    inp["dy"] = gen.fill((1, w.dim, w.seqlen), w.dtype, w.seed, DY_STREAM)
    _check(inp, w.dtype, "mamba130m batch 1")


def test_bwd_deterministic():
    inp = _case(2, 64, 300, 16, torch.bfloat16, seed=5, has_z=True)
    d = to_dev(inp)
    args = (d["u"], d["delta"], d["A"], d["B"], d["C"], d["dy"])
    kw = dict(D=d["D"], z=d["z"], delta_bias=d["delta_bias"], delta_softplus=True)
    g1 = selscan.selective_scan_bwd(*args, **kw)
    g2 = selscan.selective_scan_bwd(*args, **kw)
    torch.cuda.synchronize()
    for k in g1:
        assert torch.equal(g1[k], g2[k]), k


def test_bwd_wide_state_layer_rows():
    """64 states (16 lanes per row, one lane in two owning a step), bf16,
    a few rows of the wide-state layer shape."""
    w = W.with_shape(W.WORKLOADS["wide_state_b16_d4096_l8192_n64"], batch=1, dim=48, seqlen=1000)
    inp = W.make_inputs(w)
    inp["dy"] = gen.fill((1, 48, 1000), w.dtype, w.seed, DY_STREAM)
    _check(inp, w.dtype, "wide state N=64")


def test_bwd_softplus_linear_region():
    """delta + bias above torch's softplus threshold (20) on most steps: the
    derivative there is 1, below it sigmoid (both paths of the kernel)."""
    inp = _case(2, 24, 150, 16, torch.float32, seed=23, has_z=True)
    inp["delta_bias"] = torch.full((24,), 20.0)          # delta ~ N(0, 1): both sides of 20
    inp["A"] = (inp["A"] * 0.01).contiguous()            # keep exp(delta' A) away from underflow
    _check(inp, torch.float32, "softplus threshold")


# ---------------------------------------------------------------- sequence starts
# (ss_bwd_reset: the backward of a forward whose state is zeroed entering each
# start of the (batch, L) mask; the oracle's reset form is pinned by finite
# differences of the forward with the same starts.)

def _starts(batch, L, seed, fixed=(), p=0.0):
    m = np.zeros((batch, L), dtype=np.uint8)
    for l in fixed:
        if 0 <= l < L:
            m[:, l] = 1
    if p > 0:
        r = gen.fill((batch, L), torch.float32, seed, DY_STREAM + 1, gen.UNIFORM, 0.0, 1.0).numpy()
        m |= (r < p).astype(np.uint8)
    return m


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("N", [4, 16, 33, 64])
def test_bwd_starts_state_sizes(dtype, N):
    """Every state bucket; 203 steps (flags read byte by byte), starts at
    step 0, on and beside sub-chunk (8) and stage (64) boundaries, at the last
    step, and seeded ones; batch entries with different starts."""
    inp = _case(2, 45, 203, N, dtype, seed=N + 300, has_z=True, return_last_state=False)
    reset = _starts(2, 203, seed=N, fixed=(7, 8, 9, 63, 64, 100, 202), p=0.02)
    reset[0, 0] = 1
    _check(inp, dtype, f"starts N={N}", reset=reset)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_bwd_starts_aligned_rows(dtype):
    """256 steps (flags read as 8-byte words), starts every 32 steps plus
    seeded ones, every optional operand."""
    inp = _case(3, 40, 256, 16, dtype, seed=17, has_z=True, bias_kind="uniform_dt")
    _check(inp, dtype, "starts, aligned rows", reset=_starts(3, 256, seed=17, fixed=range(0, 256, 32), p=0.03))


def test_bwd_start_every_step():
    inp = _case(2, 20, 65, 16, torch.float32, seed=19, has_z=True)
    _check(inp, torch.float32, "a start at every step", reset=np.ones((2, 65), np.uint8))


def test_bwd_all_zero_starts_bitwise_plain():
    """The reset instance with no start set does the plain instance's arithmetic."""
    inp = _case(2, 40, 256, 16, torch.bfloat16, seed=23, has_z=True)
    d = to_dev(inp)
    args = (d["u"], d["delta"], d["A"], d["B"], d["C"], d["dy"])
    kw = dict(D=d.get("D"), z=d.get("z"), delta_bias=d.get("delta_bias"), delta_softplus=True)
    g0 = selscan.selective_scan_bwd(*args, **kw)
    g1 = selscan.selective_scan_bwd(*args, reset=torch.zeros(2, 256, dtype=torch.uint8, device="cuda"), **kw)
    torch.cuda.synchronize()
    for k, v in g0.items():
        assert (v is None and g1[k] is None) or torch.equal(v, g1[k]), k


def test_bwd_starts_mamba130m_one_batch():
    """One batch entry of the mamba-130m-shaped layer cut into 512-step sequences."""
    w = W.with_shape(W.WORKLOADS[W.MAMBA130M], batch=1)
    inp = W.make_inputs(w)
    inp["dy"] = gen.fill((1, w.dim, w.seqlen), torch.bfloat16, 77, DY_STREAM)
    _check(inp, torch.bfloat16, "starts, mamba-130m-shaped batch entry",
           reset=_starts(1, w.seqlen, seed=77, fixed=range(0, w.seqlen, 512), p=0.002))


# ---------------------------------------------------------------- initial state
# (ss_bwd_state: the backward of ss_fwd_state's forward from a given state,
# with an optional gradient on the last state, returning the gradient with
# respect to the initial state; the oracle's form is pinned by finite
# differences in tests/pins_bwd.py.)

def _check_state(inp, dtype, what, reset=None, with_h0=True, with_dlast=True, seed=0):
    batch, dim, L = inp["u"].shape
    N = inp["A"].shape[1]
    g = torch.Generator().manual_seed(seed)
    h0 = torch.randn((batch, dim, N), generator=g) if with_h0 else None
    dlast = torch.randn((batch, dim, N), generator=g) if with_dlast else None
    d = to_dev(inp)
    got = selscan.selective_scan_bwd(d["u"], d["delta"], d["A"], d["B"], d["C"], d["dy"], D=d.get("D"),
                                     z=d.get("z"), delta_bias=d.get("delta_bias"),
                                     delta_softplus=inp["delta_softplus"],
                                     reset=None if reset is None else torch.as_tensor(reset).cuda(),
                                     initial_state=None if h0 is None else h0.cuda(),
                                     d_last_state=None if dlast is None else dlast.cuda())
    torch.cuda.synchronize()
    ref = oracle.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["dy"],
                                    D=inp.get("D"), z=inp.get("z"), delta_bias=inp.get("delta_bias"),
                                    delta_softplus=inp["delta_softplus"], reset=reset, magnitudes=True,
                                    initial_state=h0 if h0 is not None else torch.zeros((batch, dim, N)),
                                    dlast_state=dlast)
    for k, want in ref.items():
        if k.startswith("mag_") or want is None:
            continue
        if k == "dinitial_state" and h0 is None and dlast is None:
            assert k not in got   # asked for only with a state or a last-state gradient
            continue
        gk = got[k].detach().to("cpu", torch.float64).numpy()
        assert np.isfinite(gk).all(), f"{what}: {k} not finite"
        if k in ELEM:
            e = float(np.max(np.abs(gk - want) / (1.0 + np.abs(want))))
            assert e <= TOL_ELEM[dtype], f"{what}: {k} max |err|/(1+|ref|) = {e:.3e}"
        elif k == "dinitial_state":
            # a sum over the row's steps of adjoint terms, each accurate to the
            # fp32/SFU rounding of its factors: per element against 1 + |ref|
            e = float(np.max(np.abs(gk - want) / (1.0 + np.abs(want))))
            assert e <= TOL_ELEM[dtype], f"{what}: dinitial_state max |err|/(1+|ref|) = {e:.3e}"
        else:
            check_summed(k, gk, want, ref["mag_" + k], TOL_SUM[dtype], what)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("N", [4, 16, 33, 64])
def test_bwd_initial_state(dtype, N):
    """From a given state with a last-state gradient: every bucket, ragged
    length and channels, every operand."""
    _check_state(_case(2, 45, 203, N, dtype, seed=N + 500, has_z=True), dtype, f"h0 N={N}", seed=N)


@pytest.mark.parametrize("with_h0,with_dlast", [(True, False), (False, True), (False, False)])
def test_bwd_initial_state_parts(with_h0, with_dlast):
    """Only the initial state, only the last-state gradient (the
    initial-state gradient of a zero start is returned), neither (plain
    ss_bwd)."""
    _check_state(_case(2, 33, 150, 16, torch.bfloat16, seed=31, has_z=True), torch.bfloat16,
                 f"h0={with_h0} dlast={with_dlast}", with_h0=with_h0, with_dlast=with_dlast, seed=3)


def test_bwd_initial_state_with_starts():
    """With sequence starts, one at step 0 in batch entry 0 (its initial
    state is cut off: zero gradient there)."""
    reset = _starts(2, 203, seed=41, fixed=(7, 64, 100), p=0.02)
    reset[0, 0] = 1
    _check_state(_case(2, 40, 203, 16, torch.float32, seed=41, has_z=True), torch.float32, "h0 + starts",
                 reset=reset, seed=41)


def test_bwd_initial_state_empty_sequence():
    """L = 0: the initial-state gradient is the last-state gradient."""
    inp = _case(2, 5, 0, 16, torch.float32, seed=1)
    d = to_dev(inp)
    dlast = torch.randn((2, 5, 16), device="cuda")
    got = selscan.selective_scan_bwd(d["u"], d["delta"], d["A"], d["B"], d["C"], d["dy"], D=d["D"],
                                     delta_bias=d["delta_bias"], delta_softplus=True,
                                     initial_state=torch.zeros_like(dlast), d_last_state=dlast)
    torch.cuda.synchronize()
    assert torch.equal(got["dinitial_state"], dlast)


def test_bwd_in_pieces_equals_whole():
    """A 1000-step sequence trained in two pieces (cut at a stage boundary,
    640): forward piece 1 from h0, piece 2 from piece 1's last state; backward
    of piece 2 from that state, then of piece 1 with piece 2's initial-state
    gradient as its last-state gradient.  The per-step gradients agree with
    the whole sequence's: per-step gradients to bf16 output rounding, the
    state-carried and summed ones to fp32 rounding of the split sums."""
    inp = _case(2, 48, 1000, 16, torch.bfloat16, seed=57, has_z=True)
    d = to_dev(inp)
    h0 = torch.randn((2, 48, 16), device="cuda")
    kw = dict(D=d["D"], z=None, delta_bias=d["delta_bias"], delta_softplus=True)
    whole = selscan.selective_scan_bwd(d["u"], d["delta"], d["A"], d["B"], d["C"], d["dy"], initial_state=h0,
                                       **dict(kw, z=d["z"]))
    cut = 640
    sl = lambda t, a, b: t[..., a:b].contiguous()  # noqa: E731
    y1 = torch.empty_like(sl(d["u"], 0, cut))
    h1 = torch.empty_like(h0)
    selscan.ss_fwd(sl(d["u"], 0, cut), sl(d["delta"], 0, cut), d["A"], sl(d["B"], 0, cut), sl(d["C"], 0, cut), y1,
                   z=sl(d["z"], 0, cut), last_state=h1, initial_state=h0, lanes_per_row=4, split_states=1,
                   warps_per_block=4, segments=1, **{k: v for k, v in kw.items() if k != "z"})
    g2 = selscan.selective_scan_bwd(sl(d["u"], cut, 1000), sl(d["delta"], cut, 1000), d["A"], sl(d["B"], cut, 1000),
                                    sl(d["C"], cut, 1000), sl(d["dy"], cut, 1000), initial_state=h1,
                                    **dict(kw, z=sl(d["z"], cut, 1000)))
    g1 = selscan.selective_scan_bwd(sl(d["u"], 0, cut), sl(d["delta"], 0, cut), d["A"], sl(d["B"], 0, cut),
                                    sl(d["C"], 0, cut), sl(d["dy"], 0, cut), initial_state=h0,
                                    d_last_state=g2["dinitial_state"], **dict(kw, z=sl(d["z"], 0, cut)))
    torch.cuda.synchronize()
    for k in ("du", "ddelta", "dz"):
        joined = torch.cat([g1[k], g2[k]], dim=-1).double()
        e = float(((joined - whole[k].double()).abs() / (1 + whole[k].double().abs())).max())
        assert e <= 1e-2, f"pieces: {k} {e:.3e}"
    for k in ("dB", "dC"):
        joined = torch.cat([g1[k], g2[k]], dim=-1)
        assert torch.allclose(joined, whole[k], rtol=1e-4, atol=1e-5 * float(whole[k].abs().max())), k
    assert torch.allclose(g1["dinitial_state"], whole["dinitial_state"], rtol=1e-4, atol=1e-5)
    for k in ("dA", "dD", "ddelta_bias"):
        assert torch.allclose(g1[k] + g2[k], whole[k], rtol=1e-4, atol=1e-5 * float(whole[k].abs().max())), k
