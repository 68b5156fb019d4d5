"""Initial state (ss_fwd_state) through the C ABI against the fp64 oracle:
every launch shape, sequence segments, a sequence run in pieces with the
state updated in place, and single-step decoding.

The walkthrough's state starts at zero; the initial state is an extension
(see the oracle), pinned there by a closed form, an unrolled sum and the
equality of a piecewise run with a single run."""
import pytest
import torch

import oracle
from gpu_util import TOL, assert_parity, to_dev
from selective_state_space_41_b200 import gen, selscan, workloads as W

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

STATE_STREAM = 8  # Philox stream of the initial state (the operands use 1..7)


def _case(batch, dim, L, N, dtype, seed, **kw):
    inp = W.make_inputs(W.custom("state", batch, dim, L, N, dtype, seed, **kw))
    inp["initial_state"] = gen.fill((batch, dim, N), torch.float32, seed, STATE_STREAM, gen.NORMAL, 0.0, 2.0)
    return inp


def _oracle(inp, h0=None, sl=slice(None)):
    cut = lambda t: None if t is None else t[..., sl]  # noqa: E731
    return oracle.selective_scan(cut(inp["u"]), cut(inp["delta"]), inp["A"], cut(inp["B"]), cut(inp["C"]),
                                 D=inp.get("D"), z=cut(inp.get("z")), delta_bias=inp.get("delta_bias"),
                                 delta_softplus=inp["delta_softplus"], return_last_state=True,
                                 initial_state=inp["initial_state"] if h0 is None else h0)


def _run(d, out_dtype, state, sl=slice(None), last=None, **cfg):
    """libselscan from `state` over steps `sl` of the device inputs `d`."""
    cut = lambda t: None if t is None else t[..., sl].contiguous()  # noqa: E731
    u = cut(d["u"])
    batch, dim, L = u.shape
    N = d["A"].shape[1]
    y = torch.empty((batch, dim, L), dtype=out_dtype, device="cuda")
    if last is None:
        last = torch.empty((batch, dim, N), dtype=torch.float32, device="cuda")
    ws = selscan.workspace_for(batch, dim, L, N, u.dtype, out_dtype, **cfg) if L else None
    selscan.ss_fwd(u, cut(d["delta"]), d["A"], cut(d["B"]), cut(d["C"]), y, D=d.get("D"), z=cut(d.get("z")),
                   delta_bias=d.get("delta_bias"), delta_softplus=d["delta_softplus"], last_state=last,
                   workspace=ws, initial_state=state, **cfg)
    return y, last


SHAPES = ([dict(lanes_per_row=w) for w in (1, 2, 4, 8, 16, 32)] +
          [dict(lanes_per_row=g, split_states=True) for g in (2, 4, 8)] +
          [dict(lanes_per_row=2, split_states=True, segments=3), dict(lanes_per_row=1, segments=2)])


@pytest.mark.parametrize("cfg", SHAPES, ids=lambda c: "-".join(f"{k}{v}" for k, v in c.items()))
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_initial_state_every_shape(cfg, dtype):
    inp = _case(2, 37, 517 if "segments" not in cfg else 4100, 16, dtype, seed=5, has_z=True)
    d = to_dev(inp)
    y, last = _run(d, dtype, d["initial_state"], warps_per_block=4, **cfg)
    torch.cuda.synchronize()
    y_ref, last_ref = _oracle(inp)
    assert_parity(y, last, y_ref, last_ref, TOL[dtype], f"initial state {cfg}")


def test_pieces_in_place_equal_one_run():
    """A sequence in three pieces (one of a single step), the state updated
    in place between them: equal to the oracle, and bitwise equal to one run
    of the same launch shape (the state passes through float32 memory
    exactly, and the shape has no segments)."""
    inp = _case(2, 64, 1000, 16, torch.bfloat16, seed=9, has_z=True, bias_kind="uniform_dt")
    d = to_dev(inp)
    cfg = dict(lanes_per_row=4, split_states=True, warps_per_block=4, segments=1)
    y_one, last_one = _run(d, torch.bfloat16, d["initial_state"], **cfg)
    state = d["initial_state"].clone()
    ys = []
    for sl in (slice(0, 300), slice(300, 301), slice(301, 1000)):
        y, _ = _run(d, torch.bfloat16, state, sl, last=state, **cfg)   # in place
        ys.append(y)
    torch.cuda.synchronize()
    y_pieces = torch.cat(ys, dim=-1)
    assert torch.equal(y_pieces, y_one)
    assert torch.equal(state, last_one)
    y_ref, last_ref = _oracle(inp)
    assert_parity(y_pieces, state, y_ref, last_ref, TOL[torch.bfloat16], "pieces")


def test_single_step_decode():
    """Recurrent decoding: 24 calls of one step each (L = 1), state in place,
    heuristic launch shape, against the oracle's 24-step run."""
    inp = _case(3, 80, 24, 16, torch.float32, seed=13, has_z=True, bias_kind="uniform_dt")
    d = to_dev(inp)
    state = d["initial_state"].clone()
    ys = []
    for t in range(24):
        y, _ = _run(d, torch.float32, state, slice(t, t + 1), last=state)
        ys.append(y)
    torch.cuda.synchronize()
    y_ref, last_ref = _oracle(inp)
    assert_parity(torch.cat(ys, dim=-1), state, y_ref, last_ref, TOL[torch.float32], "decode")


def test_empty_sequence_returns_initial_state():
    inp = _case(2, 3, 0, 5, torch.float32, seed=3)
    d = to_dev(inp)
    y, last = _run(d, torch.float32, d["initial_state"])
    torch.cuda.synchronize()
    assert torch.equal(last, d["initial_state"])


def test_initial_state_zero_equals_no_state():
    inp = _case(2, 40, 300, 16, torch.bfloat16, seed=17, has_z=True)
    d = to_dev(inp)
    y0, l0 = _run(d, torch.bfloat16, torch.zeros_like(d["initial_state"]))
    y1, l1 = _run(d, torch.bfloat16, None)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1) and torch.equal(l0, l1)


# ---------------------------------------------------------------- ss_step
def _step_loop(d, out_dtype, steps, state):
    ys = []
    for t in range(steps):
        col = lambda x: None if x is None else x[..., t].contiguous()  # noqa: E731
        y = torch.empty(d["u"].shape[:2], dtype=out_dtype, device="cuda")
        selscan.ss_step(col(d["u"]), col(d["delta"]), d["A"], col(d["B"]), col(d["C"]), state, y,
                        D=d.get("D"), z=col(d.get("z")), delta_bias=d.get("delta_bias"),
                        delta_softplus=d["delta_softplus"])
        ys.append(y)
    return torch.stack(ys, dim=-1)


@pytest.mark.parametrize("dtype,out_dtype", [(torch.float32, torch.float32), (torch.bfloat16, torch.bfloat16),
                                             (torch.bfloat16, torch.float32)])
@pytest.mark.parametrize("N", [4, 9, 16, 33, 64])
def test_step_decode_against_oracle(dtype, out_dtype, N):
    """ss_step (the decoding kernel) for 20 steps, state in place, against the
    oracle's 20-step run from the same initial state; ragged row count."""
    inp = _case(3, 37, 20, N, dtype, seed=N + 31, has_z=True, out_dtype=out_dtype)
    d = to_dev(inp)
    state = d["initial_state"].clone()
    y = _step_loop(d, out_dtype, 20, state)
    torch.cuda.synchronize()
    y_ref, last_ref = _oracle(inp)
    assert_parity(y, state, y_ref, last_ref, 1e-4 if out_dtype == torch.float32 and dtype == torch.bfloat16
                  else TOL[dtype], f"step N={N}")


@pytest.mark.parametrize("has_z,D_kind,bias_kind,softplus",
                         [(False, "none", "none", True), (True, "ones", "zeros", False)])
def test_step_optional_operands(has_z, D_kind, bias_kind, softplus):
    inp = _case(2, 50, 6, 16, torch.float32, seed=3, has_z=has_z, D_kind=D_kind, bias_kind=bias_kind,
                delta_softplus=softplus)
    d = to_dev(inp)
    state = d["initial_state"].clone()
    y = _step_loop(d, torch.float32, 6, state)
    torch.cuda.synchronize()
    y_ref, last_ref = _oracle(inp)
    assert_parity(y, state, y_ref, last_ref, TOL[torch.float32], "step operands")


def test_step_matches_forward_from_state():
    """One ss_step equals ss_fwd_state with L = 1 up to float32 summation order."""
    inp = _case(4, 64, 1, 16, torch.bfloat16, seed=41, has_z=True, out_dtype=torch.float32)
    d = to_dev(inp)
    s1 = d["initial_state"].clone()
    y1 = _step_loop(d, torch.float32, 1, s1)
    y2, s2 = _run(d, torch.float32, d["initial_state"])
    torch.cuda.synchronize()
    assert torch.allclose(y1, y2, rtol=1e-5, atol=1e-5)
    assert torch.allclose(s1, s2, rtol=1e-6, atol=1e-6)
