"""The forward that writes the backward's checkpoints (ss_fwd_ckpt) and the
backward that reads them (ss_bwd_ckpt), through the C ABI:

* y and the last state are those of the forward without checkpoints (bitwise
  in the same launch shape) and the oracle's;
* checkpoint k is the state after step 8k - 1: the oracle's last state of
  the first 8k steps (from the same initial state, with the same starts),
  element by element within 1e-4 (1 + |ref|) (an fp32 state against fp64);
  with sequence segments the fix-up's correction of segments >= 1 included;
* the backward from the checkpoints equals the backward with its own
  checkpointing pass bit for bit where neither cuts the sequence, and the
  oracle's gradients (tolerances of test_bwd_gpu.py) where both do.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from gpu_util import TOL, assert_parity, to_dev
from test_bwd_gpu import _case, _starts, ELEM, TOL_ELEM, TOL_SUM, check_summed
from selective_state_space_41_b200 import selscan

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

CK_TOL = 1e-4


def _fwd_ckpt(d, inp, h0=None, reset=None, workspace=True):
    batch, dim, L = d["u"].shape
    N = d["A"].shape[1]
    y = torch.full((batch, dim, L), float("nan"), dtype=d["u"].dtype, device="cuda")
    last = torch.full((batch, dim, N), float("nan"), device="cuda")
    ck = torch.full(selscan.ckpt_shape(batch, dim, L, N), float("nan"), device="cuda")
    ws = selscan.workspace_for(batch, dim, L, N, d["u"].dtype) if workspace else None
    selscan.ss_fwd_ckpt(d["u"], d["delta"], d["A"], d["B"], d["C"], y, ck, D=d.get("D"), z=d.get("z"),
                        delta_bias=d.get("delta_bias"), delta_softplus=inp["delta_softplus"], last_state=last,
                        initial_state=h0, reset=reset, workspace=ws)
    torch.cuda.synchronize()
    return y, last, ck


def _check_ckpts(inp, ck, ks, h0=None, reset=None, what=""):
    """Checkpoints ks against the oracle's state after 8k steps."""
    for k in ks:
        l = 8 * k
        if l == 0:
            want = np.zeros(ck.shape[:2] + (ck.shape[3],)) if h0 is None else h0.numpy().astype(np.float64)
        else:
            sl = lambda t: None if t is None else t[..., :l].contiguous()  # noqa: E731
            _, want = oracle.selective_scan(sl(inp["u"]), sl(inp["delta"]), inp["A"], sl(inp["B"]), sl(inp["C"]),
                                            D=inp.get("D"), z=sl(inp.get("z")), delta_bias=inp.get("delta_bias"),
                                            delta_softplus=inp["delta_softplus"], return_last_state=True,
                                            initial_state=h0, reset=None if reset is None else reset[:, :l])
        got = ck[:, :, k, :].to("cpu", torch.float64).numpy()
        e = float(np.max(np.abs(got - want) / (1.0 + np.abs(want))))
        assert e <= CK_TOL, f"{what}: checkpoint {k} max |err|/(1+|ref|) = {e:.3e}"


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("N", [4, 16, 33, 64])
def test_fwd_ckpt_values_and_outputs(dtype, N):
    """Every state bucket, ragged length (partial sub-chunk and stage) and
    channels; y and the last state as the plain forward's."""
    inp = _case(2, 45, 203, N, dtype, seed=N + 900, has_z=True, return_last_state=True)
    d = to_dev(inp)
    y, last, ck = _fwd_ckpt(d, inp)
    y_ref, last_ref = oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                                            z=inp["z"], delta_bias=inp["delta_bias"], delta_softplus=True,
                                            return_last_state=True)
    assert_parity(y, last, y_ref, last_ref, TOL[dtype], f"N={N}")
    assert torch.isfinite(ck).all()
    _check_ckpts(inp, ck, [0, 1, 7, 8, 15, 25], what=f"N={N}")


def test_fwd_ckpt_bitwise_equals_plain_forward():
    """One batch entry of the mamba-130m-shaped layer: the direct kernel with
    and without checkpoint stores gives the same bits (for so few rows the
    checkpointing forward takes the direct kernel's widest state split, 4
    lanes, where the plain forward would take the scan kernel, so the plain
    forward is given that launch shape)."""
    from selective_state_space_41_b200 import workloads as W
    w = W.with_shape(W.WORKLOADS[W.MAMBA130M], batch=1)
    inp = W.make_inputs(w)
    inp["return_last_state"] = True
    d = to_dev(inp)
    y, last, ck = _fwd_ckpt(d, inp, workspace=False)
    y2 = torch.empty_like(y)
    last2 = torch.empty_like(last)
    selscan.ss_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], y2, D=d["D"], z=d["z"], delta_bias=d["delta_bias"],
                   delta_softplus=True, last_state=last2, lanes_per_row=4, split_states=1, warps_per_block=4,
                   segments=1)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    assert torch.equal(last, last2)


def test_fwd_ckpt_initial_state_and_starts():
    """From a given state, with starts on and beside checkpoint steps: the
    checkpoint at a start holds the state before it is zeroed."""
    inp = _case(2, 24, 300, 16, torch.float32, seed=911, has_z=True, return_last_state=True)
    reset = _starts(2, 300, seed=911, fixed=(7, 8, 16, 100, 299), p=0.01)
    h0 = torch.randn((2, 24, 16), generator=torch.Generator().manual_seed(911))
    d = to_dev(inp)
    y, last, ck = _fwd_ckpt(d, inp, h0=h0.cuda(), reset=torch.as_tensor(reset).cuda())
    y_ref, last_ref = oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                                            z=inp["z"], delta_bias=inp["delta_bias"], delta_softplus=True,
                                            return_last_state=True, initial_state=h0, reset=reset)
    assert_parity(y, last, y_ref, last_ref, TOL[torch.float32], "h0 + starts")
    _check_ckpts(inp, ck, [0, 1, 2, 12, 13, 37], h0=h0, reset=reset, what="h0 + starts")


@pytest.mark.parametrize("softplus", [True, False])
def test_fwd_ckpt_segments(softplus):
    """Few rows and 9000 steps with a workspace (sequence segments): the
    fix-up completes the checkpoints of segments >= 1 (long memory, so the
    carried state reaches far into each segment)."""
    inp = _case(1, 8, 9000, 16, torch.float32, seed=913, has_z=True, return_last_state=True,
                delta_softplus=softplus)
    if softplus:
        inp["delta_bias"] = torch.full((8,), -6.0)
    else:
        inp["delta"] = (inp["delta"] * 0.5 - 7.0).contiguous()
    assert selscan.ss_fwd_heuristic(1, 8, 9000, 16, torch.float32, workspace_bytes=1 << 30)["segments"] > 1
    d = to_dev(inp)
    y, last, ck = _fwd_ckpt(d, inp)
    y_ref, last_ref = oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                                            z=inp["z"], delta_bias=inp["delta_bias"], delta_softplus=softplus,
                                            return_last_state=True)
    assert_parity(y, last, y_ref, last_ref, TOL[torch.float32], "segments")
    # a spread of checkpoints over every segment (long memory: the carried
    # state's share reaches through whole segments) and the last one
    ks = list(range(0, ck.shape[2], 37)) + [ck.shape[2] - 1]
    _check_ckpts(inp, ck, [k for k in ks if 0 <= k < ck.shape[2]], what="segments")


def _bwd_pair(inp, h0=None, dlast=None, reset=None):
    """(ss_bwd_state's gradients, ss_bwd_ckpt's from ss_fwd_ckpt's checkpoints)."""
    d = to_dev(inp)
    rs = None if reset is None else torch.as_tensor(reset).cuda()
    hd = None if h0 is None else h0.cuda()
    dl = None if dlast is None else dlast.cuda()
    _, _, ck = _fwd_ckpt(d, inp, h0=hd, reset=rs)
    kw = dict(D=d.get("D"), z=d.get("z"), delta_bias=d.get("delta_bias"), delta_softplus=inp["delta_softplus"],
              reset=rs, d_last_state=dl)
    plain = selscan.selective_scan_bwd(d["u"], d["delta"], d["A"], d["B"], d["C"], d["dy"], initial_state=hd, **kw)
    if hd is None and dl is None:
        plain.pop("dinitial_state", None)
    from_ck = selscan.selective_scan_bwd(d["u"], d["delta"], d["A"], d["B"], d["C"], d["dy"], ckpt=ck,
                                         initial_state=hd, **kw)
    torch.cuda.synchronize()
    return plain, from_ck


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("N", [4, 16, 64])
def test_bwd_ckpt_bitwise_equals_own_pass(dtype, N):
    """Without sequence segments the forward's checkpoints are the values
    the backward's own pass computes, so every gradient is the same bits."""
    inp = _case(2, 45, 203, N, dtype, seed=N + 920, has_z=True)
    plain, from_ck = _bwd_pair(inp)
    for k, v in plain.items():
        assert (v is None and from_ck[k] is None) or torch.equal(v, from_ck[k]), k


def test_bwd_ckpt_bitwise_with_state_and_starts():
    inp = _case(2, 40, 256, 16, torch.bfloat16, seed=925, has_z=True, bias_kind="uniform_dt")
    g = torch.Generator().manual_seed(925)
    h0, dlast = torch.randn((2, 40, 16), generator=g), torch.randn((2, 40, 16), generator=g)
    reset = _starts(2, 256, seed=925, fixed=(0, 64, 130), p=0.02)
    plain, from_ck = _bwd_pair(inp, h0=h0, dlast=dlast, reset=reset)
    for k, v in plain.items():
        assert (v is None and from_ck[k] is None) or torch.equal(v, from_ck[k]), k


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_bwd_ckpt_segments_against_oracle(dtype):
    """Few rows and 9000 steps: the forward and the backward both cut the
    sequence; the backward needs no forward summary (the checkpoints hold the
    true states) and matches the oracle."""
    inp = _case(1, 8, 9000, 16, dtype, seed=931, has_z=True)
    inp["delta_bias"] = torch.full((8,), -4.0)
    assert selscan.ss_bwd_heuristic(1, 8, 9000, 16, dtype)["segments"] > 1
    g = torch.Generator().manual_seed(931)
    h0, dlast = torch.randn((1, 8, 16), generator=g), torch.randn((1, 8, 16), generator=g)
    _, got = _bwd_pair(inp, h0=h0, dlast=dlast)
    ref = oracle.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["dy"], D=inp["D"],
                                    z=inp["z"], delta_bias=inp["delta_bias"], delta_softplus=True, magnitudes=True,
                                    initial_state=h0, dlast_state=dlast)
    for k, want in ref.items():
        if k.startswith("mag_") or want is None:
            continue
        gk = got[k].to("cpu", torch.float64).numpy()
        if k in ELEM or k == "dinitial_state":
            e = float(np.max(np.abs(gk - want) / (1.0 + np.abs(want))))
            assert e <= TOL_ELEM[dtype], f"{k}: {e:.3e}"
        else:
            check_summed(k, gk, want, ref["mag_" + k], TOL_SUM[dtype], "ckpt segments")


def test_ckpt_rejections():
    inp = _case(1, 8, 64, 16, torch.float32, seed=3)
    d = to_dev(inp)
    y = torch.empty_like(d["u"])
    with pytest.raises(ValueError):   # wrong checkpoint shape
        selscan.ss_fwd_ckpt(d["u"], d["delta"], d["A"], d["B"], d["C"], y, torch.empty((1, 8, 7, 16), device="cuda"))
    lib = selscan.lib()
    desc = selscan.make_desc(1, 8, 64, 16, torch.float32)
    args = [selscan._ptr(t) for t in (d["u"], d["delta"], d["A"], d["B"], d["C"])]
    assert lib.ss_fwd_ckpt(ctypes.byref(desc), *args, None, None, None, 0, None, None, selscan._ptr(y), None, None,
                           None, 0, None) == 1  # no checkpoint buffer
