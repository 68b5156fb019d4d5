"""selective_scan_fn, the scan as a torch autograd Function over the training
path (ss_fwd_ckpt forward, ss_bwd_ckpt backward): its gradients through
torch.autograd against the fp64 backward oracle (fp32 inputs, tolerances of
test_bwd_gpu.py) and, for bf16 inputs, bit for bit against the direct
backward call cast to the inputs' dtypes."""
import numpy as np
import pytest
import torch

import oracle
from test_bwd_gpu import ELEM, TOL_ELEM, TOL_SUM, _case, check_summed
from selective_state_space_41_b200 import selscan

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

NAMES = ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")
GRAD = {"u": "du", "delta": "ddelta", "A": "dA", "B": "dB", "C": "dC", "D": "dD", "z": "dz",
        "delta_bias": "ddelta_bias"}


def _leaves(inp):
    return {k: (inp[k].cuda().requires_grad_(True) if inp.get(k) is not None else None) for k in NAMES}


def _autograd(inp):
    t = _leaves(inp)
    y = selscan.selective_scan_fn(t["u"], t["delta"], t["A"], t["B"], t["C"], D=t["D"], z=t["z"],
                                  delta_bias=t["delta_bias"], delta_softplus=inp["delta_softplus"])
    (y.float() * inp["dy"].cuda().float()).sum().backward()
    torch.cuda.synchronize()
    return y, {GRAD[k]: (v.grad if v is not None else None) for k, v in t.items()}


@pytest.mark.parametrize("has_z,D_kind,bias_kind", [(True, "normal", "normal"), (False, "none", "none")])
def test_autograd_against_oracle(has_z, D_kind, bias_kind):
    inp = _case(2, 24, 300, 16, torch.float32, seed=951, has_z=has_z, D_kind=D_kind, bias_kind=bias_kind)
    y, got = _autograd(inp)
    y_ref = oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"], z=inp["z"],
                                  delta_bias=inp["delta_bias"], delta_softplus=inp["delta_softplus"])
    assert float(np.max(np.abs(y.detach().double().cpu().numpy() - y_ref) / (1 + np.abs(y_ref)))) <= 1e-5
    ref = oracle.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["dy"], D=inp["D"],
                                    z=inp["z"], delta_bias=inp["delta_bias"], delta_softplus=inp["delta_softplus"],
                                    magnitudes=True)
    for k, want in ref.items():
        if k.startswith("mag_"):
            continue
        if want is None:
            assert got[k] is None, k
            continue
        g = got[k].double().cpu().numpy()
        if k in ELEM:
            e = float(np.max(np.abs(g - want) / (1.0 + np.abs(want))))
            assert e <= TOL_ELEM[torch.float32], f"{k}: {e:.3e}"
        else:
            check_summed(k, g, want, ref["mag_" + k], TOL_SUM[torch.float32], "autograd")


def test_autograd_bf16_matches_the_direct_backward():
    inp = _case(2, 40, 512, 16, torch.bfloat16, seed=953, has_z=True, bias_kind="uniform_dt")
    _, got = _autograd(inp)
    d = {k: (inp[k].cuda() if inp.get(k) is not None else None) for k in NAMES}
    want = selscan.selective_scan_bwd(d["u"], d["delta"], d["A"], d["B"], d["C"], inp["dy"].cuda(), D=d["D"],
                                      z=d["z"], delta_bias=d["delta_bias"], delta_softplus=inp["delta_softplus"])
    torch.cuda.synchronize()
    for k, g in got.items():
        w = want[k]
        if k in ("dB", "dC"):
            w = w.to(torch.bfloat16)
        assert g.dtype == w.dtype and torch.equal(g, w), k


def test_no_grad_forward_is_the_plain_forward():
    """Without inputs that need gradients the Function runs ss_fwd (no
    checkpoints): y is selective_scan_fwd's, bit for bit."""
    inp = _case(2, 40, 512, 16, torch.bfloat16, seed=955, has_z=True)
    d = {k: (inp[k].cuda() if inp.get(k) is not None else None) for k in NAMES}
    kw = dict(D=d["D"], z=d["z"], delta_bias=d["delta_bias"], delta_softplus=inp["delta_softplus"])
    y = selscan.selective_scan_fn(d["u"], d["delta"], d["A"], d["B"], d["C"], **kw)
    want = selscan.selective_scan_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], **kw)
    torch.cuda.synchronize()
    assert not y.requires_grad and torch.equal(y.view(torch.int16), want.view(torch.int16))


def test_autograd_pieces_equal_whole():
    """A sequence trained in two pieces, the first piece's last state the
    second's initial state, gives the whole sequence's outputs and gradients:
    the adjoint crosses the cut through the last state's gradient and the
    initial state's.  fp32 inputs; equal up to fp32 rounding (the pieces may
    take other launch shapes, which sum a step's states in another order)."""
    inp = _case(2, 24, 512, 16, torch.float32, seed=957, has_z=True)
    t = _leaves(inp)
    dy = inp["dy"].cuda()
    kw = dict(D=t["D"], z=None, delta_bias=t["delta_bias"], delta_softplus=inp["delta_softplus"])
    y = selscan.selective_scan_fn(t["u"], t["delta"], t["A"], t["B"], t["C"], **dict(kw, z=t["z"]))
    (y * dy).sum().backward()
    whole = {k: v.grad.clone() for k, v in t.items() if v is not None}
    for v in t.values():
        if v is not None:
            v.grad = None
    cut = 256
    s1, s2 = slice(0, cut), slice(cut, None)
    y1, last1 = selscan.selective_scan_fn(t["u"][:, :, s1], t["delta"][:, :, s1], t["A"], t["B"][:, :, s1],
                                          t["C"][:, :, s1], **dict(kw, z=t["z"][:, :, s1]), return_last_state=True)
    y2 = selscan.selective_scan_fn(t["u"][:, :, s2], t["delta"][:, :, s2], t["A"], t["B"][:, :, s2], t["C"][:, :, s2],
                                   **dict(kw, z=t["z"][:, :, s2]), initial_state=last1)
    ((y1 * dy[:, :, s1]).sum() + (y2 * dy[:, :, s2]).sum()).backward()
    torch.cuda.synchronize()
    yy, y = torch.cat([y1, y2], dim=2).detach(), y.detach()
    assert float(((yy - y).abs() / (1 + y.abs())).max()) <= 1e-5
    for k, v in t.items():
        if v is None:
            continue
        err = float(((v.grad - whole[k]).abs() / (1.0 + whole[k].abs())).max())
        assert err <= 1e-4, f"{k}: {err:.3e}"


def test_autograd_starts_and_state_against_oracle():
    """Sequence starts, a given initial state and a loss on the last state:
    every gradient (the initial state's included) against the fp64 backward
    oracle; the mask's gradients equal the direct backward call's bit for bit."""
    from test_bwd_gpu import _starts
    inp = _case(2, 40, 300, 16, torch.float32, seed=959, has_z=True, bias_kind="uniform_dt")
    gen_ = torch.Generator().manual_seed(959)
    h0, dlast = torch.randn((2, 40, 16), generator=gen_), torch.randn((2, 40, 16), generator=gen_)
    reset = _starts(2, 300, seed=959, fixed=(0, 77, 128), p=0.01)
    t = _leaves(inp)
    th0 = h0.cuda().requires_grad_(True)
    y, last = selscan.selective_scan_fn(t["u"], t["delta"], t["A"], t["B"], t["C"], D=t["D"], z=t["z"],
                                        delta_bias=t["delta_bias"], delta_softplus=inp["delta_softplus"],
                                        initial_state=th0, reset=torch.as_tensor(reset).cuda(),
                                        return_last_state=True)
    ((y * inp["dy"].cuda()).sum() + (last * dlast.cuda()).sum()).backward()
    torch.cuda.synchronize()
    got = {GRAD[k]: v.grad for k, v in t.items() if v is not None}
    got["dinitial_state"] = th0.grad
    ref = oracle.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["dy"], D=inp["D"],
                                    z=inp["z"], delta_bias=inp["delta_bias"], delta_softplus=inp["delta_softplus"],
                                    magnitudes=True, reset=reset, initial_state=h0, dlast_state=dlast)
    for k, want in ref.items():
        if k.startswith("mag_") or want is None:
            continue
        g = got[k].double().cpu().numpy()
        if k in ELEM or k == "dinitial_state":
            e = float(np.max(np.abs(g - want) / (1.0 + np.abs(want))))
            assert e <= TOL_ELEM[torch.float32], f"{k}: {e:.3e}"
        else:
            check_summed(k, g, want, ref["mag_" + k], TOL_SUM[torch.float32], "autograd starts")
    d = {k: (inp[k].cuda() if inp.get(k) is not None else None) for k in NAMES}
    direct = selscan.selective_scan_bwd(d["u"], d["delta"], d["A"], d["B"], d["C"], inp["dy"].cuda(), D=d["D"],
                                        z=d["z"], delta_bias=d["delta_bias"], delta_softplus=inp["delta_softplus"],
                                        reset=torch.as_tensor(reset).cuda(), initial_state=h0.cuda(),
                                        d_last_state=dlast.cuda())
    torch.cuda.synchronize()
    for k, v in direct.items():
        assert (v is None and got.get(k) is None) or torch.equal(v, got[k]), k


def test_autograd_empty_batch_and_sequence():
    """No batch entries: empty outputs and gradients; an empty sequence
    with a returned last state: the last state is the initial one and its
    gradient reaches the initial state unchanged."""
    inp = _case(0, 8, 32, 16, torch.float32, seed=961)
    t = _leaves(inp)
    y = selscan.selective_scan_fn(t["u"], t["delta"], t["A"], t["B"], t["C"], D=t["D"],
                                  delta_bias=t["delta_bias"], delta_softplus=True)
    y.sum().backward()
    torch.cuda.synchronize()
    assert y.shape == (0, 8, 32) and t["u"].grad.shape == (0, 8, 32) and float(t["A"].grad.abs().sum()) == 0.0
    inp = _case(2, 8, 0, 16, torch.float32, seed=962)
    t = _leaves(inp)
    h0 = torch.randn((2, 8, 16), generator=torch.Generator().manual_seed(962)).cuda().requires_grad_(True)
    y, last = selscan.selective_scan_fn(t["u"], t["delta"], t["A"], t["B"], t["C"], D=t["D"],
                                        delta_bias=t["delta_bias"], delta_softplus=True, initial_state=h0,
                                        return_last_state=True)
    g = torch.randn_like(last)
    (last * g).sum().backward()
    torch.cuda.synchronize()
    assert torch.equal(last.detach(), h0.detach()) and torch.equal(h0.grad, g)
