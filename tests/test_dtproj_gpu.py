"""The forward with delta = W_dt delta_r produced inside the scan (ss_fwd_dtproj:
the dt_proj map of the mamba-minimal block, Mamba-minimal项目解析 核心组件解析
§5, on the tensor cores) through the C ABI, against the fp64 oracle's dt_proj
form (the scan fed the float64 product W_dt delta_r).  Tolerance as for bf16
inputs: max |err| <= 1e-2 (1 + |y|) (the product accumulates in fp32 from
exact bf16 products; y is rounded to bf16)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import TOL, assert_parity, to_dev
from selective_state_space_41_b200 import selscan, workloads as W

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

BF16 = torch.bfloat16


def _run(inp, out_dtype=None, workspace=False):
    d = to_dev(inp)
    batch, dim, L = d["u"].shape
    N = d["A"].shape[1]
    y = torch.full((batch, dim, L), float("nan"), dtype=out_dtype or BF16, device="cuda")
    last = torch.full((batch, dim, N), float("nan"), device="cuda") if inp["return_last_state"] else None
    ws = selscan.workspace_for(batch, dim, L, N, BF16, y.dtype) if workspace else None
    selscan.ss_fwd_dtproj(d["u"], d["delta_r"], d["W_dt"], d["A"], d["B"], d["C"], y, D=d["D"], z=d["z"],
                          delta_bias=d["delta_bias"], delta_softplus=inp["delta_softplus"], last_state=last,
                          workspace=ws)
    torch.cuda.synchronize()
    return y, last


def _oracle(inp):
    return oracle.selective_scan_dtproj(inp["u"], inp["delta_r"], inp["W_dt"], inp["A"], inp["B"], inp["C"],
                                        D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"],
                                        delta_softplus=inp["delta_softplus"], return_last_state=True)


def _case(batch, dim, L, N, R, seed, **kw):
    w = W.custom("dtproj", batch, dim, L, N, BF16, seed, **kw)
    return W.make_dtproj_inputs(w, R)


def _check(inp, what, **kw):
    y, last = _run(inp, **kw)
    y_ref, last_ref = _oracle(inp)
    assert_parity(y, last, y_ref, last_ref if inp["return_last_state"] else None,
                  1e-4 if kw.get("out_dtype") == torch.float32 else TOL[BF16], what)
    assert selscan.ss_device_status() == 0


@pytest.mark.parametrize("R", [1, 7, 16, 17, 33, 48, 64])
def test_dtproj_ranks(R):
    """dt_rank from 1 to 64 (zero-padded to a multiple of 16 in K)."""
    _check(_case(2, 70, 300, 16, R, seed=R, has_z=True, bias_kind="uniform_dt", return_last_state=True), f"R={R}")


@pytest.mark.parametrize("N", [4, 8, 9, 16, 32, 33, 64])
def test_dtproj_state_sizes(N):
    """Every state bucket (2 or 4 lanes per row, the heuristic's when it can)."""
    _check(_case(2, 45, 203, N, 48, seed=100 + N, has_z=True, return_last_state=True), f"N={N}")


@pytest.mark.parametrize("L", [1, 15, 16, 63, 64, 65, 127, 128, 129, 191, 192, 1000])
def test_dtproj_lengths(L):
    """Ragged lengths: partial stages and sub-chunks (delta_r zero-filled
    past the end), one to many stages (the product pipeline's start-up)."""
    _check(_case(3, 40, L, 16, 48, seed=L, has_z=True, return_last_state=True), f"L={L}")


def test_dtproj_exp_mode_and_f32_output():
    inp = _case(2, 33, 500, 16, 48, seed=5, has_z=False, D_kind="none", bias_kind="none",
                delta_softplus=False, return_last_state=True)
    inp["W_dt"] = (inp["W_dt"].float() * 0.5).to(BF16)   # keep exp(delta) in a sane range
    _check(inp, "exp mode, f32 out", out_dtype=torch.float32)


def test_dtproj_segments():
    """Few rows and a long sequence with a workspace: the heuristic's
    segments with the product computed per segment."""
    inp = _case(1, 64, 9000, 16, 48, seed=9, has_z=True, return_last_state=True)
    assert selscan.ss_fwd_heuristic(1, 64, 9000, 16, BF16, workspace_bytes=1 << 26)["segments"] > 1
    _check(inp, "segments", workspace=True)


def test_dtproj_mamba130m_one_batch():
    """One batch entry of the mamba-130m-shaped layer with dt_rank 48."""
    w = W.with_shape(W.WORKLOADS[W.MAMBA130M], batch=1)
    inp = W.make_dtproj_inputs(w, W.dt_rank_auto(768))
    inp["return_last_state"] = True
    _check(inp, "mamba130m batch 1")


def test_dtproj_equals_unfused_on_the_same_delta():
    """When W_dt delta_r is exactly representable in bf16 (an identity
    projection: dt_rank = dim, W_dt = I), the fused form gives the unfused
    scan of delta = delta_r bit for bit."""
    inp = _case(2, 32, 400, 16, 32, seed=11, has_z=True, return_last_state=True)
    inp["W_dt"] = torch.eye(32, dtype=BF16)
    y, last = _run(inp)
    d = to_dev(inp)
    y2 = torch.empty_like(y)
    last2 = torch.empty_like(last)
    selscan.ss_fwd(d["u"], d["delta_r"], d["A"], d["B"], d["C"], y2, D=d["D"], z=d["z"], delta_bias=d["delta_bias"],
                   delta_softplus=True, last_state=last2, lanes_per_row=4, split_states=1, warps_per_block=4,
                   segments=1)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    assert torch.equal(last, last2)


def test_dtproj_rejections():
    inp = _case(1, 8, 64, 16, 48, seed=3)
    d = to_dev(inp)
    y = torch.empty_like(d["u"])
    with pytest.raises(selscan.SelscanError):   # fp32 inputs
        selscan.ss_fwd_dtproj(d["u"].float(), d["delta_r"].float(), d["W_dt"].float(), d["A"], d["B"].float(),
                              d["C"].float(), y.float())
    big = torch.zeros((1, 65, 64), dtype=BF16, device="cuda")
    with pytest.raises(selscan.SelscanError):   # dt_rank above 64
        selscan.ss_fwd_dtproj(d["u"], big, torch.zeros((8, 65), dtype=BF16, device="cuda"), d["A"], d["B"],
                              d["C"], y)


# ---------------------------------------------------------------- x_dbl form
def _xdbl(inp):
    """x_proj's output as one (batch, dt_rank + 2 N, L) tensor: feature rows
    delta_r, then B, then C."""
    return torch.cat([inp["delta_r"], inp["B"], inp["C"]], dim=1).contiguous()


def _run_xdbl(inp, x_dbl, out_dtype=None, workspace=False):
    d = to_dev(inp)
    batch, dim, L = d["u"].shape
    N = d["A"].shape[1]
    y = torch.full((batch, dim, L), float("nan"), dtype=out_dtype or BF16, device="cuda")
    last = torch.full((batch, dim, N), float("nan"), device="cuda") if inp["return_last_state"] else None
    ws = selscan.workspace_for(batch, dim, L, N, BF16, y.dtype) if workspace else None
    selscan.ss_fwd_xdbl(d["u"], x_dbl.cuda(), d["W_dt"], d["A"], y, D=d["D"], z=d["z"],
                        delta_bias=d["delta_bias"], delta_softplus=inp["delta_softplus"], last_state=last,
                        workspace=ws)
    torch.cuda.synchronize()
    return y, last


@pytest.mark.parametrize("R,N,L", [(48, 16, 300), (7, 33, 203), (64, 64, 129), (16, 4, 1000), (1, 8, 65)])
def test_xdbl_against_oracle_and_dtproj(R, N, L):
    """delta_r, B and C read in place from x_dbl: the oracle fed the three
    row ranges of the same tensor (the x_proj split), and ss_fwd_dtproj on
    contiguous copies of them bit for bit."""
    inp = _case(3, 40, L, N, R, seed=700 + R + N, has_z=True, bias_kind="uniform_dt", return_last_state=True)
    x = _xdbl(inp)
    y, last = _run_xdbl(inp, x)
    split = dict(inp, delta_r=x[:, :R], B=x[:, R:R + N], C=x[:, R + N:])
    y_ref, last_ref = _oracle(split)
    assert_parity(y, last, y_ref, last_ref, TOL[BF16], f"x_dbl R={R} N={N} L={L}")
    y2, last2 = _run(inp)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16)) and torch.equal(last, last2)


def test_xdbl_segments_and_f32_output():
    """Few rows over a long sequence (sequence segments: the fix-up reads C
    and delta_r from x_dbl too), fp32 output."""
    inp = _case(1, 64, 9000, 16, 48, seed=777, has_z=True, return_last_state=True)
    assert selscan.ss_fwd_heuristic(1, 64, 9000, 16, BF16, workspace_bytes=1 << 26)["segments"] > 1
    x = _xdbl(inp)
    y, last = _run_xdbl(inp, x, out_dtype=torch.float32, workspace=True)
    y_ref, last_ref = _oracle(inp)
    assert_parity(y, last, y_ref, last_ref, 1e-4, "x_dbl segments")
    y2, last2 = _run(inp, out_dtype=torch.float32, workspace=True)
    assert torch.equal(y, y2) and torch.equal(last, last2)


def test_xdbl_rejections():
    inp = _case(1, 8, 64, 16, 48, seed=3)
    d = to_dev(inp)
    y = torch.empty_like(d["u"])
    x = _xdbl(inp).cuda()
    with pytest.raises(ValueError):   # feature rows do not match dt_rank + 2 N
        selscan.ss_fwd_xdbl(d["u"], x[:, :-1], d["W_dt"], d["A"], y)
    with pytest.raises(selscan.SelscanError):   # fp32 inputs
        selscan.ss_fwd_xdbl(d["u"].float(), x.float(), d["W_dt"].float(), d["A"], y.float())


@pytest.mark.parametrize("form", ["dtproj", "xdbl"])
def test_empty_sequence_and_no_rows(form):
    """L = 0 writes a zero last state (no initial state is taken here); no
    batch entries is a no-op; both for delta_r/B/C passed apart and in place."""
    inp = _case(2, 24, 0, 16, 48, seed=31, return_last_state=True)
    d = to_dev(inp)
    last = torch.full((2, 24, 16), 7.0, device="cuda")
    y = torch.empty((2, 24, 0), dtype=BF16, device="cuda")
    if form == "dtproj":
        selscan.ss_fwd_dtproj(d["u"], d["delta_r"], d["W_dt"], d["A"], d["B"], d["C"], y, last_state=last)
    else:
        selscan.ss_fwd_xdbl(d["u"], _xdbl(inp).cuda(), d["W_dt"], d["A"], y, last_state=last)
    torch.cuda.synchronize()
    assert torch.all(last == 0)
    inp = _case(0, 24, 64, 16, 48, seed=32)
    d = to_dev(inp)
    y = torch.empty((0, 24, 64), dtype=BF16, device="cuda")
    if form == "dtproj":
        selscan.ss_fwd_dtproj(d["u"], d["delta_r"], d["W_dt"], d["A"], d["B"], d["C"], y)
    else:
        selscan.ss_fwd_xdbl(d["u"], _xdbl(inp).cuda(), d["W_dt"], d["A"], y)
    torch.cuda.synchronize()
    assert selscan.ss_device_status() == 0
