"""Helpers shared by the GPU parity tests: run the CUDA path on generated
inputs and compare with the oracle under the tolerance of the input dtype."""
import numpy as np
import torch

import oracle
from selective_state_space_41_b200 import selscan

# max |err| <= TOL * (1 + |y_oracle|), per input dtype: fp32 inputs 1e-5; bf16
# inputs (fp32 state and accumulation, y rounded to bf16) 1e-2.
TOL = {torch.float32: 1e-5, torch.bfloat16: 1e-2}


def to_dev(inp, device="cuda"):
    out = {}
    for k, v in inp.items():
        out[k] = v.to(device, non_blocking=True) if isinstance(v, torch.Tensor) else v
    return out


def run_gpu(inp, out_dtype=None, lanes=None, warps=None, split=False, segments=None,
            workspace=True, device="cuda"):
    """(y, last_state) from libselscan for host inputs ``inp``.  ``workspace``:
    give the call the workspace its launch shape can use (as the benchmark and
    selective_scan_fwd do); False: no workspace (plain ss_fwd)."""
    d = to_dev(inp, device)
    u = d["u"]
    batch, dim, L = u.shape
    N = d["A"].shape[1]
    y = torch.empty((batch, dim, L), dtype=out_dtype or inp.get("out_dtype") or u.dtype,
                    device=device)
    last = (torch.empty((batch, dim, N), dtype=torch.float32, device=device)
            if inp.get("return_last_state") else None)
    cfg = {}
    if lanes is not None or warps is not None or segments is not None:
        cfg = dict(lanes_per_row=lanes, warps_per_block=warps, split_states=split, segments=segments)
    ws = (selscan.workspace_for(batch, dim, L, N, u.dtype, y.dtype, device=device, **cfg)
          if workspace else None)
    selscan.ss_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], y, D=d.get("D"), z=d.get("z"),
                   delta_bias=d.get("delta_bias"), delta_softplus=inp["delta_softplus"],
                   last_state=last, workspace=ws, **cfg)
    torch.cuda.synchronize()
    return y, last


def run_oracle(inp):
    return oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                 D=inp.get("D"), z=inp.get("z"), delta_bias=inp.get("delta_bias"),
                                 delta_softplus=inp["delta_softplus"], return_last_state=True)


def max_scaled_err(got, want):
    got = got.detach().to("cpu", torch.float64).numpy() if isinstance(got, torch.Tensor) else got
    want = np.asarray(want, np.float64)
    if want.size == 0:
        return 0.0
    return float(np.max(np.abs(got - want) / (1.0 + np.abs(want))))


def assert_parity(y, last, y_ref, last_ref, tol, what=""):
    assert torch.isfinite(y.float()).all(), f"{what}: non-finite output"
    e = max_scaled_err(y, y_ref)
    assert e <= tol, f"{what}: y max |err|/(1+|y|) = {e:.3e} > {tol:.0e}"
    if last is not None:
        e2 = max_scaled_err(last, last_ref)
        assert e2 <= tol, f"{what}: last_state max |err|/(1+|h|) = {e2:.3e} > {tol:.0e}"
    return e
