"""ss_fwd_noalloc, the entry point whose workspace is the library's static
device scratch array, against ss_fwd_ws given an allocated workspace of the
size the launch shape asks for.

The two run the same launch shape and kernels, so their outputs agree
bitwise.  Each case makes two calls in a row on different inputs through the
C ABI, so the second call runs on scratch the first one left behind.  The
file is named to be collected last: it must also pass when it runs alone,
where its first call on the device is the one that looks up the array's
address."""
import pytest
import torch

from gpu_util import to_dev
from selective_state_space_41_b200 import selscan, workloads as W

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

# (workload, whether its launch shape cuts the sequence into segments)
CASES = [
    # few rows, long sequence: 8 segments, 139 KB of scratch
    (W.custom("noalloc_bf16_b1_d256_l16384_n16", 1, 256, 16384, 16, torch.bfloat16, 9101,
              has_z=True, D_kind="ones", bias_kind="uniform_dt", return_last_state=True), True),
    # 4 x 1024 channels over 16384 steps: 8 segments, 2.2 MB of scratch
    (W.custom("noalloc_bf16_b4_d1024_l16384_n16", 4, 1024, 16384, 16, torch.bfloat16, 9102,
              D_kind="ones", bias_kind="none", return_last_state=True), True),
    # bf16 in, fp32 out, 64 states, ragged length
    (W.custom("noalloc_bf16f32_b1_d128_l8251_n64", 1, 128, 8251, 64, torch.bfloat16, 9103,
              has_z=True, return_last_state=True, out_dtype=torch.float32), True),
    # short sequence: no segments, the scratch is not used
    (W.custom("noalloc_fp32_b2_d64_l300_n16", 2, 64, 300, 16, torch.float32, 9104,
              return_last_state=True), False),
]


def _outputs(d, out_dtype):
    batch, dim, L = d["u"].shape
    N = d["A"].shape[1]
    y = torch.full((batch, dim, L), float("nan"), dtype=out_dtype, device="cuda")
    last = (torch.full((batch, dim, N), float("nan"), dtype=torch.float32, device="cuda")
            if d["return_last_state"] else None)
    return y, last


def _operands(d):
    return dict(D=d["D"], z=d["z"], delta_bias=d["delta_bias"], delta_softplus=d["delta_softplus"])


def _with_workspace(d, out_dtype):
    y, last = _outputs(d, out_dtype)
    batch, dim, L = d["u"].shape
    ws = selscan.workspace_for(batch, dim, L, d["A"].shape[1], d["u"].dtype, out_dtype)
    selscan.ss_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], y, last_state=last, workspace=ws,
                   **_operands(d))
    return y, last


def _no_alloc(d, out_dtype):
    y, last = _outputs(d, out_dtype)
    selscan.ss_fwd_noalloc(d["u"], d["delta"], d["A"], d["B"], d["C"], y, last_state=last,
                           **_operands(d))
    return y, last


@pytest.mark.parametrize("w,segmented", CASES, ids=[w.name for w, _ in CASES])
def test_no_alloc_matches_workspace_entry(w, segmented):
    out_dtype = w.out_dtype or w.dtype
    shape = selscan.ss_fwd_heuristic(w.batch, w.dim, w.seqlen, w.dstate, w.dtype, out_dtype,
                                     workspace_bytes=selscan.NOALLOC_SCRATCH_BYTES)
    need = selscan.ss_fwd_workspace_bytes(w.batch, w.dim, w.seqlen, w.dstate, w.dtype, out_dtype)
    assert (shape["segments"] > 1) == segmented and (need > 0) == segmented
    assert need <= selscan.NOALLOC_SCRATCH_BYTES

    first = to_dev(W.make_inputs(w))
    second = to_dev(W.make_inputs(W.with_shape(w, seed=w.seed + 1000)))
    want = [_with_workspace(d, out_dtype) for d in (first, second)]
    torch.cuda.synchronize()
    got = [_no_alloc(d, out_dtype) for d in (first, second)]   # two calls in a row
    torch.cuda.synchronize()
    for call, ((y, last), (y_ref, last_ref)) in enumerate(zip(got, want)):
        assert torch.equal(y, y_ref), f"{w.name}: y differs on call {call + 1}"
        assert torch.equal(last, last_ref), f"{w.name}: last_state differs on call {call + 1}"
    assert not torch.equal(got[0][0], got[1][0])   # the two calls saw different inputs


def test_no_alloc_against_oracle():
    """A segmented no-alloc call checked directly against the fp64 oracle
    (every output of a 2 x 64-channel, 9000-step, 16-state layer)."""
    import oracle
    from gpu_util import TOL, assert_parity
    w = W.custom("noalloc_oracle_b2_d64_l9000_n16", 2, 64, 9000, 16, torch.bfloat16, 9105, has_z=True,
                 D_kind="normal", bias_kind="uniform_dt", return_last_state=True)
    assert selscan.ss_fwd_heuristic(2, 64, 9000, 16, torch.bfloat16,
                                    workspace_bytes=selscan.NOALLOC_SCRATCH_BYTES)["segments"] > 1
    inp = W.make_inputs(w)
    y, last = _no_alloc(to_dev(inp), torch.bfloat16)
    torch.cuda.synchronize()
    y_ref, last_ref = oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                                            z=inp["z"], delta_bias=inp["delta_bias"], delta_softplus=True,
                                            return_last_state=True)
    assert_parity(y, last, y_ref, last_ref, TOL[torch.bfloat16], w.name)


def test_no_alloc_first_call_in_a_fresh_process():
    """The first call on a device is the one that looks up the array's
    address: run it in a new process (whatever ran before in this one), two
    calls in a row, against ss_fwd_ws."""
    import os
    import subprocess
    import sys
    code = (
        "import sys, torch\n"
        "sys.path.insert(0, %r); sys.path.insert(0, %r)\n"
        "import test_zz_no_alloc as T\n"
        "w, seg = T.CASES[0]\n"
        "T.test_no_alloc_matches_workspace_entry(w, seg)\n"
        "print('fresh ok')\n"
    ) % (os.path.dirname(os.path.dirname(os.path.abspath(__file__))), os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "fresh ok" in r.stdout, r.stdout[-2000:] + r.stderr[-2000:]
