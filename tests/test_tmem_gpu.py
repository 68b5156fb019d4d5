"""The tensor-memory-fed direct kernel (split_states = 2: B and C broadcast
into each lane's TMEM lane by a tcgen05 MMA with a 0/1 selection matrix)
through the C ABI, against the fp64 oracle and against the shared-memory
form of the same kernel (split_states = 1), which does the same fp32
arithmetic in the same order and so must agree bitwise.  Tolerance as in
test_parity_gpu.py: max |err| <= 1e-2 (1 + |y|) for bf16 inputs."""
import numpy as np
import pytest
import torch

from gpu_util import TOL, assert_parity, run_gpu, run_oracle, to_dev
from selective_state_space_41_b200 import selscan, workloads as W

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

BF16 = torch.bfloat16


def _case(batch, dim, L, N, seed, **kw):
    return W.make_inputs(W.custom("tmem", batch, dim, L, N, BF16, seed, **kw))


def _bucket(N):
    return 4 if N <= 4 else 8 if N <= 8 else 16 if N <= 16 else 32 if N <= 32 else 64


def _supported(N, lanes):
    """2 to 8 states per lane, the four TMEM buffers of a sub-chunk (16 steps
    from 4 lanes per row, 8 below) within 128 columns, and each buffer a
    multiple of 16 columns (the MMA's N)."""
    s = _bucket(N) // lanes
    sub = 16 if lanes >= 4 else 8
    return 2 <= s <= 8 and 2 * s * sub <= 128 and (2 * s * sub // 4) % 16 == 0


def _status_clear():
    assert selscan.ss_device_status() == 0, "a bounded wait of the TMEM-fed kernel ran out"


@pytest.mark.parametrize("N", [2, 4, 7, 8, 9, 16, 17, 31, 32, 33, 64])
@pytest.mark.parametrize("lanes", [2, 4, 8])
def test_tmem_state_splits(N, lanes):
    """Every (state bucket, lanes) the kernel is built for; ragged length
    (partial stage, sub-chunk and TMEM buffer) and channels (mirrored rows)."""
    if not _supported(N, lanes):
        pytest.skip("not a split the TMEM-fed kernel is built for")
    inp = _case(2, 19, 203, N, seed=N * 11 + lanes, has_z=True, return_last_state=True)
    y, last = run_gpu(inp, lanes=lanes, split=2)
    y_ref, last_ref = run_oracle(inp)
    assert_parity(y, last, y_ref, last_ref, TOL[BF16], f"N={N} lanes={lanes}")
    _status_clear()


@pytest.mark.parametrize("L", [1, 7, 8, 9, 15, 16, 17, 63, 64, 65, 127, 129, 1000, 1003])
def test_tmem_ragged_lengths(L):
    for lanes in (2, 4):
        inp = _case(3, 40, L, 16, seed=L + lanes, has_z=True, return_last_state=True)
        y, last = run_gpu(inp, lanes=lanes, split=2)
        y_ref, last_ref = run_oracle(inp)
        assert_parity(y, last, y_ref, last_ref, TOL[BF16], f"L={L} lanes={lanes}")
    _status_clear()


@pytest.mark.parametrize("has_z", [False, True])
@pytest.mark.parametrize("D_kind", ["none", "normal"])
@pytest.mark.parametrize("bias_kind", ["none", "uniform_dt"])
@pytest.mark.parametrize("softplus", [False, True])
def test_tmem_optional_operands(has_z, D_kind, bias_kind, softplus):
    inp = _case(2, 36, 300, 16, seed=5, has_z=has_z, D_kind=D_kind, bias_kind=bias_kind,
                delta_softplus=softplus, return_last_state=True)
    if not softplus:  # keep exp(delta + bias) in a sane range
        inp["delta"] = (inp["delta"].float() * 0.5 - 1.0).to(BF16)
    y, last = run_gpu(inp, lanes=4, split=2)
    y_ref, last_ref = run_oracle(inp)
    assert_parity(y, last, y_ref, last_ref, TOL[BF16], "flags")


def test_tmem_f32_output():
    inp = _case(2, 33, 500, 16, seed=8, has_z=True, return_last_state=True)
    y, last = run_gpu(inp, out_dtype=torch.float32, lanes=4, split=2)
    y_ref, last_ref = run_oracle(inp)
    assert_parity(y, last, y_ref, last_ref, 1e-4, "bf16 -> f32")


@pytest.mark.parametrize("L,segments", [(4096, 2), (3001, 3), (5000, 7), (640, 4)])
@pytest.mark.parametrize("lanes", [2, 4])
def test_tmem_segments(L, segments, lanes):
    """Sequence segments run by the TMEM-fed kernel, joined by the fix-up."""
    inp = _case(2, 70, L, 16, seed=L + segments + lanes, has_z=True, return_last_state=True)
    y, last = run_gpu(inp, lanes=lanes, split=2, segments=segments)
    y_ref, last_ref = run_oracle(inp)
    assert_parity(y, last, y_ref, last_ref, TOL[BF16], f"L={L} segments={segments} lanes={lanes}")
    _status_clear()


@pytest.mark.parametrize("name,lanes", [(W.MAMBA130M, 4), (W.GENOMIC, 2), ("wide_state_b16_d4096_l8192_n16", 2)])
def test_tmem_bitwise_equals_shared_memory_form(name, lanes):
    """The same launch with B/C through shared memory (split_states = 1) and
    through tensor memory (2): identical fp32 arithmetic, identical bits.
    One batch entry, 1000 steps (ragged), of each layer shape."""
    w = W.WORKLOADS[name]
    inp = W.make_inputs(W.with_shape(w, batch=1, seqlen=1000))
    y1, last1 = run_gpu(inp, lanes=lanes, split=1, warps=4)
    y2, last2 = run_gpu(inp, lanes=lanes, split=2)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16)), name
    if last1 is not None:
        assert torch.equal(last1, last2), name
    _status_clear()


def test_tmem_initial_state_in_place():
    """From a given state, updated in place, a sequence in two pieces equals one run."""
    inp = _case(2, 40, 600, 16, seed=13, has_z=True, return_last_state=True)
    d = to_dev(inp)
    h0 = torch.randn((2, 40, 16), device="cuda")
    cfg = dict(lanes_per_row=4, split_states=2, warps_per_block=4, segments=1)
    y = torch.empty_like(d["u"])
    last = torch.empty_like(h0)
    kw = dict(D=d["D"], z=d["z"], delta_bias=d["delta_bias"], delta_softplus=True)
    selscan.ss_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], y, last_state=last, initial_state=h0, **kw, **cfg)
    st = h0.clone()
    ys = []
    for lo, hi in ((0, 256), (256, 600)):
        sl = lambda t: t[..., lo:hi].contiguous()  # noqa: E731
        yp = torch.empty_like(sl(d["u"]))
        selscan.ss_fwd(sl(d["u"]), sl(d["delta"]), d["A"], sl(d["B"]), sl(d["C"]), yp, D=d["D"], z=sl(d["z"]),
                       delta_bias=d["delta_bias"], delta_softplus=True, last_state=st, initial_state=st, **cfg)
        ys.append(yp)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(ys, dim=-1).view(torch.int16), y.view(torch.int16))
    assert torch.equal(st, last)
    import oracle
    y_ref, last_ref = oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                                            z=inp["z"], delta_bias=inp["delta_bias"], delta_softplus=True,
                                            return_last_state=True, initial_state=h0.cpu())
    assert_parity(y, last, y_ref, last_ref, TOL[BF16], "initial state")
    _status_clear()


def test_tmem_rejections():
    """split_states = 2 only for bf16 inputs, 2..8 states per lane, 4 compute
    warps, and without sequence starts."""
    f32 = _case(1, 8, 64, 16, seed=1)
    f32 = {k: (v.float() if isinstance(v, torch.Tensor) and v.dtype == BF16 else v) for k, v in f32.items()}
    with pytest.raises(selscan.SelscanError):
        run_gpu(f32, lanes=4, split=2)
    inp = _case(1, 8, 64, 64, seed=2)
    with pytest.raises(selscan.SelscanError):
        run_gpu(inp, lanes=2, split=2)       # 32 states per lane
    inp = _case(1, 8, 64, 16, seed=3)
    with pytest.raises(selscan.SelscanError):
        run_gpu(inp, lanes=4, split=2, warps=2)
    d = to_dev(inp)
    y = torch.empty_like(d["u"])
    with pytest.raises(selscan.SelscanError):
        selscan.ss_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], y, delta_softplus=True, lanes_per_row=4,
                       split_states=2, reset=torch.zeros((1, 64), dtype=torch.uint8, device="cuda"))
