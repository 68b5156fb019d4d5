"""Seeded random cases: each seed draws a shape (batch, channels, length,
states), the input dtype (bf16 sometimes with fp32 output) and the optional
parts (z gate, D skip, delta bias, softplus or exp mode, sequence starts, an
initial state, a last-state gradient), then checks the forward (ss_fwd with
the workspace its shape can use) and the backward both ways (ss_bwd with its
own checkpointing pass; ss_fwd_ckpt then the backward from its checkpoints)
through the C ABI against the fp64 oracle, under the tolerances of
test_parity_gpu.py and test_bwd_gpu.py.  Further families draw a random
accepted launch shape, a few decoding steps from a random state, the dt_proj
form with a random rank (apart and in place from x_dbl, bit for bit equal),
and the host-buffer forward over random streams and batch ranges.  The draws
are fixed by the seed, so a failure names a reproducible case; SS_FUZZ_SEEDS
sets how many seeds run (48 by default; 300 of each family passed)."""
import os

import numpy as np
import pytest
import torch

import oracle
from gpu_util import TOL, assert_parity, to_dev
from test_bwd_gpu import ELEM, TOL_ELEM, TOL_SUM, check_summed
from selective_state_space_41_b200 import gen, selscan, workloads as W

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

SEEDS = range(int(os.environ.get("SS_FUZZ_SEEDS", "48")))


def _draw(seed):
    rng = np.random.default_rng(1000 + seed)
    batch = int(rng.integers(1, 4))
    dim = int(rng.integers(1, 49))
    L = int(rng.integers(1, 601))
    N = int(rng.choice([1, 3, 4, 8, 9, 16, 17, 32, 33, 64]))
    dtype = torch.bfloat16 if rng.random() < 0.5 else torch.float32
    softplus = bool(rng.random() < 0.75)
    kw = dict(has_z=bool(rng.random() < 0.5), D_kind=str(rng.choice(["normal", "ones", "none"])),
              bias_kind=str(rng.choice(["normal", "zeros", "uniform_dt", "none"])) if softplus else "none",
              delta_softplus=softplus, return_last_state=True)
    out_dtype = torch.float32 if dtype == torch.bfloat16 and rng.random() < 0.25 else None
    inp = W.make_inputs(W.custom(f"fuzz{seed}", batch, dim, L, N, dtype, 5000 + seed, **kw))
    inp["out_dtype"] = out_dtype
    if not softplus:  # exp mode: keep delta' = exp(delta) in a moderate range
        inp["delta"] = (inp["delta"].float() * 0.5).to(dtype)
    reset = None
    if rng.random() < 0.4:
        reset = (rng.random((batch, L)) < 0.02).astype(np.uint8)
        reset[:, int(rng.integers(0, L))] = 1
    h0 = torch.from_numpy(rng.standard_normal((batch, dim, N)).astype(np.float32)) if rng.random() < 0.4 else None
    dlast = torch.from_numpy(rng.standard_normal((batch, dim, N)).astype(np.float32)) if rng.random() < 0.4 else None
    inp["dy"] = gen.fill((batch, dim, L), out_dtype or dtype, 5000 + seed, 9)
    return inp, reset, h0, dlast


def _case_name(inp, reset, h0, dlast):
    b, d, L = inp["u"].shape
    return (f"{b}x{d}x{L} N={inp['A'].shape[1]} {str(inp['u'].dtype)[6:]} z={inp['z'] is not None} "
            f"D={inp['D'] is not None} bias={inp['delta_bias'] is not None} softplus={inp['delta_softplus']} "
            f"starts={reset is not None} h0={h0 is not None} dlast={dlast is not None} "
            f"out={'f32' if inp.get('out_dtype') else 'in'}")


@pytest.mark.parametrize("seed", SEEDS)
def test_fuzz_forward(seed):
    inp, reset, h0, _ = _draw(seed)
    what = _case_name(inp, reset, h0, None)
    d = to_dev(inp)
    b, dim, L = d["u"].shape
    N = d["A"].shape[1]
    y = torch.full((b, dim, L), float("nan"), dtype=inp["out_dtype"] or d["u"].dtype, device="cuda")
    last = torch.full((b, dim, N), float("nan"), device="cuda")
    ws = selscan.workspace_for(b, dim, L, N, d["u"].dtype, y.dtype)
    selscan.ss_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], y, D=d["D"], z=d["z"], delta_bias=d["delta_bias"],
                   delta_softplus=inp["delta_softplus"], last_state=last, workspace=ws,
                   initial_state=None if h0 is None else h0.cuda(),
                   reset=None if reset is None else torch.as_tensor(reset).cuda())
    torch.cuda.synchronize()
    y_ref, last_ref = oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                                            z=inp["z"], delta_bias=inp["delta_bias"],
                                            delta_softplus=inp["delta_softplus"], return_last_state=True,
                                            initial_state=h0, reset=reset)
    assert_parity(y, last, y_ref, last_ref, 1e-4 if inp["out_dtype"] else TOL[inp["u"].dtype], what)


@pytest.mark.parametrize("path", ["own_pass", "checkpoints"])
@pytest.mark.parametrize("seed", SEEDS)
def test_fuzz_backward(seed, path):
    """ss_bwd (its own checkpointing pass), or the training path: the
    forward that writes the checkpoints, then the backward from them."""
    inp, reset, h0, dlast = _draw(seed)
    what = _case_name(inp, reset, h0, dlast) + " " + path
    dtype = inp["u"].dtype
    d = to_dev(inp)
    rs = None if reset is None else torch.as_tensor(reset).cuda()
    hd = None if h0 is None else h0.cuda()
    ck = None
    if path == "checkpoints":
        b, dim, L = d["u"].shape
        N = d["A"].shape[1]
        y = torch.empty((b, dim, L), dtype=inp["out_dtype"] or dtype, device="cuda")
        ck = torch.empty(selscan.ckpt_shape(b, dim, L, N), device="cuda")
        selscan.ss_fwd_ckpt(d["u"], d["delta"], d["A"], d["B"], d["C"], y, ck, D=d["D"], z=d["z"],
                            delta_bias=d["delta_bias"], delta_softplus=inp["delta_softplus"], initial_state=hd,
                            reset=rs, workspace=selscan.workspace_for(b, dim, L, N, dtype, y.dtype))
    got = selscan.selective_scan_bwd(d["u"], d["delta"], d["A"], d["B"], d["C"], d["dy"], D=d["D"], z=d["z"],
                                     delta_bias=d["delta_bias"], delta_softplus=inp["delta_softplus"],
                                     reset=rs, initial_state=hd, ckpt=ck,
                                     d_last_state=None if dlast is None else dlast.cuda())
    torch.cuda.synchronize()
    ref = oracle.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["dy"], D=inp["D"],
                                    z=inp["z"], delta_bias=inp["delta_bias"], delta_softplus=inp["delta_softplus"],
                                    magnitudes=True, reset=reset, initial_state=h0, dlast_state=dlast)
    for k, want in ref.items():
        if k.startswith("mag_") or want is None:
            continue
        if k == "dinitial_state" and "dinitial_state" not in got:
            continue
        g = got[k].detach().to("cpu", torch.float64).numpy()
        assert np.isfinite(g).all(), f"{what}: {k} not finite"
        if want.size == 0:
            continue
        if k in ELEM or k == "dinitial_state":
            e = float(np.max(np.abs(g - want) / (1.0 + np.abs(want))))
            assert e <= TOL_ELEM[dtype], f"{what}: {k} max |err|/(1+|ref|) = {e:.3e}"
        else:
            check_summed(k, g, want, ref["mag_" + k], TOL_SUM[dtype], what)


# ---------------------------------------------------------------- launch shapes
# (lanes per row, split_states) pairs the forward takes: one lane per row
# (scan kernel when split_states is 0), the state split over 2/4/8 lanes in
# shared memory (1) or fed through tensor memory (2).
_SHAPES = [(1, 0), (2, 0), (4, 0), (8, 0), (16, 0), (32, 0), (1, 1), (2, 1), (4, 1), (8, 1), (2, 2), (4, 2), (8, 2)]


@pytest.mark.parametrize("seed", SEEDS)
def test_fuzz_launch_shapes(seed):
    """A random shape in a random launch shape the library accepts (lanes,
    state split, warps per block, sequence segments), with the optional
    parts drawn as above (no sequence starts or initial state: not every
    launch shape reads them)."""
    inp, _, _, _ = _draw(seed)
    rng = np.random.default_rng(7000 + seed)
    d = to_dev(inp)
    b, dim, L = d["u"].shape
    N = d["A"].shape[1]
    y = torch.full((b, dim, L), float("nan"), dtype=inp["out_dtype"] or d["u"].dtype, device="cuda")
    last = torch.full((b, dim, N), float("nan"), device="cuda")
    for attempt in range(64):
        lanes, split = _SHAPES[int(rng.integers(0, len(_SHAPES)))]
        cfg = dict(lanes_per_row=lanes, split_states=split, warps_per_block=int(rng.choice([1, 2, 4, 8])),
                   segments=int(rng.integers(1, 9)) if split == 1 or lanes == 1 else 1)
        try:
            ws = selscan.workspace_for(b, dim, L, N, d["u"].dtype, y.dtype, **cfg)
            selscan.ss_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], y, D=d["D"], z=d["z"],
                           delta_bias=d["delta_bias"], delta_softplus=inp["delta_softplus"], last_state=last,
                           workspace=ws, **cfg)
            break
        except selscan.SelscanError as e:
            if e.status != 7:  # only SS_ERR_BAD_CONFIG means "another shape"
                raise
    else:
        pytest.skip("no accepted launch shape drawn")
    torch.cuda.synchronize()
    y_ref, last_ref = oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                                            z=inp["z"], delta_bias=inp["delta_bias"],
                                            delta_softplus=inp["delta_softplus"], return_last_state=True)
    assert_parity(y, last, y_ref, last_ref, 1e-4 if inp["out_dtype"] else TOL[inp["u"].dtype],
                  _case_name(inp, None, None, None) + f" {cfg}")
    assert selscan.ss_device_status() == 0


# ---------------------------------------------------------------- other entries
@pytest.mark.parametrize("seed", SEEDS)
def test_fuzz_decode_steps(seed):
    """ss_step, a few steps with the state updated in place from a random
    initial state, against the oracle's run from that state."""
    inp, _, h0, _ = _draw(seed)
    rng = np.random.default_rng(8000 + seed)
    b, dim, L = inp["u"].shape
    steps = min(int(rng.integers(1, 9)), L)
    N = inp["A"].shape[1]
    sl = {k: (inp[k][..., :steps].contiguous() if k in ("u", "delta", "z", "B", "C") and inp[k] is not None
              else inp[k]) for k in ("u", "delta", "z", "B", "C", "A", "D", "delta_bias")}
    h0 = h0 if h0 is not None else torch.from_numpy(rng.standard_normal((b, dim, N)).astype(np.float32))
    d = to_dev(sl)
    state = h0.cuda().clone()
    out_dtype = inp["out_dtype"] or inp["u"].dtype
    ys = []
    for t in range(steps):
        y = torch.empty((b, dim), dtype=out_dtype, device="cuda")
        col = lambda k: None if d[k] is None else d[k][..., t].contiguous()  # noqa: E731
        selscan.ss_step(col("u"), col("delta"), d["A"], col("B"), col("C"), state, y, D=d["D"], z=col("z"),
                        delta_bias=d["delta_bias"], delta_softplus=inp["delta_softplus"])
        ys.append(y)
    torch.cuda.synchronize()
    y_ref, last_ref = oracle.selective_scan(sl["u"], sl["delta"], sl["A"], sl["B"], sl["C"], D=sl["D"], z=sl["z"],
                                            delta_bias=sl["delta_bias"], delta_softplus=inp["delta_softplus"],
                                            return_last_state=True, initial_state=h0)
    assert_parity(torch.stack(ys, dim=-1), state, y_ref, last_ref,
                  1e-4 if inp["out_dtype"] else TOL[inp["u"].dtype], _case_name(inp, None, h0, None) + f" {steps} steps")


@pytest.mark.parametrize("seed", SEEDS)
def test_fuzz_dtproj_and_xdbl(seed):
    """The dt_proj form with a random rank, delta_r/B/C passed apart and
    read in place from one x_dbl tensor (bf16 only): against the oracle fed
    W_dt delta_r, and the two entries bit for bit."""
    rng = np.random.default_rng(9000 + seed)
    batch, dim, L = int(rng.integers(1, 4)), int(rng.integers(1, 49)), int(rng.integers(1, 601))
    N = int(rng.choice([1, 4, 8, 9, 16, 17, 32, 64]))
    R = int(rng.integers(1, 65))
    kw = dict(has_z=bool(rng.random() < 0.5), D_kind=str(rng.choice(["normal", "ones", "none"])),
              bias_kind=str(rng.choice(["normal", "uniform_dt", "none"])), return_last_state=True)
    w = W.custom(f"fuzzdt{seed}", batch, dim, L, N, torch.bfloat16, 9500 + seed, **kw)
    inp = W.make_dtproj_inputs(w, R)
    out_dtype = torch.float32 if rng.random() < 0.25 else torch.bfloat16
    d = to_dev(inp)
    ws = selscan.workspace_for(batch, dim, L, N, torch.bfloat16, out_dtype) if rng.random() < 0.5 else None
    y = torch.empty((batch, dim, L), dtype=out_dtype, device="cuda")
    last = torch.empty((batch, dim, N), device="cuda")
    selscan.ss_fwd_dtproj(d["u"], d["delta_r"], d["W_dt"], d["A"], d["B"], d["C"], y, D=d["D"], z=d["z"],
                          delta_bias=d["delta_bias"], delta_softplus=True, last_state=last, workspace=ws)
    x = torch.cat([d["delta_r"], d["B"], d["C"]], dim=1).contiguous()
    y2, last2 = torch.empty_like(y), torch.empty_like(last)
    selscan.ss_fwd_xdbl(d["u"], x, d["W_dt"], d["A"], y2, D=d["D"], z=d["z"], delta_bias=d["delta_bias"],
                        delta_softplus=True, last_state=last2, workspace=ws)
    torch.cuda.synchronize()
    y_ref, last_ref = oracle.selective_scan_dtproj(inp["u"], inp["delta_r"], inp["W_dt"], inp["A"], inp["B"],
                                                   inp["C"], D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"],
                                                   delta_softplus=True, return_last_state=True)
    what = f"{batch}x{dim}x{L} N={N} R={R} out={out_dtype} ws={ws is not None}"
    assert_parity(y, last, y_ref, last_ref, 1e-4 if out_dtype == torch.float32 else TOL[torch.bfloat16], what)
    assert torch.equal(y.view(torch.int16) if out_dtype == torch.bfloat16 else y,
                       y2.view(torch.int16) if out_dtype == torch.bfloat16 else y2) and torch.equal(last, last2), what
    assert selscan.ss_device_status() == 0


@pytest.mark.parametrize("seed", SEEDS)
def test_fuzz_host_buffers(seed):
    """The host-buffer forward pipelined over a random number of streams and
    batch ranges, against the oracle."""
    inp, _, _, _ = _draw(seed)
    rng = np.random.default_rng(9900 + seed)
    b, dim, L = inp["u"].shape
    N = inp["A"].shape[1]
    names = ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")
    host = {k: (inp[k].pin_memory() if inp[k] is not None else None) for k in names}
    out_dtype = inp["out_dtype"] or inp["u"].dtype
    host["y"] = torch.empty((b, dim, L), dtype=out_dtype).pin_memory()
    host["last_state"] = torch.empty((b, dim, N)).pin_memory()
    dev = {k: (torch.empty_like(inp[k], device="cuda") if inp[k] is not None else None) for k in names}
    dev["y"] = torch.empty((b, dim, L), dtype=out_dtype, device="cuda")
    dev["last_state"] = torch.empty((b, dim, N), device="cuda")
    nst = int(rng.integers(1, 5))
    streams = [torch.cuda.current_stream()] + [torch.cuda.Stream() for _ in range(nst - 1)]
    ws = torch.empty(nst * max(selscan.ss_fwd_workspace_bytes(b, dim, L, N, inp["u"].dtype, out_dtype), 1) + 4096,
                     dtype=torch.uint8, device="cuda")
    selscan.ss_fwd_hostio(host, dev, delta_softplus=inp["delta_softplus"], workspace=ws, streams=streams,
                          chunks=int(rng.integers(0, 2 * b + 1)))
    torch.cuda.synchronize()
    y_ref, last_ref = oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                                            z=inp["z"], delta_bias=inp["delta_bias"],
                                            delta_softplus=inp["delta_softplus"], return_last_state=True)
    assert_parity(host["y"], host["last_state"], y_ref, last_ref, 1e-4 if inp["out_dtype"] else TOL[inp["u"].dtype],
                  _case_name(inp, None, None, None) + f" streams={nst}")
