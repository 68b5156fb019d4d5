"""CUDA path (through the C ABI) against the fp64 oracle, element by element,
on the same seeded inputs.  Tolerance: max |err| <= tol * (1 + |y|) with tol
1e-5 for fp32 inputs and 1e-2 for bf16 inputs (fp32 state and accumulation)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import TOL, assert_parity, run_gpu, run_oracle
from selective_state_space_41_b200 import selscan, workloads as W

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _case(batch, dim, L, N, dtype=torch.float32, seed=1, **kw):
    return W.make_inputs(W.custom("case", batch, dim, L, N, dtype, seed, **kw))


# ---------------------------------------------------------------- workloads
@pytest.mark.parametrize("name", ["tiny_fp32_b4_d16_l64_n32", "fp32_b32_d128_l256_n16"])
def test_small_workloads_full(name):
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w)
    y, last = run_gpu(inp)
    y_ref, last_ref = run_oracle(inp)
    assert_parity(y, last, y_ref, last_ref if inp["return_last_state"] else None, TOL[w.dtype], name)


def test_mamba130m_one_batch_full():
    """Every output of one batch entry of the mamba-130m-shaped layer."""
    w = W.with_shape(W.WORKLOADS[W.MAMBA130M], batch=1)
    inp = W.make_inputs(w)
    y, last = run_gpu(inp)
    y_ref, _ = run_oracle(inp)
    assert_parity(y, None, y_ref, None, TOL[w.dtype], w.name)


def _sample_rows(w, k, seed):
    rng = np.random.default_rng(seed)
    rows = {(0, 0), (w.batch - 1, w.dim - 1), (0, w.dim - 1), (w.batch - 1, 0)}
    for d in (31, 32, 63, 64, 127, 128):  # block and warp edges of the row tiles
        if d < w.dim:
            rows.add((int(rng.integers(w.batch)), d))
    while len(rows) < k:
        rows.add((int(rng.integers(w.batch)), int(rng.integers(w.dim))))
    return sorted(rows)


@pytest.mark.parametrize("name", [W.MAMBA130M, W.GENOMIC, "wide_state_b16_d4096_l8192_n16",
                                  "wide_state_b16_d4096_l8192_n32",
                                  "wide_state_b16_d4096_l8192_n64"])
def test_full_size_sampled_rows(name):
    """Full-size workload in the launch shape the benchmark uses; sampled
    rows against the oracle row by row, every output checked finite."""
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w)
    y, last = run_gpu(inp)
    assert torch.isfinite(y.float()).all()
    rows = _sample_rows(w, 24, w.seed)
    y_ref, last_ref = oracle.selective_scan_rows(inp, rows)
    idx_b = torch.tensor([r[0] for r in rows])
    idx_d = torch.tensor([r[1] for r in rows])
    y_rows = y[idx_b.cuda(), idx_d.cuda()]
    last_rows = last[idx_b.cuda(), idx_d.cuda()] if last is not None else None
    assert_parity(y_rows, last_rows, y_ref, last_ref, TOL[w.dtype], name)
    del y, last
    torch.cuda.empty_cache()


def test_over_2g_elements_per_tensor():
    """A layer with more than 2^31 elements per (batch, dim, L) tensor
    (1 x 1024 x 2.1M steps, bf16, 16 states): 64-bit offsets throughout,
    the segmented shape over a 2.1M-step sequence and its fix-up; rows at
    both ends and the middle against the oracle.  Inputs are drawn on the
    device from a seeded generator (no host copy of the whole layer)."""
    D, L, N = 1024, 2_100_000, 16
    assert D * L > 2**31
    g = torch.Generator(device="cuda").manual_seed(4107)
    u = torch.randn((1, D, L), generator=g, device="cuda").to(torch.bfloat16)
    delta = torch.randn((1, D, L), generator=g, device="cuda").to(torch.bfloat16)
    B = torch.randn((1, N, L), generator=g, device="cuda").to(torch.bfloat16)
    C = torch.randn((1, N, L), generator=g, device="cuda").to(torch.bfloat16)
    A = -torch.arange(1, N + 1, dtype=torch.float32, device="cuda").repeat(D, 1).contiguous()
    Dv = torch.ones(D, device="cuda")
    y = torch.empty((1, D, L), dtype=torch.bfloat16, device="cuda")
    last = torch.empty((1, D, N), dtype=torch.float32, device="cuda")
    ws = selscan.workspace_for(1, D, L, N, torch.bfloat16)
    assert ws is not None   # the segmented shape
    selscan.ss_fwd(u, delta, A, B, C, y, D=Dv, delta_softplus=True, last_state=last, workspace=ws)
    torch.cuda.synchronize()
    rows = [0, 511, D - 1]
    host = {"u": u[:, rows].cpu(), "delta": delta[:, rows].cpu(), "A": A[rows].cpu(), "B": B.cpu(),
            "C": C.cpu(), "D": Dv[rows].cpu()}
    y_ref, last_ref = oracle.selective_scan(host["u"], host["delta"], host["A"], host["B"], host["C"],
                                            D=host["D"], delta_softplus=True, return_last_state=True)
    assert_parity(y[:, rows], last[:, rows], y_ref, last_ref, TOL[torch.bfloat16], "2^31+ elements")
    del u, delta, B, C, y, last, ws
    torch.cuda.empty_cache()


# ---------------------------------------------------------------- edge cases
@pytest.mark.parametrize("L", [1, 2, 7, 8, 9, 63, 64, 65, 255, 257, 1000, 1003])
def test_ragged_lengths(L):
    for dtype in (torch.float32, torch.bfloat16):
        inp = _case(3, 5, L, 16, dtype, seed=L, has_z=True, return_last_state=True)
        y, last = run_gpu(inp)
        y_ref, last_ref = run_oracle(inp)
        assert_parity(y, last, y_ref, last_ref, TOL[dtype], f"L={L} {dtype}")


@pytest.mark.parametrize("N", [1, 2, 3, 4, 5, 8, 9, 15, 16, 17, 31, 32, 33, 48, 63, 64])
def test_state_sizes(N):
    inp = _case(2, 7, 130, N, torch.float32, seed=100 + N, has_z=(N % 2 == 0),
                return_last_state=True)
    y, last = run_gpu(inp)
    y_ref, last_ref = run_oracle(inp)
    assert_parity(y, last, y_ref, last_ref, TOL[torch.float32], f"N={N}")


@pytest.mark.parametrize("dim", [1, 3, 31, 33, 129])
def test_channel_counts(dim):
    inp = _case(2, dim, 77, 16, torch.bfloat16, seed=dim, return_last_state=True)
    y, last = run_gpu(inp)
    y_ref, last_ref = run_oracle(inp)
    assert_parity(y, last, y_ref, last_ref, TOL[torch.bfloat16], f"dim={dim}")


@pytest.mark.parametrize("has_z", [False, True])
@pytest.mark.parametrize("D_kind", ["none", "normal"])
@pytest.mark.parametrize("bias_kind", ["none", "normal"])
@pytest.mark.parametrize("softplus", [False, True])
@pytest.mark.parametrize("last", [False, True])
def test_optional_operands(has_z, D_kind, bias_kind, softplus, last):
    inp = _case(2, 6, 96, 8, torch.float32, seed=7, has_z=has_z, D_kind=D_kind,
                bias_kind=bias_kind, delta_softplus=softplus, return_last_state=last)
    if not softplus:  # keep exp(delta + bias) in a sane range
        inp["delta"] = inp["delta"] * 0.5 - 1.0
    y, lst = run_gpu(inp)
    y_ref, last_ref = run_oracle(inp)
    assert_parity(y, lst, y_ref, last_ref if last else None, TOL[torch.float32], "flags")


def test_bf16_in_f32_out():
    inp = _case(2, 9, 300, 16, torch.bfloat16, seed=3, has_z=True, return_last_state=True)
    y, last = run_gpu(inp, out_dtype=torch.float32)
    assert y.dtype == torch.float32
    y_ref, last_ref = run_oracle(inp)
    # fp32 output of bf16 inputs: only the fp32 arithmetic rounds
    assert_parity(y, last, y_ref, last_ref, 1e-4, "bf16->f32")


SHAPES = ([(w, False) for w in (1, 2, 4, 8, 16, 32)] + [(2, True), (4, True), (8, True)])


@pytest.mark.parametrize("lanes,split", SHAPES)
@pytest.mark.parametrize("warps", [1, 2, 4, 8])
def test_every_launch_shape(lanes, split, warps):
    inp = _case(2, 37, 517, 16, torch.float32, seed=lanes * 10 + warps, has_z=True,
                return_last_state=True)
    y, last = run_gpu(inp, lanes=lanes, warps=warps, split=split)
    y_ref, last_ref = run_oracle(inp)
    assert_parity(y, last, y_ref, last_ref, TOL[torch.float32],
                  f"lanes={lanes} split={split} warps={warps}")


@pytest.mark.parametrize("N", [4, 8, 9, 16, 33, 64])
@pytest.mark.parametrize("lanes", [2, 4, 8])
def test_state_split_shapes(N, lanes):
    """The state split over 2, 4 or 8 lanes, bf16, ragged length and channels."""
    bucket = 4 if N <= 4 else 8 if N <= 8 else 16 if N <= 16 else 32 if N <= 32 else 64
    if bucket // 2 < lanes:
        pytest.skip("fewer state pairs than lanes")
    inp = _case(2, 19, 203, N, torch.bfloat16, seed=N * 7 + lanes, has_z=True,
                return_last_state=True)
    y, last = run_gpu(inp, lanes=lanes, warps=2, split=True)
    y_ref, last_ref = run_oracle(inp)
    assert_parity(y, last, y_ref, last_ref, TOL[torch.bfloat16], f"N={N} lanes={lanes} split")


# ---------------------------------------------------------------- segments
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("L,segments", [(4096, 2), (3001, 3), (5000, 7), (640, 4), (129, 2)])
@pytest.mark.parametrize("lanes,split", [(1, False), (2, True), (4, True)])
def test_sequence_segments(dtype, L, segments, lanes, split):
    """Segments run from a zero state plus the fix-up of the carried state."""
    inp = _case(2, 5, L, 16, dtype, seed=L + segments + lanes, has_z=True, return_last_state=True)
    y, last = run_gpu(inp, lanes=lanes, split=split, warps=2, segments=segments)
    y_ref, last_ref = run_oracle(inp)
    assert_parity(y, last, y_ref, last_ref, TOL[dtype], f"L={L} segments={segments} lanes={lanes}")


def test_segments_long_memory():
    """delta' tiny (long memory: the carried state never decays to 0, so the
    fix-up runs through whole segments) and exp mode with large delta' (fast
    decay), each segmented."""
    inp = _case(1, 6, 2500, 8, torch.float32, seed=11, has_z=False, return_last_state=True)
    slow = dict(inp, delta=inp["delta"] * 0.1 - 7.0)            # softplus(-7) ~ 1e-3
    y, last = run_gpu(slow, lanes=2, split=True, warps=1, segments=5)
    y_ref, last_ref = run_oracle(slow)
    assert_parity(y, last, y_ref, last_ref, TOL[torch.float32], "slow decay")
    fast = dict(inp, delta=inp["delta"] * 0.3 + 1.0, delta_softplus=False)
    y, last = run_gpu(fast, lanes=2, split=True, warps=1, segments=5)
    y_ref, last_ref = run_oracle(fast)
    assert_parity(y, last, y_ref, last_ref, TOL[torch.float32], "fast decay")


def test_segments_bf16_carry_dominated():
    """bf16 output where, after the first segment, y is mostly the carried
    state's share: u large over the first 1000 steps and 1/64 of it after,
    slow decay (delta' ~ 1e-3), no skip term.  The fix-up adds a share that is
    large against the segment kernel's own (rounded) value, so y is rounded
    twice where that matters; the 1e-2 (1 + |y|) bound still holds."""
    inp = _case(2, 6, 4000, 16, torch.bfloat16, seed=29, has_z=True, D_kind="none", return_last_state=True)
    u = inp["u"].float()
    u[..., 1000:] *= 1.0 / 64
    inp["u"] = u.to(torch.bfloat16)
    inp["delta"] = (inp["delta"].float() * 0.1 - 7.0).to(torch.bfloat16)
    for segs in (3, 4):
        y, last = run_gpu(inp, lanes=2, split=True, warps=1, segments=segs)
        y_ref, last_ref = run_oracle(inp)
        assert_parity(y, last, y_ref, last_ref, TOL[torch.bfloat16], f"carry-dominated, {segs} segments")


def test_heuristic_segments_genomic_shape():
    """The genomic shape segments when given a workspace, and not without one."""
    h_ws = selscan.ss_fwd_heuristic(4, 1024, 100000, 16, torch.bfloat16, workspace_bytes=1 << 30)
    h_no = selscan.ss_fwd_heuristic(4, 1024, 100000, 16, torch.bfloat16)
    assert h_ws["segments"] > 1 and h_no["segments"] == 1


def test_unaligned_rows_take_the_scalar_path():
    """Pointers offset by one element (still element-aligned) and an odd L:
    the kernel must fall back from 16-byte vectors and still be exact."""
    inp = _case(2, 4, 64, 4, torch.bfloat16, seed=5, has_z=True, return_last_state=True)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    shifted = {}
    for k in ("u", "delta", "B", "C", "z"):
        buf = torch.empty(d[k].numel() + 1, dtype=d[k].dtype, device="cuda")
        buf[1:].copy_(d[k].reshape(-1))
        shifted[k] = buf[1:].view(d[k].shape)
        assert shifted[k].data_ptr() % 16 != 0
    y = torch.empty_like(d["u"])
    last = torch.empty(2, 4, 4, dtype=torch.float32, device="cuda")
    selscan.ss_fwd(shifted["u"], shifted["delta"], d["A"], shifted["B"], shifted["C"], y, D=d["D"],
                   z=shifted["z"], delta_bias=d["delta_bias"], delta_softplus=True, last_state=last)
    torch.cuda.synchronize()
    y_ref, last_ref = run_oracle(inp)
    assert_parity(y, last, y_ref, last_ref, TOL[torch.bfloat16], "unaligned")


def test_large_decay_and_tiny_delta():
    """Large delta' (every decay underflows to 0: y = C.(delta' B u) + D u) and
    delta' -> 0 (no state movement: y = D u)."""
    for shift in (8.0, -60.0):
        inp = _case(1, 4, 50, 16, torch.float32, seed=9, return_last_state=True)
        inp["delta"] = inp["delta"] * 0.1 + shift
        y, last = run_gpu(inp)
        y_ref, last_ref = run_oracle(inp)
        assert_parity(y, last, y_ref, last_ref, TOL[torch.float32], f"shift={shift}")


def test_hand_worked_example_fp32():
    """The golden hand-worked example, run on the GPU in fp32."""
    import json, math, os  # noqa: E401
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")))
    i = g["inputs"]
    f = lambda x: torch.tensor(x, dtype=torch.float32)  # noqa: E731
    inp = dict(u=f(i["u"]), delta=f(i["delta_softplus_mode"]), A=f(i["A"]),
               B=f(i["B_times_ln2"]) / math.log(2.0), C=f(i["C"]), D=f(i["D"]), z=None,
               delta_bias=None, delta_softplus=True, return_last_state=True)
    y, last = run_gpu(inp)
    assert_parity(y, last, np.array(g["expected"]["y"]), np.array(g["expected"]["last_state"]),
                  TOL[torch.float32], "hand-worked")


# ---------------------------------------------------------------- degenerate
def test_empty_sequence_writes_zero_state():
    inp = _case(2, 3, 0, 5, torch.float32, return_last_state=True)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    last = torch.full((2, 3, 5), 7.0, device="cuda")
    y = torch.empty((2, 3, 0), device="cuda")
    selscan.ss_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], y, D=d["D"], last_state=last,
                   delta_softplus=True)
    torch.cuda.synchronize()
    assert torch.all(last == 0)


def test_no_rows_is_a_no_op():
    inp = _case(0, 3, 10, 4, torch.float32)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    y = torch.empty((0, 3, 10), device="cuda")
    selscan.ss_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], y, delta_softplus=True)
    torch.cuda.synchronize()


def test_bitwise_deterministic():
    inp = W.make_inputs(W.with_shape(W.WORKLOADS[W.MAMBA130M], batch=2, dim=256))
    y1, _ = run_gpu(inp)
    y2, _ = run_gpu(inp)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_hostio_matches_device_path():
    w = W.with_shape(W.WORKLOADS[W.GENOMIC], dim=64, seqlen=5000)
    inp = W.make_inputs(w, pin=True)
    y_dev, last_dev = run_gpu(inp)
    host = {k: inp[k] for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}
    host["y"] = torch.empty(y_dev.shape, dtype=y_dev.dtype).pin_memory()
    host["last_state"] = torch.empty(last_dev.shape, dtype=torch.float32).pin_memory()
    dev = {k: (torch.empty_like(v, device="cuda") if v is not None else None)
           for k, v in host.items()}
    ws = selscan.workspace_for(w.batch, w.dim, w.seqlen, w.dstate, w.dtype)  # as run_gpu
    selscan.ss_fwd_hostio(host, dev, delta_softplus=True, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(host["y"].view(torch.int16), y_dev.cpu().view(torch.int16))
    assert torch.equal(host["last_state"], last_dev.cpu())


@pytest.mark.parametrize("nstreams,chunks", [(1, 0), (2, 0), (3, 5), (2, 1)])
def test_hostio_streams_against_oracle(nstreams, chunks):
    """The host-buffer form pipelined over streams by batch ranges (ragged
    ranges: 5 batch entries), two calls in a row on different inputs."""
    streams = [torch.cuda.Stream() for _ in range(nstreams)]
    for seed in (61, 62):
        inp = _case(5, 40, 700, 16, torch.bfloat16, seed=seed, has_z=True, return_last_state=True)
        host = {k: (inp[k].pin_memory() if inp[k] is not None else None)
                for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}
        host["y"] = torch.empty((5, 40, 700), dtype=torch.bfloat16).pin_memory()
        host["last_state"] = torch.empty((5, 40, 16), dtype=torch.float32).pin_memory()
        dev = {k: (torch.empty_like(v, device="cuda") if v is not None else None) for k, v in host.items()}
        ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
        selscan.ss_fwd_hostio(host, dev, delta_softplus=True, workspace=ws, streams=streams, chunks=chunks)
        for st in streams:
            st.synchronize()
        y_ref, last_ref = run_oracle(inp)
        assert_parity(host["y"], host["last_state"], y_ref, last_ref, TOL[torch.bfloat16],
                      f"streams={nstreams} chunks={chunks} seed={seed}")


def test_hostio_streams_segmented_ranges():
    """Few rows and a long sequence: every batch range runs the segmented
    shape inside its stream's share of the workspace."""
    streams = [torch.cuda.Stream() for _ in range(2)]
    inp = _case(3, 16, 6000, 16, torch.float32, seed=71, has_z=True, return_last_state=True)
    assert selscan.ss_fwd_heuristic(1, 16, 6000, 16, torch.float32, workspace_bytes=1 << 19)["segments"] > 1
    host = {k: (inp[k].pin_memory() if inp[k] is not None else None)
            for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}
    host["y"] = torch.empty((3, 16, 6000), dtype=torch.float32).pin_memory()
    host["last_state"] = torch.empty((3, 16, 16), dtype=torch.float32).pin_memory()
    dev = {k: (torch.empty_like(v, device="cuda") if v is not None else None) for k, v in host.items()}
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    selscan.ss_fwd_hostio(host, dev, delta_softplus=True, workspace=ws, streams=streams)
    for st in streams:
        st.synchronize()
    y_ref, last_ref = run_oracle(inp)
    assert_parity(host["y"], host["last_state"], y_ref, last_ref, TOL[torch.float32], "segmented ranges")


def test_convenience_wrapper():
    inp = _case(2, 4, 33, 16, torch.bfloat16, seed=2, has_z=True, return_last_state=True)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    y, last = selscan.selective_scan_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], D=d["D"],
                                         z=d["z"], delta_bias=d["delta_bias"],
                                         delta_softplus=True, return_last_state=True)
    torch.cuda.synchronize()
    y_ref, last_ref = run_oracle(inp)
    assert_parity(y, last, y_ref, last_ref, TOL[torch.bfloat16], "wrapper")
