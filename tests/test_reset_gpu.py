"""Sequence starts (ss_fwd_reset) through the C ABI against the fp64 oracle.

A nonzero reset[b, l] starts a new sequence at step l of every row of batch
entry b: the state entering step l is zero (the boundary reset of
"Mamba实战：如何用选择性状态空间模型提升你的长序列处理效率（附代码）" §2).  The
oracle's reset form is pinned on the CPU by the equality of a masked run with
independent runs of its pieces and by the memoryless closed form of a start
at every step.  Here: every direct-kernel shape, sequence segments with
starts on and around segment, stage and sub-chunk boundaries, the
heuristic's shapes, a dense mask, an all-zero mask (bitwise the plain
kernel), a rejected scan-kernel config, and sampled rows of the
mamba-130m-shaped layer cut into 512-step sequences."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import TOL, assert_parity, max_scaled_err, to_dev
from selective_state_space_41_b200 import gen, selscan, workloads as W

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

STATE_STREAM, RESET_STREAM = 8, 9  # Philox streams past the operands' 1..7


def _mask(batch, L, seed, starts=(), p=0.0):
    """(batch, L) uint8: the given starts in every batch entry, plus a seeded
    sparse draw with probability p per step."""
    m = np.zeros((batch, L), dtype=np.uint8)
    for l in starts:
        if 0 <= l < L:
            m[:, l] = 1
    if p > 0:
        r = gen.fill((batch, L), torch.float32, seed, RESET_STREAM, gen.UNIFORM, 0.0, 1.0).numpy()
        m |= (r < p).astype(np.uint8)
    return m


def _case(batch, dim, L, N, dtype, seed, state=True, **kw):
    inp = W.make_inputs(W.custom("reset", batch, dim, L, N, dtype, seed, **kw))
    inp["initial_state"] = (gen.fill((batch, dim, N), torch.float32, seed, STATE_STREAM, gen.NORMAL, 0.0, 2.0)
                            if state else None)
    return inp


def _oracle(inp, reset):
    return oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp.get("D"),
                                 z=inp.get("z"), delta_bias=inp.get("delta_bias"),
                                 delta_softplus=inp["delta_softplus"], return_last_state=True,
                                 initial_state=inp.get("initial_state"), reset=reset)


def _run(d, out_dtype, reset, workspace=True, **cfg):
    u = d["u"]
    batch, dim, L = u.shape
    N = d["A"].shape[1]
    y = torch.empty((batch, dim, L), dtype=out_dtype, device="cuda")
    last = torch.empty((batch, dim, N), dtype=torch.float32, device="cuda")
    ws = selscan.workspace_for(batch, dim, L, N, u.dtype, out_dtype, **cfg) if workspace else None
    r = None if reset is None else torch.as_tensor(reset).cuda()
    selscan.ss_fwd(u, d["delta"], d["A"], d["B"], d["C"], y, D=d.get("D"), z=d.get("z"),
                   delta_bias=d.get("delta_bias"), delta_softplus=d["delta_softplus"], last_state=last,
                   workspace=ws, initial_state=d.get("initial_state"), reset=r, **cfg)
    torch.cuda.synchronize()
    return y, last


# Starts at step 0 (overriding the initial state), on and beside 16-step
# sub-chunk and 64-step stage boundaries, and at the last step.
EDGE_STARTS = (0, 1, 15, 16, 17, 63, 64, 65, 128, 300, 516)

SHAPES = ([dict(lanes_per_row=1)] +
          [dict(lanes_per_row=g, split_states=True) for g in (2, 4, 8)] +
          [dict(lanes_per_row=g, split_states=True, warps_per_block=w) for g, w in ((4, 2), (2, 8))])


@pytest.mark.parametrize("cfg", SHAPES, ids=lambda c: "-".join(f"{k}{v}" for k, v in c.items()))
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_reset_every_direct_shape(cfg, dtype):
    inp = _case(2, 37, 517, 16, dtype, seed=7, has_z=True)
    reset = _mask(2, 517, seed=7, starts=EDGE_STARTS[1:], p=0.01)
    reset[1, 0] = 1  # batch entry 1 drops its initial state; entry 0 keeps it
    y, last = _run(to_dev(inp), dtype, reset, **cfg)
    y_ref, last_ref = _oracle(inp, reset)
    assert_parity(y, last, y_ref, last_ref, TOL[dtype], f"starts {cfg}")


@pytest.mark.parametrize("N", [4, 16, 33, 64])
def test_reset_state_buckets(N):
    inp = _case(2, 9, 300, N, torch.float32, seed=11 + N, has_z=True)
    reset = _mask(2, 300, seed=11, starts=(0, 64, 65, 299), p=0.02)
    y, last = _run(to_dev(inp), torch.float32, reset, lanes_per_row=2, split_states=True)
    y_ref, last_ref = _oracle(inp, reset)
    assert_parity(y, last, y_ref, last_ref, TOL[torch.float32], f"N={N}")


@pytest.mark.parametrize("seg_cfg", [dict(lanes_per_row=2, split_states=True, segments=3),
                                     dict(lanes_per_row=1, segments=4),
                                     dict(lanes_per_row=4, split_states=True, segments=5)],
                         ids=["g2s3", "g1s4", "g4s5"])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_reset_segments(seg_cfg, dtype):
    """Segments of 1408 / 1088 / 832 steps: starts exactly at, one before and
    one after segment starts, a segment with no start between two with
    starts, several starts in one segment; slow decay (small delta') so the
    carried state reaches far into each segment."""
    L = 4100
    inp = _case(2, 6, L, 16, dtype, seed=13, has_z=True, bias_kind="uniform_dt")
    seg_len = {3: 1408, 4: 1088, 5: 832}[seg_cfg["segments"]]
    starts = [seg_len, 2 * seg_len - 1, 2 * seg_len + 1, 2 * seg_len + 40, 2 * seg_len + 41]
    reset = _mask(2, L, seed=13, starts=starts)
    reset[1, min(3 * seg_len, L) - 5] = 1  # only batch entry 1: a start near the end of its third segment
    y, last = _run(to_dev(inp), dtype, reset, **seg_cfg)
    y_ref, last_ref = _oracle(inp, reset)
    assert_parity(y, last, y_ref, last_ref, TOL[dtype], f"segments {seg_cfg}")


def test_reset_heuristic_shapes():
    """No config: few rows and no workspace (the plain heuristic would take
    the scan kernel; with starts the rows run in the direct kernel), and the
    same with a workspace (sequence segments)."""
    inp = _case(1, 16, 9000, 16, torch.bfloat16, seed=17, has_z=False, bias_kind="none",
                return_last_state=True)
    assert selscan.ss_fwd_heuristic(1, 16, 9000, 16, torch.bfloat16)["split_states"] == 0
    reset = _mask(1, 9000, seed=17, starts=(0, 4096, 4097), p=0.001)
    d = to_dev(inp)
    y_ref, last_ref = _oracle(inp, reset)
    for ws in (False, True):
        y, last = _run(d, torch.bfloat16, reset, workspace=ws)
        assert_parity(y, last, y_ref, last_ref, TOL[torch.bfloat16], f"heuristic workspace={ws}")


def test_reset_dense_masks():
    """A start at every step (no memory at all) and at every other step."""
    inp = _case(2, 20, 130, 16, torch.float32, seed=19, has_z=True)
    d = to_dev(inp)
    for reset in (np.ones((2, 130), np.uint8), np.tile(np.array([1, 0], np.uint8), (2, 65))):
        y, last = _run(d, torch.float32, reset, lanes_per_row=4, split_states=True)
        y_ref, last_ref = _oracle(inp, reset)
        assert_parity(y, last, y_ref, last_ref, TOL[torch.float32], "dense starts")


@pytest.mark.parametrize("cfg", [dict(lanes_per_row=4, split_states=True),
                                 dict(lanes_per_row=2, split_states=True, segments=3)], ids=["g4", "g2s3"])
def test_reset_all_zero_is_bitwise_plain(cfg):
    """The reset instance with an all-zero mask does the plain instance's
    arithmetic: bitwise equal outputs."""
    inp = _case(2, 24, 4100, 16, torch.bfloat16, seed=23, has_z=True)
    d = to_dev(inp)
    y0, last0 = _run(d, torch.bfloat16, None, **cfg)
    y1, last1 = _run(d, torch.bfloat16, np.zeros((2, 4100), np.uint8), **cfg)
    assert torch.equal(y0, y1) and torch.equal(last0, last1)


def test_reset_scan_config_rejected():
    inp = _case(1, 4, 64, 4, torch.float32, seed=29)
    with pytest.raises(selscan.SelscanError) as e:
        _run(to_dev(inp), torch.float32, np.zeros((1, 64), np.uint8), lanes_per_row=4, split_states=False)
    assert e.value.status == 7


def test_reset_mamba130m_packed_sequences():
    """The mamba-130m-shaped layer (8 x 1536 x 2048 x 16, bf16, gate) cut into
    512-step sequences plus seeded extra starts, in the launch shape the
    heuristic picks: sampled rows against the oracle row by row."""
    w = W.WORKLOADS[W.MAMBA130M]
    inp = W.make_inputs(w)
    reset = _mask(w.batch, w.seqlen, seed=31, starts=range(0, w.seqlen, 512), p=0.002)
    d = to_dev(inp)
    y, last = _run(d, torch.bfloat16, reset)
    rows = [(0, 0), (3, 777), (7, 1535), (5, 1024)]
    for b, dd in rows:
        sl = lambda t: None if t is None else t[b:b + 1, dd:dd + 1]  # noqa: E731
        pd = lambda t: None if t is None else t[dd:dd + 1]  # noqa: E731
        y_ref, last_ref = oracle.selective_scan(sl(inp["u"]), sl(inp["delta"]), inp["A"][dd:dd + 1],
                                                inp["B"][b:b + 1], inp["C"][b:b + 1], D=pd(inp["D"]),
                                                z=sl(inp["z"]), delta_bias=pd(inp["delta_bias"]),
                                                delta_softplus=True, return_last_state=True,
                                                reset=reset[b:b + 1])
        assert max_scaled_err(y[b, dd], y_ref[0, 0]) <= TOL[torch.bfloat16], (b, dd)
        assert max_scaled_err(last[b, dd], last_ref[0, 0]) <= TOL[torch.bfloat16], (b, dd)
