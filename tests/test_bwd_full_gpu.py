"""Backward at the full sizes of the long and wide layers, through the C ABI,
against the fp64 backward oracle on what it can compute in seconds:

* the 100 000-step genomic-shaped layer (4 x 1024 channels, 16 states; the
  (4, 100000) genomic input of "Mamba实战" §4.1), the whole layer on the GPU;
* one batch entry of the wide-state layer with 64 states (4096 channels x
  8192 steps, z gate, D ~ N(0, 1)).

Per-row gradients du, ddelta, dz are compared element by element on sampled
rows (each row's gradients depend only on its own inputs and the batch
entry's B, C); dA, dD per channel on sampled channels (the oracle over that
channel's rows of every batch entry); dB, dC element by element for one
whole batch entry (the oracle over all its channels).  Tolerances as in
test_bwd_gpu.py: per-row gradients |err| <= 2e-2 (1 + |ref|) for bf16
inputs; summed ones |err| <= 1e-3 (S + 1e-6 max S), S the sum of |terms|.
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_41_b200 import gen, selscan, workloads as W
from test_bwd_gpu import DY_STREAM, TOL_ELEM, TOL_SUM, check_summed

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _row_slice(inp, b, d):
    sl = lambda t: None if t is None else t[b:b + 1, d:d + 1]  # noqa: E731
    pd = lambda t: None if t is None else t[d:d + 1]  # noqa: E731
    return dict(u=sl(inp["u"]), delta=sl(inp["delta"]), A=inp["A"][d:d + 1], B=inp["B"][b:b + 1],
                C=inp["C"][b:b + 1], dy=sl(inp["dy"]), D=pd(inp["D"]), z=sl(inp["z"]),
                delta_bias=pd(inp["delta_bias"]))


def _channel_slice(inp, d):
    sl = lambda t: None if t is None else t[:, d:d + 1]  # noqa: E731
    pd = lambda t: None if t is None else t[d:d + 1]  # noqa: E731
    return dict(u=sl(inp["u"]), delta=sl(inp["delta"]), A=inp["A"][d:d + 1], B=inp["B"], C=inp["C"],
                dy=sl(inp["dy"]), D=pd(inp["D"]), z=sl(inp["z"]), delta_bias=pd(inp["delta_bias"]))


def _batch_slice(inp, b):
    sl = lambda t: None if t is None else t[b:b + 1]  # noqa: E731
    return dict(u=sl(inp["u"]), delta=sl(inp["delta"]), A=inp["A"], B=sl(inp["B"]), C=sl(inp["C"]),
                dy=sl(inp["dy"]), D=inp["D"], z=sl(inp["z"]), delta_bias=inp["delta_bias"])


def _oracle(p, softplus, magnitudes=False):
    return oracle.selective_scan_bwd(p["u"], p["delta"], p["A"], p["B"], p["C"], p["dy"], D=p["D"],
                                     z=p["z"], delta_bias=p["delta_bias"], delta_softplus=softplus,
                                     magnitudes=magnitudes)


def _oracle_dBdC(p, softplus):
    """dB, dC (and their sums of |terms|) of a one-batch-entry problem: the
    oracle (which runs the channels of a batch entry in one thread) over
    disjoint channel ranges on all host cores, the partial sums then added in
    range order."""
    import concurrent.futures
    import os
    dim = p["u"].shape[1]
    workers = max(1, min(os.cpu_count() or 1, dim))
    bounds = np.linspace(0, dim, workers + 1).astype(int)

    def part(i):
        lo, hi = bounds[i], bounds[i + 1]
        sl = lambda t: None if t is None else t[:, lo:hi]  # noqa: E731
        pd = lambda t: None if t is None else t[lo:hi]  # noqa: E731
        q = dict(u=sl(p["u"]), delta=sl(p["delta"]), A=p["A"][lo:hi], B=p["B"], C=p["C"], dy=sl(p["dy"]),
                 D=pd(p["D"]), z=sl(p["z"]), delta_bias=pd(p["delta_bias"]))
        r = oracle.selective_scan_bwd(q["u"], q["delta"], q["A"], q["B"], q["C"], q["dy"], D=q["D"],
                                      z=q["z"], delta_bias=q["delta_bias"], delta_softplus=softplus,
                                      magnitudes=True, nthreads=1)
        return {k: r[k] for k in ("dB", "dC", "mag_dB", "mag_dC")}

    with concurrent.futures.ThreadPoolExecutor(workers) as ex:
        parts = list(ex.map(part, [i for i in range(workers) if bounds[i] < bounds[i + 1]]))
    return {k: sum(q[k] for q in parts) for k in ("dB", "dC", "mag_dB", "mag_dC")}


def _full_size_check(w, rows, channels, batch_entry):
    inp = W.make_inputs(w)
    inp["dy"] = gen.fill(tuple(inp["u"].shape), w.dtype, w.seed, DY_STREAM)
    dev = torch.device("cuda")
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    got = selscan.selective_scan_bwd(d["u"], d["delta"], d["A"], d["B"], d["C"], d["dy"], D=d["D"],
                                     z=d["z"], delta_bias=d["delta_bias"], delta_softplus=w.delta_softplus)
    torch.cuda.synchronize()
    got = {k: (None if v is None else v.to("cpu", torch.float64).numpy()) for k, v in got.items()}
    del d
    torch.cuda.empty_cache()
    tol_e, tol_s = TOL_ELEM[w.dtype], TOL_SUM[w.dtype]
    for k, v in got.items():
        if v is not None:
            assert np.isfinite(v).all(), f"{w.name}: {k} not finite"
    # per-row gradients on sampled rows
    for (b, dd) in rows:
        ref = _oracle(_row_slice(inp, b, dd), w.delta_softplus)
        for k in ("du", "ddelta", "dz"):
            if ref[k] is None:
                assert got[k] is None
                continue
            e = np.abs(got[k][b, dd] - ref[k][0, 0]) / (1.0 + np.abs(ref[k][0, 0]))
            assert e.max() <= tol_e, f"{w.name} row ({b}, {dd}): {k} max |err|/(1+|ref|) = {e.max():.3e}"
    # dA, dD per sampled channel (every batch entry of that channel)
    for dd in channels:
        ref = _oracle(_channel_slice(inp, dd), w.delta_softplus, magnitudes=True)
        check_summed("dA", got["dA"][dd:dd + 1], ref["dA"], ref["mag_dA"], tol_s, f"{w.name} channel {dd}")
        if ref["dD"] is not None:
            check_summed("dD", got["dD"][dd:dd + 1], ref["dD"], ref["mag_dD"], tol_s, f"{w.name} channel {dd}")
    # dB, dC over one whole batch entry
    ref = _oracle_dBdC(_batch_slice(inp, batch_entry), w.delta_softplus)
    for k in ("dB", "dC"):
        check_summed(k, got[k][batch_entry:batch_entry + 1], ref[k], ref["mag_" + k], tol_s,
                     f"{w.name} batch entry {batch_entry}")


def test_bwd_genomic_full_length():
    """The 4 x 1024 x 100000, 16-state layer, whole on the GPU."""
    w = W.WORKLOADS[W.GENOMIC]
    _full_size_check(w, rows=[(0, 0), (1, 511), (2, 777), (3, 1023)], channels=[0, 333, 1023],
                     batch_entry=2)


def test_bwd_wide_state_n64_batch_entry():
    """One batch entry (4096 channels x 8192 steps) of the 64-state wide layer."""
    w = W.with_shape(W.WORKLOADS["wide_state_b16_d4096_l8192_n64"], batch=1)
    _full_size_check(w, rows=[(0, 0), (0, 2049), (0, 4095)], channels=[0, 1234, 4095], batch_entry=0)


def test_bwd_batch_groups_equal_per_entry_runs():
    """A batch whose backward workspace exceeds one group's budget runs in
    batch groups (here 3 entries of the 64-state wide layer: groups of 2 and
    1).  Every per-entry gradient equals, bit for bit, the backward of that
    entry alone, and dA, dD (summed over the batch in batch order) equal the
    per-entry sums added in that order."""
    w = W.with_shape(W.WORKLOADS["wide_state_b16_d4096_l8192_n64"], batch=3)
    one = selscan.ss_bwd_workspace_bytes(1, w.dim, w.seqlen, w.dstate, w.dtype)
    assert selscan.ss_bwd_workspace_bytes(3, w.dim, w.seqlen, w.dstate, w.dtype) < 3 * one
    inp = W.make_inputs(w)
    inp["dy"] = gen.fill(tuple(inp["u"].shape), w.dtype, w.seed, DY_STREAM)
    dev = torch.device("cuda")
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}

    def bwd(sl):
        return selscan.selective_scan_bwd(sl(d["u"]), sl(d["delta"]), d["A"], sl(d["B"]), sl(d["C"]), sl(d["dy"]),
                                          D=d["D"], z=sl(d["z"]), delta_bias=d["delta_bias"],
                                          delta_softplus=w.delta_softplus)

    whole = bwd(lambda t: t)
    parts = [bwd(lambda t, b=b: t[b:b + 1].contiguous()) for b in range(3)]
    torch.cuda.synchronize()
    for k in ("du", "ddelta", "dz", "dB", "dC"):
        for b in range(3):
            assert torch.equal(whole[k][b:b + 1], parts[b][k]), f"{k} entry {b}"
    for k in ("dA", "dD"):
        s = parts[0][k].clone()
        for b in (1, 2):
            s = s + parts[b][k]
        assert torch.equal(whole[k], s), k
