"""Run the forward of one named workload a few times, for a profiler.

    python -m selective_state_space_41_b200.run_workload NAME [--batch B]
        [--repeat K] [--lanes G] [--split S] [--warps W] [--segments P]
        [--dt-rank R] [--backward] [--backward-ckpt]

Draws the workload's seeded inputs (optionally only its first B batch
entries, to keep a capture small), moves them to ``cuda:0`` and calls
``ss_fwd`` (or ``ss_fwd_dtproj`` with ``--dt-rank``) K times in the launch
shape given, zeros meaning the heuristic's choice.  A workspace is passed
when the shape uses sequence segments.  ``--backward`` calls ``ss_bwd`` (all
gradients, a seeded dy, its own plan) K times instead; ``--backward-ckpt``
calls ``ss_fwd_ckpt`` once, then ``ss_bwd_ckpt`` from its checkpoints K
times.  Prints ``ok`` after a final synchronize.
"""
import argparse

import torch

from . import gen, selscan, workloads as W


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("name", choices=sorted(W.WORKLOADS))
    ap.add_argument("--batch", type=int, default=0)
    ap.add_argument("--repeat", type=int, default=3)
    ap.add_argument("--lanes", type=int, default=0)
    ap.add_argument("--split", type=int, default=0)
    ap.add_argument("--warps", type=int, default=0)
    ap.add_argument("--segments", type=int, default=0)
    ap.add_argument("--dt-rank", type=int, default=0)
    ap.add_argument("--backward", action="store_true")
    ap.add_argument("--backward-ckpt", action="store_true")
    a = ap.parse_args(argv)
    w = W.WORKLOADS[a.name]
    if a.batch:
        w = W.with_shape(w, batch=a.batch)
    inp = W.make_dtproj_inputs(w, a.dt_rank) if a.dt_rank else W.make_inputs(w)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    y = torch.empty(d["u"].shape, dtype=w.out_dtype or w.dtype, device="cuda")
    last = torch.empty((w.batch, w.dim, w.dstate), device="cuda") if w.return_last_state else None
    cfg = {}
    if a.lanes or a.split or a.warps or a.segments:
        cfg = dict(lanes_per_row=a.lanes, split_states=a.split, warps_per_block=a.warps, segments=a.segments)
    kw = dict(D=d["D"], z=d["z"], delta_bias=d["delta_bias"], delta_softplus=w.delta_softplus, last_state=last)
    if a.backward_ckpt:
        dy = gen.fill(tuple(inp["u"].shape), w.out_dtype or w.dtype, w.seed, 9).cuda()
        ck = torch.empty(selscan.ckpt_shape(w.batch, w.dim, w.seqlen, w.dstate), device="cuda")
        ws = selscan.workspace_for(w.batch, w.dim, w.seqlen, w.dstate, w.dtype, y.dtype)
        selscan.ss_fwd_ckpt(d["u"], d["delta"], d["A"], d["B"], d["C"], y, ck, workspace=ws, **kw)
        for _ in range(a.repeat):
            selscan.selective_scan_bwd(d["u"], d["delta"], d["A"], d["B"], d["C"], dy, D=d["D"], z=d["z"],
                                       delta_bias=d["delta_bias"], delta_softplus=w.delta_softplus, ckpt=ck)
    elif a.backward:
        dy = gen.fill(tuple(inp["u"].shape), w.out_dtype or w.dtype, w.seed, 9).cuda()
        for _ in range(a.repeat):
            selscan.selective_scan_bwd(d["u"], d["delta"], d["A"], d["B"], d["C"], dy, D=d["D"], z=d["z"],
                                       delta_bias=d["delta_bias"], delta_softplus=w.delta_softplus)
    elif a.dt_rank:
        ws = selscan.workspace_for(w.batch, w.dim, w.seqlen, w.dstate, w.dtype, y.dtype)
        for _ in range(a.repeat):
            selscan.ss_fwd_dtproj(d["u"], d["delta_r"], d["W_dt"], d["A"], d["B"], d["C"], y, workspace=ws, **kw)
    else:
        ws = selscan.workspace_for(w.batch, w.dim, w.seqlen, w.dstate, w.dtype, y.dtype, **cfg)
        for _ in range(a.repeat):
            selscan.ss_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], y, workspace=ws, **kw, **cfg)
    torch.cuda.synchronize()
    print("ok")


if __name__ == "__main__":
    main()
