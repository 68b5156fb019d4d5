"""Host-side logic of bench.py: byte accounting, the reference arm's JSON
line, and the multi-rank plumbing (world size 2 over gloo on the CPU)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from selective_state_space_41_b200 import workloads as W  # noqa: E402


def test_algorithmic_bytes_mamba130m():
    w = W.WORKLOADS[W.MAMBA130M]
    bdl = 8 * 1536 * 2048
    want = bdl * 8 + 2 * 8 * 16 * 2048 * 2 + 1536 * 16 * 4 + 1536 * 4 * 2
    assert bench.algorithmic_bytes(w) == want
    assert abs(want / 1e6 - 202.5) < 0.5


def test_algorithmic_bytes_genomic_counts_last_state():
    w = W.WORKLOADS[W.GENOMIC]
    bdl = 4 * 1024 * 100000
    want = bdl * 6 + 2 * 4 * 16 * 100000 * 2 + 1024 * 16 * 4 + 1024 * 4 + 4 * 1024 * 16 * 4
    assert bench.algorithmic_bytes(w) == want


def test_reference_arm_prints_one_line():
    env = dict(os.environ, RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3", "--workload", W.TINY],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "updates/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["config"]["workload"] == W.TINY


def test_reference_arm_other_ranks_do_nothing():
    env = dict(os.environ, RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True, env=env,
                       timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_warmup_below_three_rejected():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--warmup", "1"], capture_output=True, text=True, timeout=120)
    assert r.returncode != 0


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(WORLD_SIZE=str(world), RANK=str(rank), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench as b
    w, r, _ = b.dist_setup(None)
    assert (w, r) == (world, rank)
    b.barrier(w)
    m = b.max_over_ranks(float(rank + 1) * 1.5, w)
    seed = b.rank_workload(W.WORKLOADS[W.TINY], r).seed
    import torch.distributed as dist
    dist.destroy_process_group()
    q.put((rank, m, seed))


@pytest.mark.skipif(torch.cuda.is_available(), reason="gloo path runs where CUDA is absent")
def test_two_ranks_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [m for _, m, _ in res] == [3.0, 3.0]           # max over ranks
    assert res[0][2] != res[1][2]                          # independent problems per rank

