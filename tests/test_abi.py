"""The C-ABI library: it loads, exports every entry point the header declares,
and rejects bad arguments on the host, before any CUDA call (so these run
without a GPU: no pointer given here is ever dereferenced)."""
import ctypes
import os
import re
import types

import pytest

from selective_state_space_41_b200 import build, selscan

HEADER = os.path.join(build.INCLUDE, "selscan.h")


@pytest.fixture(scope="module")
def lib():
    build.build_selscan()
    return selscan.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\**\s*(ss_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_binding_exports():
    assert sorted(selscan.EXPORTS) == declared_functions()


def declared_arity():
    """Number of parameters of each function prototype in the header."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = {}
    for name, params in re.findall(r"^\s*(?:const\s+)?\w+\s*\**\s*(ss_\w+)\s*\(([^)]*)\)\s*;", text, flags=re.M):
        params = params.strip()
        out[name] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_argtypes_match_the_prototypes(lib):
    """Every ctypes signature the binding sets has as many arguments as the
    header's prototype (a wrong count fails only at call time, on a GPU)."""
    arity = declared_arity()
    assert sorted(arity) == declared_functions()
    for name, n in arity.items():
        assert len(getattr(lib, name).argtypes) == n, name


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} not exported"


def test_header_is_c_and_links(lib, tmp_path):
    """The header compiles as C99 with every warning an error, every function
    it declares resolves when a C program links the library, and the
    host-only calls answer from C."""
    import subprocess
    funcs = declared_functions()
    src = tmp_path / "uses_header.c"
    src.write_text(
        "#include <stdio.h>\n#include <string.h>\n#include \"selscan.h\"\n"
        "typedef void (*any_fn)(void);\n"
        "int main(void) {\n"
        "    any_fn fns[] = {" + ", ".join(f"(any_fn)&{f}" for f in funcs) + "};\n"
        "    for (size_t i = 0; i < sizeof fns / sizeof fns[0]; ++i)\n"
        "        if (!fns[i]) return 2;\n"
        "    if (ss_version() != SS_VERSION) return 3;\n"
        "    if (strlen(ss_status_string(SS_ERR_NULL_POINTER)) == 0) return 4;\n"
        "    printf(\"%d\\n\", ss_version());\n"
        "    return 0;\n"
        "}\n")
    exe = tmp_path / "uses_header"
    libdir = os.path.dirname(selscan.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", build.INCLUDE,
                    str(src), "-o", str(exe), "-L", libdir, "-lselscan", "-Wl,-rpath," + libdir],
                   check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    assert int(out) == lib.ss_version()


def test_version_and_strings(lib):
    assert selscan.ss_version() == 100
    for code, name in selscan.STATUS_NAMES.items():
        assert selscan.ss_status_string(code) and selscan.ss_status_string(code) != "unknown status"
    assert selscan.ss_status_string(99) == "unknown status"


def _desc(**kw):
    d = dict(batch=2, dim=3, seqlen=16, dstate=4, in_dtype=0, out_dtype=0)
    d.update(kw)
    return selscan.Desc(**d)


FAKE = ctypes.c_void_p(0x10000)      # 64 KiB-aligned, never dereferenced
ODD = ctypes.c_void_p(0x10001)       # not aligned to any element size


def _call(lib, desc, u=FAKE, delta=FAKE, A=FAKE, B=FAKE, C=FAKE, D=None, z=None, bias=None,
          y=FAKE, last=None):
    return lib.ss_fwd(ctypes.byref(desc) if desc is not None else None, u, delta, A, B, C, D, z,
                      bias, 1, y, last, None)


def test_rejections_before_any_launch(lib):
    assert _call(lib, None) == 1                                   # NULL descriptor
    assert _call(lib, _desc(seqlen=-1)) == 2                       # negative size
    assert _call(lib, _desc(batch=1 << 40, dim=1 << 40)) == 2      # overflow
    assert _call(lib, _desc(dstate=0)) == 4
    assert _call(lib, _desc(dstate=65)) == 4
    assert _call(lib, _desc(in_dtype=0, out_dtype=1)) == 3         # f32 -> bf16 not offered
    assert _call(lib, _desc(in_dtype=2)) == 3
    assert _call(lib, _desc(), u=None) == 1
    assert _call(lib, _desc(), A=None) == 1
    assert _call(lib, _desc(), y=None) == 1
    assert _call(lib, _desc(), u=ODD) == 5
    assert _call(lib, _desc(), D=ODD) == 5
    assert _call(lib, _desc(in_dtype=1, out_dtype=1), z=ctypes.c_void_p(0x10003)) == 5
    # empty problems need no pointers at all
    assert _call(lib, _desc(batch=0), u=None, delta=None, A=None, B=None, C=None, y=None) == 0
    assert _call(lib, _desc(seqlen=0), u=None, delta=None, B=None, C=None, y=None) == 0
    assert lib.ss_status_string(8) == b"workspace missing or too small"


def _cfg(lanes=0, split=0, warps=0, segments=0):
    return ctypes.byref(selscan.LaunchConfig(lanes, split, warps, segments))


def test_bad_launch_shapes_rejected(lib):
    # Every call here must be rejected before any launch: the pointers are fake.
    d = _desc(seqlen=4096)
    args = (ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, 1, FAKE, None)
    assert lib.ss_fwd_with_config(*args, _cfg(3, 0, 4), None, 0, None) == 7
    assert lib.ss_fwd_with_config(*args, _cfg(64, 0, 4), None, 0, None) == 7
    assert lib.ss_fwd_with_config(*args, _cfg(4, 0, 3), None, 0, None) == 7
    assert lib.ss_fwd_with_config(*args, _cfg(4, 2, 4), None, 0, None) == 7
    assert lib.ss_fwd_with_config(*args, _cfg(16, 1, 4), None, 0, None) == 7   # 16-way state split
    assert lib.ss_fwd_with_config(*args, _cfg(4, 0, 4, 3), None, 0, None) == 7  # segments need split
    assert lib.ss_fwd_with_config(*args, _cfg(segments=-1), None, 0, None) == 7
    assert lib.ss_fwd_with_config(*args, None, None, 0, None) == 1


def test_workspace_sizes(lib):
    """Workspace query: segments need (segments x rows x (N + 1)) floats."""
    d = _desc(batch=2, dim=3, seqlen=4096, dstate=4)
    assert lib.ss_fwd_workspace_bytes(ctypes.byref(d), _cfg(2, 1, 4, 1)) == 0
    # 4096 steps in about 4 segments of 1024 steps: 4 segments
    assert lib.ss_fwd_workspace_bytes(ctypes.byref(d), _cfg(2, 1, 4, 4)) == 4 * 6 * 5 * 4
    # 3 segments: 1366 rounded up to 1408 (a multiple of 64): 3 segments
    assert lib.ss_fwd_workspace_bytes(ctypes.byref(d), _cfg(1, 0, 4, 3)) == 3 * 6 * 5 * 4
    assert lib.ss_fwd_workspace_bytes(ctypes.byref(d), _cfg(4, 0, 4, 2)) == 0   # invalid: no split
    assert lib.ss_fwd_workspace_bytes(None, None) == 0


def test_segmented_call_without_workspace_rejected(lib):
    d = _desc(batch=2, dim=3, seqlen=4096, dstate=4)
    args = (ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, 1, FAKE, None)
    assert lib.ss_fwd_with_config(*args, _cfg(2, 1, 4, 4), None, 0, None) == 8
    assert lib.ss_fwd_with_config(*args, _cfg(2, 1, 4, 4), FAKE, 100, None) == 8


def test_noalloc_rejections_before_any_launch(lib):
    """ss_fwd_noalloc rejects a bad descriptor, and a launch shape needing
    more than the static scratch array, before any CUDA call."""
    args = (FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, 1, FAKE, None, None)
    assert lib.ss_fwd_noalloc(None, *args) == 1
    assert lib.ss_fwd_noalloc(ctypes.byref(_desc(dstate=0)), *args) == 4
    assert lib.ss_fwd_noalloc(ctypes.byref(_desc(in_dtype=0, out_dtype=1)), *args) == 3
    # 64 rows x 4M steps x 64 states: about 1025 segments, 17 MB of scratch
    big = _desc(batch=1, dim=64, seqlen=4_000_000, dstate=64)
    assert lib.ss_fwd_workspace_bytes(ctypes.byref(big), None) > selscan.NOALLOC_SCRATCH_BYTES
    assert lib.ss_fwd_noalloc(ctypes.byref(big), *args) == 9
    assert "scratch" in selscan.ss_status_string(9)


def test_noalloc_scratch_covers_the_genomic_layer(lib):
    """The figure the header gives for the 4 x 1024 x 100000, 16-state bf16
    layer is what ss_fwd_workspace_bytes reports for its default shape, and
    it fits the static scratch array."""
    d = _desc(batch=4, dim=1024, seqlen=100_000, dstate=16, in_dtype=1, out_dtype=1)
    n = lib.ss_fwd_workspace_bytes(ctypes.byref(d), None)
    assert n == 4_456_448
    assert n <= selscan.NOALLOC_SCRATCH_BYTES


def test_bwd_workspace_bounded_by_batch_groups(lib):
    """The backward's workspace grows with one batch group, not the batch: the
    16 x 4096 x 8192 layers stay under 8 GB at every state size, and a batch
    whose entries each fit alone needs no more than the whole batch would."""
    for n in (16, 32, 64):
        d = _desc(batch=16, dim=4096, seqlen=8192, dstate=n, in_dtype=1, out_dtype=1)
        assert 0 < lib.ss_bwd_workspace_bytes(ctypes.byref(d)) < 8_000_000_000, n
    one = lib.ss_bwd_workspace_bytes(ctypes.byref(_desc(batch=1, dim=4096, seqlen=8192, dstate=64,
                                                        in_dtype=1, out_dtype=1)))
    three = lib.ss_bwd_workspace_bytes(ctypes.byref(_desc(batch=3, dim=4096, seqlen=8192, dstate=64,
                                                          in_dtype=1, out_dtype=1)))
    assert one < three < 3 * one
    small = [lib.ss_bwd_workspace_bytes(ctypes.byref(_desc(batch=b, dim=1536, seqlen=2048, dstate=16,
                                                           in_dtype=1, out_dtype=1))) for b in (1, 8)]
    assert small[1] > 7 * small[0] - 8 * 4096   # small batches run whole: the workspace scales with B


def test_state_entry_rejections(lib):
    """ss_fwd_state: a misaligned initial state or a bad config is rejected
    before any launch."""
    d = _desc(seqlen=64, dstate=4)
    head = (ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, 1)
    assert lib.ss_fwd_state(*head, ODD, FAKE, None, None, None, 0, None) == 5
    assert lib.ss_fwd_state(*head, FAKE, FAKE, None, _cfg(3, 0, 4), None, 0, None) == 7
    assert lib.ss_fwd_state(None, *head[1:], FAKE, FAKE, None, None, None, 0, None) == 1


def test_reset_entry_rejections(lib):
    """ss_fwd_reset: no mask for a non-empty problem, a config asking for the
    scan kernel (which reads no sequence starts), a misaligned initial state
    and no descriptor are rejected before any launch; an empty problem needs
    no mask."""
    d = _desc(seqlen=64, dstate=4)
    head = (ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, 1)
    assert lib.ss_fwd_reset(*head, None, None, FAKE, None, None, None, 0, None) == 1
    assert lib.ss_fwd_reset(*head, FAKE, None, FAKE, None, _cfg(4, 0, 4), None, 0, None) == 7
    assert lib.ss_fwd_reset(*head, FAKE, ODD, FAKE, None, None, None, 0, None) == 5
    assert lib.ss_fwd_reset(None, *head[1:], FAKE, None, FAKE, None, None, None, 0, None) == 1
    empty = _desc(batch=0, seqlen=64, dstate=4)
    assert lib.ss_fwd_reset(ctypes.byref(empty), *head[1:], None, None, None, None, None, None, 0,
                            None) == 0


def test_reset_mask_checked_by_the_binding():
    """The binding rejects a start mask of the wrong shape or dtype before it
    calls the library (CPU tensors; nothing reaches a device)."""
    import torch
    t = torch.zeros(1, 2, 8)
    A, BC = torch.zeros(2, 4), torch.zeros(1, 4, 8)
    s0 = types.SimpleNamespace(cuda_stream=0)
    for bad in (torch.zeros(1, 7, dtype=torch.uint8), torch.zeros(2, 8, dtype=torch.uint8),
                torch.zeros(1, 8, dtype=torch.int32)):
        with pytest.raises(ValueError):
            selscan.ss_fwd(t, t, A, BC, BC, t, stream=s0, reset=bad)
        with pytest.raises(ValueError):
            selscan.ss_bwd(t, t, A, BC, BC, t, {"du": t, "ddelta": t, "dA": A, "dB": BC, "dC": BC},
                           workspace=torch.zeros(16, dtype=torch.uint8), stream=s0, reset=bad)


@pytest.mark.parametrize("shape,want", [
    # (B, D, L, N), (batch entries per launch, sequence segments) on 148 SMs
    ((8, 1536, 2048, 16), (8, 1)),        # mamba-130m-shaped layer: 384 blocks, whole batch
    ((4, 1024, 100000, 16), (4, 7)),      # genomic: 128 blocks -> 7 segments of 14 336 steps
    ((16, 4096, 8192, 16), (16, 1)),      # wide layers: groups within 7 GiB of workspace
    ((16, 4096, 8192, 32), (6, 1)),
    ((16, 4096, 8192, 64), (2, 1)),
    ((1, 8, 9000, 16), (1, 4)),           # few rows: segments capped at L / 2048
    ((1, 8, 4095, 16), (1, 1)),           # too short to cut
])
def test_bwd_plan(shape, want):
    """The backward's plan for the measured layers and the segment limits."""
    plan = selscan.ss_bwd_heuristic(*shape, selscan.SS_BF16)
    assert (plan["batch_group"], plan["segments"]) == want


def test_bwd_plan_rejections(lib):
    g, s = ctypes.c_int64(0), ctypes.c_int(0)
    assert lib.ss_bwd_heuristic(None, ctypes.byref(g), ctypes.byref(s)) == 1
    assert lib.ss_bwd_heuristic(ctypes.byref(_desc(dstate=65)), ctypes.byref(g), ctypes.byref(s)) == 4
    assert lib.ss_bwd_heuristic(ctypes.byref(_desc()), None, ctypes.byref(s)) == 1


def test_bwd_segment_records_in_the_workspace(lib):
    """A segmented plan adds its per-segment records to the unsegmented
    layout: the forward summary's end states and delta' sums ((N + 1) floats
    per piece and row; 4 segments of 2304 steps, each cut into four 576-step
    pieces), the adjoint summaries and their fold (2 N floats per segment and
    row), and per-segment row partials (N + 2)."""
    d = _desc(batch=1, dim=8, seqlen=9000, dstate=16, in_dtype=1, out_dtype=1)
    n = lib.ss_bwd_workspace_bytes(ctypes.byref(d))
    rows, N, segs, pieces, nsub = 8, 16, 4, 4, (9000 + 7) // 8
    base = rows * nsub * N * 4 + 1 * 2 * N * 9000 * 4   # checkpoints + one tile's dB/dC partials
    extra = segs * pieces * rows * (N + 1) * 4 + segs * rows * 2 * N * 4 + segs * rows * (N + 2) * 4
    assert base + extra <= n <= base + extra + 16 * 256  # 256-byte alignment of each region


@pytest.mark.parametrize("shape,ws,want", [
    # (B, D, L, N), workspace bytes, (lanes_per_row, split_states, warps_per_block, segments)
    ((8, 1536, 2048, 16), 0, (4, 1, 4, 1)),          # mamba-130m-shaped layer: measured best 4s/4
    ((4, 1024, 100000, 16), 1 << 30, (2, 1, 4, 16)),  # 100k genomic, with workspace: 2s/4, 16 segments
    ((16, 4096, 8192, 16), 0, (2, 1, 4, 1)),          # wide layers: 2s/4 at 16, 32 and 64 states
    ((16, 4096, 8192, 32), 0, (2, 1, 4, 1)),
    ((16, 4096, 8192, 64), 0, (2, 1, 4, 1)),
])
def test_heuristic_picks_the_measured_shapes(shape, ws, want):
    """The launch heuristic (host logic, 148 SMs when no device answers)
    chooses, for the benchmark workloads, the shapes the sweeps measured
    fastest on a B200."""
    import torch
    h = selscan.ss_fwd_heuristic(*shape, torch.bfloat16, workspace_bytes=ws)
    assert (h["lanes_per_row"], h["split_states"], h["warps_per_block"], h["segments"]) == want


def test_heuristic_genomic_without_workspace_and_its_workspace():
    """Without a workspace the 100k-step genomic layer takes the scan kernel;
    with one, 16 segments need nseg x rows x (N + 1) floats."""
    import torch
    h = selscan.ss_fwd_heuristic(4, 1024, 100000, 16, torch.bfloat16)
    assert h["split_states"] == 0 and h["segments"] == 1
    assert selscan.ss_fwd_workspace_bytes(4, 1024, 100000, 16, torch.bfloat16) == 16 * 4096 * 17 * 4


def test_ckpt_entry_rejections(lib):
    """The checkpoint entries reject before any launch (fake pointers): no
    checkpoint buffer, a misaligned one; the backward from checkpoints needs
    no checkpoint region in its workspace."""
    P = FAKE
    d = _desc(seqlen=64, dstate=16)
    fwd_head = (ctypes.byref(d), P, P, P, P, P, None, None, None, 1, None, None, P, None)
    assert lib.ss_fwd_ckpt(*fwd_head, None, None, 0, None) == 1
    assert lib.ss_fwd_ckpt(*fwd_head, ODD, None, 0, None) == 5
    grads = (P, P, P, P, P, None, None, None)
    bwd_head = (ctypes.byref(d), P, P, P, P, P, None, None, None, 1, None)
    assert lib.ss_bwd_ckpt(*bwd_head, None, None, P, *grads, None, None, 0, None) == 1
    assert lib.ss_bwd_ckpt(*bwd_head, ODD, None, P, *grads, None, None, 0, None) == 5
    assert lib.ss_bwd_ckpt(*bwd_head, P, None, P, *grads, None, None, 0, None) == 8   # no workspace
    for shape in ((8, 1536, 2048, 16), (4, 1024, 100000, 16), (1, 8, 9000, 64)):
        big = _desc(batch=shape[0], dim=shape[1], seqlen=shape[2], dstate=shape[3], in_dtype=1, out_dtype=1)
        full = lib.ss_bwd_workspace_bytes(ctypes.byref(big))
        ck = lib.ss_bwd_ckpt_workspace_bytes(ctypes.byref(big))
        rows, nsub = shape[0] * shape[1], -(-shape[2] // 8)
        assert 0 < ck < full and full - ck >= rows * nsub * shape[3] * 4 - 256, shape


def test_xdbl_entry_rejections(lib):
    """ss_fwd_xdbl rejects before any launch (fake pointers): dt_rank outside
    1..64, fp32 inputs, no x_dbl."""
    P = FAKE
    d = _desc(seqlen=64, dstate=16, in_dtype=1, out_dtype=1)
    tail = (P, P, P, P, None, None, None, 1, P, None, None, 0, None)   # u, x_dbl, W_dt, A, D, z, bias, sp, y, ...
    assert lib.ss_fwd_xdbl(ctypes.byref(d), 0, *tail) == 2
    assert lib.ss_fwd_xdbl(ctypes.byref(d), 65, *tail) == 2
    assert lib.ss_fwd_xdbl(ctypes.byref(_desc(seqlen=64, dstate=16)), 48, *tail) == 3
    assert lib.ss_fwd_xdbl(ctypes.byref(d), 48, P, None, P, P, None, None, None, 1, P, None, None, 0, None) == 1
    assert lib.ss_fwd_xdbl(None, 48, *tail) == 1


def test_bwd_rejections(lib):
    """ss_bwd rejects before any launch (the pointers are fake): no
    descriptor, more than 64 states, a missing gradient output, no workspace.
    Also goes through the binding's argument list once (its call is rejected
    on the state count before any pointer is used)."""
    P = FAKE
    args = (P, P, P, P, P, None, None, None, 1, P, P, P, P, P, P, None, None, None)
    assert lib.ss_bwd(None, *args, None, 0, None) == 1
    assert lib.ss_bwd(ctypes.byref(_desc(dstate=65)), *args, None, 0, None) == 4
    d = _desc(dstate=16)
    missing = (P, P, P, P, P, None, None, None, 1, P, None, P, P, P, P, None, None, None)
    assert lib.ss_bwd(ctypes.byref(d), *missing, None, 0, None) == 1
    withD = (P, P, P, P, P, P, None, None, 1, P, P, P, P, P, P, None, None, None)   # D without dD
    assert lib.ss_bwd(ctypes.byref(d), *withD, None, 0, None) == 1
    assert lib.ss_bwd(ctypes.byref(d), *args, None, 0, None) == 8
    assert lib.ss_bwd_workspace_bytes(ctypes.byref(d)) > 0
    assert lib.ss_bwd_workspace_bytes(ctypes.byref(_desc(dstate=64))) > 0
    assert lib.ss_bwd_workspace_bytes(ctypes.byref(_desc(dstate=65))) == 0
    import torch
    t = torch.zeros(1, 2, 4)
    with pytest.raises(selscan.SelscanError) as e:
        selscan.ss_bwd(t, t, torch.zeros(2, 65), torch.zeros(1, 65, 4), torch.zeros(1, 65, 4), t,
                       {"du": t, "ddelta": t, "dA": t, "dB": t, "dC": t},
                       workspace=torch.zeros(16, dtype=torch.uint8),
                       stream=types.SimpleNamespace(cuda_stream=0))
    assert e.value.status == 4


def test_bwd_reset_rejections(lib):
    """ss_bwd_reset: no mask for a non-empty problem, and the ss_bwd
    rejections, before any launch; the binding passes its mask through (the
    call is rejected on the state count before any pointer is used)."""
    P = FAKE
    head = (P, P, P, P, P, None, None, None, 1)
    tail = (P, P, P, P, P, P, None, None, None)
    d = _desc(dstate=16)
    assert lib.ss_bwd_reset(ctypes.byref(d), *head, None, *tail, None, 0, None) == 1
    assert lib.ss_bwd_reset(None, *head, P, *tail, None, 0, None) == 1
    assert lib.ss_bwd_reset(ctypes.byref(_desc(dstate=65)), *head, P, *tail, None, 0, None) == 4
    assert lib.ss_bwd_reset(ctypes.byref(d), *head, P, *tail, None, 0, None) == 8
    import torch
    t = torch.zeros(1, 2, 4)
    with pytest.raises(selscan.SelscanError) as e:
        selscan.ss_bwd(t, t, torch.zeros(2, 65), torch.zeros(1, 65, 4), torch.zeros(1, 65, 4), t,
                       {"du": t, "ddelta": t, "dA": t, "dB": t, "dC": t},
                       workspace=torch.zeros(16, dtype=torch.uint8),
                       stream=types.SimpleNamespace(cuda_stream=0), reset=torch.zeros(1, 4, dtype=torch.uint8))
    assert e.value.status == 4


def test_step_rejections(lib):
    """ss_step: one step only, required pointers, alignment; before any launch."""
    P = FAKE
    d = _desc(seqlen=1, dstate=16)
    args = (P, P, P, P, P, None, None, None, 1, P, P, None)
    assert lib.ss_step(ctypes.byref(_desc(seqlen=2)), *args) == 2
    assert lib.ss_step(ctypes.byref(d), P, P, P, P, P, None, None, None, 1, None, P, None) == 1
    assert lib.ss_step(ctypes.byref(d), P, P, P, P, P, None, None, None, 1, ODD, P, None) == 5
    assert lib.ss_step(ctypes.byref(_desc(seqlen=1, batch=0)), *args) == 0


def test_hostio_streams_rejections(lib):
    d = _desc()
    P = FAKE
    host = [P, P, P, P, P, None, None, None]
    dev = [P, P, P, P, P, None, None, None, P, None]
    streams = (ctypes.c_void_p * 2)(None, None)
    args = (ctypes.byref(d), *host, 1, P, None, *dev, None, 0)
    assert lib.ss_fwd_hostio_streams(*args, None, 2, 0) == 7
    assert lib.ss_fwd_hostio_streams(*args, streams, 0, 0) == 7
    assert lib.ss_fwd_hostio_streams(*args, streams, 17, 0) == 7
    assert lib.ss_fwd_hostio_streams(*args, streams, 2, -1) == 7
    assert lib.ss_fwd_hostio_streams(None, *args[1:], streams, 2, 0) == 1


def test_hostio_rejections(lib):
    d = _desc()
    P = FAKE
    base = [P, P, P, P, P, None, None, None]   # h_u h_delta h_A h_B h_C h_D h_z h_bias
    dev = [P, P, P, P, P, None, None, None, P, None]
    # D given on the host but not on the device
    base_d = [P, P, P, P, P, P, None, None]
    assert lib.ss_fwd_hostio(ctypes.byref(d), *base_d, 1, P, None, *dev, None, 0, None) == 1
    assert lib.ss_fwd_hostio(None, *base, 1, P, None, *dev, None, 0, None) == 1
