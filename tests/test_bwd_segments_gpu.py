"""Backward over sequence segments (few rows, long sequences: the segment
summaries, their folds and the segmented adjoint kernel) through the C ABI,
against the fp64 backward oracle.  Shapes are chosen so that the plan cuts
the sequence (asserted); tolerances as in test_bwd_gpu.py."""
import numpy as np
import pytest
import torch

from test_bwd_gpu import _case, _check, _check_state, _starts
from selective_state_space_41_b200 import selscan

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _segments(inp):
    batch, dim, L = inp["u"].shape
    return selscan.ss_bwd_heuristic(batch, dim, L, inp["A"].shape[1], inp["u"].dtype)["segments"]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("N", [4, 16, 33, 64])
def test_bwd_segments_state_sizes(dtype, N):
    """Every state bucket, 8 rows over 9000 steps (4 segments of 2304)."""
    inp = _case(1, 8, 9000, N, dtype, seed=N + 700, has_z=True)
    assert _segments(inp) == 4
    _check(inp, dtype, f"segments N={N}")


def test_bwd_segments_ragged_rows_and_length():
    """5003 steps (a partial last stage and sub-chunk), 5 channels (mirrored
    rows in the tile), two batch entries."""
    inp = _case(2, 5, 5003, 16, torch.bfloat16, seed=71, has_z=True, bias_kind="normal")
    assert _segments(inp) > 1
    _check(inp, torch.bfloat16, "segments, ragged")


@pytest.mark.parametrize("softplus", [True, False])
def test_bwd_segments_long_memory(softplus):
    """delta' near 0 (bias -7 under softplus; exp mode with small delta): the
    state and the adjoint carry across whole segments, so the folds matter."""
    inp = _case(1, 8, 9000, 16, torch.float32, seed=73, has_z=True, delta_softplus=softplus)
    if softplus:
        inp["delta_bias"] = torch.full((8,), -7.0)
    else:
        inp["delta"] = (inp["delta"] * 0.5 - 8.0).contiguous()
    assert _segments(inp) == 4
    _check(inp, torch.float32, f"segments, long memory (softplus={softplus})")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_bwd_segments_starts(dtype):
    """Sequence starts on and beside the segment boundaries (2304, 4608,
    6912), at step 0 of one batch entry, at the last step, and seeded ones."""
    inp = _case(2, 8, 9000, 16, dtype, seed=79, has_z=True)
    assert _segments(inp) == 4
    reset = _starts(2, 9000, seed=79, fixed=(2303, 2304, 4608, 4609, 6911, 8999), p=0.0005)
    reset[0, 0] = 1
    _check(inp, dtype, "segments with starts", reset=reset)


def test_bwd_segments_segment_without_start_between_starts():
    """Starts only in the first and last segments: the middle segments pass
    state and adjoint on (P > 0) while the outer ones cut them."""
    inp = _case(1, 8, 9000, 16, torch.float32, seed=83, has_z=False, bias_kind="zeros")
    inp["delta_bias"] = torch.full((8,), -5.0)
    reset = np.zeros((1, 9000), np.uint8)
    reset[0, 1000] = 1
    reset[0, 8000] = 1
    _check(inp, torch.float32, "segments, starts in the outer segments", reset=reset)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_bwd_segments_initial_state(dtype):
    """From a given state with a last-state gradient: the initial-state
    gradient comes out of segment 0 after the adjoint fold."""
    inp = _case(1, 8, 9000, 16, dtype, seed=89, has_z=True)
    inp["delta_bias"] = torch.full((8,), -4.0)  # carries reach across segments
    assert _segments(inp) == 4
    _check_state(inp, dtype, "segments, h0 and dlast", seed=89)


def test_bwd_segments_initial_state_with_starts():
    inp = _case(2, 8, 9000, 16, torch.float32, seed=97, has_z=True)
    reset = _starts(2, 9000, seed=97, fixed=(2304, 7000), p=0.0002)
    _check_state(inp, torch.float32, "segments, h0 + starts", reset=reset, seed=97)
