"""Seeded input generator: Philox4x32-10 known answers, determinism, stream
independence, distribution sanity and bf16 rounding."""
import numpy as np
import pytest
import torch

from selective_state_space_41_b200 import gen, workloads


def test_philox_known_answers():
    # Known-answer vectors published with the Random123 library (Salmon et al., SC'11).
    kat = [
        ([0, 0, 0, 0], [0, 0], [0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8]),
        ([0xFFFFFFFF] * 4, [0xFFFFFFFF] * 2, [0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD]),
        ([0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344], [0xA4093822, 0x299F31D0],
         [0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1]),
    ]
    for ctr, key, want in kat:
        assert gen.philox4x32_10(ctr, key) == want


def test_deterministic_and_thread_independent():
    a = gen.fill((1001,), torch.float32, 42, 3, nthreads=1)
    b = gen.fill((1001,), torch.float32, 42, 3, nthreads=4)
    assert torch.equal(a, b)
    c = gen.fill((1001,), torch.float32, 42, 4)
    assert not torch.equal(a, c)
    # element i does not depend on the tensor's length
    d = gen.fill((37,), torch.float32, 42, 3)
    assert torch.equal(a[:37], d)


def test_normal_and_uniform_moments():
    x = gen.fill((400000,), torch.float32, 9, 1).double()
    assert abs(x.mean().item()) < 0.01 and abs(x.std().item() - 1) < 0.01
    assert abs(((x - x.mean()) ** 3).mean().item()) < 0.03
    y = gen.fill((400000,), torch.float32, 9, 2, gen.NORMAL, 3.0, 0.5).double()
    assert abs(y.mean().item() - 3) < 0.01 and abs(y.std().item() - 0.5) < 0.01
    w = gen.fill((400000,), torch.float32, 9, 3, gen.UNIFORM, -2.0, 5.0).double()
    assert w.min().item() >= -2.0 and w.max().item() < 5.0
    assert abs(w.mean().item() - 1.5) < 0.02


def test_bf16_is_round_to_nearest_even_of_the_f32_draw():
    f = gen.fill((100000,), torch.float32, 5, 1)
    b = gen.fill((100000,), torch.bfloat16, 5, 1)
    assert torch.equal(f.to(torch.bfloat16).view(torch.int16), b.view(torch.int16))
    # ties: 1 + 2^-8 is halfway between bf16 neighbours 1 and 1 + 2^-7 -> even (1.0)
    assert gen.f32_to_bf16_bits(1.0 + 2.0 ** -8) == 0x3F80
    assert gen.f32_to_bf16_bits(1.0 + 3 * 2.0 ** -8) == 0x3F82


def test_workload_recipes():
    w = workloads.WORKLOADS[workloads.MAMBA130M]
    small = workloads.with_shape(w, batch=1, dim=8, seqlen=16)
    inp = workloads.make_inputs(small)
    assert inp["u"].dtype == torch.bfloat16 and inp["z"] is not None
    assert torch.equal(inp["A"][3], -torch.arange(1, 17, dtype=torch.float32))
    sp = torch.nn.functional.softplus(inp["delta_bias"].double())
    assert sp.min() >= 1e-3 - 1e-9 and sp.max() <= 0.1 + 1e-9
    g = workloads.WORKLOADS[workloads.GENOMIC]
    assert g.updates == 4 * 1024 * 100000 * 16
