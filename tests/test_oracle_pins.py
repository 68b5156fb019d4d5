"""The fp64 oracle against facts that do not come from it (see tests/pins.py)."""
import numpy as np
import pytest

import oracle
import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(oracle.selective_scan)


def test_differs_from_cumprod_cumsum_form():
    """The walkthrough's §4.2 / §6 "parallel" body (cumprod of dA, cumsum of
    dB*dA_cum, then times u at the current step) is not the §3.2 loop; the
    oracle follows the loop, so on random inputs the two must disagree."""
    rng = np.random.default_rng(1)
    Bt, Dm, L, N = 2, 3, 16, 4
    u = rng.standard_normal((Bt, Dm, L))
    delta = rng.standard_normal((Bt, Dm, L))
    A = -rng.uniform(0.2, 1.5, (Dm, N))
    B = rng.standard_normal((Bt, N, L))
    C = rng.standard_normal((Bt, N, L))
    y = oracle.selective_scan(u, delta, A, B, C, delta_softplus=True)
    dl = np.log1p(np.exp(delta))
    dA = np.exp(np.einsum("bdl,dn->bdln", dl, A))
    dB = np.einsum("bdl,bnl->bdln", dl, B)
    dA_cum = np.cumprod(dA, axis=2)
    state = np.cumsum(dB * dA_cum, axis=2) * u[..., None]
    y_wrong = np.einsum("bdln,bnl->bdl", state, C)
    assert np.max(np.abs(y - y_wrong)) > 0.1


def test_rejects_bad_arguments():
    with pytest.raises(ValueError):
        oracle.selective_scan(np.zeros((1, 1, 3)), np.zeros((1, 1, 4)), np.zeros((1, 2)),
                              np.zeros((1, 2, 3)), np.zeros((1, 2, 3)))
    with pytest.raises(ValueError):
        oracle.selective_scan(np.zeros((1, 1, 3)), np.zeros((1, 1, 3)), np.zeros((1, 2)),
                              np.zeros((1, 3, 3)), np.zeros((1, 2, 3)))


def test_threads_do_not_change_results():
    rng = np.random.default_rng(2)
    args = (rng.standard_normal((3, 5, 33)), rng.standard_normal((3, 5, 33)),
            -rng.uniform(0.1, 2, (5, 7)), rng.standard_normal((3, 7, 33)),
            rng.standard_normal((3, 7, 33)))
    y1 = oracle.selective_scan(*args, delta_softplus=True, nthreads=1)
    y4 = oracle.selective_scan(*args, delta_softplus=True, nthreads=4)
    assert np.array_equal(y1, y4)


def test_rows_helper_matches_full_problem():
    rng = np.random.default_rng(12)
    Bt, Dm, L, N = 2, 4, 21, 3
    inp = dict(u=rng.standard_normal((Bt, Dm, L)), delta=rng.standard_normal((Bt, Dm, L)),
               A=-rng.uniform(0.1, 2, (Dm, N)), B=rng.standard_normal((Bt, N, L)),
               C=rng.standard_normal((Bt, N, L)), D=rng.standard_normal(Dm),
               z=rng.standard_normal((Bt, Dm, L)), delta_bias=rng.standard_normal(Dm),
               delta_softplus=True, return_last_state=True)
    y, last = oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                    D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"],
                                    delta_softplus=True, return_last_state=True)
    rows = [(0, 0), (1, 3), (0, 2)]
    yr, lr = oracle.selective_scan_rows(inp, rows)
    for i, (b, d) in enumerate(rows):
        assert np.array_equal(yr[i], y[b, d])
        assert np.array_equal(lr[i], last[b, d])


def test_dt_projection_against_torch_linear():
    """The dt_proj form (delta = W_dt delta_r, Mamba-minimal项目解析 核心组件解析
    §5 ssm) against torch's own Linear (no bias; the scan adds delta_bias),
    in float64: the same numbers up to summation order."""
    import torch
    rng = np.random.default_rng(71)
    r = rng.standard_normal((3, 48, 37))
    w = rng.uniform(-48 ** -0.5, 48 ** -0.5, (20, 48))
    ref = torch.nn.functional.linear(torch.from_numpy(r).transpose(1, 2), torch.from_numpy(w)).transpose(1, 2)
    got = oracle.delta_from_projection(r, w)
    assert got.shape == (3, 20, 37)
    assert np.max(np.abs(got - ref.numpy())) <= 1e-13 * (1 + np.max(np.abs(got)))


def test_dt_projection_special_cases():
    """An identity projection (dt_rank = dim) gives the unfused scan of
    delta_r exactly; the projection is linear in W_dt; a zero projection
    with a large negative bias gives y = D u (delta' -> 0)."""
    rng = np.random.default_rng(73)
    Bt, Dm, L, N = 2, 5, 30, 4
    u = rng.standard_normal((Bt, Dm, L))
    r = rng.standard_normal((Bt, Dm, L))
    A = -rng.uniform(0.2, 1.5, (Dm, N))
    B = rng.standard_normal((Bt, N, L))
    C = rng.standard_normal((Bt, N, L))
    D = rng.standard_normal(Dm)
    y_id = oracle.selective_scan_dtproj(u, r, np.eye(Dm), A, B, C, D=D, delta_softplus=True)
    y = oracle.selective_scan(u, r, A, B, C, D=D, delta_softplus=True)
    assert np.array_equal(y_id, y)
    r3 = rng.standard_normal((Bt, 7, L))
    w1, w2 = rng.standard_normal((Dm, 7)), rng.standard_normal((Dm, 7))
    lhs = oracle.delta_from_projection(r3, 2.5 * w1 + w2)
    rhs = 2.5 * oracle.delta_from_projection(r3, w1) + oracle.delta_from_projection(r3, w2)
    assert np.max(np.abs(lhs - rhs)) <= 1e-12 * (1 + np.max(np.abs(lhs)))
    y0 = oracle.selective_scan_dtproj(u, r3, np.zeros((Dm, 7)), A, B, C, D=D, delta_bias=np.full(Dm, -1e4),
                                      delta_softplus=True)
    assert np.array_equal(y0, u * D[None, :, None])
