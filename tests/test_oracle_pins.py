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
