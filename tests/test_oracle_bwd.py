"""The fp64 backward oracle against its pins (finite differences of the
pinned forward oracle), and planted mistakes that the pins must catch."""
import os
import subprocess

import numpy as np
import pytest

import oracle
import pins_bwd

SRC = os.path.join(os.path.dirname(oracle.__file__), "ss_oracle_bwd.c")


def _grad(lib=None):
    def g(*a, **k):
        return oracle.selective_scan_bwd(*a, lib=lib, **k)
    return g


@pytest.mark.parametrize("pin", pins_bwd.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(_grad(), oracle.selective_scan)


def test_threads_do_not_change_results():
    rng = np.random.default_rng(5)
    p = pins_bwd._problem(rng, 3, 5, 40, 6)
    dy = rng.standard_normal((3, 5, 40))
    args = (p["u"], p["delta"], p["A"], p["B"], p["C"], dy)
    kw = dict(D=p["D"], z=p["z"], delta_bias=p["delta_bias"], delta_softplus=True)
    g1 = oracle.selective_scan_bwd(*args, nthreads=1, **kw)
    g4 = oracle.selective_scan_bwd(*args, nthreads=4, **kw)
    for k in g1:
        assert np.array_equal(g1[k], g4[k]), k


MUTANTS = {
    "carry_without_decay": ("carry[n] = keep ? a * lam : 0.0;", "carry[n] = keep ? lam : 0.0;"),
    "start_passes_adjoint": ("carry[n] = keep ? a * lam : 0.0;", "carry[n] = a * lam;"),
    "start_keeps_old_state": ("a * (keep ? h[l * N + n] : 0.0)", "a * h[l * N + n]"),
    "start_keeps_dA_term": ("const double da = keep ? lam * h[l * N + n] : 0.0;",
                            "const double da = lam * h[l * N + n];"),
    "silu_grad_sign": ("(1.0 + z[idx] * (1.0 - sg))", "(1.0 - z[idx] * (1.0 - sg))"),
    "softplus_grad_missing": ("ddl * (xs[l] > 20.0 ? 1.0 : sigmoid(xs[l]))", "ddl"),
    "dB_uses_B": ("dB[bn] += lam * dl[l] * u[idx];", "dB[bn] += lam * dl[l] * B[bn];"),
    "dC_uses_old_state": ("dC[bn] += g * h[(l + 1) * N + n];", "dC[bn] += g * h[l * N + n];"),
    "dA_missing_delta": ("pA[row * N + n] += da * a * dl[l];", "pA[row * N + n] += da * a;"),
    "du_missing_skip": ("double dui = D ? g * D[d] : 0.0;", "double dui = 0.0;"),
    "exp_mode_grad": (": ddl * dl[l];", ": ddl;"),
    "initial_state_ignored": ("h[n] = h0 ? h0[row * N + n] : 0.0;", "h[n] = 0.0;"),
    "initial_state_grad_without_decay": ("dh0[row * N + n] = L > 0 ? carry[n] :",
                                         "dh0[row * N + n] = L > 0 ? carry[n] / exp(dl[0] * A[d * N + n]) :"),
    "magnitude_of_sum": ("mB[bn] += lam_m * fabs(dl[l] * u[idx]);", "mB[bn] += lam * dl[l] * u[idx];"),
    "magnitude_without_recursion": ("const double lam_m = fabs(g * C[bn]) + cm[n];",
                                    "const double lam_m = fabs(g * C[bn] + carry[n]);"),
    "last_state_gradient_ignored": ("carry[n] = dlast ? dlast[row * N + n] : 0.0;", "carry[n] = 0.0;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    source = open(SRC).read()
    assert source.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    src = tmp_path / "mutant_bwd.c"
    src.write_text(source.replace(old, new))
    lib = tmp_path / "libmutant.so"
    fwd = os.path.join(os.path.dirname(oracle.__file__), "ss_oracle.c")
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
                    fwd, str(src), "-o", str(lib), "-lm"], check=True)
    caught = []
    for pin in pins_bwd.ALL_PINS:
        try:
            pin(_grad(str(lib)), oracle.selective_scan)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"planted mistake {name} passed every pin"
