"""Each plausible mistake planted in a copy of the oracle's C source (on the
CPU, in a temporary directory) must be caught by at least one pin."""
import os
import subprocess

import pytest

import oracle
import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "ss_oracle.c")

MUTANTS = {
    "drop_skip_D": ("yv += ul * D[d];", ";"),
    "exp_sign": ("exp(dl * A[d * dstate + n])", "exp(-dl * A[d * dstate + n])"),
    "A_transposed": ("A[d * dstate + n]", "A[n * dim + d]"),
    "B_index_transposed": ("const double dB = dl * B[bn];",
                           "const double dB = dl * B[(b * seqlen + l) * dstate + n];"),
    "drop_u": ("dB * ul;", "dB;"),
    "y_before_update": ("h[n] = dA * h[n] + dB * ul;                      /* §3.2 */\n"
                        "                yv += h[n] * C[bn];                              /* §3.2 */",
                        "yv += h[n] * C[bn];\n                h[n] = dA * h[n] + dB * ul;"),
    "gate_before_skip": ("            if (D)\n                yv += ul * D[d]; /* §3.3 skip connection */\n"
                         "            if (z)\n                yv *= silu(z[idx]); /* §3.3 gate */",
                         "            if (z)\n                yv *= silu(z[idx]);\n"
                         "            if (D)\n                yv += ul * D[d];"),
    "softplus_threshold": ("if (x > 20.0)", "if (x > 2.0)"),
    "exp_mode_uses_softplus": ("delta_softplus ? softplus_default(x) : exp(x)", "softplus_default(x)"),
    "drop_bias": ("x += delta_bias[d];", ";"),
    "silu_sign": ("z / (1.0 + exp(-z))", "z / (1.0 + exp(z))"),
    "last_state_wrong_index": ("last_state[row * dstate + n] = h[n];",
                               "last_state[row * dstate + n] = h[0];"),
    "initial_state_ignored": ("h[n] = initial_state ? initial_state[row * dstate + n] : 0.0;",
                              "h[n] = 0.0;"),
    "initial_state_transposed": ("initial_state[row * dstate + n]", "initial_state[n * dim * batch + row]"),
    "reset_ignored": ("if (reset && reset[b * seqlen + l])", "if (0)"),
    "reset_one_step_late": ("reset[b * seqlen + l])", "reset[b * seqlen + (l > 0 ? l - 1 : 0)])"),
    "reset_wrong_batch_entry": ("reset[b * seqlen + l])", "reset[(batch - 1 - b) * seqlen + l])"),
    "reset_keeps_one_state": ("                for (int64_t n = 0; n < dstate; ++n)\n                    h[n] = 0.0;",
                              "                for (int64_t n = 1; n < dstate; ++n)\n                    h[n] = 0.0;"),
}


@pytest.fixture(scope="module")
def source():
    return open(SRC).read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, source, tmp_path):
    old, new = MUTANTS[name]
    assert source.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mutated = source.replace(old, new)
    src = tmp_path / "mutant.c"
    lib = tmp_path / "libmutant.so"
    src.write_text(mutated)
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
                    str(src), "-o", str(lib), "-lm"], check=True)

    def scan(*a, **k):
        return oracle.selective_scan(*a, lib=str(lib), **k)

    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(scan)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake {name}"
