"""The oracle's pins are sensitive: each plausible mistake, planted in a copy of
the oracle's C source and compiled on the CPU, makes at least one pin fail."""
import os
import subprocess

import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "ssd_oracle.c")

MUTATIONS = {
    "decays_own_input": ("Sp[n] = a * Sp[n] + u * Bt[n];", "Sp[n] = a * (Sp[n] + u * Bt[n]);"),
    "reads_state_before_update": ("Sp[n] = a * Sp[n] + u * Bt[n];\n            acc += Ct[n] * Sp[n];",
                                  "acc += Ct[n] * Sp[n];\n            Sp[n] = a * Sp[n] + u * Bt[n];"),
    "drops_D": ("yt[p] = acc + Dh * xt[p];", "yt[p] = acc;"),
    "D_on_scaled_x": ("yt[p] = acc + Dh * xt[p];", "yt[p] = acc + Dh * u;"),
    "decay_sign": ("const double a = exp(dtt * A[h]);\n        const double* xt",
                   "const double a = exp(-dtt * A[h]);\n        const double* xt"),
    "group_modulo": ("return head_group ? (int64_t)head_group[h] : h / (H / G);",
                     "return head_group ? (int64_t)head_group[h] : h % G;"),
    "input_not_dt_scaled": ("const double u = dtt * xt[p];", "const double u = xt[p];"),
    "ignores_init": ("if (init)\n        memcpy", "if (0)\n        memcpy"),
}

PINS = [
    lambda: pins.test_dense_semiseparable_matrix(48, 4, 3, 4, 2),
    pins.test_unit_decay_is_causal_linear_attention,
    pins.test_zero_decay_is_diagonal,
    pins.test_free_response_closed_form,
    pins.test_group_mapping_contiguous_heads,
    lambda: pins.test_recurrence_equals_chunked_algorithm(16),
    pins.test_linear_in_input_and_initial_state,
    pins.test_single_token_closed_form,
]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path):
    before, after = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(before) == 1, "mutation anchor drifted from the oracle source"
    mutated = tmp_path / "mut.c"
    mutated.write_text(src.replace(before, after))
    lib = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", str(lib), str(mutated),
                           "-lm"])
    caught = 0
    with oracle.using_library(str(lib)):
        for pin in PINS:
            try:
                pin()
            except (AssertionError, RuntimeError, FloatingPointError):
                caught += 1
    assert caught > 0, f"no pin detects the planted mistake {name!r}"
