"""The pins of the oracle's next-row functions (step-size prologue, causal conv1d + SiLU,
gated RMSNorm) are sensitive: each plausible mistake, planted in a stand-in for the
oracle function on the CPU, makes at least one of their pins fail."""
import numpy as np
import pytest

import oracle
import test_oracle_pins as pins


def _silu(v):
    return v / (1.0 + np.exp(-v))


def dt_no_softplus(dt_raw, dt_bias=None, softplus=True, dt_min=0.0, dt_max=np.inf):
    v = np.asarray(dt_raw, float) + (0.0 if dt_bias is None else np.asarray(dt_bias, float))
    return np.clip(v, dt_min, dt_max)


def dt_bias_after_softplus(dt_raw, dt_bias=None, softplus=True, dt_min=0.0, dt_max=np.inf):
    v = np.asarray(dt_raw, float)
    if softplus:
        v = np.logaddexp(0.0, v)
    return np.clip(v + (0.0 if dt_bias is None else np.asarray(dt_bias, float)), dt_min, dt_max)


def conv_tap_shift(x, weight, bias=None, seq_offsets=None):
    # window shifted by one token: in[t - 2 + k] instead of in[t - 3 + k]
    x, w = np.asarray(x, float), np.asarray(weight, float)
    T, ch = x.shape
    offs = [0, T] if seq_offsets is None else list(seq_offsets)
    out = np.zeros((T, ch))
    for s in range(len(offs) - 1):
        a, e = int(offs[s]), int(offs[s + 1])
        for t in range(a, e):
            acc = np.zeros(ch) if bias is None else np.asarray(bias, float).copy()
            for k in range(4):
                src = t - 2 + k
                if a <= src < e:
                    acc += w[:, k] * x[src]
            out[t] = _silu(acc)
    return out


def norm_before_gate(y, z, weight, eps=1e-5):
    y, z, w = (np.asarray(v, float) for v in (y, z, weight))
    n = y / np.sqrt(np.mean(y * y, axis=-1, keepdims=True) + eps)
    return n * _silu(z) * w


def norm_no_weight(y, z, weight, eps=1e-5):
    y, z = np.asarray(y, float), np.asarray(z, float)
    g = y * _silu(z)
    return g / np.sqrt(np.mean(g * g, axis=-1, keepdims=True) + eps)


MUTANTS = {
    "dt_no_softplus": ("dt_prologue", dt_no_softplus),
    "dt_bias_after_softplus": ("dt_prologue", dt_bias_after_softplus),
    "conv_tap_shift": ("causal_conv1d_silu", conv_tap_shift),
    "conv_no_reset": ("causal_conv1d_silu", None),
    "norm_before_gate": ("gated_rmsnorm", norm_before_gate),
    "norm_no_weight": ("gated_rmsnorm", norm_no_weight),
}

PINS = {
    "dt_prologue": [pins.test_dt_prologue_closed_forms, pins.test_dt_prologue_forward_equals_forward_on_inverse_softplus],
    "causal_conv1d_silu": [pins.test_conv_impulse_response_and_sequence_reset, pins.test_conv_equals_library_convolution],
    "gated_rmsnorm": [pins.test_gated_rmsnorm_closed_forms],
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, monkeypatch):
    fn_name, mutant = MUTANTS[name]
    if name == "conv_no_reset":
        good = oracle.causal_conv1d_silu
        mutant = lambda x, w, b=None, seq_offsets=None: good(x, w, b, None)  # one sequence: no reset
    monkeypatch.setattr(oracle, fn_name, mutant)
    failed = 0
    for pin in PINS[fn_name]:
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed >= 1, f"no pin caught the planted mistake {name}"


def test_unmutated_pins_pass():
    for fns in PINS.values():
        for pin in fns:
            pin()
