"""GPU parity of the recurrent decode step (one token per sequence and head, the
pages' generation mode) against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import ssd_sequence_mixing_b200 as ssd
import workloads
from harness import assert_close, check, to_device

pytestmark = pytest.mark.gpu

CASES = [
    # batch, T, H, P, N, G, dtype, with D
    (3, 6, 4, 64, 128, 2, "bf16", True),
    (2, 5, 6, 17, 36, 3, "f32", False),
    (1, 3, 80, 64, 256, 1, "bf16", True),
    (5, 4, 8, 64, 64, 8, "f32", True),
    (2, 3, 4, 200, 4, 1, "f32", True),
]


def step_inputs(d, t):
    return [d[k][:, t].contiguous() for k in ("x", "dt", "B", "C")]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b{}_T{}_H{}_P{}_N{}_G{}_{}_D{}".format(*c))
def test_decode_steps_match_oracle(case):
    b, T, H, P, N, G, dtype, with_d = case
    wl = workloads.custom(b, T, H, P, N, G, chunk=64, dtype=dtype, init=True)
    prob = workloads.generate(wl, seed=21)
    if not with_d:
        prob.D = None
    d = to_device(prob)
    state = d["init_state"].clone()
    st_ref = prob.init_state.double().numpy()
    f64 = lambda v: None if v is None else v.double().numpy()
    for t in range(T):
        x, dt, B, C = step_inputs(d, t)
        y = ssd.ssd_decode_step(x, dt, d["A"], B, C, d["D"], state)
        torch.cuda.synchronize()
        y_ref, st_ref = oracle.decode_step(f64(prob.x[:, t].float()), f64(prob.dt[:, t]), f64(prob.A),
                                           f64(prob.B[:, t].float()), f64(prob.C[:, t].float()), f64(prob.D), st_ref)
        assert y.dtype == x.dtype
        assert_close(f"y step {t}", y.float().cpu().numpy(), y_ref, dtype)
    assert_close("state", state.cpu().numpy(), st_ref, dtype)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_sequence_equals_forward_pass(dtype):
    """T decode steps from the initial state reproduce the forward pass: y of every
    token and the final state, checked against the oracle's forward recurrence."""
    wl = workloads.custom(4, 300, H=8, P=64, N=128, G=2, chunk=256, dtype=dtype, init=True)
    prob = workloads.generate(wl, seed=22)
    d = to_device(prob)
    state = d["init_state"].clone()
    ys = []
    for t in range(wl.seqlen):
        x, dt, B, C = step_inputs(d, t)
        ys.append(ssd.ssd_decode_step(x, dt, d["A"], B, C, d["D"], state))
    y = torch.stack(ys, dim=1)
    torch.cuda.synchronize()
    check(prob, y, state)
    y_fwd, fin_fwd = ssd.ssd_forward(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["init_state"], None, 256)
    torch.cuda.synchronize()
    scale = float(y_fwd.float().abs().max())
    assert float((y.float() - y_fwd.float()).abs().max()) <= 3e-2 * scale
    assert float((state - fin_fwd).abs().max()) <= 3e-2 * float(fin_fwd.abs().max())


def test_decode_state_in_place_and_no_side_effects():
    wl = workloads.custom(2, 1, H=4, P=64, N=64, G=1, chunk=64, dtype="bf16", init=True)
    prob = workloads.generate(wl, seed=23)
    d = to_device(prob)
    x, dt, B, C = step_inputs(d, 0)
    snapshot = {k: v.clone() for k, v in d.items() if v is not None}
    state = d["init_state"].clone()
    ptr = state.data_ptr()
    y1 = ssd.ssd_decode_step(x, dt, d["A"], B, C, d["D"], state)
    assert state.data_ptr() == ptr and not torch.equal(state, d["init_state"])
    for k, v in snapshot.items():
        assert torch.equal(v, d[k]), k
    # deterministic: the same step from the same state gives the same bits
    state2 = d["init_state"].clone()
    y2 = ssd.ssd_decode_step(x, dt, d["A"], B, C, d["D"], state2)
    assert torch.equal(y1, y2) and torch.equal(state, state2)
