"""The failure path of the tensor-core kernel's bounded waits, made to run on purpose
without faulting the GPU: CTAs withhold the flag that hands their state on, or CTA 0 its
flag of the barrier after the split's tile weights, so the CTAs that wait for it give up
after a short limit.  The call must return, the device must report
SSD_ERR_DEVICE_TIMEOUT, and the next normal call on the same stream must be correct
against the oracle (the context stays usable)."""
import pytest
import torch

import ssd_sequence_mixing_b200 as ssd
import workloads
from harness import check, run, to_device

pytestmark = pytest.mark.gpu


def test_withheld_hand_on_times_out_and_next_call_is_correct():
    # one packed 8192-token sequence and two head pairs: 128 tiles spread over the SMs, so
    # nearly every CTA waits for the state of the one before it (a dense batch this long
    # would be cut into segments, whose CTAs hand nothing on)
    lens = [8192]
    wl = workloads.custom(1, 0, H=4, P=64, N=128, G=1, chunk=256, dtype="bf16", init=True, lengths=lens)
    prob = workloads.generate(wl, seed=21, lengths=lens)
    dev = to_device(prob)
    shape = ssd.make_shape(dev["x"], dev["B"], dev["cu_seqlens"])
    if ssd.select_path(shape, wl.chunk) != ssd.PATH_TC:
        pytest.skip("shape not on the tensor-core path")
    assert ssd.query_status() == 0
    ssd.set_test_hooks(wait_limit_cycles=20_000_000, withhold_carry=True)  # about 10 ms per wait
    try:
        run(prob, dev=dev)
    finally:
        ssd.set_test_hooks()
    assert ssd.query_status() == 5  # SSD_ERR_DEVICE_TIMEOUT
    assert ssd.query_status() == 0  # read and cleared
    y, fin = run(prob, dev=dev)
    assert ssd.query_status() == 0
    check(prob, y, fin)


def test_withheld_weight_flag_times_out_and_next_call_is_correct():
    # 4 x 2048 tokens, 64 heads: 64 sequence tiles and 128 units, one launch of the fused
    # kernel (no segments), whose CTAs weigh the tiles themselves and meet at the flag
    # barrier; CTA 0 never sets its flag, so every CTA's wait there gives up and no CTA
    # takes any work
    wl = workloads.custom(4, 2048, H=64, P=64, N=128, G=1, chunk=256, dtype="bf16")
    prob = workloads.generate(wl, seed=22)
    dev = to_device(prob)
    shape = ssd.make_shape(dev["x"], dev["B"], dev["cu_seqlens"])
    if ssd.select_path(shape, wl.chunk) != ssd.PATH_TC:
        pytest.skip("shape not on the tensor-core path")
    assert ssd.query_status() == 0
    ssd.set_test_hooks(wait_limit_cycles=20_000_000, withhold_split=True)  # about 10 ms per wait
    try:
        run(prob, dev=dev)
    finally:
        ssd.set_test_hooks()
    assert ssd.query_status() == 5  # SSD_ERR_DEVICE_TIMEOUT
    assert ssd.query_status() == 0  # read and cleared
    y, fin = run(prob, dev=dev)
    assert ssd.query_status() == 0
    check(prob, y, fin)
