"""ssd_forward_noalloc: the entry point for callers that cannot allocate device memory.

A caller that owns the GPU's memory through its own pool (for example a server that
hands HBM to weights and KV caches up front) cannot let the library call
cudaMallocAsync.  This entry point takes its scratch from a static device array
instead.  The GPU test calls it through the C ABI twice in a row, on two different
problems (so the second call runs over the first call's leftover scratch), and checks
each result against ssd_forward's on the same inputs.  This file is named to be
collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import ssd_sequence_mixing_b200 as ssd
import workloads
from harness import TOL, check, errors, to_device


def _call_raw(dev, wl, y, fin):
    """Call the C entry point directly with ctypes (y, final_state preallocated)."""
    shape = ssd.make_shape(dev["x"], dev["B"], dev["cu_seqlens"])
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return ssd.library().ssd_forward_noalloc(ctypes.byref(shape), p(dev["x"]), p(dev["dt"]), p(dev["A"]),
                                             p(dev["B"]), p(dev["C"]), p(dev["D"]), p(dev["init_state"]),
                                             p(dev["cu_seqlens"]), wl.chunk, p(y), p(fin), stream)


def _within(got, ref, dtype):
    tol = TOL[dtype]
    rel, mx, ref_max = errors(got.double().cpu().numpy(), ref.double().cpu().numpy())
    ok = rel <= tol["rel_l2"] and (tol["max_abs_frac"] is None or mx <= tol["max_abs_frac"] * ref_max)
    return ok, rel, mx


@pytest.mark.gpu
def test_noalloc_matches_forward_on_two_calls_in_a_row():
    problems = [
        workloads.generate(workloads.custom(2, 700, H=4, P=64, N=128, G=2, chunk=256, dtype="bf16", init=True),
                           seed=11),
        workloads.generate(workloads.custom(1, 0, H=4, P=64, N=64, G=1, chunk=128, dtype="bf16", init=True,
                                            lengths=[5, 300, 0, 129]), seed=12, lengths=[5, 300, 0, 129]),
    ]
    for prob in problems:
        wl = prob.wl
        dev = to_device(prob)
        y_ref, f_ref = ssd.ssd_forward(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"],
                                       dev["init_state"], dev["cu_seqlens"], wl.chunk)
        y = torch.full_like(dev["x"], float("nan"))
        fin = torch.full_like(f_ref, float("nan"))
        assert _call_raw(dev, wl, y, fin) == 0
        torch.cuda.synchronize()
        assert ssd.query_status() == 0
        for name, got, ref in (("y", y, y_ref), ("final_state", fin, f_ref)):
            ok, rel, mx = _within(got, ref, wl.dtype)
            assert ok, f"{wl.name} {name}: rel-L2 {rel:.3e}, max-abs {mx:.3e}"
        check(prob, y, fin)  # and against the fp64 oracle directly


@pytest.mark.gpu
def test_noalloc_all_sequences_empty_takes_null_inputs():
    """No tokens at all: x, dt, B, C and y may be NULL, as for ssd_forward, and every
    final state is its initial state."""
    lens = [0, 0, 0]
    wl = workloads.custom(1, 0, H=4, P=64, N=64, G=1, chunk=128, dtype="bf16", init=True, lengths=lens)
    prob = workloads.generate(wl, seed=13, lengths=lens)
    dev = to_device(prob)
    shape = ssd.make_shape(dev["x"], dev["B"], dev["cu_seqlens"])
    fin = torch.full_like(dev["init_state"], float("nan"))
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = ssd.library().ssd_forward_noalloc(ctypes.byref(shape), None, None, p(dev["A"]), None, None, p(dev["D"]),
                                           p(dev["init_state"]), p(dev["cu_seqlens"]), wl.chunk, None, p(fin),
                                           stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert ssd.query_status() == 0
    assert torch.equal(fin, dev["init_state"])


def test_noalloc_rejects_shapes_beyond_its_scratch():
    """Checked on the host before anything touches the GPU: no GPU needed."""
    shape = ssd.SsdShape(8, 2048, 80, 64, 128, 1, 0, ssd.SSD_BF16, None)
    fake = ctypes.c_void_p(1 << 20)
    rc = ssd.library().ssd_forward_noalloc(ctypes.byref(shape), fake, fake, fake, fake, fake, None, None, None, 256,
                                           fake, None, None)
    assert rc == 7  # SSD_ERR_SCRATCH_LIMIT
    assert "scratch" in ssd.library().ssd_status_string(7).decode()
