"""Sequence-parallel steps on one GPU: the segments of one sequence are run as the ranks
would run them (zero-start final-state-only pass, segment log-decay, start-state
recurrence, the segment's pass from its start state), in one process; the stitched result
is checked against the fp64 oracle's single pass.  The orchestration itself
(forward_sequence_parallel) runs on a one-rank NCCL group with the library's kernels."""
import os
import socket

import numpy as np
import pytest
import torch

import ssd_sequence_mixing_b200 as ssd
import workloads
from harness import check, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cuts", [[0, 300, 301, 1024, 1500], [0, 750, 1500]], ids=["four_ragged", "two"])
def test_sequence_parallel_steps_match_one_pass(cuts):
    wl = workloads.custom(1, 1500, H=8, P=64, N=128, G=1, chunk=256, dtype="bf16", init=True)
    prob = workloads.generate(wl, seed=31)
    d = to_device(prob)
    R = len(cuts) - 1
    seg = lambda v, r: v[:, cuts[r]:cuts[r + 1]].contiguous()
    states, lams = [], []
    for r in range(R):
        s_r = ssd.ssd_final_state(seg(d["x"], r), seg(d["dt"], r), d["A"], seg(d["B"], r), None, None, 256)
        _, s_full = ssd.ssd_forward(seg(d["x"], r), seg(d["dt"], r), d["A"], seg(d["B"], r), seg(d["C"], r), None,
                                    None, None, 256)
        torch.cuda.synchronize()
        assert torch.equal(s_r, s_full)  # the final-state-only pass is the same computation
        lam = ssd.segment_logdecay(seg(d["dt"], r), d["A"])
        ref = seg(d["dt"], r)[0].double().sum(0) * d["A"].double()
        assert torch.allclose(lam.double(), ref, rtol=1e-5, atol=1e-6)
        states.append(s_r)
        lams.append(lam)
    S, L = torch.cat(states, 0).contiguous(), torch.stack(lams, 0).contiguous()
    init = d["init_state"][0].contiguous()
    ys, fin = [], None
    h = init.clone()
    for r in range(R):
        h_r = ssd.state_prefix(r, S, L, init)
        assert torch.allclose(h_r, h, rtol=1e-5, atol=1e-6)  # the recurrence, step by step in torch
        h = torch.exp(L[r])[:, None, None] * h + S[r]
        y_r, fin = ssd.ssd_forward(seg(d["x"], r), seg(d["dt"], r), d["A"], seg(d["B"], r), seg(d["C"], r),
                                   d["D"], h_r[None].contiguous(), None, 256)
        ys.append(y_r)
    torch.cuda.synchronize()
    check(prob, torch.cat(ys, 1), fin)


def test_forward_sequence_parallel_on_one_rank_nccl_group():
    import torch.distributed as dist
    from ssd_sequence_mixing_b200.sequence_parallel import forward_sequence_parallel

    wl = workloads.custom(1, 1500, H=8, P=64, N=128, G=1, chunk=256, dtype="bf16", init=True)
    prob = workloads.generate(wl, seed=32)
    d = to_device(prob)
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        y, fin = forward_sequence_parallel(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["init_state"], 256)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    check(prob, y, fin)
