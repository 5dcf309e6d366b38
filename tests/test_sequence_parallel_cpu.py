"""Sequence-parallel SSD on CPU: two and three gloo ranks each hold a contiguous segment of
one sequence; the exchange (all-gather of segment end states and log-decays) and the
start-state recurrence must give the single-pass result.  The per-segment kernels are
stood in for by the fp64 oracle (the GPU test runs the library's kernels)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from ssd_sequence_mixing_b200.sequence_parallel import forward_sequence_parallel


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def oracle_steps():
    def forward(x, dt, A, B, C, D, init, chunk):
        state_only = C is None  # the end state does not depend on C
        Cv = np.zeros_like(B[0].numpy()) if state_only else C[0].numpy()
        y, fin = oracle.ssd_forward(x[0].numpy(), dt[0].numpy(), A.numpy(), B[0].numpy(), Cv,
                                    None if D is None else D.numpy(), None if init is None else init.numpy())
        return (None if state_only else torch.from_numpy(y)[None]), torch.from_numpy(fin)

    def logdecay(dt2d, A):
        return dt2d.sum(0) * A

    def prefix(rank, states, lams, init):
        h = torch.zeros_like(states[0]) if init is None else init.clone()
        for q in range(rank):
            h = torch.exp(lams[q])[:, None, None] * h + states[q]
        return h

    return forward, logdecay, prefix


def problem(seed, T=90, H=3, P=4, N=5, G=1):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((1, T, H, P))
    dt = rng.uniform(0.01, 0.5, (1, T, H))
    A = -rng.uniform(0.2, 2.0, H)
    B = rng.standard_normal((1, T, G, N)) / np.sqrt(N)
    C = rng.standard_normal((1, T, G, N)) / np.sqrt(N)
    D = rng.standard_normal(H)
    init = 0.1 * rng.standard_normal((1, H, P, N))
    return [torch.from_numpy(v) for v in (x, dt, A, B, C, D, init)]


def _rank(rank, world, port, cuts, variant, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x, dt, A, B, C, D, init = problem(7, **variant)
        if variant.get("G") == 2:
            init, D = None, None  # no initial state, no skip
        a, e = cuts[rank], cuts[rank + 1]
        seg = lambda v: v[:, a:e].contiguous()
        y, fin = forward_sequence_parallel(seg(x), seg(dt), A, seg(B), seg(C), D, init, steps=oracle_steps())
        out[rank] = (y.numpy(), fin.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cuts,variant", [([0, 40, 90], {}), ([0, 1, 60, 90], {}), ([0, 30, 30, 90], {}),
                                          ([0, 45, 90], {"H": 4, "G": 2})],
                         ids=["two", "three", "empty_middle", "two_groups_no_init_no_skip"])
def test_sequence_parallel_equals_one_pass(cuts, variant):
    world = len(cuts) - 1
    out = mp.Manager().dict()
    mp.spawn(_rank, args=(world, _free_port(), cuts, variant, out), nprocs=world, join=True)
    x, dt, A, B, C, D, init = problem(7, **variant)
    if variant.get("G") == 2:
        init, D = None, None
    y_ref, fin_ref = oracle.ssd_forward(x[0].numpy(), dt[0].numpy(), A.numpy(), B[0].numpy(), C[0].numpy(),
                                        None if D is None else D.numpy(), None if init is None else init.numpy())
    y = np.concatenate([out[r][0][0] for r in range(world)], 0)
    assert np.allclose(y, y_ref, rtol=1e-10, atol=1e-12)
    assert np.allclose(out[world - 1][1], fin_ref, rtol=1e-10, atol=1e-12)
