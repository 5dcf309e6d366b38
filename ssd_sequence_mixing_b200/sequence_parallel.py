"""Sequence-parallel SSD forward: one long sequence split into contiguous segments, one
per rank (one process per GPU).

The state passes from segment to segment as it passes from chunk to chunk in the
chunked algorithm ("Transformers are SSMs", the wikillm.com card, Method step 5: the
centre factor).  Each rank

1. computes only its segment's end state from a zero state, s_r (H, P, N), with the
   final-state-only form of the forward pass (it reads x, dt and B, not C, and writes no
   y), and the segment log-decay lambda_r[h] = A[h] * sum_t dt[t, h];
2. all-gathers (s, lambda) over the process group: H*P*N + H fp32 per rank, the only
   exchange;
3. forms its start state h_r by the recurrence h_{q+1} = exp(lambda_q) h_q + s_q over the
   preceding segments, from h_0 = init (a library kernel);
4. runs its segment from h_r: its y rows and, on the last rank, the final state.

Step 1 reads the segment's x a first time; nothing else of it is repeated, so a rank
moves about 1.5 times the bytes of one pass (x is about half of them) instead of 2.

The steps are passed in as callables so that the same exchange and ordering can run
with other implementations of the kernels; by default they are this package's.
"""
from __future__ import annotations

from typing import Callable, Optional, Tuple

import torch
import torch.distributed as dist


def _library_steps():
    from . import segment_logdecay, ssd_final_state, ssd_forward, state_prefix

    def forward(x, dt, A, B, C, D, init, chunk):
        if C is None:  # only the end state is wanted
            return None, ssd_final_state(x, dt, A, B, init, None, chunk)
        return ssd_forward(x, dt, A, B, C, D, init, None, chunk)

    return forward, segment_logdecay, state_prefix


def forward_sequence_parallel(x, dt, A, B, C, D=None, init_state=None, chunk: int = 256, group=None,
                              steps: Optional[Tuple[Callable, Callable, Callable]] = None):
    """This rank's segment (batch 1): x (1, T_r, H, P), dt (1, T_r, H), B and C (1, T_r, G, N),
    init_state (1, H, P, N) or None: the sequence's initial state, the same on every rank.
    Returns (y, final_state): y for this segment; final_state (1, H, P, N) is the state after
    this segment (on the last rank, the sequence's final state).

    ``steps`` = (forward, logdecay, prefix) replaces the library kernels:
    forward(x, dt, A, B, C, D, init, chunk) -> (y, final), where C = None asks for the final
    state only (y may then be None); logdecay(dt2d, A) -> (H,);
    prefix(rank, states, logdecays, init) -> (H, P, N)."""
    forward, logdecay, prefix = steps or _library_steps()
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    H = x.shape[2]
    # 1. this segment's end state from a zero state (no C, no y)
    _, s_r = forward(x, dt, A, B, None, None, None, chunk)
    lam_r = logdecay(dt.reshape(-1, H), A)
    # 2. one exchange: every rank's (end state, log-decay)
    states = [torch.empty_like(s_r) for _ in range(world)]
    lams = [torch.empty_like(lam_r) for _ in range(world)]
    dist.all_gather(states, s_r.contiguous(), group=group)
    dist.all_gather(lams, lam_r.contiguous(), group=group)
    init0 = None if init_state is None else init_state.reshape(init_state.shape[-3:]).contiguous()
    # 3. this segment's start state
    h_r = prefix(rank, torch.cat(states, 0).contiguous(), torch.stack(lams, 0).contiguous(), init0)
    # 4. the segment again, from its true start state
    return forward(x, dt, A, B, C, D, h_r.unsqueeze(0).contiguous(), chunk)
