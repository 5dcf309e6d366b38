"""Chunked SSD in plain numpy fp64 -- TEST INFRASTRUCTURE, not the product.

An independent restatement of the chunked (block-decomposed) algorithm of
"Transformers are SSMs" (wikillm.com card, Method step 5, sec. 6: diagonal
blocks, right factors, centre factors, left factors), used to pin the
sequential recurrence in ``ssd_oracle.c``: both must agree for every chunk
length.  It follows the steps in the pages' order with whole-array numpy
operations and no blocking beyond the chunking the algorithm itself defines.

Inputs are one sequence of length T (a partial last chunk is allowed):
  xs   (T, H, P)  the dt-scaled input dt * x
  l    (T, H)     log decay dt * A  (<= 0)
  B, C (T, H, N)  per-head B and C (group sharing is expanded by the caller)
  h0   (H, P, N)  initial state or None
Returns (Y (T, H, P), final state (H, P, N)), without the D skip.
"""
from __future__ import annotations

import numpy as np


def segsum(l_chunk: np.ndarray) -> np.ndarray:
    """seg[h, i, j] = sum_{r=j+1..i} l[r, h] for i >= j, -inf above the diagonal.

    The -inf mask is applied before any exponential (card, Pitfalls: mask before exp).
    """
    Qc, H = l_chunk.shape
    cs = np.cumsum(l_chunk, axis=0)  # (Qc, H), inclusive, restarted in the chunk
    seg = cs.T[:, :, None] - cs.T[:, None, :]  # (H, i, j) = cs_i - cs_j
    tri = np.tril(np.ones((Qc, Qc), dtype=bool))
    return np.where(tri[None], seg, -np.inf)


def ssd_chunked(xs, l, B, C, Q, h0=None):
    T, H, P = xs.shape
    N = B.shape[-1]
    bounds = list(range(0, T, Q)) + [T]
    K = len(bounds) - 1
    Y = np.zeros((T, H, P))
    chunk_states = np.zeros((K, H, P, N))
    chunk_decay = np.zeros((K, H))
    cs_all = []
    # diagonal blocks and right factors, chunk by chunk (the chunks are independent)
    for k in range(K):
        t0, t1 = bounds[k], bounds[k + 1]
        lk, xk, Bk, Ck = l[t0:t1], xs[t0:t1], B[t0:t1], C[t0:t1]
        cs = np.cumsum(lk, axis=0)  # (Qc, H) decay cumsum restarted per chunk
        cs_all.append(cs)
        Lmask = np.exp(segsum(lk))  # (H, Qc, Qc)
        CB = np.einsum("ihn,jhn->hij", Ck, Bk)  # (H, Qc, Qc)
        Y[t0:t1] = np.einsum("hij,jhp->ihp", Lmask * CB, xk)  # diagonal block
        decay_to_end = np.exp(cs[-1][None, :] - cs)  # (Qc, H)
        chunk_states[k] = np.einsum("jhn,jh,jhp->hpn", Bk, decay_to_end, xk)  # right factor
        chunk_decay[k] = np.exp(cs[-1])
    # centre factors: scalar recurrence over the chunk states
    state = np.zeros((H, P, N)) if h0 is None else np.array(h0, dtype=np.float64)
    start_states = np.zeros((K, H, P, N))
    for k in range(K):
        start_states[k] = state
        state = chunk_decay[k][:, None, None] * state + chunk_states[k]
    # left factors: contribution of the carried-in state
    for k in range(K):
        t0, t1 = bounds[k], bounds[k + 1]
        decay_from_start = np.exp(cs_all[k])  # (Qc, H)
        Y[t0:t1] += np.einsum("ihn,hpn,ih->ihp", C[t0:t1], start_states[k], decay_from_start)
    return Y, state
