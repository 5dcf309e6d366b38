"""Seeded synthetic inputs for the chunked SSD forward pass.

This module is shared by the tests, the bench and the oracle harness.  It holds
the workload shapes and the input distributions and nothing of the SSD
arithmetic itself: it draws numbers and rounds them to the I/O dtypes.

Distributions (Mamba-2 initialisation used as the synthetic input recipe; see
"Transformers are SSMs", wikillm.com card, "Paper vs code" item 8, and the
Mamba-2 block sketch in Method step 6):

* x ~ N(0, 1), shape (tokens, H, P)
* dt = softplus(0.5 * N(0, 1) + b_h), b_h = softplus^-1(dt0_h),
  dt0_h log-uniform in [1e-3, 1e-1]; shape (tokens, H), fp32
* A_h = -exp(U[log 1, log 16]), fp32
* B, C ~ N(0, 1) / sqrt(N), shape (tokens, G, N)
* D_h ~ N(0, 1), fp32
* init_state ~ N(0, 0.1^2) per sequence where the workload asks for one
* packed lengths ~ U{64..8192}, drawn until the total is reached, last truncated

Every tensor comes from its own counter-keyed stream
``numpy.random.default_rng([seed, tensor_id, block])`` in float32 blocks of
``BLOCK_TOKENS`` tokens, so a tensor's values do not depend on the shape or
draw order of any other tensor, and huge inputs are generated block by block.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import numpy as np
import torch

BLOCK_TOKENS = 4096

# stream ids, one per tensor
_SID = {"x": 1, "dt_noise": 2, "dt0": 3, "A": 4, "B": 5, "C": 6, "D": 7, "init": 8, "lengths": 9}


@dataclasses.dataclass
class Workload:
    """A synthetic SSD problem description (no data)."""

    name: str
    batch: int
    seqlen: int  # tokens per sequence (dense) or total tokens (packed)
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    chunk: int
    dtype: str  # "f32" or "bf16": dtype of x, B, C, y
    init: bool = False  # nonzero initial states
    packed: bool = False  # variable-length packed batch (batch == 1)
    min_len: int = 64
    max_len: int = 8192

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen


def _cfg(name, **kw) -> Workload:
    return Workload(name=name, **kw)


# The five workloads (0: tiny parity case; 1: Mamba-2-2.7B-like layer, the
# throughput workload; 2: state-size sweep; 3: sequence-length sweep at fixed
# tokens; 4: packed variable-length with grouped B/C and initial states).
TINY = _cfg("tiny_b1_L256_H2_P16_N16_fp32", batch=1, seqlen=256, nheads=2, headdim=16, dstate=16,
            ngroups=1, chunk=64, dtype="f32")
MAMBA2_2P7B = _cfg("mamba2_2.7b_layer_b8_L2048_H80_P64_N128_bf16", batch=8, seqlen=2048, nheads=80,
                   headdim=64, dstate=128, ngroups=1, chunk=256, dtype="bf16")
STATE_SWEEP = [_cfg(f"state_sweep_b4_L4096_H32_P64_N{n}_bf16", batch=4, seqlen=4096, nheads=32,
                    headdim=64, dstate=n, ngroups=1, chunk=256, dtype="bf16")
               for n in (16, 32, 64, 128, 256)]
LENGTH_SWEEP = [_cfg(f"length_sweep_b{b}_L{L}_H64_P64_N64_bf16", batch=b, seqlen=L, nheads=64,
                     headdim=64, dstate=64, ngroups=1, chunk=256, dtype="bf16")
                for (b, L) in ((256, 512), (64, 2048), (16, 8192), (8, 16384), (2, 65536))]
PACKED = _cfg("packed_varlen_T262144_H64_P64_N128_G8_bf16", batch=1, seqlen=262144, nheads=64,
              headdim=64, dstate=128, ngroups=8, chunk=256, dtype="bf16", init=True, packed=True)

ALL = [TINY, MAMBA2_2P7B] + STATE_SWEEP + LENGTH_SWEEP + [PACKED]
BY_NAME = {w.name: w for w in ALL}


@dataclasses.dataclass
class Problem:
    """Concrete inputs on the host (torch CPU tensors in their I/O dtypes)."""

    wl: Workload
    x: torch.Tensor  # (batch, T, H, P) io dtype
    dt: torch.Tensor  # (batch, T, H) fp32
    A: torch.Tensor  # (H,) fp32
    B: torch.Tensor  # (batch, T, G, N) io dtype
    C: torch.Tensor  # (batch, T, G, N) io dtype
    D: Optional[torch.Tensor]  # (H,) fp32
    init_state: Optional[torch.Tensor]  # (nseq, H, P, N) fp32
    cu_seqlens: Optional[torch.Tensor]  # (nseq+1,) int32 for packed problems
    seq_offsets: List[int]  # token offsets of every sequence, nseq+1 (dense rows too)

    @property
    def nseq(self) -> int:
        return len(self.seq_offsets) - 1


def _rng(seed: int, name: str, block: int = 0) -> np.random.Generator:
    return np.random.default_rng([seed, _SID[name], block])


def _normal_tokens(seed, name, tokens, inner, scale=1.0):
    """float32 N(0, scale^2) of shape (tokens, inner), drawn per token block."""
    out = np.empty((tokens, inner), dtype=np.float32)
    for blk, t0 in enumerate(range(0, tokens, BLOCK_TOKENS)):
        t1 = min(tokens, t0 + BLOCK_TOKENS)
        out[t0:t1] = _rng(seed, name, blk).standard_normal((t1 - t0, inner), dtype=np.float32)
    if scale != 1.0:
        out *= np.float32(scale)
    return out


def _softplus64(v: np.ndarray) -> np.ndarray:
    return np.maximum(v, 0.0) + np.log1p(np.exp(-np.abs(v)))


def packed_lengths(seed: int, total: int, lo: int, hi: int) -> List[int]:
    """Integer lengths U{lo..hi} drawn until they reach ``total``; the last is truncated."""
    rng = _rng(seed, "lengths")
    out, acc = [], 0
    while acc < total:
        n = int(rng.integers(lo, hi + 1))
        n = min(n, total - acc)
        out.append(n)
        acc += n
    return out


def head_params(seed: int, H: int):
    """Per-head dt bias b_h, A_h and D_h in float64."""
    dt0 = np.exp(_rng(seed, "dt0").uniform(math.log(1e-3), math.log(1e-1), size=H))
    bias = np.log(np.expm1(dt0))  # softplus^-1(dt0)
    A = -np.exp(_rng(seed, "A").uniform(0.0, math.log(16.0), size=H))
    D = _rng(seed, "D").standard_normal(H)
    return bias, A, D


def to_io(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def generate(wl: Workload, seed: int = 0, lengths: Optional[Sequence[int]] = None,
             dt_scale: float = 1.0, A_override: Optional[Sequence[float]] = None) -> Problem:
    """Draw the inputs of ``wl``.

    ``lengths`` overrides the packed lengths (packed problems only).  ``dt_scale``
    multiplies dt and ``A_override`` replaces A; both exist for edge-case tests.
    """
    H, P, N, G = wl.nheads, wl.headdim, wl.dstate, wl.ngroups
    tokens = wl.tokens
    if wl.packed:
        assert wl.batch == 1
        lens = list(lengths) if lengths is not None else packed_lengths(seed, wl.seqlen, wl.min_len, wl.max_len)
        assert sum(lens) == wl.seqlen, (sum(lens), wl.seqlen)
        offs = [0]
        for n in lens:
            offs.append(offs[-1] + n)
        cu = torch.tensor(offs, dtype=torch.int32)
    else:
        offs = [b * wl.seqlen for b in range(wl.batch + 1)]
        cu = None
    nseq = len(offs) - 1

    x = _normal_tokens(seed, "x", tokens, H * P)
    bias, A, D = head_params(seed, H)
    if A_override is not None:
        A = np.asarray(A_override, dtype=np.float64)
    z = _normal_tokens(seed, "dt_noise", tokens, H).astype(np.float64)
    dt = _softplus64(0.5 * z + bias[None, :]) * dt_scale
    Bm = _normal_tokens(seed, "B", tokens, G * N, scale=1.0 / math.sqrt(N))
    Cm = _normal_tokens(seed, "C", tokens, G * N, scale=1.0 / math.sqrt(N))
    init = None
    if wl.init:
        init = torch.from_numpy(_normal_tokens(seed, "init", nseq * H, P * N, scale=0.1)).reshape(nseq, H, P, N)

    bt = (wl.batch, wl.seqlen)
    return Problem(
        wl=wl,
        x=to_io(x, wl.dtype).reshape(*bt, H, P),
        dt=torch.from_numpy(dt.astype(np.float32)).reshape(*bt, H),
        A=torch.from_numpy(A.astype(np.float32)),
        B=to_io(Bm, wl.dtype).reshape(*bt, G, N),
        C=to_io(Cm, wl.dtype).reshape(*bt, G, N),
        D=torch.from_numpy(D.astype(np.float32)),
        init_state=init,
        cu_seqlens=cu,
        seq_offsets=offs,
    )


def custom(batch, seqlen, H, P, N, G=1, chunk=64, dtype="f32", init=False, lengths=None, name="custom"):
    """A workload of arbitrary shape with the standard distributions (tests)."""
    packed = lengths is not None
    if packed:
        return Workload(name=name, batch=1, seqlen=int(sum(lengths)), nheads=H, headdim=P, dstate=N,
                        ngroups=G, chunk=chunk, dtype=dtype, init=init, packed=True)
    return Workload(name=name, batch=batch, seqlen=seqlen, nheads=H, headdim=P, dstate=N, ngroups=G,
                    chunk=chunk, dtype=dtype, init=init)
