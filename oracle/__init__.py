"""The SSD oracle -- TEST INFRASTRUCTURE, not the product.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  It shares no code with the CUDA path.

* ``ssd_forward``: the fp64 sequential recurrence (``ssd_oracle.c``, OpenMP over
  sequence x head), following "Transformers are SSMs" (wikillm.com card, Method
  steps 1-3 and 6-7).
* ``ssd_forward_problem``: the same on a ``workloads.Problem``, optionally only
  on sampled (sequence, head) pairs so that full-size problems stay cheap.
* ``chunked.ssd_chunked``: the pages' chunked algorithm restated in numpy
  (Method step 5, sec. 6), used to pin the recurrence.
* ``decode_step``: one recurrent generation step (Method step 8, sec. 6.3).
* ``dt_prologue``: the step size from the raw projection, dt = softplus(raw + bias)
  (the Mamba-2 block sketch of sec. 7.1 and Method note 7 "Discretisation").
* ``causal_conv1d_silu`` and ``gated_rmsnorm``: the block's steps before and after the
  SSD (the Mamba-2 block sketch of sec. 7.1; "Paper vs code" 1, 2 and 9).

Pins (``tests/test_oracle_pins.py``): ``ssd_forward`` against a dense semiseparable
brute force, textbook special cases, closed forms, hand-worked values and the
chunked restatement; ``decode_step`` against the dense matrix; ``dt_prologue``
against softplus closed forms and the inverse softplus; ``causal_conv1d_silu``
against an impulse response, a sequence reset and numpy's convolution;
``gated_rmsnorm`` against closed forms (gate off, constant gate, unit RMS).  No
function here is unpinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Iterable, Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_LIB = os.path.join(_HERE, "libssd_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``ssd_oracle.c`` with gcc (fp64, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", _LIB, _SRC, "-lm"])
    return _LIB


def _load():
    global _lib
    if _lib is None:
        _lib = _open(build())
    return _lib


def _open(path: str):
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    lib.oracle_ssd_forward.argtypes = [I64, P, I64, I64, I64, I64, P, P, P, P, P, P, P, P, P, P, ctypes.c_int]
    lib.oracle_ssd_forward.restype = ctypes.c_int
    lib.oracle_ssd_decode_step.argtypes = [I64, I64, I64, I64, I64, P, P, P, P, P, P, P, P]
    lib.oracle_ssd_decode_step.restype = ctypes.c_int
    return lib


class using_library:
    """Temporarily route this module through another build of the oracle source.

    Used only by the mutation test, which compiles deliberately broken copies of
    ``ssd_oracle.c`` to show that the pins detect each planted mistake."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        self.saved = _load()
        _lib = _open(self.path)
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def ssd_forward(x, dt, A, B, C, D=None, init=None, seq_offsets=None, head_group=None, nthreads: int = 0
                ) -> Tuple[np.ndarray, np.ndarray]:
    """fp64 recurrence on numpy arrays.

    x (T, H, P); dt (T, H); A (H,); B, C (T, G, N); D (H,) or None;
    init (nseq, H, P, N) or None; seq_offsets (nseq+1) token offsets (default:
    one sequence of T tokens); head_group (H,) int or None (default h // (H/G)).
    Returns y (T, H, P) and final (nseq, H, P, N), both fp64.
    """
    x, dt, A, B, C = _f64(x), _f64(dt), _f64(A), _f64(B), _f64(C)
    T, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    offs = np.ascontiguousarray([0, T] if seq_offsets is None else seq_offsets, dtype=np.int64)
    nseq = len(offs) - 1
    D = None if D is None else _f64(D)
    init = None if init is None else _f64(init)
    hg = None if head_group is None else np.ascontiguousarray(head_group, dtype=np.int32)
    y = np.zeros((T, H, P))
    fin = np.zeros((nseq, H, P, N))
    rc = _load().oracle_ssd_forward(nseq, _ptr(offs), H, P, N, G, _ptr(hg), _ptr(x), _ptr(dt), _ptr(A), _ptr(B),
                                    _ptr(C), _ptr(D), _ptr(init), _ptr(y), _ptr(fin), int(nthreads))
    if rc:
        raise RuntimeError(f"oracle_ssd_forward failed ({rc})")
    return y, fin


def ssd_forward_problem(prob, pairs: Optional[Iterable[Tuple[int, int]]] = None, nthreads: int = 0):
    """Run the oracle on a ``workloads.Problem`` (torch CPU tensors, already rounded).

    With ``pairs`` = [(seq, head), ...] only those are computed: the sequences and
    heads involved are gathered into a compact sub-problem (every sampled sequence
    x every sampled head), so full-size workloads cost only what is sampled.
    Returns (y, final) with y shaped like the full (tokens, H, P) problem but only
    the sampled rows filled (NaN elsewhere), and final (nseq, H, P, N) likewise.
    """
    wl = prob.wl
    H, P, N, G = wl.nheads, wl.headdim, wl.dstate, wl.ngroups
    T = wl.tokens
    offs = prob.seq_offsets
    nseq = len(offs) - 1
    x = prob.x.reshape(T, H, P)
    dt = prob.dt.reshape(T, H)
    B = prob.B.reshape(T, G, N)
    C = prob.C.reshape(T, G, N)
    if pairs is None:
        seqs, heads = list(range(nseq)), list(range(H))
    else:
        pairs = list(pairs)
        seqs = sorted({s for s, _ in pairs})
        heads = sorted({h for _, h in pairs})
    hpg = H // G
    groups = sorted({h // hpg for h in heads})
    gidx = {g: i for i, g in enumerate(groups)}
    head_group = [gidx[h // hpg] for h in heads]
    # token index list of the selected sequences, in order
    tok = np.concatenate([np.arange(offs[s], offs[s + 1]) for s in seqs]) if seqs else np.zeros(0, np.int64)
    sub_offs = np.cumsum([0] + [offs[s + 1] - offs[s] for s in seqs])
    hs = np.asarray(heads)
    gs = np.asarray(groups)
    xs = x[tok][:, hs].double().numpy()
    dts = dt[tok][:, hs].double().numpy()
    Bs = B[tok][:, gs].double().numpy()
    Cs = C[tok][:, gs].double().numpy()
    As = prob.A[hs].double().numpy()
    Ds = None if prob.D is None else prob.D[hs].double().numpy()
    init = None
    if prob.init_state is not None:
        init = prob.init_state[np.asarray(seqs)][:, hs].double().numpy()
    ys, fs = ssd_forward(xs, dts, As, Bs, Cs, Ds, init, sub_offs, head_group, nthreads)
    y = np.full((T, H, P), np.nan)
    fin = np.full((nseq, H, P, N), np.nan)
    for si, s in enumerate(seqs):
        for hi, h in enumerate(heads):
            if pairs is not None and (s, h) not in set(pairs):
                continue
            y[offs[s]:offs[s + 1], h] = ys[sub_offs[si]:sub_offs[si + 1], hi]
            fin[s, h] = fs[si, hi]
    return y, fin


def dt_prologue(dt_raw, dt_bias=None, softplus: bool = True, dt_min: float = 0.0, dt_max: float = np.inf):
    """The pages' discretisation of the step size, in fp64: v = dt_raw + dt_bias (bias per head,
    the last axis), dt = log(1 + exp(v)) when ``softplus``, then clamped to [dt_min, dt_max]."""
    v = _f64(dt_raw) + (0.0 if dt_bias is None else _f64(dt_bias))
    if softplus:
        v = np.logaddexp(0.0, v)  # log(exp(0) + exp(v)) = log(1 + exp(v))
    return np.clip(v, dt_min, dt_max)


def causal_conv1d_silu(x, weight, bias=None, seq_offsets=None):
    """Depthwise causal convolution of kernel K = weight.shape[1] along time, then SiLU, in
    fp64: out[t, c] = silu(bias[c] + sum_k weight[c, k] x[t - (K-1) + k, c]) with x = 0
    before each sequence's first token; silu(v) = v / (1 + exp(-v)).
    x (T, channels); seq_offsets (nseq + 1) token offsets (default: one sequence)."""
    x, w = _f64(x), _f64(weight)
    T, ch = x.shape
    K = w.shape[1]
    offs = [0, T] if seq_offsets is None else list(seq_offsets)
    out = np.zeros((T, ch))
    for s in range(len(offs) - 1):
        a, e = int(offs[s]), int(offs[s + 1])
        for t in range(a, e):
            acc = np.zeros(ch) if bias is None else _f64(bias).copy()
            for k in range(K):
                src = t - (K - 1) + k
                if src >= a:
                    acc += w[:, k] * x[src]
            out[t] = acc / (1.0 + np.exp(-acc))
    return out


def gated_rmsnorm(y, z, weight, eps: float = 1e-5):
    """Gate first, then RMSNorm over the last axis, in fp64: g = y * silu(z),
    out = g / sqrt(mean(g^2) + eps) * weight."""
    y, z, w = _f64(y), _f64(z), _f64(weight)
    g = y * (z / (1.0 + np.exp(-z)))
    return g / np.sqrt(np.mean(g * g, axis=-1, keepdims=True) + eps) * w


def decode_step(x, dt, A, B, C, D, state):
    """One recurrent step in fp64; returns (y, new_state) without touching ``state``.

    x (batch, H, P); dt (batch, H); A, D (H,); B, C (batch, G, N); state (batch, H, P, N).
    """
    x, dt, A, B, C = _f64(x), _f64(dt), _f64(A), _f64(B), _f64(C)
    D = None if D is None else _f64(D)
    st = np.array(state, dtype=np.float64, copy=True)
    bsz, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    y = np.zeros((bsz, H, P))
    rc = _load().oracle_ssd_decode_step(bsz, H, P, N, G, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                        _ptr(st), _ptr(y))
    if rc:
        raise RuntimeError(f"oracle_ssd_decode_step failed ({rc})")
    return y, st
