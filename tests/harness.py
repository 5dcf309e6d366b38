"""Shared helpers for the GPU parity tests: move a workloads.Problem to the device,
run the library through its C ABI, and compare with the fp64 oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import ssd_sequence_mixing_b200 as ssd

# Tolerances for y and final_state against the fp64 oracle (the oracle consumes
# the already-rounded inputs, so only the GPU arithmetic is measured):
#   fp32 I/O: relative L2 <= 1e-4
#   bf16 I/O: relative L2 <= 5e-3 and max-abs <= 3e-2 * max|reference|
TOL = {"f32": dict(rel_l2=1e-4, max_abs_frac=None), "bf16": dict(rel_l2=5e-3, max_abs_frac=3e-2)}


def to_device(prob, device="cuda"):
    d = {}
    for k in ("x", "dt", "A", "B", "C", "D", "init_state", "cu_seqlens"):
        v = getattr(prob, k)
        d[k] = None if v is None else v.to(device).contiguous()
    return d


def run(prob, chunk=None, path=ssd.PATH_AUTO, dev=None, return_final=True):
    dev = dev or to_device(prob)
    old = ssd.set_path(path)
    try:
        y, fin = ssd.ssd_forward(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["init_state"],
                                 dev["cu_seqlens"], chunk or prob.wl.chunk, return_final=return_final)
    finally:
        ssd.set_path(old)
    torch.cuda.synchronize()
    return y, fin


def errors(got: np.ndarray, ref: np.ndarray):
    m = ~np.isnan(ref)
    g, r = got[m].astype(np.float64), ref[m]
    rel = float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-300))
    mx = float(np.abs(g - r).max()) if g.size else 0.0
    ref_max = float(np.abs(r).max()) if r.size else 0.0
    return rel, mx, ref_max


def assert_close(name, got, ref, dtype):
    tol = TOL[dtype]
    rel, mx, ref_max = errors(got, ref)
    assert np.isfinite(got[~np.isnan(ref)]).all(), f"{name}: non-finite values"
    assert rel <= tol["rel_l2"], f"{name}: relative L2 {rel:.3e} > {tol['rel_l2']:.1e}"
    if tol["max_abs_frac"] is not None:
        assert mx <= tol["max_abs_frac"] * ref_max, f"{name}: max-abs {mx:.3e} > {tol['max_abs_frac']} * {ref_max:.3e}"
    return rel, mx


def check(prob, y, fin, pairs=None):
    """Compare device outputs with the oracle (all pairs, or only ``pairs``)."""
    y_ref, f_ref = oracle.ssd_forward_problem(prob, pairs=pairs)
    wl = prob.wl
    y_np = y.float().cpu().numpy().reshape(wl.tokens, wl.nheads, wl.headdim)
    ry = assert_close("y", y_np, y_ref, wl.dtype)
    rf = None
    if fin is not None:
        rf = assert_close("final_state", fin.cpu().numpy(), f_ref, wl.dtype)
    return ry, rf


def sample_pairs(prob, k=6, seed=0):
    """(sequence, head) pairs: the corners plus seeded random picks."""
    rng = np.random.default_rng(seed)
    nseq, H = prob.nseq, prob.wl.nheads
    pairs = {(0, 0), (nseq - 1, H - 1)}
    while len(pairs) < min(k, nseq * H):
        pairs.add((int(rng.integers(nseq)), int(rng.integers(H))))
    return sorted(pairs)
