"""Shared helpers for the GPU parity tests: move a workloads.Problem to the device,
run the library through its C ABI, and compare with the fp64 oracle."""
from __future__ import annotations

import warnings

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


class ParityMargin(UserWarning):
    """Carries a full-size comparison's errors and tolerances into the pytest summary."""


def check_every_pair(prob, y, fin, head_block=16, seq_block_tokens=1 << 16):
    """Compare the device outputs with the oracle on EVERY (sequence, head) pair, one block
    of whole sequences x ``head_block`` heads at a time, so that the fp64 reference never
    needs a full-size buffer.  Asserts the tolerances on the accumulated relative L2 and
    max-abs errors of y and final_state, and reports them as a ParityMargin warning."""
    wl = prob.wl
    T, H, P, N, G = wl.tokens, wl.nheads, wl.headdim, wl.dstate, wl.ngroups
    hpg = H // G
    offs = prob.seq_offsets
    nseq = len(offs) - 1
    x = prob.x.reshape(T, H, P)
    dt = prob.dt.reshape(T, H)
    B = prob.B.reshape(T, G, N)
    C = prob.C.reshape(T, G, N)
    yd = y.reshape(T, H, P)
    acc = {"y": np.zeros(4), "final_state": np.zeros(4)}  # sum sq err, sum sq ref, max err, max ref

    def add(name, got, ref):
        a = acc[name]
        d = got - ref
        a[0] += float((d * d).sum())
        a[1] += float((ref * ref).sum())
        a[2] = max(a[2], float(np.abs(d).max()) if d.size else 0.0)
        a[3] = max(a[3], float(np.abs(ref).max()) if ref.size else 0.0)
        if not np.isfinite(got).all():
            raise AssertionError(f"{name}: non-finite values")

    s0 = 0
    while s0 < nseq:  # whole sequences, about seq_block_tokens tokens per block
        s1 = s0 + 1
        while s1 < nseq and offs[s1 + 1] - offs[s0] <= seq_block_tokens:
            s1 += 1
        a, b = offs[s0], offs[s1]
        sub_offs = np.asarray([o - a for o in offs[s0:s1 + 1]], dtype=np.int64)
        for h0 in range(0, H, head_block):
            hs = np.arange(h0, min(H, h0 + head_block))
            groups = sorted({int(h) // hpg for h in hs})
            gidx = {g: i for i, g in enumerate(groups)}
            init = None if prob.init_state is None else prob.init_state[s0:s1][:, hs].double().numpy()
            ys, fs = oracle.ssd_forward(x[a:b][:, hs].double().numpy(), dt[a:b][:, hs].double().numpy(),
                                        prob.A[hs].double().numpy(), B[a:b][:, groups].double().numpy(),
                                        C[a:b][:, groups].double().numpy(),
                                        None if prob.D is None else prob.D[hs].double().numpy(), init, sub_offs,
                                        [gidx[int(h) // hpg] for h in hs])
            add("y", yd[a:b, h0:h0 + len(hs)].double().cpu().numpy(), ys)
            if fin is not None:
                add("final_state", fin[s0:s1, h0:h0 + len(hs)].double().cpu().numpy(), fs)
        s0 = s1
    tol = TOL[wl.dtype]
    report = []
    for name, a in acc.items():
        if name == "final_state" and fin is None:
            continue
        rel = float(np.sqrt(a[0] / max(a[1], 1e-300)))
        frac = a[2] / max(a[3], 1e-300)
        report.append(f"{name}: rel-L2 {rel:.2e} (tol {tol['rel_l2']:.0e}), max-abs/max|ref| {frac:.2e}"
                      + (f" (tol {tol['max_abs_frac']:.0e})" if tol["max_abs_frac"] else ""))
        assert rel <= tol["rel_l2"], f"{wl.name} {name}: relative L2 {rel:.3e} > {tol['rel_l2']:.1e}"
        if tol["max_abs_frac"] is not None:
            assert frac <= tol["max_abs_frac"], f"{wl.name} {name}: max-abs {a[2]:.3e} > {tol['max_abs_frac']} * {a[3]:.3e}"
    warnings.warn(ParityMargin(f"{wl.name}, all {nseq} x {H} (sequence, head) pairs: " + "; ".join(report)))
    return acc
