"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the same
seeded inputs, at sizes the oracle finishes in seconds (several chunks and a ragged
tail) and at the five full-size workloads on every (sequence, head) pair."""
import numpy as np
import pytest
import torch

import oracle
import ssd_sequence_mixing_b200 as ssd
import workloads
from harness import assert_close, check, check_every_pair, run, sample_pairs, to_device

pytestmark = pytest.mark.gpu

PATHS = {"simt": ssd.PATH_SIMT, "auto": ssd.PATH_AUTO}


def tc_available(prob, chunk):
    s = ssd.make_shape(prob.x, prob.B, prob.cu_seqlens)
    old = ssd.set_path(ssd.PATH_TC)
    try:
        return ssd.select_path(s, chunk) == ssd.PATH_TC
    finally:
        ssd.set_path(old)


def paths_for(prob, chunk):
    out = [("simt", ssd.PATH_SIMT)]
    if tc_available(prob, chunk):
        out.append(("tc", ssd.PATH_TC))
    return out


# ------------------------------------------------------------------ small cases
def test_tiny_fp32_workload():
    prob = workloads.generate(workloads.TINY, seed=0)
    for name, path in paths_for(prob, 64):
        y, fin = run(prob, path=path)
        check(prob, y, fin)


SMALL = [
    # batch, T, H, P, N, G, chunk, dtype, init
    (2, 700, 4, 64, 128, 2, 256, "bf16", True),
    (1, 513, 3, 64, 64, 1, 128, "bf16", False),
    (3, 130, 2, 64, 128, 1, 64, "bf16", True),
    (2, 300, 4, 32, 16, 4, 64, "f32", True),
    (1, 257, 2, 17, 33, 2, 128, "f32", False),
    (2, 200, 2, 64, 256, 1, 256, "bf16", False),
    (1, 1, 4, 64, 128, 1, 256, "bf16", True),
    # one long sequence and two head pairs: their 128 tiles are spread over many CTAs,
    # which hand the state on to one another
    (1, 8192, 4, 64, 128, 1, 256, "bf16", True),
    (1, 2048, 2, 64, 128, 1, 256, "bf16", True),  # 2 heads: no 4-head dt rows, SIMT path
    (3, 1000, 16, 64, 64, 2, 128, "bf16", True),
    # state sizes the tensor-core path pads (16, 32, 96) or splits in column halves (256)
    (2, 700, 4, 64, 16, 1, 256, "bf16", True),
    (1, 900, 8, 64, 32, 2, 128, "bf16", True),
    (2, 333, 4, 64, 96, 1, 256, "bf16", True),
    (2, 700, 4, 64, 256, 1, 256, "bf16", True),
    (1, 1100, 8, 64, 256, 2, 64, "bf16", False),
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "b{}_T{}_H{}_P{}_N{}_G{}_Q{}_{}_init{}".format(*c))
def test_small_dense(case):
    b, T, H, P, N, G, Q, dt, init = case
    wl = workloads.custom(b, T, H, P, N, G, chunk=Q, dtype=dt, init=init)
    prob = workloads.generate(wl, seed=1)
    for name, path in paths_for(prob, Q):
        y, fin = run(prob, path=path)
        check(prob, y, fin)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_small_packed_with_resets(dtype):
    lens = [1, 63, 64, 65, 0, 300, 257, 511, 2]
    wl = workloads.custom(1, 0, H=4, P=64, N=128, G=2, chunk=128, dtype=dtype, init=True, lengths=lens)
    prob = workloads.generate(wl, seed=2, lengths=lens)
    for name, path in paths_for(prob, 128):
        y, fin = run(prob, path=path)
        check(prob, y, fin)


@pytest.mark.parametrize("lengths", [[8192], [300, 12000, 5]], ids=["one_long", "long_between_short"])
def test_packed_long_sequence_hands_state_between_ctas(lengths):
    """A packed sequence far longer than one CTA's share of the tiles: its tiles are cut
    across many CTAs, each waiting for the state the one before it hands on."""
    wl = workloads.custom(1, 0, H=4, P=64, N=128, G=1, chunk=256, dtype="bf16", init=True, lengths=lengths)
    prob = workloads.generate(wl, seed=15, lengths=lengths)
    for name, path in paths_for(prob, 256):
        y, fin = run(prob, path=path)
        check(prob, y, fin)


@pytest.mark.parametrize("case", [(1, 20000, 4, 128), (3, 9000, 8, 64), (2, 4097, 2 * 4, 128)],
                         ids=["b1_T20000_H4", "b3_T9000_H8_N64", "b2_T4097_H8"])
def test_dense_long_sequences_in_segments(case):
    """Dense batches whose units are much longer than one CTA's share: the library cuts the
    sequences into segments (a final-state-only pass, the segments' start states, the full
    pass); every y row and final state must match the single-pass oracle."""
    b, T, H, N = case
    wl = workloads.custom(b, T, H=H, P=64, N=N, G=1, chunk=256, dtype="bf16", init=True)
    prob = workloads.generate(wl, seed=16)
    y, fin = run(prob)
    check(prob, y, fin)


@pytest.mark.parametrize("case", [(4, 1024, 64, 128, 8), (2, 1536, 128, 64, 4)], ids=["H64_G8_N128", "H128_G4_N64"])
def test_dense_many_tiles_per_cta(case):
    """Enough heads that no sequence is cut into segments and every CTA runs several tiles
    in a row (its ring of B/C tiles, both x stages and both S/P buffers in turn) and hands
    the state on inside units."""
    b, T, H, N, G = case
    wl = workloads.custom(b, T, H=H, P=64, N=N, G=G, chunk=256, dtype="bf16", init=True)
    prob = workloads.generate(wl, seed=18)
    y, fin = run(prob)
    check(prob, y, fin)


@pytest.mark.parametrize("batch", [18, 19], ids=["in_kernel", "weight_kernel"])
def test_split_weights_either_side_of_the_threshold(batch):
    """The work split's tile weights come from the fused kernel's own CTAs (one flag barrier)
    while there are at most two sequence tiles per SM, and from a kernel of their own beyond
    that: batch 18 x 16 tiles (288) and 19 x 16 (304) fall either side of 2 x 148."""
    if torch.cuda.get_device_properties(0).multi_processor_count != 148:
        pytest.skip("the threshold is set for 148 SMs")
    wl = workloads.custom(batch, 2048, H=64, P=64, N=128, G=1, chunk=256, dtype="bf16", init=True)
    prob = workloads.generate(wl, seed=23)
    dev = to_device(prob)
    assert ssd.select_path(ssd.make_shape(dev["x"], dev["B"], dev["cu_seqlens"]), wl.chunk) == ssd.PATH_TC
    y, fin = run(prob, dev=dev)
    check(prob, y, fin, pairs=sample_pairs(prob, k=8))


def test_packed_passes_and_hand_ons():
    """Heads that decay too fast for one pass per tile (A = -1e4 and -60), in packed
    sequences long enough to be cut across CTAs."""
    lens = [700, 2500, 64, 1800]
    wl = workloads.custom(1, 0, H=8, P=64, N=128, G=2, chunk=256, dtype="bf16", init=True, lengths=lens)
    prob = workloads.generate(wl, seed=19, lengths=lens, A_override=[-1e4, -1.0, -60.0, -2.0, -0.5, -30.0, -8.0, -1e-3])
    for name, path in paths_for(prob, 256):
        y, fin = run(prob, path=path)
        check(prob, y, fin)


def test_final_state_only_matches_full_pass():
    """y = NULL: only the final states, without reading C or D; equal to the full pass's."""
    wl = workloads.custom(3, 700, H=8, P=64, N=128, G=2, chunk=256, dtype="bf16", init=True)
    prob = workloads.generate(wl, seed=17)
    dev = to_device(prob)
    for name, path in paths_for(prob, 256):
        old = ssd.set_path(path)
        try:
            _, fin = ssd.ssd_forward(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["init_state"],
                                     None, 256)
            fin_only = ssd.ssd_final_state(dev["x"], dev["dt"], dev["A"], dev["B"], dev["init_state"], None, 256)
        finally:
            ssd.set_path(old)
        torch.cuda.synchronize()
        assert torch.equal(fin, fin_only), name
        _, f_ref = oracle.ssd_forward_problem(prob)
        assert_close("final_state", fin_only.cpu().numpy(), f_ref, "bf16")


def test_packed_many_sequences_grouped():
    """Many packed sequences of mixed lengths (some shorter than a tile, some empty) with
    8 heads per B/C group: the flat tile list is cut across CTAs mid-sequence."""
    rng = np.random.default_rng(9)
    lens = [int(v) for v in rng.integers(0, 700, 40)]
    wl = workloads.custom(1, 0, H=16, P=64, N=128, G=2, chunk=256, dtype="bf16", init=True, lengths=lens)
    prob = workloads.generate(wl, seed=9, lengths=lens)
    for name, path in paths_for(prob, 256):
        y, fin = run(prob, path=path)
        check(prob, y, fin, pairs=sample_pairs(prob, k=12))


@pytest.mark.parametrize("Q", [64, 128, 256])
def test_chunk_lengths_agree(Q):
    wl = workloads.custom(2, 600, H=4, P=64, N=64, G=1, chunk=Q, dtype="bf16", init=True)
    prob = workloads.generate(wl, seed=3)
    for name, path in paths_for(prob, Q):
        y, fin = run(prob, chunk=Q, path=path)
        check(prob, y, fin)


def test_tiny_dt_and_strong_decay():
    """dt scaled down 1000x (decay ~1, long memory) and A = -1e4 (decay underflows to 0)."""
    wl = workloads.custom(1, 400, H=4, P=64, N=128, G=1, chunk=256, dtype="bf16", init=True)
    for kw in (dict(dt_scale=1e-3), dict(A_override=[-1e4, -1.0, -50.0, -1e-3])):
        prob = workloads.generate(wl, seed=4, **kw)
        for name, path in paths_for(prob, 256):
            y, fin = run(prob, path=path)
            check(prob, y, fin)


@pytest.mark.parametrize("case", [(2, 700, 4, 64, 128, 2, 256, "bf16", True, 1e-3, 0.3),
                                  (1, 300, 3, 32, 16, 1, 64, "f32", True, 0.0, float("inf")),
                                  (2, 260, 8, 64, 64, 2, 128, "bf16", False, 0.0, float("inf"))],
                         ids=["bf16_softplus_clamp", "f32_softplus", "bf16_bias_only"])
def test_fused_dt_prologue(case):
    """ssd_forward_dt makes dt = clamp(softplus(dt_raw + dt_bias)) inside the kernels; the
    oracle runs on the same raw values through its own fp64 prologue."""
    b, T, H, P, N, G, Q, dtype, softplus, lo, hi = case
    wl = workloads.custom(b, T, H, P, N, G, chunk=Q, dtype=dtype, init=True)
    prob = workloads.generate(wl, seed=12)
    rng = np.random.default_rng(12)
    mean = -3.0 if softplus else 0.05
    raw = torch.from_numpy(rng.normal(mean, 1.0 if softplus else 0.01, tuple(prob.dt.shape)).astype(np.float32))
    bias = torch.from_numpy(rng.uniform(-1, 1, H).astype(np.float32) * (1.0 if softplus else 0.01))
    if not softplus:
        raw = raw.abs()
    ref_dt = oracle.dt_prologue(raw.double().numpy(), bias.double().numpy(), softplus, lo, hi)
    prob.dt = torch.from_numpy(ref_dt)  # the oracle reads dt from the problem (fp64 here)
    dev = to_device(prob)
    raw_d, bias_d = raw.cuda(), bias.cuda()
    for name, path in paths_for(prob, Q):
        old = ssd.set_path(path)
        try:
            y, fin = ssd.ssd_forward_dt(dev["x"], raw_d, dev["A"], dev["B"], dev["C"], dev["D"], dev["init_state"],
                                        None, Q, dt_bias=bias_d, softplus=softplus, dt_min=lo, dt_max=hi)
        finally:
            ssd.set_path(old)
        torch.cuda.synchronize()
        check(prob, y, fin)


def test_no_skip_no_init_no_final():
    wl = workloads.custom(1, 300, H=4, P=64, N=64, G=1, chunk=128, dtype="bf16")
    prob = workloads.generate(wl, seed=5)
    prob.D = None
    for name, path in paths_for(prob, 128):
        y, fin = run(prob, path=path, return_final=False)
        assert fin is None
        check(prob, y, None)


def test_deterministic():
    wl = workloads.custom(2, 700, H=4, P=64, N=128, G=2, chunk=256, dtype="bf16", init=True)
    prob = workloads.generate(wl, seed=6)
    dev = to_device(prob)
    for name, path in paths_for(prob, 256):
        y1, f1 = run(prob, path=path, dev=dev)
        y2, f2 = run(prob, path=path, dev=dev)
        assert torch.equal(y1, y2) and torch.equal(f1, f2), name


def test_host_entry_point_matches_device():
    wl = workloads.custom(1, 500, H=4, P=64, N=64, G=2, chunk=128, dtype="bf16", init=True,
                          lengths=[100, 0, 400])
    prob = workloads.generate(wl, seed=7, lengths=[100, 0, 400])
    y, fin = run(prob)
    pin = lambda t: None if t is None else t.pin_memory()
    yh, fh = ssd.ssd_forward_host(pin(prob.x), pin(prob.dt), pin(prob.A), pin(prob.B), pin(prob.C), pin(prob.D),
                                  pin(prob.init_state), pin(prob.cu_seqlens), chunk=128)
    assert torch.equal(yh, y.cpu()) and torch.equal(fh, fin.cpu())


@pytest.mark.parametrize("lengths", [None, [700, 0, 1, 300, 129, 2048, 64, 5, 900, 33]], ids=["dense", "packed"])
def test_host_entry_point_groups_match_device(lengths):
    """The host entry point copies in, computes and copies out by groups of whole sequences;
    every sequence's outputs match the oracle and the single device call's (each group is
    its own launch, so the CTA split, and with it the rounding, may differ)."""
    if lengths is None:
        wl = workloads.custom(6, 500, H=8, P=64, N=128, G=2, chunk=256, dtype="bf16", init=True)
        prob = workloads.generate(wl, seed=11)
    else:
        wl = workloads.custom(1, 0, H=8, P=64, N=64, G=1, chunk=128, dtype="bf16", init=True, lengths=lengths)
        prob = workloads.generate(wl, seed=11, lengths=lengths)
    y, fin = run(prob, chunk=wl.chunk)
    pin = lambda t: None if t is None else t.pin_memory()
    yh, fh = ssd.ssd_forward_host(pin(prob.x), pin(prob.dt), pin(prob.A), pin(prob.B), pin(prob.C), pin(prob.D),
                                  pin(prob.init_state), pin(prob.cu_seqlens), chunk=wl.chunk)
    check(prob, yh, fh)
    assert_close("y vs device call", yh.float().numpy(), y.float().cpu().double().numpy(), "bf16")
    assert_close("final vs device call", fh.numpy(), fin.cpu().double().numpy(), "bf16")


def test_bad_device_seqlens_sets_status_and_writes_nothing():
    wl = workloads.custom(1, 300, H=4, P=64, N=64, G=1, chunk=128, dtype="bf16", lengths=[100, 200])
    prob = workloads.generate(wl, seed=8, lengths=[100, 200])
    dev = to_device(prob)
    dev["cu_seqlens"] = torch.tensor([0, 250, 200], dtype=torch.int32, device="cuda")  # not monotone
    assert ssd.query_status() == 0
    y = torch.full_like(dev["x"], 7.0)
    fin = torch.full((2, 4, 64, 64), 7.0, device="cuda")
    ssd.ssd_forward(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], None, dev["cu_seqlens"], 128,
                    y=y, final_state=fin)
    assert ssd.query_status() == 6
    assert ssd.query_status() == 0  # cleared by the read
    assert bool((y == 7.0).all()) and bool((fin == 7.0).all())


# ----------------------------------------------------------- full-size workloads
FULL = [workloads.TINY, workloads.MAMBA2_2P7B] + workloads.STATE_SWEEP + workloads.LENGTH_SWEEP + [workloads.PACKED]


@pytest.mark.parametrize("wl", FULL, ids=lambda w: w.name)
def test_full_size_every_pair(wl):
    """Full-size inputs in the launch configuration the bench times (auto path), checked
    against the oracle on every (sequence, head) pair: every output element of y and of
    the final states, including the tiles where CTAs hand the state on."""
    prob = workloads.generate(wl, seed=0)
    y, fin = run(prob)
    check_every_pair(prob, y, fin)


# ------------------------------------------------------------------ edge cases
def test_all_sequences_empty_gives_init_as_final():
    """Packed sequences that are all empty: no y rows; every final state equals its init."""
    lens = [0, 0, 0]
    wl = workloads.custom(1, 0, H=4, P=64, N=64, G=1, chunk=128, dtype="bf16", init=True, lengths=lens)
    prob = workloads.generate(wl, seed=13, lengths=lens)
    dev = to_device(prob)
    for name, path in [("simt", ssd.PATH_SIMT), ("auto", ssd.PATH_AUTO)]:
        old = ssd.set_path(path)
        try:
            y, fin = ssd.ssd_forward(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["init_state"],
                                     dev["cu_seqlens"], 128)
        finally:
            ssd.set_path(old)
        torch.cuda.synchronize()
        assert y.numel() == 0 and ssd.query_status() == 0
        assert torch.equal(fin, dev["init_state"]), name


def test_largest_head_and_state_sizes():
    """P = N = 256 (the largest the boundary takes) on the SIMT path, fp32 and bf16."""
    for dtype in ("f32", "bf16"):
        wl = workloads.custom(1, 200, H=2, P=256, N=256, G=1, chunk=64, dtype=dtype, init=True)
        prob = workloads.generate(wl, seed=14)
        y, fin = run(prob)
        check(prob, y, fin)


SWEEP = np.random.default_rng(2024)


def _sweep_cases(n=10):
    cases = []
    for k in range(n):
        G = int(SWEEP.choice([1, 2]))
        H = G * int(SWEEP.choice([2, 4]))
        P = int(SWEEP.choice([16, 32, 64]))
        N = int(SWEEP.choice([16, 64, 128]))
        Q = int(SWEEP.choice([64, 128, 256]))
        dtype = str(SWEEP.choice(["bf16", "f32"]))
        lens = [int(v) for v in SWEEP.integers(0, 600, int(SWEEP.integers(1, 5)))]
        cases.append((k, H, P, N, G, Q, dtype, lens))
    return cases


@pytest.mark.parametrize("case", _sweep_cases(), ids=lambda c: "sweep{}_H{}_P{}_N{}_G{}_Q{}_{}".format(*c[:7]))
def test_seeded_shape_sweep(case):
    """Seeded random shapes, chunk lengths, dtypes and packed length mixes, every path."""
    k, H, P, N, G, Q, dtype, lens = case
    if sum(lens) == 0:
        lens = lens + [1]
    wl = workloads.custom(1, 0, H=H, P=P, N=N, G=G, chunk=Q, dtype=dtype, init=bool(k % 2), lengths=lens)
    prob = workloads.generate(wl, seed=100 + k, lengths=lens)
    for name, path in paths_for(prob, Q):
        y, fin = run(prob, path=path)
        check(prob, y, fin)


def test_final_state_only_repeated_with_resets():
    """The final-state-only variant at a size where its warps run ahead of the MMA warp:
    heads that re-centre every tile (A = -60, -1e4) and long dense units (segments), run
    repeatedly; every call must end without a wait giving up and match the full pass."""
    wl = workloads.custom(4, 3000, H=16, P=64, N=128, G=2, chunk=256, dtype="bf16", init=True)
    A = [-1e4, -1.0, -60.0, -2.0, -0.5, -30.0, -8.0, -1e-3] * 2
    prob = workloads.generate(wl, seed=23, A_override=A)
    dev = to_device(prob)
    _, fin = ssd.ssd_forward(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["init_state"], None, 256)
    for _ in range(5):
        fin_only = ssd.ssd_final_state(dev["x"], dev["dt"], dev["A"], dev["B"], dev["init_state"], None, 256)
        torch.cuda.synchronize()
        assert ssd.query_status() == 0
        assert torch.equal(fin, fin_only)
    _, f_ref = oracle.ssd_forward_problem(prob)
    assert_close("final_state", fin_only.cpu().numpy(), f_ref, "bf16")
