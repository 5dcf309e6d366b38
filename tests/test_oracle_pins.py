"""Pins for the fp64 oracle, checked against what the pages and the mathematics fix.

Each test uses code independent of the oracle's recurrence: a dense
brute-force semiseparable matrix, textbook special cases, closed forms, the
pages' chunked algorithm (numpy restatement) and hand-worked values.
Source: "Transformers are SSMs" (wikillm.com card, Method steps 1-8).
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle.chunked import ssd_chunked

HERE = os.path.dirname(os.path.abspath(__file__))


def rand_problem(rng, T, H, P, N, G, nseq=1):
    x = rng.standard_normal((T, H, P))
    dt = rng.uniform(0.01, 0.6, (T, H))
    A = -rng.uniform(0.5, 3.0, H)
    B = rng.standard_normal((T, G, N)) / math.sqrt(N)
    C = rng.standard_normal((T, G, N)) / math.sqrt(N)
    D = rng.standard_normal(H)
    return x, dt, A, B, C, D


def rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


# ---------------------------------------------------------------- brute force
def dense_M(dt, A, B, C, h, g):
    """Dense lower-triangular M for one head (Method steps 1-2: M = L o (C B^T),
    L[j, i] = prod_{r=i+1..j} a_r), with the dt input scaling folded into column i.
    The decay product is formed by repeated multiplication, not by cumsum/exp differences."""
    T = dt.shape[0]
    a = np.exp(dt[:, h] * A[h])
    M = np.zeros((T, T))
    for j in range(T):
        prod = 1.0
        for i in range(j, -1, -1):
            M[j, i] = (C[j, g] @ B[i, g]) * prod * dt[i, h]
            prod *= a[i]
    return M


@pytest.mark.parametrize("T,H,P,N,G", [(1, 1, 1, 1, 1), (17, 2, 3, 5, 1), (48, 4, 3, 4, 2), (64, 2, 5, 3, 2)])
def test_dense_semiseparable_matrix(T, H, P, N, G):
    rng = np.random.default_rng(T * 100 + H)
    x, dt, A, B, C, D = rand_problem(rng, T, H, P, N, G)
    y, fin = oracle.ssd_forward(x, dt, A, B, C, D)
    for h in range(H):
        g = h // (H // G)
        M = dense_M(dt, A, B, C, h, g)
        y_ref = M @ x[:, h, :] + D[h] * x[:, h, :]
        assert rel(y[:, h, :], y_ref) < 1e-12
        # final state = sum_i (prod_{r>i} a_r) dt_i x_i B_i^T
        a = np.exp(dt[:, h] * A[h])
        S = np.zeros((P, N))
        for i in range(T):
            S += np.prod(a[i + 1:]) * dt[i, h] * np.outer(x[i, h], B[i, g])
        assert rel(fin[0, h], S) < 1e-12


# ------------------------------------------------------------ special cases
def test_unit_decay_is_causal_linear_attention():
    """a_t == 1 (A = 0): the layer is causal linear attention (Method step 3, sec. 5.2)."""
    rng = np.random.default_rng(1)
    T, H, P, N, G = 40, 3, 4, 6, 1
    x, dt, A, B, C, D = rand_problem(rng, T, H, P, N, G)
    A = np.zeros(H)
    y, _ = oracle.ssd_forward(x, dt, A, B, C, D)
    K = B[:, 0, :]  # keys
    Qm = C[:, 0, :]  # queries
    scores = np.tril(Qm @ K.T)  # causal, unnormalised
    for h in range(H):
        V = dt[:, h:h + 1] * x[:, h, :]
        assert rel(y[:, h, :], scores @ V + D[h] * x[:, h, :]) < 1e-12


def test_zero_decay_is_diagonal():
    """a_t == 0: only the token's own term survives, y_t = (C_t . B_t) dt_t x_t + D x_t."""
    rng = np.random.default_rng(2)
    T, H, P, N, G = 25, 2, 3, 4, 1
    x, _, _, B, C, D = rand_problem(rng, T, H, P, N, G)
    dt = rng.uniform(0.5, 1.0, (T, H))
    A = np.full(H, -2000.0)  # dt*A <= -1000: exp underflows to exactly 0 in fp64
    assert np.all(np.exp(dt * A[None]) == 0.0)
    y, fin = oracle.ssd_forward(x, dt, A, B, C, D)
    cb = np.einsum("tn,tn->t", C[:, 0], B[:, 0])
    y_ref = (cb * dt.T).T[:, :, None] * x + D[None, :, None] * x
    assert rel(y, y_ref) < 1e-13
    for h in range(H):
        assert rel(fin[0, h], dt[-1, h] * np.outer(x[-1, h], B[-1, 0])) < 1e-13


def test_skip_only_when_B_is_zero():
    rng = np.random.default_rng(3)
    x, dt, A, B, C, D = rand_problem(rng, 20, 2, 3, 4, 1)
    y, fin = oracle.ssd_forward(x, dt, A, np.zeros_like(B), C, D)
    assert np.array_equal(y, D[None, :, None] * x)
    assert not fin.any()


def test_free_response_closed_form():
    """x = 0 with initial state h0: y_t = exp(sum_{r<=t} dt_r A) (h0 C_t)."""
    rng = np.random.default_rng(4)
    T, H, P, N = 30, 2, 3, 5
    _, dt, A, B, C, D = rand_problem(rng, T, H, P, N, 1)
    h0 = rng.standard_normal((1, H, P, N))
    y, fin = oracle.ssd_forward(np.zeros((T, H, P)), dt, A, B, C, D, h0)
    for h in range(H):
        dec = np.exp(np.cumsum(dt[:, h] * A[h]))
        y_ref = dec[:, None] * (C[:, 0] @ h0[0, h].T)
        assert rel(y[:, h], y_ref) < 1e-12
        assert rel(fin[0, h], dec[-1] * h0[0, h]) < 1e-12


def test_group_mapping_contiguous_heads():
    """Heads h share group h // (H/G): zeroing group 1's B silences heads 2 and 3 only."""
    rng = np.random.default_rng(5)
    T, H, P, N, G = 16, 4, 2, 3, 2
    x, dt, A, B, C, D = rand_problem(rng, T, H, P, N, G)
    B[:, 1] = 0.0
    y, _ = oracle.ssd_forward(x, dt, A, B, C, D)
    for h in (2, 3):
        assert np.array_equal(y[:, h], D[h] * x[:, h])
    for h in (0, 1):
        assert np.abs(y[:, h] - D[h] * x[:, h]).max() > 1e-3


@pytest.mark.parametrize("case", json.load(open(os.path.join(HERE, "golden", "handworked.json")))["cases"],
                         ids=lambda c: c["name"])
def test_handworked_golden(case):
    T, H, P, N, G = case["T"], case["H"], case["P"], case["N"], case["G"]
    x = np.asarray(case["x"], dtype=np.float64).reshape(T, H, P)
    dt = np.asarray(case["dt"]).reshape(T, H)
    B = np.asarray(case["B"]).reshape(T, G, N)
    C = np.asarray(case["C"]).reshape(T, G, N)
    y, fin = oracle.ssd_forward(x, dt, case["A"], B, C, case["D"])
    np.testing.assert_allclose(y.reshape(-1), np.asarray(case["y"]).reshape(-1), rtol=0, atol=1e-12)
    np.testing.assert_allclose(fin.reshape(-1), np.asarray(case["final"]).reshape(-1), rtol=0, atol=1e-12)


# -------------------------------------------------- chunked algorithm (pages)
@pytest.mark.parametrize("Q", [1, 4, 7, 16, 64, 100])
def test_recurrence_equals_chunked_algorithm(Q):
    """The chunked SSD (diag blocks + right/centre/left factors) equals the recurrence
    for every chunk length, including a partial last chunk (Q = 7, 100)."""
    rng = np.random.default_rng(6)
    T, H, P, N, G = 96, 4, 3, 5, 2
    x, dt, A, B, C, D = rand_problem(rng, T, H, P, N, G)
    h0 = rng.standard_normal((1, H, P, N))
    y, fin = oracle.ssd_forward(x, dt, A, B, C, D, h0)
    gmap = np.arange(H) // (H // G)
    Yc, Sc = ssd_chunked(dt[:, :, None] * x, dt * A[None], B[:, gmap], C[:, gmap], Q, h0[0])
    Yc = Yc + D[None, :, None] * x
    assert rel(y, Yc) < 1e-12
    assert rel(fin[0], Sc) < 1e-12


# ------------------------------------------------------- structural invariants
def test_split_and_carry_equals_one_pass():
    rng = np.random.default_rng(7)
    T, H, P, N = 50, 2, 3, 4
    x, dt, A, B, C, D = rand_problem(rng, T, H, P, N, 1)
    y, fin = oracle.ssd_forward(x, dt, A, B, C, D)
    t0 = 19
    y1, f1 = oracle.ssd_forward(x[:t0], dt[:t0], A, B[:t0], C[:t0], D)
    y2, f2 = oracle.ssd_forward(x[t0:], dt[t0:], A, B[t0:], C[t0:], D, f1)
    assert rel(np.concatenate([y1, y2]), y) < 1e-12
    assert rel(f2, fin) < 1e-12


def test_linear_in_input_and_initial_state():
    rng = np.random.default_rng(8)
    T, H, P, N = 33, 2, 4, 3
    x, dt, A, B, C, D = rand_problem(rng, T, H, P, N, 1)
    h0 = rng.standard_normal((1, H, P, N))
    y, f = oracle.ssd_forward(x, dt, A, B, C, D, h0)
    ya, fa = oracle.ssd_forward(x, dt, A, B, C, D, None)
    yb, fb = oracle.ssd_forward(np.zeros_like(x), dt, A, B, C, None, h0)
    assert rel(y, ya + yb) < 1e-12
    assert rel(f, fa + fb) < 1e-12


def test_packed_equals_independent_sequences():
    """Packed variable-length input: state resets at each boundary (zero-length sequence included)."""
    rng = np.random.default_rng(9)
    lens = [5, 0, 17, 1, 30]
    offs = np.cumsum([0] + lens)
    T, H, P, N, G = int(offs[-1]), 4, 3, 4, 2
    x, dt, A, B, C, D = rand_problem(rng, T, H, P, N, G)
    h0 = rng.standard_normal((len(lens), H, P, N))
    y, fin = oracle.ssd_forward(x, dt, A, B, C, D, h0, offs)
    for s, n in enumerate(lens):
        a, b = offs[s], offs[s + 1]
        ys, fs = oracle.ssd_forward(x[a:b], dt[a:b], A, B[a:b], C[a:b], D, h0[s:s + 1])
        assert np.array_equal(y[a:b], ys)
        assert np.array_equal(fin[s], fs[0])
    assert np.array_equal(fin[1], h0[1])  # empty sequence: final = init


def test_single_token_closed_form():
    rng = np.random.default_rng(10)
    x, dt, A, B, C, D = rand_problem(rng, 1, 2, 3, 4, 1)
    h0 = rng.standard_normal((1, 2, 3, 4))
    y, fin = oracle.ssd_forward(x, dt, A, B, C, D, h0)
    for h in range(2):
        S = math.exp(dt[0, h] * A[h]) * h0[0, h] + dt[0, h] * np.outer(x[0, h], B[0, 0])
        assert rel(fin[0, h], S) < 1e-14
        assert rel(y[0, h], S @ C[0, 0] + D[h] * x[0, h]) < 1e-14


# ---------------------------------------------------------------- decode step
def test_decode_steps_equal_dense_matrix():
    """Repeated generation steps (Method step 8, sec. 6.3) reproduce the dense M x + D x."""
    rng = np.random.default_rng(11)
    T, H, P, N, G = 12, 4, 3, 5, 2
    x, dt, A, B, C, D = rand_problem(rng, T, H, P, N, G)
    state = np.zeros((1, H, P, N))
    ys = []
    for t in range(T):
        yt, state = oracle.decode_step(x[t:t + 1], dt[t:t + 1], A, B[t:t + 1], C[t:t + 1], D, state)
        ys.append(yt[0])
    ys = np.stack(ys)
    for h in range(H):
        M = dense_M(dt, A, B, C, h, h // (H // G))
        assert rel(ys[:, h], M @ x[:, h] + D[h] * x[:, h]) < 1e-12


# ------------------------------------------------- step-size prologue (NEXT-1)
def test_dt_prologue_closed_forms():
    """softplus(0) = ln 2; softplus(ln(e - 1)) = 1; softplus(v) -> v for large v and
    -> exp(v) for very negative v; the bias is per head (last axis); the clamp bounds."""
    dt = oracle.dt_prologue(np.array([[0.0, math.log(math.e - 1.0), 40.0, -40.0]]))
    assert dt[0, 0] == pytest.approx(math.log(2.0), rel=1e-15)
    assert dt[0, 1] == pytest.approx(1.0, rel=1e-15)
    assert dt[0, 2] == pytest.approx(40.0, rel=1e-15)
    assert dt[0, 3] == pytest.approx(math.exp(-40.0), rel=1e-12)
    raw = np.zeros((3, 2))
    got = oracle.dt_prologue(raw, dt_bias=np.array([0.0, math.log(math.e ** 2 - 1.0)]))
    assert np.allclose(got[:, 0], math.log(2.0)) and np.allclose(got[:, 1], 2.0)
    assert np.array_equal(oracle.dt_prologue(raw + 0.3, softplus=False), raw + 0.3)
    assert np.all(oracle.dt_prologue(raw, dt_min=0.9) == 0.9)
    assert np.all(oracle.dt_prologue(raw, dt_max=0.25) == 0.25)


def test_dt_prologue_forward_equals_forward_on_inverse_softplus():
    """Raw values built with the inverse softplus ln(e^d - 1) of a chosen dt give the
    forward pass on that dt (and a clamp gives the forward pass on the clamped dt)."""
    rng = np.random.default_rng(31)
    x, dt, A, B, C, D = rand_problem(rng, 40, 3, 5, 6, 1)
    bias = rng.uniform(-0.5, 0.5, 3)
    raw = np.log(np.expm1(dt)) - bias
    y0, f0 = oracle.ssd_forward(x, dt, A, B, C, D)
    y1, f1 = oracle.ssd_forward(x, oracle.dt_prologue(raw, bias), A, B, C, D)
    assert np.allclose(y1, y0, rtol=1e-12, atol=1e-12) and np.allclose(f1, f0, rtol=1e-12, atol=1e-12)
    y2, f2 = oracle.ssd_forward(x, np.full_like(dt, 0.2), A, B, C, D)
    y3, f3 = oracle.ssd_forward(x, oracle.dt_prologue(raw, bias, dt_min=0.2, dt_max=0.2), A, B, C, D)
    assert np.array_equal(y3, y2) and np.array_equal(f3, f2)


# ------------------------------------------ block steps around the SSD (NEXT-3)
def silu_ref(v):
    return v / (1.0 + np.exp(-v))


def test_conv_impulse_response_and_sequence_reset():
    """A unit impulse at token t0 of channel c gives pre-activations w[c, 3 - j] at
    t0 + j (j < 4) and 0 elsewhere; an impulse on a sequence's last token does not
    reach the next sequence."""
    rng = np.random.default_rng(41)
    w = rng.standard_normal((3, 4))
    x = np.zeros((12, 3))
    x[5, 1] = 1.0
    out = oracle.causal_conv1d_silu(x, w)
    expect = np.zeros((12, 3))
    for j in range(4):
        expect[5 + j, 1] = silu_ref(w[1, 3 - j])
    assert np.allclose(out, expect, rtol=1e-15, atol=1e-300)
    x2 = np.zeros((12, 3))
    x2[6, 0] = 1.0  # last token of the first sequence [0, 7)
    bias = np.array([0.25, -0.5, 0.0])
    out2 = oracle.causal_conv1d_silu(x2, w, bias, seq_offsets=[0, 7, 7, 12])
    assert np.allclose(out2[7:], silu_ref(bias)[None, :].repeat(5, 0))
    assert out2[6, 0] == pytest.approx(silu_ref(w[0, 3] + 0.25))


def test_conv_equals_library_convolution():
    rng = np.random.default_rng(42)
    T, ch = 50, 4
    x = rng.standard_normal((T, ch))
    w = rng.standard_normal((ch, 4))
    b = rng.standard_normal(ch)
    out = oracle.causal_conv1d_silu(x, w, b)
    for c in range(ch):
        pre = np.convolve(x[:, c], w[c, ::-1])[:T] + b[c]  # causal: out[t] = sum_k w[k] x[t-3+k]
        assert np.allclose(out[:, c], silu_ref(pre), rtol=1e-13, atol=1e-13)


def test_gated_rmsnorm_closed_forms():
    rng = np.random.default_rng(43)
    y = rng.standard_normal((5, 16))
    w = rng.uniform(0.5, 2.0, 16)
    # z = 0 gates everything off: g = 0, out = 0
    assert np.array_equal(oracle.gated_rmsnorm(y, np.zeros_like(y), w), np.zeros_like(y))
    # a constant gate cancels in the norm: out = y / sqrt(mean(y^2) + eps / s^2) * w, s = silu(z)
    s = silu_ref(3.0)
    got = oracle.gated_rmsnorm(y, np.full_like(y, 3.0), w, eps=1e-5)
    expect = y / np.sqrt(np.mean(y * y, axis=1, keepdims=True) + 1e-5 / s ** 2) * w
    assert np.allclose(got, expect, rtol=1e-13)
    # eps = 0, unit weight: every token's output has RMS 1
    out = oracle.gated_rmsnorm(y, rng.standard_normal(y.shape), np.ones(16), eps=0.0)
    assert np.allclose(np.sqrt(np.mean(out * out, axis=1)), 1.0, rtol=1e-13)


# ------------------------------------------------------- workload generator
def test_sampled_problem_matches_full():
    """The sampled-pairs harness returns exactly the full oracle's rows."""
    import workloads
    wl = workloads.custom(3, 40, H=4, P=4, N=8, G=2, chunk=16, dtype="bf16", init=True)
    prob = workloads.generate(wl, seed=0)
    y, f = oracle.ssd_forward_problem(prob)
    ys, fs = oracle.ssd_forward_problem(prob, pairs=[(0, 1), (2, 3)])
    assert np.array_equal(ys[0:40, 1], y[0:40, 1]) and np.array_equal(ys[80:120, 3], y[80:120, 3])
    assert np.array_equal(fs[2, 3], f[2, 3])
    assert np.isnan(ys[40:80]).all()
