"""Pins for the fp64 CPU oracle (CPU only).

The oracle is checked against things other than itself: closed forms of the
recurrences, special cases that reduce to a textbook operation computed here
with plain numpy / torch (linear attention, a gradient step of the delta-rule
loss), hand-derived worked examples under ``tests/golden/``, the number-format
encoders against torch's casts, and the ReplaySSM invariants (replay equals the
eager state's output, commit-then-continue equals never committing, rollback
equals recomputing the truncated input) by brute force on tiny inputs.
Each case is chosen so that a dropped term, a wrong sign or index, or a
transposed operand in the oracle fails at least one test.
"""
import json
import os

import numpy as np
import pytest

import oracle
from oracle.replay_model import GdnReplay, Mamba2Replay, RingPointers, ERR_OVERFLOW, ERR_ROLLBACK

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RTOL = 1e-12


def rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


def rand_mamba2(rng, T, P, N):
    x = rng.standard_normal((T, P))
    dt = np.log1p(np.exp(rng.standard_normal(T) * 0.5 - 2.0))
    B = rng.standard_normal((T, N)) / np.sqrt(N)
    C = rng.standard_normal((T, N)) / np.sqrt(N)
    A = -np.exp(rng.uniform(0, np.log(16)))
    D = rng.standard_normal()
    return A, D, x, dt, B, C


def rand_gdn(rng, T, dk, dv):
    q = rng.standard_normal((T, dk))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((T, dk))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal(T)))
    alpha = np.exp(-rng.uniform(0.01, 0.5, T))
    return q, k, v, alpha, beta


# ---------------------------------------------------------------- Mamba-2 ---

def test_mamba2_golden_worked_examples():
    with open(os.path.join(GOLDEN, "mamba2_worked.json")) as f:
        g = json.load(f)
    for case in g["cases"]:
        y, h = oracle.mamba2_eager(case["A"], case["D"], case["x"], case["dt"], case["B"],
                                   case["C"])
        assert rel(y, case["y"]) < 1e-14, case["name"]
        assert rel(h, case["h_final"]) < 1e-14, case["name"]


def test_mamba2_scalar_geometric_closed_form():
    # P = N = 1, constant inputs: h_t = b (1 - a^t) / (1 - a), a = exp(dt A), b = dt x B.
    A, D, dt, x, Bv, Cv, T = -0.7, 0.3, 0.25, 1.5, -0.8, 1.1, 40
    y, h = oracle.mamba2_eager(A, D, np.full((T, 1), x), np.full(T, dt), np.full((T, 1), Bv),
                               np.full((T, 1), Cv))
    a, b = np.exp(dt * A), dt * x * Bv
    t = np.arange(1, T + 1)
    h_ref = b * (1 - a ** t) / (1 - a)
    assert rel(y[:, 0], h_ref * Cv + D * x) < 1e-13
    assert rel(h[0, 0], h_ref[-1]) < 1e-13


def test_mamba2_no_decay_is_causal_linear_attention():
    # A = 0, D = 0: y_t = sum_{i<=t} dt_i (B_i . C_t) x_i  -- masked (C B^T) times x.
    rng = np.random.default_rng(1)
    T, P, N = 9, 3, 5
    _, _, x, dt, B, C = rand_mamba2(rng, T, P, N)
    y, _ = oracle.mamba2_eager(0.0, 0.0, x, dt, B, C)
    scores = np.tril(C @ B.T) * dt[None, :]
    assert rel(y, scores @ x) < RTOL


def test_mamba2_skip_only():
    rng = np.random.default_rng(2)
    A, D, x, dt, B, C = rand_mamba2(rng, 6, 4, 3)
    y, h = oracle.mamba2_eager(A, D, x, dt, np.zeros_like(B), C)
    assert rel(y, D * x) < 1e-15 and np.all(h == 0)


def test_mamba2_pure_decay_of_a_state():
    # x = 0: h_t = exp(A sum_{j<=t} dt_j) h_0 and y_t = h_t C_t.
    rng = np.random.default_rng(3)
    T, P, N = 7, 3, 4
    A, D, x, dt, B, C = rand_mamba2(rng, T, P, N)
    h0 = rng.standard_normal((P, N))
    y, h = oracle.mamba2_eager(A, D, np.zeros((T, P)), dt, B, C, h0=h0)
    cum = np.cumsum(dt)
    y_ref = np.stack([np.exp(A * cum[t]) * (h0 @ C[t]) for t in range(T)])
    assert rel(y, y_ref) < RTOL
    assert rel(h, np.exp(A * cum[-1]) * h0) < RTOL


def test_mamba2_state_is_outer_product_sum():
    # Closed form of the whole recurrence: h_T = sum_i exp(A sum_{j>i} dt_j) dt_i x_i B_i^T.
    rng = np.random.default_rng(4)
    T, P, N = 6, 2, 5
    A, D, x, dt, B, C = rand_mamba2(rng, T, P, N)
    _, h = oracle.mamba2_eager(A, D, x, dt, B, C)
    ref = np.zeros((P, N))
    for i in range(T):
        ref += np.exp(A * dt[i + 1:].sum()) * dt[i] * np.outer(x[i], B[i])
    assert rel(h, ref) < RTOL


@pytest.mark.parametrize("L", range(1, 10))
def test_mamba2_replay_equals_eager(L):
    rng = np.random.default_rng(10 + L)
    P, N = 3, 4
    A, D, x, dt, B, C = rand_mamba2(rng, 12 + L, P, N)
    # checkpoint = eager state after a 12-step prefix
    _, S0 = oracle.mamba2_eager(A, D, x[:12], dt[:12], B[:12], C[:12])
    y_eager, _ = oracle.mamba2_eager(A, D, x[12:], dt[12:], B[12:], C[12:], h0=S0)
    y_replay = oracle.mamba2_replay(A, D, S0, x[12:], dt[12:], B[12:], C[12:])
    assert rel(y_replay, y_eager[-1]) < RTOL


def test_mamba2_commit_schedule_invariance_and_rollback():
    rng = np.random.default_rng(20)
    P, N, T = 3, 4, 30
    A, D, x, dt, B, C = rand_mamba2(rng, T, P, N)
    y_ref, _ = oracle.mamba2_eager(A, D, x, dt, B, C)
    for K in (1, 2, 3, 5, 7, 64):
        m = Mamba2Replay(A, D, np.zeros((P, N)))
        for t in range(T):
            m.append(x[t], dt[t], B[t], C[t])
            assert rel(m.output(), y_ref[t]) < RTOL
            if len(m) >= K:
                m.commit()
    # rollback: append junk, roll it back, continue == never having seen it
    m = Mamba2Replay(A, D, np.zeros((P, N)))
    junk = rand_mamba2(np.random.default_rng(21), 3, P, N)
    for t in range(T):
        m.append(x[t], dt[t], B[t], C[t])
        if t % 4 == 1:
            for j in range(3):
                m.append(junk[2][j], junk[3][j], junk[4][j], junk[5][j])
            m.rollback(3)
        assert rel(m.output(), y_ref[t]) < RTOL
        if len(m) >= 5:
            m.commit()


# ---------------------------------------------------------------- GDN -------

def test_gdn_golden_worked_example():
    with open(os.path.join(GOLDEN, "gdn_worked.json")) as f:
        g = json.load(f)
    o, S = oracle.gdn_eager(g["q"], g["k"], g["v"], g["alpha"], g["beta"])
    assert rel(o, g["o"]) < 1e-14
    assert rel(S, g["S_final"]) < 1e-14


def test_gdn_beta_zero_is_pure_decay():
    rng = np.random.default_rng(30)
    T, dk, dv = 6, 5, 3
    q, k, v, alpha, _ = rand_gdn(rng, T, dk, dv)
    S0 = rng.standard_normal((dv, dk))
    o, S = oracle.gdn_eager(q, k, v, alpha, np.zeros(T), S0=S0)
    cum = np.cumprod(alpha)
    assert rel(o, np.stack([cum[t] * S0 @ q[t] for t in range(T)])) < RTOL
    assert rel(S, cum[-1] * S0) < RTOL


def test_gdn_unit_key_beta_one_stores_v_exactly():
    # beta = 1, |k| = 1: S_t k_t = alpha (S k - (S k)(k.k)) + v = v for any alpha, S_{t-1}.
    rng = np.random.default_rng(31)
    dk, dv = 6, 4
    S = rng.standard_normal((dv, dk))
    for t in range(8):
        q, k, v, alpha, _ = rand_gdn(rng, 1, dk, dv)
        _, S = oracle.gdn_eager(k, k, v, alpha, np.ones(1), S0=S)   # query = key
        assert rel(S @ k[0], v[0]) < 1e-13


def test_gdn_orthonormal_keys_reduce_to_linear_attention():
    rng = np.random.default_rng(32)
    dk, dv = 5, 3
    Q, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Q.T                                  # rows orthonormal
    T = dk
    v = rng.standard_normal((T, dv))
    q = rng.standard_normal((T, dk))
    o, S = oracle.gdn_eager(q, k, v, np.ones(T), np.ones(T))
    ref = np.stack([sum(v[i] * (k[i] @ q[t]) for i in range(t + 1)) for t in range(T)])
    assert rel(o, ref) < 1e-12
    assert rel(S, v.T @ k) < 1e-12


def test_gdn_alpha_one_is_a_gradient_step_on_the_delta_loss():
    # With alpha = 1 the update is S <- S - beta * grad_S 0.5 |S k - v|^2.
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(33)
    dk, dv = 4, 3
    S0 = rng.standard_normal((dv, dk))
    q, k, v, _, beta = rand_gdn(rng, 1, dk, dv)
    St = torch.tensor(S0, dtype=torch.float64, requires_grad=True)
    loss = 0.5 * ((St @ torch.tensor(k[0]) - torch.tensor(v[0])) ** 2).sum()
    loss.backward()
    ref = S0 - beta[0] * St.grad.numpy()
    o, S = oracle.gdn_eager(q, k, v, np.ones(1), beta, S0=S0, scale=0.5)
    assert rel(S, ref) < RTOL
    assert rel(o[0], 0.5 * ref @ q[0]) < RTOL


def test_gdn_alpha_does_not_scale_the_write():
    # From S_{t-1} = 0 the new state is beta v k^T whatever alpha is.
    rng = np.random.default_rng(34)
    q, k, v, _, beta = rand_gdn(rng, 1, 5, 4)
    for a in (0.1, 0.7, 1.0):
        _, S = oracle.gdn_eager(q, k, v, np.array([a]), beta)
        assert rel(S, beta[0] * np.outer(v[0], k[0])) < 1e-15


@pytest.mark.parametrize("L", range(1, 10))
def test_gdn_replay_equals_eager(L):
    rng = np.random.default_rng(40 + L)
    dk, dv = 4, 3
    q, k, v, alpha, beta = rand_gdn(rng, 10 + L, dk, dv)
    _, S0 = oracle.gdn_eager(q[:10], k[:10], v[:10], alpha[:10], beta[:10])
    o_eager, _ = oracle.gdn_eager(q[10:], k[10:], v[10:], alpha[10:], beta[10:], S0=S0, scale=0.7)
    o_rep = oracle.gdn_replay(S0, k[10:], v[10:], alpha[10:], beta[10:], q[-1], scale=0.7)
    assert rel(o_rep, o_eager[-1]) < RTOL


def test_gdn_commit_schedule_invariance_and_rollback():
    rng = np.random.default_rng(50)
    dk, dv, T = 4, 3, 30
    q, k, v, alpha, beta = rand_gdn(rng, T, dk, dv)
    o_ref, _ = oracle.gdn_eager(q, k, v, alpha, beta)
    for K in (1, 2, 4, 6, 64):
        m = GdnReplay(np.zeros((dv, dk)))
        for t in range(T):
            m.append(q[t], k[t], v[t], alpha[t], beta[t])
            assert rel(m.output(), o_ref[t]) < RTOL
            if len(m) >= K:
                m.commit()
    m = GdnReplay(np.zeros((dv, dk)))
    junk = rand_gdn(np.random.default_rng(51), 2, dk, dv)
    for t in range(T):
        m.append(q[t], k[t], v[t], alpha[t], beta[t])
        if t % 3 == 0:
            for j in range(2):
                m.append(*(a[j] for a in junk))
            # outputs at the speculative positions equal the eager outputs of that extension
            m.rollback(2)
        assert rel(m.output(), o_ref[t]) < RTOL
        if len(m) >= 4:
            m.commit()


def test_verify_positions_equal_eager_outputs_of_each_prefix():
    rng = np.random.default_rng(52)
    dk, dv = 4, 3
    q, k, v, alpha, beta = rand_gdn(rng, 12, dk, dv)
    o_ref, S_mid = oracle.gdn_eager(q[:7], k[:7], v[:7], alpha[:7], beta[:7])
    o_all, _ = oracle.gdn_eager(q, k, v, alpha, beta)
    m = GdnReplay(S_mid)
    for t in range(7, 12):
        m.append(q[t], k[t], v[t], alpha[t], beta[t])
    for p in range(5):
        assert rel(m.output(upto=p), o_all[7 + p]) < RTOL


# ---------------------------------------------------- batched == single ----

def test_batched_drivers_match_single_pair():
    rng = np.random.default_rng(60)
    n, T, P, N = 5, 7, 3, 4
    cases = [rand_mamba2(rng, T, P, N) for _ in range(n)]
    A = np.array([c[0] for c in cases]); D = np.array([c[1] for c in cases])
    xs, dts, Bs, Cs = (np.stack([c[i] for c in cases]) for i in range(2, 6))
    y, h = oracle.mamba2_eager_batch(A, D, xs, dts, Bs, Cs, nthreads=3)
    for i in range(n):
        yi, hi = oracle.mamba2_eager(A[i], D[i], xs[i], dts[i], Bs[i], Cs[i])
        assert np.array_equal(y[i], yi) and np.array_equal(h[i], hi)
    g = [rand_gdn(rng, T, 4, 3) for _ in range(n)]
    qs, ks, vs, al, be = (np.stack([c[i] for c in g]) for i in range(5))
    o, S = oracle.gdn_eager_batch(qs, ks, vs, al, be, scale=0.5, nthreads=2)
    for i in range(n):
        oi, Si = oracle.gdn_eager(qs[i], ks[i], vs[i], al[i], be[i], scale=0.5)
        assert np.array_equal(o[i], oi) and np.array_equal(S[i], Si)


# --------------------------------------------------------- number formats --

def test_bf16_rne_matches_torch_cast():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(70)
    a = (rng.standard_normal(200000) * np.exp(rng.uniform(-30, 30, 200000))).astype(np.float32)
    ties = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 0.0, -0.0], dtype=np.float32)
    a = np.concatenate([a, ties])
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.bf16_rne(a), ref)
    assert oracle.bf16_rne(np.float32(1 + 2 ** -8)) == 0x3F80          # tie -> even
    assert oracle.bf16_rne(np.float32(1 + 3 * 2 ** -8)) == 0x3F82      # tie -> even (up)


def test_e4m3_hand_derived_codes():
    with open(os.path.join(GOLDEN, "e4m3_codes.json")) as f:
        g = json.load(f)
    vals = np.array([c[0] for c in g["cases"]], np.float32)
    codes = np.array([c[1] for c in g["cases"]], np.uint8)
    assert np.array_equal(oracle.e4m3_rne_satfinite(vals), codes)


def test_e4m3_matches_torch_cast_in_range_and_decodes():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(71)
    a = (rng.standard_normal(200000) * np.exp(rng.uniform(-14, 6, 200000))).astype(np.float32)
    a = a[np.abs(a) <= 448]
    ref = torch.from_numpy(a).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_rne_satfinite(a)
    assert np.array_equal(got, ref)
    all_codes = np.arange(256, dtype=np.uint8)
    dec = oracle.e4m3_decode(all_codes)
    tdec = torch.from_numpy(all_codes).view(torch.float8_e4m3fn).float().numpy()
    finite = ~np.isnan(tdec)
    assert np.array_equal(np.isnan(dec), ~finite)
    assert np.array_equal(dec[finite], tdec[finite])
    # every finite code round-trips
    assert np.array_equal(oracle.e4m3_rne_satfinite(dec[finite]), all_codes[finite])


def test_e4m3_tile_quantisation_bounds():
    rng = np.random.default_rng(72)
    m = (rng.standard_normal((16, 32)) * 3).astype(np.float32)
    codes, scale = oracle.e4m3_quantize_tile(m)
    amax = np.abs(m).max()
    assert scale == np.float32(amax / np.float32(448.0))
    assert codes.reshape(-1)[np.argmax(np.abs(m))] & 0x7F == 0x7E
    back = oracle.e4m3_decode(codes) * scale
    normal = np.abs(m) >= 2.0 ** -6 * scale
    assert np.all(np.abs(back - m)[normal] <= 2.0 ** -4 * np.abs(m)[normal] * (1 + 1e-6))
    assert np.all(np.abs(back - m)[~normal] <= 2.0 ** -10 * scale * (1 + 1e-6))
    z_codes, z_scale = oracle.e4m3_quantize_tile(np.zeros((4, 4), np.float32))
    assert z_scale == 1.0 and np.all(z_codes == 0)


# ---------------------------------------------------------- ring pointers --

def test_ring_pointer_model():
    r = RingPointers(3, cap=8)
    r.append(5)
    assert list(r.tail) == [5, 5, 5] and list(r.length) == [5, 5, 5]
    r.append(4)                       # 9 > 8: refused, sticky error, pointers unchanged
    assert list(r.tail) == [5, 5, 5] and np.all(r.err == ERR_OVERFLOW)
    r.rollback(np.array([0, 2, 6]))   # 6 > len: refused for sequence 2
    assert list(r.tail) == [5, 3, 5] and r.err[2] == ERR_OVERFLOW | ERR_ROLLBACK
    sel = r.commit(min_len=4)
    assert list(sel) == [True, False, True] and list(r.head) == [5, 0, 5]
    r.append(3)
    assert r.slots(0) == [5, 6, 7] and list(r.length) == [3, 6, 3]
    r.append(3)
    assert r.slots(0) == [5, 6, 7, 0, 1, 2]        # wraps modulo cap
