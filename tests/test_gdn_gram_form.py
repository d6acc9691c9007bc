"""The GDN verification prep (bf16 inputs, rings of up to 32 slots) evaluates
the backward sweep of the replay in a Gram form.  With E_j(l) = alpha_l ...
alpha_{e_j} (1 for l > e_j) the sweep's vector before step i is
E_j(i + 1) (q_j - sum_{i<m<=e_j} h_m k_m) with h_m = c_m / E_j(m + 1), so

    h_i = beta_i (k_i . q_j - sum_{i<m<=e_j} h_m (k_i . k_m)),
    coef_j[i] = scale h_i E_j(i + 1),   vec_j = E_j(0) (q_j - sum_m h_m k_m),
    y_j = scale (S0 vec_j) + sum_{i<=e_j} coef_j[i] v_i.

This CPU test restates that form in fp64 and checks the outputs it gives
against the oracle's eager Gated DeltaNet recurrence ("ReplaySSM for hybrid
SSM-Transformer stacks", How ReplaySSM works, step 4: the output from the
checkpoint and the buffered inputs equals the eager one), over random buffer
lengths, output positions and decays, including decays whose products
underflow.  It pins the derivation the kernel relies on; the GPU parity tests
pin the kernel itself."""
import numpy as np

import oracle


def gram_outputs(S0, K, V, Q, alpha, beta, npos, scale):
    L = K.shape[0]
    G = K @ K.T
    P = Q @ K.T   # P[j, i] = k_i . q_j
    ys = []
    for j in range(npos):
        e = L - npos + j
        h = np.zeros(L)
        for i in range(e, -1, -1):
            h[i] = beta[i] * (P[j, i] - sum(h[m] * G[i, m] for m in range(i + 1, e + 1)))
        E = np.ones(L + 1)   # E[l] = alpha_l ... alpha_e
        for l in range(e, -1, -1):
            E[l] = alpha[l] * E[l + 1]
        coef = np.array([scale * h[i] * E[i + 1] if i <= e else 0.0 for i in range(L)])
        vec = E[0] * (Q[j] - h @ K)
        ys.append(scale * (S0 @ vec) + coef @ V)
    return np.array(ys)


def test_gram_form_matches_the_eager_recurrence():
    rng = np.random.default_rng(20)
    worst = 0.0
    for trial in range(60):
        L = int(rng.integers(1, 33))
        npos = int(rng.integers(1, min(8, L) + 1))
        dk, dv = int(rng.choice([8, 16, 32])), int(rng.choice([8, 24]))
        K = rng.standard_normal((L, dk))
        K /= np.linalg.norm(K, axis=1, keepdims=True)
        V = rng.standard_normal((L, dv))
        qs = rng.standard_normal((L, dk)) / np.sqrt(dk)
        alpha = np.exp(-rng.exponential(0.4, L))
        if trial % 5 == 0:
            alpha[rng.integers(0, L)] = 1e-200   # products underflow to 0 in fp64
        beta = rng.uniform(0.0, 1.0, L)
        S0 = rng.standard_normal((dv, dk))
        scale = float(rng.uniform(0.3, 1.5))
        o, _ = oracle.gdn_eager(qs, K, V, alpha, beta, S0=S0, scale=scale)
        Q = qs[L - npos:]   # the queries of the verified positions
        y = gram_outputs(S0, K, V, Q, alpha, beta, npos, scale)
        ref = o[L - npos:]
        err = np.abs(y - ref).max() / max(np.abs(ref).max(), 1e-300)
        worst = max(worst, err)
    assert worst < 1e-10, worst


def test_gram_form_single_entry_closed_form():
    # one entry, one position: c_0 = beta (k . q), vec = alpha (q - c_0 k)
    k = np.array([0.6, 0.8])
    q = np.array([1.0, -2.0])
    v = np.array([3.0])
    alpha, beta, scale = 0.5, 0.25, 2.0
    S0 = np.array([[1.0, 1.0]])
    y = gram_outputs(S0, k[None], v[None], q[None], np.array([alpha]), np.array([beta]), 1, scale)[0]
    c0 = beta * (k @ q)
    expect = scale * (S0 @ (alpha * (q - c0 * k))) + scale * c0 * v
    assert np.allclose(y, expect, rtol=0, atol=1e-15)
