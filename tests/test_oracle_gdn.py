"""Pins for the oracle's gated delta-rule recurrence (CPU only).

What fixes them, independently of the token loop:
  * beta = 0 leaves only the decay: S_t = exp(sum g) S_0 in closed form;
  * with alpha = 1 and beta = 1 a write overwrites along the key: afterwards
    S k = v exactly and S x is unchanged for every x orthogonal to k (the
    pages' description of the delta rule);
  * orthonormal keys and S_0 = 0 reduce the rule to textbook linear attention,
    o_t = sum_{j<=t} beta_j (k_j . q_t) v_j;
  * d_k = d_v = 1 has a scalar closed form (a first-order linear recurrence);
  * an algebraically different evaluation, the chunked form (the keys' Gram
    matrix inverted with a dense linear solve, then matrix products per chunk),
    gives the same outputs and final state;
  * the state norm obeys |S_t|_F <= alpha_t |S_{t-1}|_F + beta_t |v_t|;
  * a perturbation of the state along k_t is erased exactly by a beta = 1
    write along k_t;
  * value heads that share a query/key head equal runs with the q/k repeated.
"""
import numpy as np

from oracle import nvfp4_oracle as o


def _inputs(rng, T, H, hk, dk, dv, g_scale=1.0):
    q = rng.standard_normal((T, hk, dk))
    k = rng.standard_normal((T, hk, dk))
    v = rng.standard_normal((T, H, dv))
    beta = rng.uniform(0.0, 1.0, (T, H))
    g = -g_scale * rng.uniform(0.0, 1.0, (T, H))
    return q, k, v, beta, g


def test_pure_decay_closed_form():
    rng = np.random.default_rng(1)
    T, H, dk, dv = 12, 3, 8, 5
    q, k, v, _, g = _inputs(rng, T, H, H, dk, dv)
    h0 = rng.standard_normal((H, dv, dk))
    out, S = o.gdn_recurrence(q, k, v, np.zeros((T, H)), g, h0=h0)
    qn = o.l2_normalise(q) * dk ** -0.5
    cum = np.cumsum(g, axis=0)
    for t in range(T):
        want = np.exp(cum[t])[:, None] * np.einsum("hvk,hk->hv", h0, qn[t])
        np.testing.assert_allclose(out[t], want, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(S, np.exp(cum[-1])[:, None, None] * h0, rtol=1e-12)


def test_write_overwrites_along_the_key():
    rng = np.random.default_rng(2)
    H, dk, dv = 2, 16, 7
    h0 = rng.standard_normal((H, dv, dk))
    q = rng.standard_normal((1, H, dk))
    k = rng.standard_normal((1, H, dk))
    v = rng.standard_normal((1, H, dv))
    _, S1 = o.gdn_recurrence(q, k, v, np.ones((1, H)), np.zeros((1, H)), h0=h0, eps=0.0)
    kn = k[0] / np.linalg.norm(k[0], axis=1, keepdims=True)
    for h in range(H):
        np.testing.assert_allclose(S1[h] @ kn[h], v[0, h], rtol=1e-12, atol=1e-12)
        x = rng.standard_normal(dk)
        x -= (x @ kn[h]) * kn[h]  # orthogonal to the key
        np.testing.assert_allclose(S1[h] @ x, h0[h] @ x, rtol=1e-12, atol=1e-12)


def test_orthonormal_keys_give_linear_attention():
    rng = np.random.default_rng(3)
    T, H, dk, dv = 9, 2, 16, 4
    perm = rng.permutation(dk)[:T]
    k = np.zeros((T, H, dk))
    for t in range(T):
        k[t, :, perm[t]] = rng.uniform(0.5, 2.0)  # any positive length: normalised to e_perm[t]
    q = rng.standard_normal((T, H, dk))
    v = rng.standard_normal((T, H, dv))
    beta = rng.uniform(0.0, 1.0, (T, H))
    out, _ = o.gdn_recurrence(q, k, v, beta, np.zeros((T, H)), eps=0.0, scale=1.0)
    qn = q / np.linalg.norm(q, axis=2, keepdims=True)
    for t in range(T):
        for h in range(H):
            want = sum(beta[j, h] * qn[t, h, perm[j]] * v[j, h] for j in range(t + 1))
            np.testing.assert_allclose(out[t, h], want, rtol=1e-12, atol=1e-13)


def test_scalar_closed_form():
    rng = np.random.default_rng(4)
    T = 40
    k = rng.choice([-3.0, 2.0], size=(T, 1, 1))  # unit after normalisation: +-1
    q = rng.choice([-1.0, 0.5], size=(T, 1, 1))
    v = rng.standard_normal((T, 1, 1))
    beta = rng.uniform(0.0, 1.0, (T, 1))
    g = -rng.uniform(0.0, 0.5, (T, 1))
    s0 = 0.7
    out, S = o.gdn_recurrence(q, k, v, beta, g, h0=np.full((1, 1, 1), s0), eps=0.0, scale=1.0)
    a = np.exp(g[:, 0])
    kn = np.sign(k[:, 0, 0])
    qn = np.sign(q[:, 0, 0])
    # s_t = a_t (1 - beta_t) s_{t-1} + beta_t v_t kn_t, solved as a sum over writes
    f = a * (1.0 - beta[:, 0])
    for t in range(T):
        s = s0 * np.prod(f[:t + 1])
        for j in range(t + 1):
            s += beta[j, 0] * v[j, 0, 0] * kn[j] * np.prod(f[j + 1:t + 1])
        assert abs(out[t, 0, 0] - s * qn[t]) <= 1e-12 * (1 + abs(s))
    assert abs(S[0, 0, 0] - out[-1, 0, 0] * qn[-1]) <= 1e-12


def _chunked(q, k, v, beta, g, h0, C, scale):
    """The same recurrence evaluated chunk by chunk in matrix form:
    A[t, j] = beta_t exp(gam_t - gam_j) (k_t . k_j) for j < t, L = (I + A)^-1,
    U = L diag(beta) V - L diag(beta e^gam) K S0^T,
    O = diag(e^gam) Q S0^T + mask_{t>=j}(Q K^T e^(gam_t - gam_j)) U,
    S_C = e^gam_C S0 + U^T diag(e^(gam_C - gam)) K."""
    T, H, dv = v.shape
    dk = q.shape[2]
    qn = o.l2_normalise(q) * scale
    kn = o.l2_normalise(k)
    out = np.zeros((T, H, dv))
    S = h0.copy()
    for c0 in range(0, T, C):
        c1 = min(T, c0 + C)
        for h in range(H):
            Q, K, V = qn[c0:c1, h], kn[c0:c1, h], v[c0:c1, h]
            b = beta[c0:c1, h]
            gam = np.cumsum(g[c0:c1, h])
            n = c1 - c0
            D = np.exp(gam[:, None] - gam[None, :])
            A = np.tril(b[:, None] * D * (K @ K.T), -1)
            L = np.linalg.solve(np.eye(n) + A, np.eye(n))
            U = L @ (b[:, None] * V) - L @ ((b * np.exp(gam))[:, None] * K) @ S[h].T
            P = np.tril((Q @ K.T) * D)
            out[c0:c1, h] = np.exp(gam)[:, None] * (Q @ S[h].T) + P @ U
            S[h] = np.exp(gam[-1]) * S[h] + U.T @ (np.exp(gam[-1] - gam)[:, None] * K)
    return out, S


def test_chunked_form_agrees():
    rng = np.random.default_rng(5)
    T, H, dk, dv = 150, 3, 16, 12  # several chunks and a ragged tail
    q, k, v, beta, g = _inputs(rng, T, H, H, dk, dv, g_scale=0.3)
    h0 = 0.5 * rng.standard_normal((H, dv, dk))
    out, S = o.gdn_recurrence(q, k, v, beta, g, h0=h0)
    for C in (16, 64):
        oc, Sc = _chunked(q, k, v, beta, g, h0, C, dk ** -0.5)
        np.testing.assert_allclose(oc, out, rtol=1e-9, atol=1e-11)
        np.testing.assert_allclose(Sc, S, rtol=1e-9, atol=1e-11)


def test_state_norm_bound():
    rng = np.random.default_rng(6)
    T, H, dk, dv = 60, 2, 8, 8
    q, k, v, beta, g = _inputs(rng, T, H, H, dk, dv)
    S = rng.standard_normal((H, dv, dk))
    for t in range(T):
        _, S1 = o.gdn_recurrence(q[t:t + 1], k[t:t + 1], v[t:t + 1], beta[t:t + 1], g[t:t + 1], h0=S)
        for h in range(H):
            bound = np.exp(g[t, h]) * np.linalg.norm(S[h]) + beta[t, h] * np.linalg.norm(v[t, h])
            assert np.linalg.norm(S1[h]) <= bound * (1 + 1e-12)
        S = S1


def test_full_write_erases_a_perturbation_along_the_key():
    rng = np.random.default_rng(7)
    H, dk, dv = 2, 12, 6
    h0 = rng.standard_normal((H, dv, dk))
    q = rng.standard_normal((1, H, dk))
    k = rng.standard_normal((1, H, dk))
    v = rng.standard_normal((1, H, dv))
    kn = k[0] / np.linalg.norm(k[0], axis=1, keepdims=True)
    delta = 0.01 * rng.standard_normal((H, dv))[:, :, None] * kn[:, None, :]
    args = (q, k, v, np.ones((1, H)), np.full((1, H), -0.2))
    _, Sa = o.gdn_recurrence(*args, h0=h0, eps=0.0)
    _, Sb = o.gdn_recurrence(*args, h0=h0 + delta, eps=0.0)
    np.testing.assert_allclose(Sa, Sb, rtol=0, atol=1e-14)
    # a perturbation orthogonal to the key survives, scaled by the decay
    x = rng.standard_normal(dk)
    x -= (x @ kn[0]) * kn[0]
    d2 = np.zeros((H, dv, dk))
    d2[0] = 0.01 * np.outer(rng.standard_normal(dv), x)
    _, Sc = o.gdn_recurrence(*args, h0=h0 + d2, eps=0.0)
    np.testing.assert_allclose(Sc - Sa, np.exp(-0.2) * d2, rtol=1e-10, atol=1e-15)


def test_shared_query_key_heads():
    rng = np.random.default_rng(8)
    T, H, hk, dk, dv = 20, 4, 2, 8, 6
    q, k, v, beta, g = _inputs(rng, T, H, hk, dk, dv)
    out, S = o.gdn_recurrence(q, k, v, beta, g)
    out2, S2 = o.gdn_recurrence(np.repeat(q, 2, axis=1), np.repeat(k, 2, axis=1), v, beta, g)
    np.testing.assert_array_equal(out, out2)
    np.testing.assert_array_equal(S, S2)
    # and head 1 reads q/k head 0, head 2 reads head 1
    o1, _ = o.gdn_recurrence(q[:, 0:1], k[:, 0:1], v[:, 1:2], beta[:, 1:2], g[:, 1:2])
    o2, _ = o.gdn_recurrence(q[:, 1:2], k[:, 1:2], v[:, 2:3], beta[:, 2:3], g[:, 2:3])
    np.testing.assert_array_equal(out[:, 1:2], o1)
    np.testing.assert_array_equal(out[:, 2:3], o2)


def test_row_norms_bound_the_output():
    rng = np.random.default_rng(9)
    T, H, dk, dv = 30, 2, 8, 5
    q, k, v, beta, g = _inputs(rng, T, H, H, dk, dv)
    out, _, rn = o.gdn_recurrence(q, k, v, beta, g, row_norms=True)
    qn = np.linalg.norm(o.l2_normalise(q) * dk ** -0.5, axis=2)  # [T, H]
    assert np.all(np.abs(out) <= rn * qn[:, :, None] * (1 + 1e-12) + 1e-15)


def _max_inverse_norm(q, k, beta, g, H, hk, C=64):
    """Largest spectral norm of L = (I + A)^-1 over every (chunk, head), with
    A[t][j] = beta_t exp(gam_t - gam_j) k_t.k_j (j < t) from unit keys."""
    T = beta.shape[0]
    kn = o.l2_normalise(np.repeat(k.reshape(T, hk, -1), H // hk, axis=1))
    worst = 0.0
    for c0 in range(0, T, C):
        c1 = min(T, c0 + C)
        n = c1 - c0
        for h in range(H):
            K = kn[c0:c1, h]
            gam = np.cumsum(g[c0:c1, h].astype(np.float64))
            A = np.tril(beta[c0:c1, h][:, None] * np.exp(gam[:, None] - gam[None, :]) * (K @ K.T), -1)
            L = np.linalg.inv(np.eye(n) + A)
            worst = max(worst, float(np.linalg.norm(L, 2)))
    return worst


def test_recurrence_tolerance_premise():
    """The GPU tolerance of the chunked recurrence (2^-7 |S_t[i,:]| |q_t|) assumes
    |(I + A)^-1| <= 2 for every chunk; check it on the parity cases' inputs."""
    from bit_quantized_linear_nvfp4_b200 import workloads as wl
    cases = [(150, 4, 2, 150 + 68, False), (321, 2, 2, 321 + 34, False), (64, 3, 3, 64 + 51, False),
             (1, 2, 1, 1 + 34, False), (40, 8, 2, 40 + 136, False), (2000, 2, 2, 5, True), (200, 2, 2, 6, False),
             (225, 2, 2, 7, False), (100, 2, 2, 9, False), (150, 2, 2, 21, False)]
    for T, H, hk, seed, slow in cases:
        q, k, v, beta, g = wl.make_recurrence_inputs(T, H, hk, seed, "bf16", slow)
        assert _max_inverse_norm(q, k, beta, g, H, hk) <= 2.0, (T, H, seed)
    # the full-length case: 32768 tokens x 32 heads
    q, k, v, beta, g = wl.make_recurrence_inputs(32768, 32, 32, 11, "bf16")
    assert _max_inverse_norm(q, k, beta, g, 32, 32) <= 2.0
