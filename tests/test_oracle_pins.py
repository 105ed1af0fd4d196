"""Pins for the fp64 oracle: facts the paper and the mathematics fix, independent of the
oracle's own code.  Each test names the passage of "Kaczmarz Linear Attention" it follows.
Shapes use d_k != d_v wherever possible so that a transposed operand cannot pass.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def _rand_inputs(rng, B, T, H, Dk, Dv, key_lo=0.3, key_hi=3.0, g_lo=-0.5, g_hi=0.0, s0=0.1):
    q = rng.standard_normal((B, T, H, Dk))
    z = rng.standard_normal((B, T, H, Dk))
    s = np.exp(rng.uniform(np.log(key_lo), np.log(key_hi), (B, T, H, 1)))
    k = s * z
    v = rng.standard_normal((B, T, H, Dv))
    eta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    g = rng.uniform(g_lo, g_hi, (B, T, H))
    S0 = s0 * rng.standard_normal((B, H, Dk, Dv))
    return q, k, v, eta, g, S0


def _steps(oracle_mod, q, k, v, eta, g, eps, S0):
    """Run the oracle one token at a time (decode entry point); return the states S_1..S_T."""
    B, T, H, Dk = k.shape
    S = S0.copy()
    states, outs = [], []
    for t in range(T):
        o, S = oracle_mod.decode_step(q[:, t], k[:, t], v[:, t], eta[:, t], g[:, t], eps, S)
        states.append(S.copy())
        outs.append(o)
    return states, outs


# ---------------------------------------------------------------------------------------
# Golden hand-worked example (Eq. 3, Algorithm 1 left panel)
# ---------------------------------------------------------------------------------------
def test_golden_hand_example(oracle_mod):
    rows = [list(map(float, ln.split())) for ln in open(os.path.join(HERE, "golden", "kla_hand_example.txt"))
            if ln.strip() and not ln.startswith("#")]
    S = np.zeros((1, 1, 2, 2))
    for r in rows:
        _, alpha, eta, eps, k0, k1, v0, v1, q0, q1, o0, o1, s00, s01, s10, s11 = r
        o, S = oracle_mod.decode_step(np.array([[[q0, q1]]]), np.array([[[k0, k1]]]), np.array([[[v0, v1]]]),
                                      np.array([[eta]]), np.array([[math.log(alpha)]]), eps, S)
        np.testing.assert_allclose(o[0, 0], [o0, o1], rtol=0, atol=1e-14)
        np.testing.assert_allclose(S[0, 0], [[s00, s01], [s10, s11]], rtol=0, atol=1e-14)


# ---------------------------------------------------------------------------------------
# Theorem 1 / Eq. (11): eta = 1, eps = 0 is an exact projection, S_t^T k_t = v_t, any alpha
# ---------------------------------------------------------------------------------------
def test_hard_projection_every_step(oracle_mod):
    rng = np.random.default_rng(1)
    q, k, v, _, g, S0 = _rand_inputs(rng, 2, 12, 3, 5, 4, key_lo=0.1, key_hi=10.0, g_lo=-2.0)
    eta = np.ones(g.shape)
    states, _ = _steps(oracle_mod, q, k, v, eta, g, 0.0, S0)
    for t, S in enumerate(states):
        readout = np.einsum("bhij,bhi->bhj", S, k[:, t])
        np.testing.assert_allclose(readout, v[:, t], rtol=0, atol=1e-12 * (1 + np.abs(v[:, t]).max()))


# ---------------------------------------------------------------------------------------
# Proposition 2 / Eq. (5): residual contraction, i.e. the relaxed interpolation
#   S_t^T k = (1 - c) Sbar^T k + c v,  c = eta n / (n + eps)
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("eps", [0.0, 1e-6, 0.5])
def test_relaxed_interpolation(oracle_mod, eps):
    rng = np.random.default_rng(2)
    q, k, v, eta, g, S0 = _rand_inputs(rng, 1, 10, 2, 6, 3, key_lo=0.05, key_hi=5.0)
    states, _ = _steps(oracle_mod, q, k, v, eta, g, eps, S0)
    prev = S0
    for t, S in enumerate(states):
        kt = k[:, t]
        n = (kt * kt).sum(-1)
        c = eta[:, t] * n / (n + eps)
        sbar_k = np.exp(g[:, t])[..., None] * np.einsum("bhij,bhi->bhj", prev, kt)
        want = (1 - c)[..., None] * sbar_k + c[..., None] * v[:, t]
        got = np.einsum("bhij,bhi->bhj", S, kt)
        np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-12)
        prev = S


# ---------------------------------------------------------------------------------------
# Eq. (4): along S(tau) = Sbar + tau k e^T the loss is (1 - tau n)^2 |e|^2 / 2; the step the
# oracle takes (tau = eta/(n+eps)) leaves loss (1 - eta n/(n+eps))^2 |e|^2 / 2, and with
# eta = 1, eps = 0 it is the line-search minimiser tau* = 1/n found by a dense scan.
# ---------------------------------------------------------------------------------------
def test_line_search(oracle_mod):
    rng = np.random.default_rng(3)
    Dk, Dv = 4, 3
    S = rng.standard_normal((1, 1, Dk, Dv))
    k = rng.standard_normal((1, 1, Dk)) * 1.7
    v = rng.standard_normal((1, 1, Dv))
    q = rng.standard_normal((1, 1, Dk))
    g = np.array([[-0.3]])
    sbar = np.exp(g[0, 0]) * S[0, 0]
    e = v[0, 0] - sbar.T @ k[0, 0]
    n = float(k[0, 0] @ k[0, 0])
    taus = np.linspace(0.0, 2.0 / n, 20001)
    losses = [0.5 * np.sum((v[0, 0] - (sbar + t * np.outer(k[0, 0], e)).T @ k[0, 0]) ** 2) for t in taus]
    tau_best = taus[int(np.argmin(losses))]
    assert abs(tau_best - 1.0 / n) <= (taus[1] - taus[0])
    _, S1 = oracle_mod.decode_step(q, k, v, np.array([[1.0]]), g, 0.0, S)
    np.testing.assert_allclose(S1[0, 0], sbar + np.outer(k[0, 0], e) / n, rtol=1e-12, atol=1e-13)
    for eta, eps in [(0.3, 0.0), (0.8, 0.2)]:
        _, S1 = oracle_mod.decode_step(q, k, v, np.array([[eta]]), g, eps, S)
        loss = 0.5 * np.sum((v[0, 0] - S1[0, 0].T @ k[0, 0]) ** 2)
        want = 0.5 * (1 - eta * n / (n + eps)) ** 2 * np.sum(e * e)
        assert abs(loss - want) <= 1e-12 * max(1.0, want)


# ---------------------------------------------------------------------------------------
# Proposition 1 (Eq. 15): the relaxed update is the exact minimiser of
#   1/2 |S - Sbar|_F^2 + mu/2 |S^T k - v|^2,  mu = eta / ((1 - eta) n + eps).
# The minimiser is computed here by numpy's least-squares solver on vec(S).
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("eta,eps", [(0.4, 0.0), (0.9, 1e-3), (0.25, 2.0)])
def test_proximal_form(oracle_mod, eta, eps):
    rng = np.random.default_rng(4)
    Dk, Dv = 5, 3
    S = rng.standard_normal((1, 1, Dk, Dv))
    k = rng.standard_normal((1, 1, Dk))
    v = rng.standard_normal((1, 1, Dv))
    q = rng.standard_normal((1, 1, Dk))
    g = np.array([[-0.7]])
    sbar = np.exp(-0.7) * S[0, 0]
    n = float(k[0, 0] @ k[0, 0])
    mu = eta / ((1 - eta) * n + eps)
    # unknown x = vec(S) in row-major order (index i*Dv + j); rows: identity block, then
    # sqrt(mu) * (S^T k)_j = sqrt(mu) * sum_i k_i S_ij
    top = np.eye(Dk * Dv)
    bot = np.zeros((Dv, Dk * Dv))
    for j in range(Dv):
        for i in range(Dk):
            bot[j, i * Dv + j] = k[0, 0, i]
    Amat = np.vstack([top, np.sqrt(mu) * bot])
    rhs = np.concatenate([sbar.reshape(-1), np.sqrt(mu) * v[0, 0]])
    x, *_ = np.linalg.lstsq(Amat, rhs, rcond=None)
    _, S1 = oracle_mod.decode_step(q, k, v, np.array([[eta]]), g, eps, S)
    np.testing.assert_allclose(S1[0, 0], x.reshape(Dk, Dv), rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------------------------------
# Classical Kaczmarz (reference [15] of the paper; section 3.1): with alpha = 1, eta = 1,
# eps = 0 and keys cycling through the rows of a consistent system A X = Y, the state
# from S0 = 0 converges to the minimum-norm solution pinv(A) Y (numpy lstsq); with
# orthonormal rows one sweep is exact.
# ---------------------------------------------------------------------------------------
def test_classical_kaczmarz_min_norm(oracle_mod):
    rng = np.random.default_rng(5)
    m, Dk, Dv = 4, 7, 3
    A = rng.standard_normal((m, Dk))
    X = rng.standard_normal((Dk, Dv))
    Y = A @ X
    sweeps = 300
    T = m * sweeps
    k = np.tile(A, (sweeps, 1))[None, :, None, :]
    v = np.tile(Y, (sweeps, 1))[None, :, None, :]
    q = np.zeros((1, T, 1, Dk))
    eta = np.ones((1, T, 1))
    g = np.zeros((1, T, 1))
    _, ST = oracle_mod.forward(q, k, v, eta, g, 0.0, None)
    Xmin, *_ = np.linalg.lstsq(A, Y, rcond=None)
    np.testing.assert_allclose(ST[0, 0], Xmin, rtol=0, atol=1e-9)


def test_classical_kaczmarz_orthonormal_one_sweep(oracle_mod):
    rng = np.random.default_rng(6)
    m, Dk, Dv = 3, 6, 4
    Qm, _ = np.linalg.qr(rng.standard_normal((Dk, m)))
    A = Qm.T  # orthonormal rows
    Y = rng.standard_normal((m, Dv))
    k = A[None, :, None, :]
    v = Y[None, :, None, :]
    _, ST = oracle_mod.forward(np.zeros_like(k), k, v, np.ones((1, m, 1)), np.zeros((1, m, 1)), 0.0, None)
    np.testing.assert_allclose(ST[0, 0], A.T @ Y, rtol=0, atol=1e-13)


# ---------------------------------------------------------------------------------------
# eta = 0 (no write): S_t = gamma_t S0 and o_t = gamma_t S0^T q_t  (gamma_t = prod alpha)
# ---------------------------------------------------------------------------------------
def test_eta_zero_pure_decay(oracle_mod):
    rng = np.random.default_rng(7)
    q, k, v, _, g, S0 = _rand_inputs(rng, 2, 9, 2, 4, 5)
    eta = np.zeros(g.shape)
    o, ST = oracle_mod.forward(q, k, v, eta, g, 1e-6, S0)
    gam = np.exp(np.cumsum(g, axis=1))  # [B,T,H]
    want_o = gam[..., None] * np.einsum("bhij,bthi->bthj", S0, q)
    np.testing.assert_allclose(o, want_o, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(ST, gam[:, -1][..., None, None] * S0, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------------------------------
# Table 6 (KLA row) / Appendix B: the recurrent form as an explicit sum of products,
#   o_t = q_t^T P_t S0 + sum_{j<=t} (q_t^T M_t M_{t-1} .. M_{j+1} k_j) beta_j v_j,
#   M_s = alpha_s (I - beta_s k_s k_s^T),  P_t = M_t .. M_1,  S_T = P_T S0 + sum_j (..) k_j v_j^T
# With alpha = 1 this is the DeltaNet row.
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("decay", [True, False])
def test_table6_product_form(oracle_mod, decay):
    rng = np.random.default_rng(8)
    B, T, H, Dk, Dv = 1, 8, 2, 4, 3
    q, k, v, eta, g, S0 = _rand_inputs(rng, B, T, H, Dk, Dv)
    if not decay:
        g = np.zeros_like(g)
    eps = 0.05
    o, ST = oracle_mod.forward(q, k, v, eta, g, eps, S0)
    for h in range(H):
        ks, vs, qs = k[0, :, h], v[0, :, h], q[0, :, h]
        betas = [eta[0, s, h] / (ks[s] @ ks[s] + eps) for s in range(T)]
        Ms = [np.exp(g[0, s, h]) * (np.eye(Dk) - betas[s] * np.outer(ks[s], ks[s])) for s in range(T)]

        def prod(lo, hi):  # M_hi M_{hi-1} .. M_lo  (identity when lo > hi)
            P = np.eye(Dk)
            for s in range(lo, hi + 1):
                P = Ms[s] @ P
            return P

        for t in range(T):
            want = qs[t] @ prod(0, t) @ S0[0, h]
            for j in range(t + 1):
                want = want + (qs[t] @ prod(j + 1, t) @ ks[j]) * betas[j] * vs[j]
            np.testing.assert_allclose(o[0, t, h], want, rtol=1e-11, atol=1e-12)
        S_want = prod(0, T - 1) @ S0[0, h]
        for j in range(T):
            S_want = S_want + np.outer(prod(j + 1, T - 1) @ ks[j], betas[j] * vs[j])
        np.testing.assert_allclose(ST[0, h], S_want, rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------------------------------
# Section 4 / Propositions 3-4: the chunkwise form equals the token recurrence for any
# chunk length, including a ragged last chunk.
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("C", [1, 2, 3, 8, 64])
def test_chunk_form_matches_token_form(oracle_mod, C):
    rng = np.random.default_rng(9)
    q, k, v, eta, g, S0 = _rand_inputs(rng, 2, 70, 2, 6, 5)
    o, ST = oracle_mod.forward(q, k, v, eta, g, 1e-6, S0)
    oc, STc = oracle_mod.chunk_forward(q, k, v, eta, g, 1e-6, S0, chunk=C)
    scale_o = np.sqrt(np.mean(o * o))
    assert np.abs(oc - o).max() <= 1e-12 * max(scale_o, 1.0) * 10
    assert np.abs(STc - ST).max() <= 1e-12 * max(np.abs(ST).max(), 1.0) * 10


# ---------------------------------------------------------------------------------------
# Exact rational brute force (Appendix B product form, Fractions) on a tiny case: the fp64
# oracle must agree to ~1e-14.  alpha is rational, passed to the oracle as g = log(alpha).
# ---------------------------------------------------------------------------------------
def test_exact_rational_bruteforce(oracle_mod):
    F = Fraction
    Dk, Dv, T = 2, 3, 4
    ks = [[F(1), F(2)], [F(-3, 2), F(1, 2)], [F(2), F(0)], [F(1, 3), F(-1)]]
    vs = [[F(1), F(0), F(-2)], [F(3, 4), F(1), F(1)], [F(0), F(-1), F(5, 2)], [F(2), F(1, 3), F(0)]]
    qs = [[F(1), F(-1)], [F(2), F(1, 2)], [F(0), F(1)], [F(-1), F(3)]]
    etas = [F(1), F(1, 2), F(3, 4), F(1, 5)]
    alphas = [F(1), F(1, 2), F(4, 5), F(9, 10)]
    # R_t = alpha_t R_{t-1} (I - beta k k^T) + beta v k^T  (Eq. 6), exactly
    R = [[F(0)] * Dk for _ in range(Dv)]
    outs = []
    for t in range(T):
        k, v, q = ks[t], vs[t], qs[t]
        beta = etas[t] / sum(x * x for x in k)
        Rk = [sum(R[a][i] * k[i] for i in range(Dk)) for a in range(Dv)]
        R = [[alphas[t] * (R[a][i] - beta * Rk[a] * k[i]) + beta * v[a] * k[i] for i in range(Dk)]
             for a in range(Dv)]
        outs.append([sum(R[a][i] * q[i] for i in range(Dk)) for a in range(Dv)])
    f = lambda rows: np.array([[float(x) for x in r] for r in rows])
    o, ST = oracle_mod.forward(f(qs)[None, :, None], f(ks)[None, :, None], f(vs)[None, :, None],
                               np.array([[float(e)] for e in etas])[None, :, :, ].reshape(1, T, 1),
                               np.log(np.array([float(a) for a in alphas])).reshape(1, T, 1), 0.0, None)
    np.testing.assert_allclose(o[0, :, 0], f(outs), rtol=0, atol=1e-14 * 10)
    np.testing.assert_allclose(ST[0, 0], f(R).T, rtol=0, atol=1e-14 * 10)


# ---------------------------------------------------------------------------------------
# KLA as GDN on unit keys (coefficient substitution, Appendix B.4):
#   KLA(k, v, eta) == GDN(k/|k|, v/|k|, beta = eta n/(n+eps))
# ---------------------------------------------------------------------------------------
def test_kla_equals_gdn_on_unit_keys(oracle_mod):
    rng = np.random.default_rng(10)
    q, k, v, eta, g, S0 = _rand_inputs(rng, 1, 15, 2, 5, 4, key_lo=0.1, key_hi=10.0)
    eps = 1e-3
    o, ST = oracle_mod.forward(q, k, v, eta, g, eps, S0)
    for h in range(2):
        S = S0[0, h].copy()
        for t in range(15):
            kt, vt = k[0, t, h], v[0, t, h]
            n = kt @ kt
            kh = kt / np.sqrt(n)
            bh = eta[0, t, h] * n / (n + eps)
            Sb = np.exp(g[0, t, h]) * S
            S = Sb + bh * np.outer(kh, vt / np.sqrt(n) - Sb.T @ kh)  # GDN write, beta = bh
            np.testing.assert_allclose(o[0, t, h], S.T @ q[0, t, h], rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(ST[0, h], S, rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------------------------------
# Symmetries: o is linear in q; (o, S_T) jointly linear in (V, S0); at eps = 0,
# S(c k; S0) = S(k; c S0) / c.
# ---------------------------------------------------------------------------------------
def test_symmetries(oracle_mod):
    rng = np.random.default_rng(11)
    q, k, v, eta, g, S0 = _rand_inputs(rng, 1, 13, 2, 4, 6)
    q2 = rng.standard_normal(q.shape)
    o1, _ = oracle_mod.forward(q, k, v, eta, g, 0.01, S0)
    o2, _ = oracle_mod.forward(q2, k, v, eta, g, 0.01, S0)
    o3, _ = oracle_mod.forward(2 * q - 3 * q2, k, v, eta, g, 0.01, S0)
    np.testing.assert_allclose(o3, 2 * o1 - 3 * o2, rtol=1e-10, atol=1e-11)
    v2 = rng.standard_normal(v.shape)
    S02 = rng.standard_normal(S0.shape)
    oa, Sa = oracle_mod.forward(q, k, v, eta, g, 0.01, S0)
    ob, Sb = oracle_mod.forward(q, k, v2, eta, g, 0.01, S02)
    oc, Sc = oracle_mod.forward(q, k, 0.5 * v - v2, eta, g, 0.01, 0.5 * S0 - S02)
    np.testing.assert_allclose(oc, 0.5 * oa - ob, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(Sc, 0.5 * Sa - Sb, rtol=1e-10, atol=1e-11)
    c = 3.7
    _, Sk = oracle_mod.forward(q, c * k, v, eta, g, 0.0, S0)
    _, Sref = oracle_mod.forward(q, k, v, eta, g, 0.0, c * S0)
    np.testing.assert_allclose(Sk, Sref / c, rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------------------------------
# Tie-break for a zero denominator (paper silent): k = 0 and eps = 0 skip the write,
# so the state only decays.
# ---------------------------------------------------------------------------------------
def test_zero_key_zero_eps_skips_write(oracle_mod):
    rng = np.random.default_rng(12)
    S = rng.standard_normal((1, 1, 3, 2))
    o, S1 = oracle_mod.decode_step(np.ones((1, 1, 3)), np.zeros((1, 1, 3)), np.ones((1, 1, 2)),
                                   np.array([[0.7]]), np.array([[-0.2]]), 0.0, S)
    np.testing.assert_allclose(S1, np.exp(-0.2) * S, rtol=1e-15)
    assert np.all(np.isfinite(o))


def test_decode_step_equals_forward_T1(oracle_mod):
    rng = np.random.default_rng(13)
    q, k, v, eta, g, S0 = _rand_inputs(rng, 2, 1, 3, 4, 5)
    o, ST = oracle_mod.forward(q, k, v, eta, g, 1e-6, S0)
    o2, S2 = oracle_mod.decode_step(q[:, 0], k[:, 0], v[:, 0], eta[:, 0], g[:, 0], 1e-6, S0)
    np.testing.assert_array_equal(o[:, 0], o2)
    np.testing.assert_array_equal(ST, S2)


def test_empty_sequence_returns_initial_state(oracle_mod):
    rng = np.random.default_rng(14)
    S0 = rng.standard_normal((2, 3, 4, 5))
    z = np.zeros((2, 0, 3, 4))
    o, ST = oracle_mod.forward(z, z, np.zeros((2, 0, 3, 5)), np.zeros((2, 0, 3)), np.zeros((2, 0, 3)), 1e-6, S0)
    assert o.shape == (2, 0, 3, 5)
    np.testing.assert_array_equal(ST, S0)


# ---------------------------------------------------------------------------------------
# Backward (paper silent; hand-derived): central finite differences of
#   L = <o, dO> + <S_T, dS_T>  w.r.t. every input, fp64.
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("T,ckpt,eps", [(7, 3, 1e-2), (12, 64, 0.3), (5, 1, 1e-6)])
def test_backward_finite_differences(oracle_mod, T, ckpt, eps):
    rng = np.random.default_rng(100 + T)
    B, H, Dk, Dv = 1, 2, 3, 4
    q, k, v, eta, g, S0 = _rand_inputs(rng, B, T, H, Dk, Dv, key_lo=0.5, key_hi=2.0, s0=0.5)
    dO = rng.standard_normal((B, T, H, Dv))
    dST = rng.standard_normal((B, H, Dk, Dv))
    grads = oracle_mod.backward(q, k, v, eta, g, eps, S0, dO, dST, ckpt=ckpt)
    args = dict(q=q, k=k, v=v, eta=eta, g=g, S0=S0)

    def loss(a):
        o, ST = oracle_mod.forward(a["q"], a["k"], a["v"], a["eta"], a["g"], eps, a["S0"])
        return float(np.sum(o * dO) + np.sum(ST * dST))

    hstep = 1e-6
    for name in args:
        x = args[name]
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            a_p = {kk: vv.copy() for kk, vv in args.items()}
            a_m = {kk: vv.copy() for kk, vv in args.items()}
            a_p[name][idx] += hstep
            a_m[name][idx] -= hstep
            fd[idx] = (loss(a_p) - loss(a_m)) / (2 * hstep)
        got = grads["d" + name]
        err = np.abs(got - fd).max() / max(np.abs(fd).max(), 1e-3)
        assert err <= 1e-6, (name, err)


@pytest.mark.parametrize("beta,eps", [("kaczmarz", 0.3), ("kaczmarz", 1e-2), ("direct", 0.0)])
def test_backward_zero_norm_key_finite_differences(oracle_mod, beta, eps):
    """At a key of exactly zero norm the write vanishes, but dk there is not zero:
    dk_t = beta_t Gbar_t v_t (the only first-order term of beta k e^T).  Central differences
    around k_t = 0 in every direction."""
    rng = np.random.default_rng(420 + int(eps * 100))
    B, T, H, Dk, Dv = 1, 6, 1, 3, 4
    q, k, v, eta, g, S0 = _rand_inputs(rng, B, T, H, Dk, Dv, key_lo=0.5, key_hi=1.5, s0=0.5)
    if beta == "direct":
        eta = 0.3 * eta
    zt = (1, 4)
    for t in zt:
        k[0, t, 0] = 0.0
    dO = rng.standard_normal((B, T, H, Dv))
    dST = rng.standard_normal((B, H, Dk, Dv))
    grads = oracle_mod.backward(q, k, v, eta, g, eps, S0, dO, dST, beta=beta)

    def loss(kk):
        o, ST = oracle_mod.forward(q, kk, v, eta, g, eps, S0, beta=beta)
        return float(np.sum(o * dO) + np.sum(ST * dST))

    hstep = 1e-6
    for t in zt:
        fd = np.zeros(Dk)
        for c in range(Dk):
            kp, km = k.copy(), k.copy()
            kp[0, t, 0, c] += hstep
            km[0, t, 0, c] -= hstep
            fd[c] = (loss(kp) - loss(km)) / (2 * hstep)
        got = grads["dk"][0, t, 0]
        assert np.abs(fd).max() > 1e-3  # the gradient there is genuinely nonzero
        assert np.abs(got - fd).max() <= 1e-6 * np.abs(fd).max(), (t, got, fd)


def test_backward_without_dST_and_zero_S0(oracle_mod):
    rng = np.random.default_rng(200)
    q, k, v, eta, g, _ = _rand_inputs(rng, 1, 6, 1, 3, 2)
    dO = rng.standard_normal((1, 6, 1, 2))
    g1 = oracle_mod.backward(q, k, v, eta, g, 1e-3, None, dO, None)
    g2 = oracle_mod.backward(q, k, v, eta, g, 1e-3, np.zeros((1, 1, 3, 2)), dO, np.zeros((1, 1, 3, 2)))
    for key in g1:
        np.testing.assert_array_equal(g1[key], g2[key])
    # o is linear in q, so <dq, q> = <o, dO> exactly
    o, _ = oracle_mod.forward(q, k, v, eta, g, 1e-3, None)
    assert abs(np.sum(g1["dq"] * q) - np.sum(o * dO)) <= 1e-12 * max(1.0, abs(np.sum(o * dO)))


# ---------------------------------------------------------------------------------------
# Direct write strength (beta_t = eta_t as given: the Gated DeltaNet update KLA starts
# from, section 3.3).  Pinned against the Kaczmarz mode, which the pins above fix:
#   direct(eta' = eta / (||k||^2 + eps)) == Kaczmarz(eta), token by token.
# ---------------------------------------------------------------------------------------
def test_direct_mode_with_kaczmarz_eta_equals_kaczmarz_mode(oracle_mod):
    rng = np.random.default_rng(300)
    q, k, v, eta, g, S0 = _rand_inputs(rng, 2, 11, 3, 5, 4, key_lo=0.1, key_hi=10.0)
    for eps in (0.0, 1e-3, 0.7):
        n = np.sum(k * k, axis=-1)
        o1, S1 = oracle_mod.forward(q, k, v, eta, g, eps, S0)
        o2, S2 = oracle_mod.forward(q, k, v, eta / (n + eps), g, 123.0, S0, beta="direct")  # eps unused
        np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(S2, S1, rtol=1e-12, atol=1e-12)
        c1, cS1 = oracle_mod.chunk_forward(q, k, v, eta / (n + eps), g, 5.0, S0, chunk=4, beta="direct")
        np.testing.assert_allclose(c1, o1, rtol=1e-10, atol=1e-11)
        np.testing.assert_allclose(cS1, S1, rtol=1e-10, atol=1e-11)


# Gated DeltaNet as a projection: with beta_t = 1 / ||k_t||^2 the write is the exact
# projection S_t^T k_t = v_t (Theorem 1 read for GDN), for any decay.
def test_direct_mode_inverse_norm_beta_projects(oracle_mod):
    rng = np.random.default_rng(301)
    q, k, v, _, g, S0 = _rand_inputs(rng, 2, 10, 2, 6, 3, key_lo=0.2, key_hi=5.0, g_lo=-1.5)
    beta = 1.0 / np.sum(k * k, axis=-1)
    S = S0.copy()
    for t in range(k.shape[1]):
        _, S = oracle_mod.decode_step(q[:, t], k[:, t], v[:, t], beta[:, t], g[:, t], 0.0, S, beta="direct")
        readout = np.einsum("bhij,bhi->bhj", S, k[:, t])
        np.testing.assert_allclose(readout, v[:, t], rtol=0, atol=1e-12 * (1 + np.abs(v[:, t]).max()))


def test_direct_decode_step_equals_forward_T1(oracle_mod):
    rng = np.random.default_rng(302)
    q, k, v, eta, g, S0 = _rand_inputs(rng, 2, 1, 3, 4, 5)
    o, ST = oracle_mod.forward(q, k, v, eta, g, 1e-6, S0, beta="direct")
    o2, S2 = oracle_mod.decode_step(q[:, 0], k[:, 0], v[:, 0], eta[:, 0], g[:, 0], 1e-6, S0, beta="direct")
    np.testing.assert_array_equal(o[:, 0], o2)
    np.testing.assert_array_equal(ST, S2)


@pytest.mark.parametrize("T,ckpt", [(7, 3), (5, 64)])
def test_direct_backward_finite_differences(oracle_mod, T, ckpt):
    rng = np.random.default_rng(310 + T)
    B, H, Dk, Dv = 1, 2, 3, 4
    q, k, v, eta, g, S0 = _rand_inputs(rng, B, T, H, Dk, Dv, key_lo=0.5, key_hi=1.5, s0=0.5)
    eta = 0.3 * eta  # beta = eta as given: keep the writes contractive for these key norms
    dO = rng.standard_normal((B, T, H, Dv))
    dST = rng.standard_normal((B, H, Dk, Dv))
    grads = oracle_mod.backward(q, k, v, eta, g, 0.0, S0, dO, dST, ckpt=ckpt, beta="direct")
    args = dict(q=q, k=k, v=v, eta=eta, g=g, S0=S0)

    def loss(a):
        o, ST = oracle_mod.forward(a["q"], a["k"], a["v"], a["eta"], a["g"], 0.0, a["S0"], beta="direct")
        return float(np.sum(o * dO) + np.sum(ST * dST))

    hstep = 1e-6
    for name in args:
        x = args[name]
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            a_p = {kk: vv.copy() for kk, vv in args.items()}
            a_m = {kk: vv.copy() for kk, vv in args.items()}
            a_p[name][idx] += hstep
            a_m[name][idx] -= hstep
            fd[idx] = (loss(a_p) - loss(a_m)) / (2 * hstep)
        got = grads["d" + name]
        err = np.abs(got - fd).max() / max(np.abs(fd).max(), 1e-3)
        assert err <= 1e-6, (name, err)


# ---------------------------------------------------------------------------------------
# Diagonal gating (Appendix A.5 and B.5): the decay Diag(exp(g_t)) per key channel.  The
# oracle's diagonal-gated functions are pinned by: equality with the scalar-gated oracle when
# every channel decays alike (forward, chunk form, backward with dg summed over channels),
# Theorem 1's projection and Proposition 2's interpolation for any per-channel decay (A.5:
# the derivation never uses how the decayed state was produced), the chunk form of B.5, and
# finite differences.
# ---------------------------------------------------------------------------------------
def _diag_g(rng, shape_btH, Dk, lo=-1.0):
    return rng.uniform(lo, 0.0, shape_btH + (Dk,))


@pytest.mark.parametrize("beta", ["kaczmarz", "direct"])
def test_diag_uniform_channels_equal_scalar_gating(oracle_mod, beta):
    rng = np.random.default_rng(400)
    q, k, v, eta, g, S0 = _rand_inputs(rng, 2, 9, 2, 5, 3, key_lo=0.4, key_hi=2.0, s0=0.5)
    if beta == "direct":
        eta = 0.3 * eta
    gd = np.repeat(g[..., None], 5, axis=-1)
    eps = 1e-3
    o1, S1 = oracle_mod.forward(q, k, v, eta, g, eps, S0, beta=beta)
    o2, S2 = oracle_mod.forward_diag(q, k, v, eta, gd, eps, S0, beta=beta)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S2, S1, rtol=1e-12, atol=1e-13)
    o3, S3 = oracle_mod.chunk_forward_diag(q, k, v, eta, gd, eps, S0, chunk=4, beta=beta)
    np.testing.assert_allclose(o3, o1, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(S3, S1, rtol=1e-10, atol=1e-11)
    dO = rng.standard_normal(o1.shape)
    dST = rng.standard_normal(S1.shape)
    r1 = oracle_mod.backward(q, k, v, eta, g, eps, S0, dO, dST, beta=beta)
    r2 = oracle_mod.backward_diag(q, k, v, eta, gd, eps, S0, dO, dST, beta=beta)
    for name in ("dq", "dk", "dv", "deta", "dS0"):
        np.testing.assert_allclose(r2[name], r1[name], rtol=1e-10, atol=1e-11, err_msg=name)
    np.testing.assert_allclose(r2["dg"].sum(-1), r1["dg"], rtol=1e-10, atol=1e-11)


def test_diag_hard_projection_any_decay(oracle_mod):
    rng = np.random.default_rng(401)
    q, k, v, _, _, S0 = _rand_inputs(rng, 2, 10, 2, 6, 3, key_lo=0.1, key_hi=10.0)
    g = _diag_g(rng, k.shape[:3], 6, lo=-3.0)
    eta = np.ones(k.shape[:3])
    S = S0.copy()
    for t in range(k.shape[1]):
        _, S = oracle_mod.decode_step_diag(q[:, t], k[:, t], v[:, t], eta[:, t], g[:, t], 0.0, S)
        readout = np.einsum("bhij,bhi->bhj", S, k[:, t])
        np.testing.assert_allclose(readout, v[:, t], rtol=0, atol=1e-12 * (1 + np.abs(v[:, t]).max()))


@pytest.mark.parametrize("eps", [1e-6, 0.5])
def test_diag_relaxed_interpolation(oracle_mod, eps):
    rng = np.random.default_rng(402)
    q, k, v, eta, _, S0 = _rand_inputs(rng, 1, 8, 3, 4, 5)
    g = _diag_g(rng, k.shape[:3], 4, lo=-2.0)
    S = S0.copy()
    for t in range(k.shape[1]):
        Sdec = np.exp(g[:, t])[..., None] * S      # the decayed state, Diag(alpha_t) S_{t-1}
        _, S = oracle_mod.decode_step_diag(q[:, t], k[:, t], v[:, t], eta[:, t], g[:, t], eps, S)
        n = np.sum(k[:, t] ** 2, axis=-1)
        c = (eta[:, t] * n / (n + eps))[..., None]
        lhs = np.einsum("bhij,bhi->bhj", S, k[:, t])
        rhs = (1 - c) * np.einsum("bhij,bhi->bhj", Sdec, k[:, t]) + c * v[:, t]
        np.testing.assert_allclose(lhs, rhs, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("C", [1, 3, 8, 64])
def test_diag_chunk_form_matches_token_form(oracle_mod, C):
    rng = np.random.default_rng(403 + C)
    q, k, v, eta, _, S0 = _rand_inputs(rng, 2, 70, 2, 5, 4, key_lo=0.3, key_hi=3.0)
    g = _diag_g(rng, k.shape[:3], 5, lo=-1.5)
    o1, S1 = oracle_mod.forward_diag(q, k, v, eta, g, 1e-6, S0)
    o2, S2 = oracle_mod.chunk_forward_diag(q, k, v, eta, g, 1e-6, S0, chunk=C)
    np.testing.assert_allclose(o2, o1, rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(S2, S1, rtol=1e-9, atol=1e-10)


def test_diag_decode_step_equals_forward_T1(oracle_mod):
    rng = np.random.default_rng(404)
    q, k, v, eta, _, S0 = _rand_inputs(rng, 2, 1, 3, 4, 5)
    g = _diag_g(rng, k.shape[:3], 4)
    o, ST = oracle_mod.forward_diag(q, k, v, eta, g, 1e-6, S0)
    o2, S2 = oracle_mod.decode_step_diag(q[:, 0], k[:, 0], v[:, 0], eta[:, 0], g[:, 0], 1e-6, S0)
    np.testing.assert_array_equal(o[:, 0], o2)
    np.testing.assert_array_equal(ST, S2)


@pytest.mark.parametrize("beta,eps", [("kaczmarz", 1e-2), ("direct", 0.0)])
def test_diag_backward_finite_differences(oracle_mod, beta, eps):
    rng = np.random.default_rng(410)
    B, T, H, Dk, Dv = 1, 6, 2, 3, 4
    q, k, v, eta, _, S0 = _rand_inputs(rng, B, T, H, Dk, Dv, key_lo=0.5, key_hi=1.5, s0=0.5)
    g = _diag_g(rng, (B, T, H), Dk, lo=-1.0)
    if beta == "direct":
        eta = 0.3 * eta
    dO = rng.standard_normal((B, T, H, Dv))
    dST = rng.standard_normal((B, H, Dk, Dv))
    grads = oracle_mod.backward_diag(q, k, v, eta, g, eps, S0, dO, dST, beta=beta)
    args = dict(q=q, k=k, v=v, eta=eta, g=g, S0=S0)

    def loss(a):
        o, ST = oracle_mod.forward_diag(a["q"], a["k"], a["v"], a["eta"], a["g"], eps, a["S0"], beta=beta)
        return float(np.sum(o * dO) + np.sum(ST * dST))

    hstep = 1e-6
    for name in args:
        x = args[name]
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            a_p = {kk: vv.copy() for kk, vv in args.items()}
            a_m = {kk: vv.copy() for kk, vv in args.items()}
            a_p[name][idx] += hstep
            a_m[name][idx] -= hstep
            fd[idx] = (loss(a_p) - loss(a_m)) / (2 * hstep)
        got = grads["d" + name]
        err = np.abs(got - fd).max() / max(np.abs(fd).max(), 1e-3)
        assert err <= 1e-6, (name, err)
