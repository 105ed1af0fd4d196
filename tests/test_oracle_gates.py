"""Pins of the gate-prologue oracle (oracle/gates.py) against what the pages and the mathematics
fix, independent of the oracle's own formulas:

  * closed forms: sigmoid(0) = 1/2, sigmoid(log 3) = 3/4, softplus(0) = log 2,
    softplus(log(e - 1)) = 1;
  * asymptotics of both activations far out on either side (a dropped sign or term fails);
  * the logits are affine in the token and each head reads only its own projection row;
  * Algorithm 1's readout o_t = S_t^T q_t / ||q_t|| equals the KLA oracle's readout on qhat;
  * central finite differences for every gradient.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import gates as og


def _rand(rng, N=7, D=5, H=3):
    x = rng.standard_normal((N, D))
    W = 0.7 * rng.standard_normal((2 * H, D))
    b = rng.standard_normal(2 * H)
    return x, W, b


def check_closed_forms(og):
    x = np.zeros((2, 4))
    W = np.zeros((4, 4))
    eta, g = og.gates(x, W, np.zeros(4), 2)
    assert np.all(eta == 0.5)
    assert np.allclose(g, -math.log(2.0), rtol=0, atol=1e-15)
    b = np.array([math.log(3.0), 0.0, math.log(math.e - 1.0), 0.0])
    eta, g = og.gates(x, W, b, 2)
    assert abs(eta[0, 0] - 0.75) < 1e-15 and abs(g[0, 0] + 1.0) < 1e-15


def check_asymptotics(og, z):
    x = np.ones((1, 1))
    W = np.array([[z], [-z], [z], [-z]])
    eta, g = og.gates(x, W, np.zeros(4), 2)
    # eta: 1 - e^-z on the right, e^-z on the left; g = -softplus: ~ -z on the right, -e^-z on the left
    assert abs((1.0 - eta[0, 0]) - math.exp(-z)) <= math.exp(-z) + 1e-16  # 1 - eta is below fp64's step
    assert abs(eta[0, 1] - math.exp(-z)) <= 1e-10 * math.exp(-z) + 1e-300
    assert abs(g[0, 0] + z) <= 1e-12 * z
    assert abs(g[0, 1] + math.exp(-z)) <= 1e-10 * math.exp(-z) + 1e-300
    assert np.all(g <= 0) and np.all(eta >= 0) and np.all(eta <= 1)


def check_logits_affine_in_the_token_and_per_head(og):
    rng = np.random.default_rng(1)
    x, W, b = _rand(rng)
    H = 3
    logit = lambda e: np.log(e / (1.0 - e))
    inv_sp = lambda g: np.log(np.expm1(-g))  # z with -softplus(z) = g
    e1, g1 = og.gates(x[:1], W, b, H)
    e2, g2 = og.gates(x[1:2], W, b, H)
    e12, g12 = og.gates(x[:1] + x[1:2], W, b, H)
    e0, g0 = og.gates(np.zeros((1, x.shape[1])), W, b, H)
    assert np.allclose(logit(e1) + logit(e2) - logit(e0), logit(e12), atol=1e-10)
    assert np.allclose(inv_sp(g1) + inv_sp(g2) - inv_sp(g0), inv_sp(g12), atol=1e-9)
    W2 = W.copy()
    W2[1] += 1.0  # eta projection of head 1 only
    W2[H + 2] -= 1.0  # decay projection of head 2 only
    e3, g3 = og.gates(x, W2, b, H)
    e4, g4 = og.gates(x, W, b, H)
    assert np.array_equal(e3[:, [0, 2]], e4[:, [0, 2]]) and not np.allclose(e3[:, 1], e4[:, 1])
    assert np.array_equal(g3[:, [0, 1]], g4[:, [0, 1]]) and not np.allclose(g3[:, 2], g4[:, 2])


def check_normalized_readout_is_algorithm1_line6(og, oracle_mod):
    """o computed from qhat equals o computed from q divided by ||q_t|| (per token and head),
    and qhat is invariant to positive rescaling of q; a zero query reads out zero."""
    rng = np.random.default_rng(2)
    B, T, H, Dk, Dv = 1, 9, 2, 4, 3
    q = rng.standard_normal((B, T, H, Dk))
    q[0, 3, 1] = 0.0
    k = rng.standard_normal((B, T, H, Dk))
    v = rng.standard_normal((B, T, H, Dv))
    eta = rng.uniform(0.1, 0.9, (B, T, H))
    g = rng.uniform(-0.5, 0.0, (B, T, H))
    qh = og.normalize_q(q)
    n = np.linalg.norm(q, axis=-1)
    assert np.allclose(np.linalg.norm(qh, axis=-1)[n > 0], 1.0, atol=1e-15)
    assert np.all(qh[0, 3, 1] == 0.0)
    assert np.allclose(og.normalize_q(q * rng.uniform(0.1, 10.0, (B, T, H, 1))), qh, atol=1e-15)
    o_hat, _ = oracle_mod.forward(qh, k, v, eta, g, 1e-6, None)
    o_raw, _ = oracle_mod.forward(q, k, v, eta, g, 1e-6, None)
    nz = n > 0
    assert np.allclose(o_hat[nz], o_raw[nz] / n[nz][:, None], atol=1e-12)
    assert np.all(o_hat[0, 3, 1] == 0.0)


def check_gates_backward_finite_differences(og):
    rng = np.random.default_rng(3)
    H = 3
    x, W, b = _rand(rng, H=H)
    deta = rng.standard_normal((x.shape[0], H))
    dg = rng.standard_normal((x.shape[0], H))
    gr = og.gates_backward(x, W, b, H, deta, dg)

    def loss(xx, WW, bb):
        e, gg = og.gates(xx, WW, bb, H)
        return float(np.sum(e * deta) + np.sum(gg * dg))

    h = 1e-6
    for name, arr in (("dx", x), ("dW", W), ("db", b)):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            p, m = arr.copy(), arr.copy()
            p[idx] += h
            m[idx] -= h
            args_p = {"dx": (p, W, b), "dW": (x, p, b), "db": (x, W, p)}[name]
            args_m = {"dx": (m, W, b), "dW": (x, m, b), "db": (x, W, m)}[name]
            fd[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        assert np.abs(gr[name] - fd).max() <= 1e-7 * max(1.0, np.abs(fd).max()), name


def check_normalize_q_backward_finite_differences(og):
    rng = np.random.default_rng(4)
    q = rng.standard_normal((3, 2, 5))
    q[1, 0] = 0.0
    dqh = rng.standard_normal(q.shape)
    dq = og.normalize_q_backward(q, dqh)
    h = 1e-6
    fd = np.zeros_like(q)
    for idx in np.ndindex(q.shape):
        if idx[:2] == (1, 0):
            continue  # not differentiable at zero; the tie-break returns zero there
        p, m = q.copy(), q.copy()
        p[idx] += h
        m[idx] -= h
        fd[idx] = (np.sum(og.normalize_q(p) * dqh) - np.sum(og.normalize_q(m) * dqh)) / (2 * h)
    assert np.abs(dq - fd).max() <= 1e-7
    assert np.all(dq[1, 0] == 0.0)


def test_closed_forms():
    check_closed_forms(og)


@pytest.mark.parametrize("z", [40.0, 700.0])
def test_asymptotics(z):
    check_asymptotics(og, z)


def test_logits_affine_in_the_token_and_per_head():
    check_logits_affine_in_the_token_and_per_head(og)


def test_normalized_readout_is_algorithm1_line6(oracle_mod):
    check_normalized_readout_is_algorithm1_line6(og, oracle_mod)


def test_gates_backward_finite_differences():
    check_gates_backward_finite_differences(og)


def test_normalize_q_backward_finite_differences():
    check_normalize_q_backward_finite_differences(og)


# ---------------------------------------------------------------------------------------
# Planted mistakes: each copy of oracle/gates.py below carries one plausible error; at least
# one of the checks above must fail on it (so the pins above do pin the oracle).
# ---------------------------------------------------------------------------------------
MUTATIONS = [
    ("sigmoid sign", "return np.where(z >= 0, 1.0 / (1.0 + e), e / (1.0 + e))",
     "return np.where(z >= 0, e / (1.0 + e), 1.0 / (1.0 + e))"),
    ("softplus drops max(z, 0)", "return np.maximum(z, 0.0) + np.log1p(np.exp(-np.abs(z)))",
     "return np.log1p(np.exp(-np.abs(z)))"),
    ("g without the minus", "return _sigmoid(z[:, :H]), -_softplus(z[:, H:])",
     "return _sigmoid(z[:, :H]), _softplus(z[:, H:])"),
    ("eta and g rows swapped", "return _sigmoid(z[:, :H]), -_softplus(z[:, H:])",
     "return _sigmoid(z[:, H:]), -_softplus(z[:, :H])"),
    ("bias dropped", "z = x @ W.T + bias\n    return _sigmoid", "z = x @ W.T\n    return _sigmoid"),
    ("norm without sqrt", "n = np.sqrt(np.sum(q * q, axis=-1, keepdims=True))\n    return np.where",
     "n = np.sum(q * q, axis=-1, keepdims=True)\n    return np.where"),
    ("sigmoid' without (1 - s)", "deta * s_eta * (1.0 - s_eta)", "deta * s_eta"),
    ("softplus' sign", "-dg * _sigmoid(z[:, H:])", "dg * _sigmoid(z[:, H:])"),
    ("dW transposed product", "dW=dz.T @ x", "dW=(x.T @ dz).T * 0.5"),
    ("dq without the projection", "dq = (dqhat - qh * np.sum(qh * dqhat, axis=-1, keepdims=True)) / safe",
     "dq = dqhat / safe"),
]


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(oracle_mod, name, old, new):
    import importlib.util
    import os
    src = open(os.path.join(os.path.dirname(og.__file__), "gates.py")).read()
    old, new = old.replace("\\n", "\n"), new.replace("\\n", "\n")
    assert old in src, name
    spec = importlib.util.spec_from_loader("gates_mutant", loader=None)
    mut = importlib.util.module_from_spec(spec)
    exec(compile(src.replace(old, new), "gates_mutant", "exec"), mut.__dict__)
    checks = [lambda: check_closed_forms(mut), lambda: check_asymptotics(mut, 40.0),
              lambda: check_asymptotics(mut, 700.0), lambda: check_logits_affine_in_the_token_and_per_head(mut),
              lambda: check_normalized_readout_is_algorithm1_line6(mut, oracle_mod),
              lambda: check_gates_backward_finite_differences(mut),
              lambda: check_normalize_q_backward_finite_differences(mut)]
    caught = 0
    for c in checks:
        try:
            with np.errstate(all="ignore"):
                c()
        except (AssertionError, FloatingPointError, ValueError):
            caught += 1
    assert caught > 0, f"planted mistake not caught: {name}"
