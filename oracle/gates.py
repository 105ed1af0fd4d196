"""fp64 CPU oracle of the gate prologue (TEST INFRASTRUCTURE ONLY).

The step before the KLA recurrence: the per-token gates and the query normalisation that feed
it.  Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may use
this module; the CUDA library shares no code with it.

Sources ("Kaczmarz Linear Attention"):
  * section 3.3: the write gate eta_t is a sigmoid-activated linear projection of the input
    token:  eta_t = sigmoid(x_t . w_eta + b_eta), one gate per head.
  * the decay: alpha_t = exp(g_t) (the blog "From Gated DeltaNet to Kaczmarz", section 2).  The
    pages do not print g's projection; the reading taken here is the plainest one that keeps
    g a log-decay (g <= 0) and is itself a linear projection of the token through a fixed
    activation: g_t = -softplus(x_t . w_g + b_g).
  * Algorithm 1 (left panel), line 6: the readout divides by ||q_t||.  Because o is linear in
    q, that readout is the library's readout on qhat_t = q_t / ||q_t|| (per head); at q_t = 0
    the readout is taken as zero (qhat_t = 0), the pages being silent there.

Layouts: x [N, D] (N = B * T tokens), W [2H, D] (rows 0..H-1 the eta projections of the H
heads, rows H..2H-1 the decay projections), bias [2H]; eta, g [N, H]; q, qhat [N, H, Dk].
"""
import numpy as np


def _f64(a):
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").double().numpy()
    return np.asarray(a, dtype=np.float64)


def _sigmoid(z):
    # 1 / (1 + e^-z) without overflow for large |z|
    e = np.exp(-np.abs(z))
    return np.where(z >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def _softplus(z):
    # log(1 + e^z) = max(z, 0) + log(1 + e^-|z|)
    return np.maximum(z, 0.0) + np.log1p(np.exp(-np.abs(z)))


def gates(x, W, bias, H):
    """eta = sigmoid(x W_eta^T + b_eta), g = -softplus(x W_g^T + b_g); returns (eta, g) [N, H]."""
    x, W, bias = _f64(x), _f64(W), _f64(bias)
    z = x @ W.T + bias
    return _sigmoid(z[:, :H]), -_softplus(z[:, H:])


def normalize_q(q):
    """qhat = q / ||q|| over the last axis; zero where q is zero."""
    q = _f64(q)
    n = np.sqrt(np.sum(q * q, axis=-1, keepdims=True))
    return np.where(n > 0, q / np.where(n > 0, n, 1.0), 0.0)


def gates_backward(x, W, bias, H, deta, dg):
    """Gradients of <eta, deta> + <g, dg> with respect to x, W and bias (chain rule:
    d sigmoid(z) = sigmoid(z) (1 - sigmoid(z)) dz, d softplus(z) = sigmoid(z) dz).
    Returns dict(dx [N, D], dW [2H, D], db [2H])."""
    x, W, bias, deta, dg = _f64(x), _f64(W), _f64(bias), _f64(deta), _f64(dg)
    z = x @ W.T + bias
    s_eta = _sigmoid(z[:, :H])
    dz = np.concatenate([deta * s_eta * (1.0 - s_eta), -dg * _sigmoid(z[:, H:])], axis=1)
    return dict(dx=dz @ W, dW=dz.T @ x, db=dz.sum(axis=0))


def normalize_q_backward(q, dqhat):
    """Gradient of <qhat, dqhat> with respect to q: (dqhat - qhat (qhat . dqhat)) / ||q||
    (zero where q is zero, where the map is not differentiable)."""
    q, dqhat = _f64(q), _f64(dqhat)
    n = np.sqrt(np.sum(q * q, axis=-1, keepdims=True))
    safe = np.where(n > 0, n, 1.0)
    qh = q / safe
    dq = (dqhat - qh * np.sum(qh * dqhat, axis=-1, keepdims=True)) / safe
    return np.where(n > 0, dq, 0.0)
