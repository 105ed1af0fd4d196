"""fp64 CPU oracle for Kaczmarz Linear Attention (TEST INFRASTRUCTURE ONLY).

The oracle is a plain, slow, token-by-token implementation of the KLA recurrence
("Kaczmarz Linear Attention", section 3.3, Algorithm 1 left panel, with the
coefficient of Eq. (3)), a hand-derived backward of that recurrence, and the
chunkwise form of section 4 (Propositions 3 and 4) used only to cross-check the
tokenwise form.  The arithmetic lives in ``kla_oracle.c``; this module only
marshals numpy arrays.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package.  The CUDA library shares no code with it.

Parity status: forward pinned (Theorem 1, Propositions 1-2, Eq. (4), the
recurrent form of Table 6, classical Kaczmarz, the chunk form, a hand-worked
example, exact rational arithmetic); backward pinned by finite differences only.

``oracle.gates`` (plain numpy, fp64) is the oracle of the gate prologue: the write gate
eta_t = sigmoid(x_t . w_eta + b_eta) of section 3.3, the log-decay g_t = -softplus(x_t . w_g +
b_g) (a reading: the pages print no projection for g) and the query normalisation of
Algorithm 1's readout; pinned by closed forms, asymptotics, affinity of the logits, the
normalised readout against this package's recurrence, and finite differences.
"""
import ctypes
import os

import numpy as np

from . import build as _build


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _check(rc, name):
    if rc != 0:
        raise RuntimeError(f"{name} failed with code {rc}")


def _direct(beta):
    if beta not in ("kaczmarz", "direct"):
        raise ValueError(f"beta must be 'kaczmarz' or 'direct', got {beta!r}")
    return 1 if beta == "direct" else 0


class OracleLib:
    """ctypes view of one build of kla_oracle.c."""

    def __init__(self, path):
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        i = ctypes.c_int
        d = ctypes.c_double
        # each takes `int direct` after eps: beta_t = eta_t as given instead of Eq. (3)
        lib.kla_oracle_forward.argtypes = [i, i, i, i, i, dp, dp, dp, dp, dp, d, i, dp, dp, dp]
        lib.kla_oracle_decode_step.argtypes = [i, i, i, i, dp, dp, dp, dp, dp, d, i, dp, dp]
        lib.kla_oracle_backward.argtypes = [i, i, i, i, i, dp, dp, dp, dp, dp, d, i, dp, dp, dp,
                                            dp, dp, dp, dp, dp, dp, i]
        lib.kla_oracle_chunk_forward.argtypes = [i, i, i, i, i, dp, dp, dp, dp, dp, d, i, dp, i, dp, dp]
        # diagonal gating: g is [B, T, H, Dk] (decode: [B, H, Dk]); the backward has no checkpoints
        lib.kla_oracle_forward_diag.argtypes = [i, i, i, i, i, dp, dp, dp, dp, dp, d, i, dp, dp, dp]
        lib.kla_oracle_decode_step_diag.argtypes = [i, i, i, i, dp, dp, dp, dp, dp, d, i, dp, dp]
        lib.kla_oracle_backward_diag.argtypes = [i, i, i, i, i, dp, dp, dp, dp, dp, d, i, dp, dp, dp,
                                                 dp, dp, dp, dp, dp, dp]
        lib.kla_oracle_chunk_forward_diag.argtypes = [i, i, i, i, i, dp, dp, dp, dp, dp, d, i, dp, i, dp, dp]
        for f in (lib.kla_oracle_forward, lib.kla_oracle_decode_step, lib.kla_oracle_backward,
                  lib.kla_oracle_chunk_forward, lib.kla_oracle_forward_diag, lib.kla_oracle_decode_step_diag,
                  lib.kla_oracle_backward_diag, lib.kla_oracle_chunk_forward_diag):
            f.restype = ctypes.c_int
        self.lib = lib
        self.path = path

    def forward(self, q, k, v, eta, g, eps, S0=None, beta="kaczmarz"):
        """Token recurrence. q,k [B,T,H,Dk]; v [B,T,H,Dv]; eta,g [B,T,H]; S0 [B,H,Dk,Dv].
        beta="direct" takes beta_t = eta_t as given (the Gated DeltaNet update) instead of
        Eq. (3); the other methods take the same keyword.

        Returns (o [B,T,H,Dv], S_T [B,H,Dk,Dv]) in float64.
        """
        q, k, v, eta, g, S0 = map(_f64, (q, k, v, eta, g, S0))
        B, T, H, Dk = k.shape
        Dv = v.shape[-1]
        o = np.zeros((B, T, H, Dv))
        ST = np.zeros((B, H, Dk, Dv))
        rc = self.lib.kla_oracle_forward(B, T, H, Dk, Dv, _ptr(q), _ptr(k), _ptr(v), _ptr(eta),
                                         _ptr(g), float(eps), _direct(beta), _ptr(S0), _ptr(o), _ptr(ST))
        _check(rc, "kla_oracle_forward")
        return o, ST

    def decode_step(self, q, k, v, eta, g, eps, S, beta="kaczmarz"):
        """One token step per head. q,k [B,H,Dk]; v [B,H,Dv]; eta,g [B,H]; S [B,H,Dk,Dv].

        Returns (o [B,H,Dv], S_new) without modifying the argument S.
        """
        q, k, v, eta, g = map(_f64, (q, k, v, eta, g))
        S = _f64(S).copy()
        B, H, Dk = k.shape
        Dv = v.shape[-1]
        o = np.zeros((B, H, Dv))
        rc = self.lib.kla_oracle_decode_step(B, H, Dk, Dv, _ptr(q), _ptr(k), _ptr(v), _ptr(eta),
                                             _ptr(g), float(eps), _direct(beta), _ptr(S), _ptr(o))
        _check(rc, "kla_oracle_decode_step")
        return o, S

    def backward(self, q, k, v, eta, g, eps, S0, dO, dS_T=None, ckpt=64, beta="kaczmarz"):
        """Gradients of <o, dO> + <S_T, dS_T> w.r.t. every input.

        Returns a dict with dq, dk, dv, deta, dg, dS0 (float64).
        """
        q, k, v, eta, g, S0, dO, dS_T = map(_f64, (q, k, v, eta, g, S0, dO, dS_T))
        B, T, H, Dk = k.shape
        Dv = v.shape[-1]
        out = dict(dq=np.zeros((B, T, H, Dk)), dk=np.zeros((B, T, H, Dk)), dv=np.zeros((B, T, H, Dv)),
                   deta=np.zeros((B, T, H)), dg=np.zeros((B, T, H)), dS0=np.zeros((B, H, Dk, Dv)))
        rc = self.lib.kla_oracle_backward(B, T, H, Dk, Dv, _ptr(q), _ptr(k), _ptr(v), _ptr(eta),
                                          _ptr(g), float(eps), _direct(beta), _ptr(S0), _ptr(dO), _ptr(dS_T),
                                          _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                                          _ptr(out["deta"]), _ptr(out["dg"]), _ptr(out["dS0"]),
                                          int(ckpt))
        _check(rc, "kla_oracle_backward")
        return out

    def chunk_forward(self, q, k, v, eta, g, eps, S0=None, chunk=64, beta="kaczmarz"):
        """Chunkwise form (Eqs. 7-9) in fp64; used only to cross-check `forward`."""
        q, k, v, eta, g, S0 = map(_f64, (q, k, v, eta, g, S0))
        B, T, H, Dk = k.shape
        Dv = v.shape[-1]
        o = np.zeros((B, T, H, Dv))
        ST = np.zeros((B, H, Dk, Dv))
        rc = self.lib.kla_oracle_chunk_forward(B, T, H, Dk, Dv, _ptr(q), _ptr(k), _ptr(v), _ptr(eta),
                                               _ptr(g), float(eps), _direct(beta), _ptr(S0), int(chunk), _ptr(o),
                                               _ptr(ST))
        _check(rc, "kla_oracle_chunk_forward")
        return o, ST

    # ---- diagonal gating ("Kaczmarz Linear Attention", App. A.5, B.5): g per key channel ----
    def forward_diag(self, q, k, v, eta, g, eps, S0=None, beta="kaczmarz"):
        """Token recurrence with the decay Diag(exp(g_t)), g [B,T,H,Dk]; returns (o, S_T)."""
        q, k, v, eta, g, S0 = map(_f64, (q, k, v, eta, g, S0))
        B, T, H, Dk = k.shape
        Dv = v.shape[-1]
        o = np.zeros((B, T, H, Dv))
        ST = np.zeros((B, H, Dk, Dv))
        rc = self.lib.kla_oracle_forward_diag(B, T, H, Dk, Dv, _ptr(q), _ptr(k), _ptr(v), _ptr(eta), _ptr(g),
                                              float(eps), _direct(beta), _ptr(S0), _ptr(o), _ptr(ST))
        _check(rc, "kla_oracle_forward_diag")
        return o, ST

    def decode_step_diag(self, q, k, v, eta, g, eps, S, beta="kaczmarz"):
        """One diagonal-gated token step per head, g [B,H,Dk]; returns (o, S_new)."""
        q, k, v, eta, g = map(_f64, (q, k, v, eta, g))
        S = _f64(S).copy()
        B, H, Dk = k.shape
        Dv = v.shape[-1]
        o = np.zeros((B, H, Dv))
        rc = self.lib.kla_oracle_decode_step_diag(B, H, Dk, Dv, _ptr(q), _ptr(k), _ptr(v), _ptr(eta), _ptr(g),
                                                  float(eps), _direct(beta), _ptr(S), _ptr(o))
        _check(rc, "kla_oracle_decode_step_diag")
        return o, S

    def backward_diag(self, q, k, v, eta, g, eps, S0, dO, dS_T=None, beta="kaczmarz"):
        """Gradients of <o, dO> + <S_T, dS_T>; dg is [B,T,H,Dk]."""
        q, k, v, eta, g, S0, dO, dS_T = map(_f64, (q, k, v, eta, g, S0, dO, dS_T))
        B, T, H, Dk = k.shape
        Dv = v.shape[-1]
        out = dict(dq=np.zeros((B, T, H, Dk)), dk=np.zeros((B, T, H, Dk)), dv=np.zeros((B, T, H, Dv)),
                   deta=np.zeros((B, T, H)), dg=np.zeros((B, T, H, Dk)), dS0=np.zeros((B, H, Dk, Dv)))
        rc = self.lib.kla_oracle_backward_diag(B, T, H, Dk, Dv, _ptr(q), _ptr(k), _ptr(v), _ptr(eta), _ptr(g),
                                               float(eps), _direct(beta), _ptr(S0), _ptr(dO), _ptr(dS_T),
                                               _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                                               _ptr(out["deta"]), _ptr(out["dg"]), _ptr(out["dS0"]))
        _check(rc, "kla_oracle_backward_diag")
        return out

    def chunk_forward_diag(self, q, k, v, eta, g, eps, S0=None, chunk=64, beta="kaczmarz"):
        """Chunk form of the diagonal-gated recurrence; used only to cross-check forward_diag."""
        q, k, v, eta, g, S0 = map(_f64, (q, k, v, eta, g, S0))
        B, T, H, Dk = k.shape
        Dv = v.shape[-1]
        o = np.zeros((B, T, H, Dv))
        ST = np.zeros((B, H, Dk, Dv))
        rc = self.lib.kla_oracle_chunk_forward_diag(B, T, H, Dk, Dv, _ptr(q), _ptr(k), _ptr(v), _ptr(eta), _ptr(g),
                                                    float(eps), _direct(beta), _ptr(S0), int(chunk), _ptr(o),
                                                    _ptr(ST))
        _check(rc, "kla_oracle_chunk_forward_diag")
        return o, ST


_default = None


def _load() -> OracleLib:
    global _default
    if _default is None:
        _default = OracleLib(_build.build())
    return _default


def forward(*a, **kw):
    return _load().forward(*a, **kw)


def decode_step(*a, **kw):
    return _load().decode_step(*a, **kw)


def backward(*a, **kw):
    return _load().backward(*a, **kw)


def chunk_forward(*a, **kw):
    return _load().chunk_forward(*a, **kw)


def forward_diag(*a, **kw):
    return _load().forward_diag(*a, **kw)


def decode_step_diag(*a, **kw):
    return _load().decode_step_diag(*a, **kw)


def backward_diag(*a, **kw):
    return _load().backward_diag(*a, **kw)


def chunk_forward_diag(*a, **kw):
    return _load().chunk_forward_diag(*a, **kw)


def threads() -> int:
    """Threads the oracle's OpenMP loops use (OMP_NUM_THREADS, else the host's cores)."""
    env = os.environ.get("OMP_NUM_THREADS")
    if env and env.isdigit():
        return int(env)
    return os.cpu_count() or 1
