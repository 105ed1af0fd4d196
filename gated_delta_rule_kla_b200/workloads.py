"""Seeded synthetic inputs for the KLA workloads.

This module draws random inputs and nothing else: it holds none of the method's
arithmetic.  Both the CUDA-path tests/benchmark and the fp64 oracle are fed from
here, so the two sides always see the same values.

Shapes follow the model of "Kaczmarz Linear Attention" (Appendix C: 8 heads of
dimension 128) and the contexts of its section 5 (4K training context, 32K decode,
65K long-context evaluation).  The paper trains on SlimPajama; no dataset or
trained weights are used here, these seeded draws stand in for them.

Draw order per workload (one CPU ``torch.Generator`` seeded with the workload's
seed, fp64): q, z_k, s_k, v, eta-logit, g, S0, dO.  Then q, k, v are cast to the
workload dtype (round-to-nearest-even for bf16); eta, g, S0, dO stay fp32.

  q, v        ~ N(0, 1)
  k           = s * z                 (key_mode "scaled", ||k|| ~ s * sqrt(d))
              = s * z / ||z||         (key_mode "unit_scaled", ||k|| = s)
                with z ~ N(0, I), ln s ~ U(ln 0.1, ln 10) per token
  eta         = sigmoid(N(0, 1))
  g           ~ U(-0.5, 0)            (gate_mode "uniform")
              = -softplus(N(0,1))*0.1 (gate_mode "softplus")
              ~ U(gate_lo, 0) per key channel, shape [..., Dk]
                                      (gate_mode "diag": diagonal gating, App. A.5)
  S0          = 0 or 0.02 * N(0, 1)
  dO          ~ N(0, 1)               (training workload only)

Gate prologue (make_gate_inputs): token vectors x ~ N(0, 1) [N, D]; projections
W ~ N(0, 1/D) [2H, D] (unit-variance logits); bias_eta ~ N(0, 1), bias_g ~ N(0, 1) - 2 (so
that -softplus keeps most decays mild); q ~ N(0, 1) [N, H, Dk] with a spread of norms
(each row times a log-uniform factor on [0.1, 10]).
"""
from dataclasses import dataclass, replace
import math

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str  # "fwd", "decode" or "train"
    B: int
    T: int  # tokens per sequence (decode: number of sequential steps)
    H: int
    Dk: int
    Dv: int
    dtype: str  # "f32" or "bf16"
    key_mode: str
    gate_mode: str
    s0: str  # "zero" or "normal"
    seed: int
    eps: float = 1e-6
    chunk: int = 64
    gate_lo: float = -0.5  # lower end of the per-channel log-decays (gate_mode "diag")

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


WORKLOADS = {
    "tiny_fwd_f32": Workload("tiny_fwd_f32", "fwd", B=1, T=256, H=2, Dk=64, Dv=64, dtype="f32",
                             key_mode="scaled", gate_mode="uniform", s0="zero", seed=0),
    "prefill_b8_t2048_h8_d128": Workload("prefill_b8_t2048_h8_d128", "fwd", B=8, T=2048, H=8,
                                         Dk=128, Dv=128, dtype="bf16", key_mode="unit_scaled",
                                         gate_mode="softplus", s0="zero", seed=1),
    "prefill_b1_t65536_h16_d128": Workload("prefill_b1_t65536_h16_d128", "fwd", B=1, T=65536, H=16,
                                           Dk=128, Dv=128, dtype="bf16", key_mode="scaled",
                                           gate_mode="uniform", s0="normal", seed=2),
    "decode_b64_h16_d128_x1024": Workload("decode_b64_h16_d128_x1024", "decode", B=64, T=1024, H=16,
                                          Dk=128, Dv=128, dtype="bf16", key_mode="scaled",
                                          gate_mode="uniform", s0="normal", seed=3),
    "train_b4_t4096_h16_d128": Workload("train_b4_t4096_h16_d128", "train", B=4, T=4096, H=16,
                                        Dk=128, Dv=128, dtype="bf16", key_mode="scaled",
                                        gate_mode="uniform", s0="zero", seed=4),
    # diagonal (per-key-channel) gating on the prefill and decode shapes above
    "prefill_diag_b8_t2048_h8_d128": Workload("prefill_diag_b8_t2048_h8_d128", "fwd", B=8, T=2048, H=8,
                                              Dk=128, Dv=128, dtype="bf16", key_mode="unit_scaled",
                                              gate_mode="diag", s0="zero", seed=5),
    "decode_diag_b64_h16_d128_x1024": Workload("decode_diag_b64_h16_d128_x1024", "decode", B=64, T=1024,
                                               H=16, Dk=128, Dv=128, dtype="bf16", key_mode="scaled",
                                               gate_mode="diag", s0="normal", seed=6),
}


def make_inputs(w: Workload, device=None):
    """Draw the inputs of workload `w`.

    Sequence workloads return q, k [B,T,H,Dk], v [B,T,H,Dv], eta, g [B,T,H] (diagonal gating:
    g [B,T,H,Dk]),
    S0 [B,H,Dk,Dv] (None when zero) and, for training, dO [B,T,H,Dv].
    Decode returns the same tensors with the step axis first: q, k [T,B,H,Dk],
    v [T,B,H,Dv], eta, g [T,B,H].
    """
    gen = torch.Generator(device="cpu").manual_seed(w.seed)
    f64 = torch.float64
    if w.kind == "decode":
        tok = (w.T, w.B, w.H)
    else:
        tok = (w.B, w.T, w.H)
    q = torch.randn(*tok, w.Dk, generator=gen, dtype=f64)
    z = torch.randn(*tok, w.Dk, generator=gen, dtype=f64)
    s = torch.exp(torch.empty(*tok, 1, dtype=f64).uniform_(math.log(0.1), math.log(10.0), generator=gen))
    if w.key_mode == "scaled":
        k = s * z
    elif w.key_mode == "unit_scaled":
        k = s * z / z.norm(dim=-1, keepdim=True)
    else:
        raise ValueError(w.key_mode)
    del z
    v = torch.randn(*tok, w.Dv, generator=gen, dtype=f64)
    eta = torch.sigmoid(torch.randn(*tok, generator=gen, dtype=f64))
    if w.gate_mode == "uniform":
        g = torch.empty(*tok, dtype=f64).uniform_(-0.5, 0.0, generator=gen)
    elif w.gate_mode == "softplus":
        g = -torch.nn.functional.softplus(torch.randn(*tok, generator=gen, dtype=f64)) * 0.1
    elif w.gate_mode == "diag":
        g = torch.empty(*tok, w.Dk, dtype=f64).uniform_(w.gate_lo, 0.0, generator=gen)
    else:
        raise ValueError(w.gate_mode)
    if w.s0 == "normal":
        S0 = (torch.randn(w.B, w.H, w.Dk, w.Dv, generator=gen, dtype=f64) * 0.02).float()
    else:
        S0 = None
    out = dict(q=q.to(w.torch_dtype), k=k.to(w.torch_dtype), v=v.to(w.torch_dtype),
               eta=eta.float(), g=g.float(), S0=S0)
    del q, k, v
    if w.kind == "train":
        out["dO"] = torch.randn(w.B, w.T, w.H, w.Dv, generator=gen, dtype=f64).float()
    if device is not None:
        out = {key: (t.to(device) if t is not None else None) for key, t in out.items()}
    return out


def make_gate_inputs(N, D, H, Dk, dtype, seed, device=None):
    """Seeded inputs of the gate prologue (see the module docstring): x [N, D], W [2H, D] and
    q [N, H, Dk] in `dtype` ("f32" or "bf16"), bias [2H] fp32."""
    gen = torch.Generator(device="cpu").manual_seed(seed)
    f64 = torch.float64
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    x = torch.randn(N, D, generator=gen, dtype=f64)
    W = torch.randn(2 * H, D, generator=gen, dtype=f64) / math.sqrt(D)
    bias = torch.randn(2 * H, generator=gen, dtype=f64)
    bias[H:] -= 2.0
    q = torch.randn(N, H, Dk, generator=gen, dtype=f64)
    q = q * torch.exp(torch.empty(N, H, 1, dtype=f64).uniform_(math.log(0.1), math.log(10.0), generator=gen))
    out = dict(x=x.to(tdt), W=W.to(tdt), bias=bias.float(), q=q.to(tdt))
    if device is not None:
        out = {key: t.to(device) for key, t in out.items()}
    return out
