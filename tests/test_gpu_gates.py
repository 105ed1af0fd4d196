"""GPU parity of the gate prologue (kla_gate_prologue / kla_gate_prologue_bwd, through the
binding and the C ABI) against the fp64 oracle of oracle/gates.py on identical seeded inputs,
and the prologue feeding the recurrence end to end.

Bars (max|gpu - oracle| / rms(oracle)): eta, g and every gradient are fp32 results of exact
dtype-rounded inputs, 1e-4; qhat is stored in the input dtype, so bf16 adds one rounding
(2^-9 relative) and takes the bf16 bar 2e-2 (fp32: 1e-4).
"""
import math

import numpy as np
import pytest
import torch

from gated_delta_rule_kla_b200.workloads import Workload, make_gate_inputs, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kla():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gated_delta_rule_kla_b200 as kla
    kla.lib()
    return kla


def rel_err(got, ref):
    got = got.detach().double().cpu().numpy() if isinstance(got, torch.Tensor) else np.asarray(got)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got))
    rms = math.sqrt(float(np.mean(ref * ref)))
    return float(np.abs(got - ref).max()) / rms


def np64(t):
    return t.detach().double().cpu().numpy()


def assert_qhat_one_rounding(qhat, ref, dtype):
    """qhat is stored in the input dtype: each element within one unit in the last place of the
    exact value (bf16 carries 8 significant bits, so one ulp is at most 2^-7 of the value; the
    fp32 normalisation before the rounding adds ~1e-7; fp32 storage: 1e-6)."""
    got = np64(qhat)
    bound = (2.0 ** -7 if dtype == "bf16" else 1e-6) * np.abs(ref) + 1e-30
    assert np.all(np.abs(got - ref) <= bound)


CASES = [
    # N, D, H, Dk, dtype   (tensor cores: bf16, D % 64 == 0, H % 8 == 0)
    (300, 1024, 8, 128, "bf16"),   # tensor cores, ragged last tile
    (128, 2048, 16, 64, "bf16"),   # tensor cores, N = 2H = 32
    (77, 512, 64, 64, "bf16"),     # tensor cores, N = 2H = 128
    (50, 96, 6, 128, "bf16"),      # CUDA cores (H % 8 != 0)
    (33, 104, 3, 64, "f32"),       # CUDA cores, fp32
]


@pytest.mark.parametrize("N,D,H,Dk,dtype", CASES)
def test_gate_prologue_matches_oracle(kla, N, D, H, Dk, dtype):
    from oracle import gates as og
    inp = make_gate_inputs(N, D, H, Dk, dtype, seed=N + D + H)
    d = {k: v.cuda() for k, v in inp.items()}
    eta, g, qhat = kla.gate_prologue(d["x"], d["W"], d["bias"], d["q"])
    eta2, g2 = kla.gate_prologue(d["x"], d["W"], d["bias"])
    torch.cuda.synchronize()
    kla.check_device_error()
    re, rg = og.gates(np64(inp["x"]), np64(inp["W"]), np64(inp["bias"]), H)
    assert rel_err(eta, re) <= 1e-4 and rel_err(g, rg) <= 1e-4
    assert torch.equal(eta, eta2) and torch.equal(g, g2)
    assert float(g.max()) <= 0.0 and float(eta.min()) >= 0.0 and float(eta.max()) <= 1.0
    assert_qhat_one_rounding(qhat, og.normalize_q(np64(inp["q"])), dtype)


def test_gate_prologue_zero_query_and_empty(kla):
    inp = make_gate_inputs(10, 128, 8, 64, "bf16", seed=3)
    inp["q"][4, 2] = 0
    d = {k: v.cuda() for k, v in inp.items()}
    _, _, qhat = kla.gate_prologue(d["x"], d["W"], d["bias"], d["q"])
    e0, g0 = kla.gate_prologue(d["x"][:0], d["W"], d["bias"])
    torch.cuda.synchronize()
    assert torch.all(qhat[4, 2] == 0)
    assert e0.shape == (0, 8) and g0.shape == (0, 8)


@pytest.mark.parametrize("N,D,H,Dk,dtype", [(300, 1024, 8, 128, "bf16"), (70, 104, 3, 64, "f32"),
                                            (65, 256, 16, 128, "bf16")])
def test_gate_prologue_bwd_matches_oracle(kla, N, D, H, Dk, dtype):
    from oracle import gates as og
    inp = make_gate_inputs(N, D, H, Dk, dtype, seed=7 * N + H)
    inp["q"][3, 1] = 0
    gen = torch.Generator().manual_seed(N)
    deta = torch.randn(N, H, generator=gen)
    dg = torch.randn(N, H, generator=gen)
    dqh = torch.randn(N, H, Dk, generator=gen)
    d = {k: v.cuda() for k, v in inp.items()}
    eta, g = kla.gate_prologue(d["x"], d["W"], d["bias"])
    gr = kla.gate_prologue_bwd(d["x"], d["W"], eta, g, deta.cuda(), dg.cuda(), d["q"], dqh.cuda())
    gr2 = kla.gate_prologue_bwd(d["x"], d["W"], eta, g, deta.cuda(), dg.cuda(), d["q"], dqh.cuda())
    torch.cuda.synchronize()
    ref = og.gates_backward(np64(inp["x"]), np64(inp["W"]), np64(inp["bias"]), H, np64(deta), np64(dg))
    assert rel_err(gr["dx"], ref["dx"]) <= 1e-4
    assert rel_err(gr["dW"], ref["dW"]) <= 1e-4
    assert rel_err(gr["dbias"], ref["db"]) <= 1e-4
    assert rel_err(gr["dq"], og.normalize_q_backward(np64(inp["q"]), np64(dqh))) <= 1e-4
    for key in gr:  # fixed-order reductions: the same bits every call
        assert torch.equal(gr[key], gr2[key]), key


def test_prologue_feeds_the_recurrence_end_to_end(kla, oracle_mod):
    """x, W, bias and raw q -> (eta, g, qhat) -> kla_chunk_fwd (split tensor-core path) against
    the oracle's gates -> token recurrence, i.e. Algorithm 1 with its normalised readout.  qhat
    enters the recurrence in bf16 (the dtype of k and v), one rounding of the exact q/||q||: the
    oracle is fed that same rounded qhat (the rounding itself is checked elementwise), and its
    own eta and g from the exact inputs."""
    from oracle import gates as og
    B, T, H, D, Dk = 2, 150, 8, 1024, 128
    gi = make_gate_inputs(B * T, D, H, Dk, "bf16", seed=21)
    w = Workload("e2e", "fwd", B=B, T=T, H=H, Dk=Dk, Dv=Dk, dtype="bf16", key_mode="scaled",
                 gate_mode="uniform", s0="normal", seed=22)
    rec = make_inputs(w)
    d = {k: v.cuda() for k, v in gi.items()}
    eta, g, qhat = kla.gate_prologue(d["x"].view(B, T, D), d["W"], d["bias"], d["q"].view(B, T, H, Dk))
    o, ST = kla.chunk_fwd(qhat, rec["k"].cuda(), rec["v"].cuda(), eta, g, w.eps, rec["S0"].cuda())
    torch.cuda.synchronize()
    re, rg = og.gates(np64(gi["x"]), np64(gi["W"]), np64(gi["bias"]), H)
    assert_qhat_one_rounding(qhat, og.normalize_q(np64(gi["q"])).reshape(B, T, H, Dk), "bf16")
    ro, rST = oracle_mod.forward(np64(qhat), np64(rec["k"]), np64(rec["v"]), re.reshape(B, T, H),
                                 rg.reshape(B, T, H), w.eps, np64(rec["S0"]))
    assert rel_err(o, ro) <= 2e-2
    assert rel_err(ST, rST) <= 2e-2
