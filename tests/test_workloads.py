"""The input recipe: the seeded generators produce the shapes, layouts, dtypes and
distributions the workloads are documented with (CPU only, shortened copies of each
workload: the properties do not depend on the sizes)."""
import math

import pytest
import torch

from gated_delta_rule_kla_b200.workloads import WORKLOADS, make_inputs


def small(name, **kw):
    w = WORKLOADS[name]
    return w.with_(**kw)


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_shapes_layout_and_dtypes(name):
    w = WORKLOADS[name]
    ws = w.with_(T=min(w.T, 96), B=min(w.B, 3))
    d = make_inputs(ws)
    tok = (ws.T, ws.B, ws.H) if ws.kind == "decode" else (ws.B, ws.T, ws.H)
    dt = torch.bfloat16 if ws.dtype == "bf16" else torch.float32
    assert d["q"].shape == tok + (ws.Dk,) and d["k"].shape == tok + (ws.Dk,) and d["v"].shape == tok + (ws.Dv,)
    assert d["q"].dtype == d["k"].dtype == d["v"].dtype == dt
    gshape = tok + (ws.Dk,) if ws.gate_mode == "diag" else tok
    assert d["eta"].shape == tok and d["g"].shape == gshape
    assert d["eta"].dtype == d["g"].dtype == torch.float32
    if ws.s0 == "normal":
        assert d["S0"].shape == (ws.B, ws.H, ws.Dk, ws.Dv) and d["S0"].dtype == torch.float32
    else:
        assert d["S0"] is None
    if ws.kind == "train":
        assert d["dO"].shape == (ws.B, ws.T, ws.H, ws.Dv) and d["dO"].dtype == torch.float32
    else:
        assert "dO" not in d


def test_same_seed_same_draws_and_seeds_differ():
    w = small("prefill_b8_t2048_h8_d128", T=128, B=2)
    a, b = make_inputs(w), make_inputs(w)
    for key in ("q", "k", "v", "eta", "g"):
        assert torch.equal(a[key], b[key])
    c = make_inputs(w.with_(seed=w.seed + 1))
    assert not torch.equal(a["q"], c["q"])


def test_key_norms_log_uniform_on_0p1_to_10():
    # unit_scaled: ||k|| = s exactly (before the bf16 rounding), ln s ~ U(ln 0.1, ln 10)
    w = small("prefill_b8_t2048_h8_d128", T=512, B=4)
    k = make_inputs(w)["k"].double()
    n = k.norm(dim=-1)
    assert n.min() >= 0.1 * 0.99 and n.max() <= 10.0 * 1.01
    ln = n.log()
    assert abs(float(ln.mean())) < 0.05                                    # centre of U(ln .1, ln 10)
    assert abs(float(ln.std()) - math.log(100.0) / math.sqrt(12.0)) < 0.05  # its spread
    # scaled: ||k|| ~ s sqrt(d), the same log-uniform factor times a chi-distributed norm
    w2 = small("train_b4_t4096_h16_d128", T=256, B=2)
    k2 = make_inputs(w2)["k"].double()
    ln2 = (k2.norm(dim=-1) / math.sqrt(w2.Dk)).log()
    assert abs(float(ln2.mean())) < 0.05
    assert float(ln2.min()) > math.log(0.1) - 0.3 and float(ln2.max()) < math.log(10.0) + 0.3


def test_gates_eta_and_initial_state():
    d = make_inputs(small("train_b4_t4096_h16_d128", T=512, B=2))  # uniform gates
    assert float(d["eta"].min()) > 0.0 and float(d["eta"].max()) < 1.0
    assert abs(float(d["eta"].double().mean()) - 0.5) < 0.02        # sigmoid(N(0,1)) is symmetric
    g = d["g"].double()
    assert float(g.min()) >= -0.5 and float(g.max()) <= 0.0
    assert abs(float(g.mean()) + 0.25) < 0.01
    gs = make_inputs(small("prefill_b8_t2048_h8_d128", T=512, B=2))["g"].double()  # -softplus(N(0,1)) * 0.1
    assert float(gs.max()) < 0.0
    assert abs(float(gs.mean()) + 0.08066) < 0.003                   # -0.1 E[softplus(N(0,1))]
    S0 = make_inputs(small("decode_b64_h16_d128_x1024", T=4))["S0"].double()
    assert abs(float(S0.std()) - 0.02) < 0.001 and abs(float(S0.mean())) < 0.001


def test_diagonal_gates_per_channel_uniform():
    w = small("prefill_diag_b8_t2048_h8_d128", T=256, B=2)
    g = make_inputs(w)["g"].double()
    assert g.shape == (2, 256, w.H, w.Dk)
    assert float(g.min()) >= w.gate_lo and float(g.max()) <= 0.0
    assert abs(float(g.mean()) - w.gate_lo / 2) < 0.01
    # channels are drawn independently: the decay differs across the key channels of a token
    assert float(g.std(dim=-1).mean()) > 0.1
    g4 = make_inputs(w.with_(gate_lo=-4.0))["g"].double()
    assert float(g4.min()) >= -4.0 and abs(float(g4.mean()) + 2.0) < 0.05
