"""GPU parity for diagonal (per-key-channel) gating ("Kaczmarz Linear Attention", App. A.5 and
B.5): kla_chunk_fwd_diag, kla_chunk_bwd_diag and kla_decode_step_diag through the binding and
the C ABI, against the fp64 oracle's diagonal-gated functions on identical seeded inputs.

Metric per output tensor: max|gpu - oracle| / rms(oracle); bars 1e-4 (fp32 inputs) and 2e-2
(bf16 inputs).  Decays cover U(-0.5, 0) and U(-4, 0) per channel (the latter drives a 16-token
chunk's decay to ~e^-32 per channel on average and far below e^-80 over a 64-token span).
"""
import math

import numpy as np
import pytest
import torch

from gated_delta_rule_kla_b200.workloads import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}
GRADS = ("dq", "dk", "dv", "deta", "dg", "dS0")


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
    assert np.all(np.isfinite(got)), "non-finite GPU output"
    rms = math.sqrt(float(np.mean(ref * ref))) if ref.size else 0.0
    if rms == 0.0:
        return float(np.abs(got - ref).max()) if ref.size else 0.0
    return float(np.abs(got - ref).max()) / rms


def np64(t):
    return None if t is None else t.detach().double().cpu().numpy()


def diag_inputs(B, T, H, Dk, Dv, dtype, seed, gate_lo=-0.5, s0=True, kind="train"):
    w = Workload("diag", kind, B=B, T=T, H=H, Dk=Dk, Dv=Dv, dtype=dtype, key_mode="scaled",
                 gate_mode="diag", s0="normal" if s0 else "zero", seed=seed, gate_lo=gate_lo)
    return w, make_inputs(w)


def direct_eta(inp):
    k = inp["k"].double()
    return (inp["eta"].double() / ((k * k).sum(-1) + 1.0)).float()


FWD_CASES = [
    # B, T, H, Dk, Dv, dtype, gate_lo, s0, beta
    (1, 1, 1, 64, 64, "f32", -0.5, True, "kaczmarz"),
    (1, 50, 2, 64, 64, "f32", -0.5, True, "kaczmarz"),
    (2, 77, 3, 128, 64, "f32", -4.0, True, "kaczmarz"),
    (1, 40, 2, 64, 128, "f32", -0.5, False, "direct"),
    (2, 130, 2, 128, 128, "bf16", -0.5, True, "kaczmarz"),
    (1, 200, 2, 128, 128, "bf16", -4.0, True, "kaczmarz"),
    (1, 150, 3, 128, 128, "bf16", -0.05, True, "kaczmarz"),  # long memory: S0 matters to the end
    (1, 100, 2, 128, 128, "bf16", -0.5, True, "direct"),
    # bf16 at Dk = Dv = 128 runs on the tensor cores over 64-token chunks; log-decays down to -5
    # and -12 a token make some or all chunks span 160 or more in some channel, where the
    # preparation forms the pairwise decay factors exactly instead of around a reference
    (1, 130, 2, 128, 128, "bf16", -5.0, True, "kaczmarz"),
    (1, 70, 1, 128, 128, "bf16", -12.0, False, "kaczmarz"),
    (2, 640, 16, 128, 128, "bf16", -0.5, True, "kaczmarz"),  # two slabs (5 and 5 chunks)
    (1, 4100, 1, 128, 128, "bf16", -0.5, True, "kaczmarz"),  # parallel segments and the scan
]


@pytest.mark.parametrize("B,T,H,Dk,Dv,dtype,gate_lo,s0,beta", FWD_CASES)
def test_fwd_diag_matches_oracle(kla, oracle_mod, B, T, H, Dk, Dv, dtype, gate_lo, s0, beta):
    w, inp = diag_inputs(B, T, H, Dk, Dv, dtype, seed=T + 3 * H + Dk, gate_lo=gate_lo, s0=s0)
    if beta == "direct":
        inp["eta"] = direct_eta(inp)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    o, ST = kla.chunk_fwd_diag(d["q"], d["k"], d["v"], d["eta"], d["g"], w.eps, d["S0"], beta=beta)
    torch.cuda.synchronize()
    ro, rST = oracle_mod.forward_diag(*(np64(inp[k]) for k in ("q", "k", "v", "eta", "g")), w.eps, np64(inp["S0"]),
                                      beta=beta)
    assert rel_err(o, ro) <= TOL[dtype]
    assert rel_err(ST, rST) <= TOL[dtype]


@pytest.mark.parametrize("B,T,H,Dk,Dv,dtype,gate_lo", [(1, 50, 2, 64, 64, "f32", -0.5),
                                                       (2, 77, 3, 128, 64, "f32", -4.0),
                                                       (1, 200, 2, 128, 128, "bf16", -4.0),
                                                       (1, 40, 2, 64, 128, "bf16", -0.5)])
def test_fwd_diag_one_kernel_path_matches_oracle(kla, oracle_mod, B, T, H, Dk, Dv, dtype, gate_lo):
    """Without a workspace the forward runs as one kernel per (head, 64 value columns); with one
    (the default above) as the chunk-parallel preparation plus the state pass."""
    w, inp = diag_inputs(B, T, H, Dk, Dv, dtype, seed=T + H + 1, gate_lo=gate_lo)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    o1, S1 = kla.chunk_fwd_diag(d["q"], d["k"], d["v"], d["eta"], d["g"], w.eps, d["S0"], fused=True)
    o2, S2 = kla.chunk_fwd_diag(d["q"], d["k"], d["v"], d["eta"], d["g"], w.eps, d["S0"])
    torch.cuda.synchronize()
    kla.check_device_error()
    ro, rST = oracle_mod.forward_diag(*(np64(inp[k]) for k in ("q", "k", "v", "eta", "g")), w.eps, np64(inp["S0"]))
    for o, ST in ((o1, S1), (o2, S2)):
        assert rel_err(o, ro) <= TOL[dtype]
        assert rel_err(ST, rST) <= TOL[dtype]


def test_fwd_diag_uniform_channels_equal_scalar_gating(kla):
    """When every channel decays alike the diagonal-gated forward is the scalar-gated one
    (fp32, CUDA cores on both sides)."""
    w, inp = diag_inputs(2, 150, 2, 128, 128, "f32", seed=5)
    gs = inp["g"][..., 0].contiguous()
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    gd = gs.cuda()[..., None].expand(-1, -1, -1, 128).contiguous()
    o1, S1 = kla.chunk_fwd_diag(d["q"], d["k"], d["v"], d["eta"], gd, w.eps, d["S0"])
    o2, S2 = kla.chunk_fwd(d["q"], d["k"], d["v"], d["eta"], gs.cuda(), w.eps, d["S0"])
    torch.cuda.synchronize()
    assert rel_err(o1, np64(o2)) <= 1e-5
    assert rel_err(S1, np64(S2)) <= 1e-5


def test_fwd_diag_bf16_output_and_aliased_state(kla, oracle_mod):
    w, inp = diag_inputs(1, 90, 2, 128, 128, "bf16", seed=11)
    d = {k: v.cuda() for k, v in inp.items()}
    o32, S32 = kla.chunk_fwd_diag(d["q"], d["k"], d["v"], d["eta"], d["g"], w.eps, d["S0"])
    S = d["S0"].clone()
    o16, _ = kla.chunk_fwd_diag(d["q"], d["k"], d["v"], d["eta"], d["g"], w.eps, S, S_T=S,
                                out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(o16, o32.to(torch.bfloat16))
    assert torch.equal(S, S32)


def test_fwd_diag_empty_sequence(kla):
    S0 = torch.randn(1, 2, 64, 64, device="cuda")
    q = torch.empty(1, 0, 2, 64, device="cuda")
    o, ST = kla.chunk_fwd_diag(q, q, q, torch.empty(1, 0, 2, device="cuda"), torch.empty(1, 0, 2, 64, device="cuda"),
                               1e-6, S0)
    torch.cuda.synchronize()
    assert o.shape == (1, 0, 2, 64) and torch.equal(ST, S0)


def test_fwd_diag_prefill_workload_sampled_heads(kla, oracle_mod):
    """The full B=8 T=2048 H=8 d=128 diagonal-gated prefill; the oracle checks 3 (b, h) pairs."""
    w = WORKLOADS["prefill_diag_b8_t2048_h8_d128"]
    inp = make_inputs(w)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    o, ST = kla.chunk_fwd_diag(d["q"], d["k"], d["v"], d["eta"], d["g"], w.eps, d["S0"])
    torch.cuda.synchronize()
    for b, h in [(0, 0), (7, 7), (3, 5)]:
        sl = lambda x: np.ascontiguousarray(np64(x)[b:b + 1, :, h:h + 1])
        ro, rST = oracle_mod.forward_diag(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["eta"]), sl(inp["g"]),
                                          w.eps, None)
        assert rel_err(o[b:b + 1, :, h:h + 1], ro) <= 2e-2
        assert rel_err(ST[b:b + 1, h:h + 1], rST) <= 2e-2


BWD_CASES = [
    # B, T, H, Dk, Dv, dtype, gate_lo, with_dST, beta
    (1, 45, 2, 64, 64, "f32", -0.5, True, "kaczmarz"),
    (1, 33, 1, 128, 64, "f32", -4.0, False, "kaczmarz"),
    (1, 40, 2, 64, 128, "f32", -0.5, True, "direct"),
    (1, 70, 2, 128, 128, "bf16", -0.5, True, "kaczmarz"),
    (2, 100, 2, 128, 128, "bf16", -4.0, True, "kaczmarz"),
    (1, 64, 2, 128, 128, "bf16", -0.05, False, "direct"),
    # log-decays down to -12 a token: in-chunk |G| passes 80, so the backward forms every pairwise
    # factor exactly instead of as exp(G_i) exp(-G_j)
    (1, 50, 2, 128, 128, "bf16", -12.0, True, "kaczmarz"),
    (1, 37, 1, 64, 64, "f32", -12.0, False, "kaczmarz"),
]


@pytest.mark.parametrize("B,T,H,Dk,Dv,dtype,gate_lo,with_dST,beta", BWD_CASES)
def test_bwd_diag_matches_oracle(kla, oracle_mod, B, T, H, Dk, Dv, dtype, gate_lo, with_dST, beta):
    w, inp = diag_inputs(B, T, H, Dk, Dv, dtype, seed=2 * T + H, gate_lo=gate_lo)
    if beta == "direct":
        inp["eta"] = direct_eta(inp)
    gen = torch.Generator().manual_seed(T + 17)
    dO = torch.randn(B, T, H, Dv, generator=gen).to(inp["q"].dtype)
    dST = torch.randn(B, H, Dk, Dv, generator=gen) if with_dST else None
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    gr = kla.chunk_bwd_diag(d["q"], d["k"], d["v"], d["eta"], d["g"], dO.cuda(), w.eps, d["S0"],
                            dST.cuda() if dST is not None else None, beta=beta)
    torch.cuda.synchronize()
    ref = oracle_mod.backward_diag(*(np64(inp[k]) for k in ("q", "k", "v", "eta", "g")), w.eps, np64(inp["S0"]),
                                   np64(dO), np64(dST), beta=beta)
    for name in GRADS:
        assert rel_err(gr[name], ref[name]) <= TOL[dtype], name


def test_fwd_diag_tensor_cores_zero_keys_zero_eta_and_T1(kla, oracle_mod):
    """The tensor-core forward (bf16, Dk = Dv = 128) with keys of zero norm (they write nothing),
    eta = 0 tokens, a ragged last chunk, S_T aliasing S0, and a one-token sequence."""
    w, inp = diag_inputs(2, 75, 2, 128, 128, "bf16", seed=31, gate_lo=-1.0)
    for b, t, h in ((0, 0, 0), (0, 63, 1), (1, 64, 0), (1, 74, 1), (0, 30, 0)):
        inp["k"][b, t, h] = 0
    inp["eta"][:, 5::9] = 0
    d = {k: v.cuda() for k, v in inp.items()}
    S = d["S0"].clone()
    o, _ = kla.chunk_fwd_diag(d["q"], d["k"], d["v"], d["eta"], d["g"], w.eps, S, S_T=S)
    torch.cuda.synchronize()
    kla.check_device_error()
    ro, rST = oracle_mod.forward_diag(*(np64(inp[k]) for k in ("q", "k", "v", "eta", "g")), w.eps, np64(inp["S0"]))
    assert rel_err(o, ro) <= 2e-2
    assert rel_err(S, rST) <= 2e-2
    w1, inp1 = diag_inputs(1, 1, 3, 128, 128, "bf16", seed=32)
    d1 = {k: v.cuda() for k, v in inp1.items()}
    o1, S1 = kla.chunk_fwd_diag(d1["q"], d1["k"], d1["v"], d1["eta"], d1["g"], w1.eps, d1["S0"])
    torch.cuda.synchronize()
    ro1, rS1 = oracle_mod.forward_diag(*(np64(inp1[k]) for k in ("q", "k", "v", "eta", "g")), w1.eps,
                                       np64(inp1["S0"]))
    assert rel_err(o1, ro1) <= 2e-2
    assert rel_err(S1, rS1) <= 2e-2


def test_bwd_diag_zero_norm_keys_exact(kla, oracle_mod):
    """dk at keys of zero norm is beta_t Gbar_t v_t (compared on its own scale)."""
    w, inp = diag_inputs(1, 60, 2, 128, 128, "f32", seed=23, gate_lo=-1.0)
    zk = ((0, 3, 0), (0, 20, 1), (0, 21, 1), (0, 59, 0))
    for b, t, h in zk:
        inp["k"][b, t, h] = 0
    gen = torch.Generator().manual_seed(3)
    dO = torch.randn(1, 60, 2, 128, generator=gen)
    dST = torch.randn(1, 2, 128, 128, generator=gen)
    d = {k: v.cuda() for k, v in inp.items()}
    gr = kla.chunk_bwd_diag(d["q"], d["k"], d["v"], d["eta"], d["g"], dO.cuda(), w.eps, d["S0"], dST.cuda())
    torch.cuda.synchronize()
    ref = oracle_mod.backward_diag(*(np64(inp[k]) for k in ("q", "k", "v", "eta", "g")), w.eps, np64(inp["S0"]),
                                   np64(dO), np64(dST))
    z = np.zeros((1, 60, 2), dtype=bool)
    for b, t, h in zk:
        z[b, t, h] = True
    for name in GRADS:
        if name == "dk":
            got, want = np64(gr["dk"]), np.asarray(ref["dk"])
            assert rel_err(got[~z], want[~z]) <= 1e-4
            assert np.abs(want[z]).max() > 0 and rel_err(got[z], want[z]) <= 1e-4
        else:
            assert rel_err(gr[name], ref[name]) <= 1e-4, name


def test_bwd_diag_empty_sequence(kla):
    dST = torch.randn(1, 2, 64, 64, device="cuda")
    e = torch.empty(1, 0, 2, 64, device="cuda")
    gr = kla.chunk_bwd_diag(e, e, e, torch.empty(1, 0, 2, device="cuda"), torch.empty(1, 0, 2, 64, device="cuda"),
                            e, 1e-6, None, dST)
    torch.cuda.synchronize()
    assert torch.equal(gr["dS0"], dST)


@pytest.mark.parametrize("Dk,Dv,dtype,beta", [(128, 128, "bf16", "kaczmarz"), (64, 128, "f32", "kaczmarz"),
                                              (128, 64, "bf16", "direct")])
def test_decode_diag_matches_oracle(kla, oracle_mod, Dk, Dv, dtype, beta):
    w = Workload("dec", "decode", B=3, T=12, H=5, Dk=Dk, Dv=Dv, dtype=dtype, key_mode="scaled",
                 gate_mode="diag", s0="normal", seed=Dk + Dv + 1, gate_lo=-1.0)
    inp = make_inputs(w)
    if beta == "direct":
        inp["eta"] = direct_eta(inp)
    S = inp["S0"].cuda().clone()
    Sref = np64(inp["S0"])
    for t in range(w.T):
        o = kla.decode_step_diag(inp["q"][t].cuda(), inp["k"][t].cuda(), inp["v"][t].cuda(), inp["eta"][t].cuda(),
                                 inp["g"][t].cuda(), S, w.eps, beta=beta)
        ro, Sref = oracle_mod.decode_step_diag(np64(inp["q"][t]), np64(inp["k"][t]), np64(inp["v"][t]),
                                               np64(inp["eta"][t]), np64(inp["g"][t]), w.eps, Sref, beta=beta)
        assert rel_err(o, ro) <= TOL[dtype]
    assert rel_err(S, Sref) <= TOL[dtype]


def test_decode_diag_workload_sampled_heads(kla, oracle_mod):
    """The B=64 H=16 d=128 decode shape with per-channel decays: 64 steps on the full batch,
    every output and the final state of 3 (b, h) pairs against the oracle."""
    w = WORKLOADS["decode_diag_b64_h16_d128_x1024"].with_(T=64)
    inp = make_inputs(w)
    S = inp["S0"].cuda().clone()
    pairs = [(0, 0), (63, 15), (17, 9)]
    Sref = {p: np64(inp["S0"])[p[0]:p[0] + 1, p[1]:p[1] + 1] for p in pairs}
    dev = {k: v.cuda() for k, v in inp.items()}
    for t in range(w.T):
        o = kla.decode_step_diag(dev["q"][t], dev["k"][t], dev["v"][t], dev["eta"][t], dev["g"][t], S, w.eps)
        for (b, h) in pairs:
            sl = lambda x: np.ascontiguousarray(np64(x[t])[b:b + 1, h:h + 1])
            ro, Sref[(b, h)] = oracle_mod.decode_step_diag(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["eta"]),
                                                           sl(inp["g"]), w.eps, Sref[(b, h)])
            assert rel_err(o[b:b + 1, h:h + 1], ro) <= 2e-2
    torch.cuda.synchronize()
    for (b, h) in pairs:
        assert rel_err(S[b:b + 1, h:h + 1], Sref[(b, h)]) <= 2e-2


def test_decode_diag_equals_forward_T1(kla):
    """One decode step is the forward at T = 1: to fp32 rounding against the CUDA-core forward
    (one kernel, fp32 arithmetic), and within the bf16 bar against the tensor-core split forward
    (its W and Q o Gam operands are single bf16 roundings)."""
    w, inp = diag_inputs(2, 1, 3, 128, 128, "bf16", seed=9)
    d = {k: v.cuda() for k, v in inp.items()}
    o, ST = kla.chunk_fwd_diag(d["q"], d["k"], d["v"], d["eta"], d["g"], w.eps, d["S0"], fused=True)
    ot, STt = kla.chunk_fwd_diag(d["q"], d["k"], d["v"], d["eta"], d["g"], w.eps, d["S0"])
    S = d["S0"].clone()
    od = kla.decode_step_diag(d["q"][:, 0].contiguous(), d["k"][:, 0].contiguous(), d["v"][:, 0].contiguous(),
                              d["eta"][:, 0].contiguous(), d["g"][:, 0].contiguous(), S, w.eps)
    torch.cuda.synchronize()
    assert rel_err(od, np64(o[:, 0])) <= 1e-4
    assert rel_err(S, np64(ST)) <= 1e-4
    assert rel_err(od, np64(ot[:, 0])) <= 2e-2
    assert rel_err(S, np64(STt)) <= 2e-2
