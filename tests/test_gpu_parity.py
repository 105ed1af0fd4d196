"""GPU parity: the CUDA path (through the C ABI, via the thin binding) against the fp64
oracle on identical seeded inputs.

Metric per output tensor: max|gpu - oracle| / rms(oracle).  Bars: 1e-4 for fp32 inputs,
2e-2 for bf16 inputs (state always fp32).  The oracle sees the exact dtype-rounded values
the GPU sees, upcast to fp64.  At full workload sizes the oracle runs on a sample of the
independent (batch, head) pairs; every output of those pairs is compared.
"""
import math

import numpy as np
import pytest
import torch

from gated_delta_rule_kla_b200.workloads import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


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


def heads_slice(x, pairs, state=False):
    """Select (b, h) pairs of a [B,T,H,...] (or state [B,H,...]) array into [n,T,1,...]."""
    if x is None:
        return None
    if state:
        return np.ascontiguousarray(np.stack([x[b, h] for b, h in pairs])[:, None])
    return np.ascontiguousarray(np.stack([x[b, :, h] for b, h in pairs])[:, :, None])


def run_fwd(kla, inp, eps, dev="cuda"):
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    o, ST = kla.chunk_fwd(d["q"], d["k"], d["v"], d["eta"], d["g"], eps, d["S0"])
    torch.cuda.synchronize()
    return o, ST


def small_inputs(B, T, H, Dk, Dv, dtype, seed, s0=True, g_lo=-0.5, key_mode="scaled"):
    w = Workload("small", "train", B=B, T=T, H=H, Dk=Dk, Dv=Dv, dtype=dtype, key_mode=key_mode,
                 gate_mode="uniform", s0="normal" if s0 else "zero", seed=seed)
    inp = make_inputs(w)
    if g_lo != -0.5:
        gen = torch.Generator().manual_seed(seed + 1000)
        inp["g"] = (torch.rand(B, T, H, generator=gen, dtype=torch.float64) * g_lo).float()
    return inp


# ---------------------------------------------------------------------------------------
# forward
# ---------------------------------------------------------------------------------------
FWD_CASES = [
    # B, T, H, Dk, Dv, dtype, s0, g_lo
    (1, 1, 1, 64, 64, "f32", True, -0.5),
    (1, 63, 2, 64, 64, "f32", True, -0.5),
    (2, 64, 1, 128, 128, "f32", False, -0.5),
    (1, 65, 3, 128, 64, "f32", True, -0.5),
    (2, 200, 2, 64, 128, "f32", True, -0.01),   # long memory: S0 matters to the end
    (1, 333, 2, 128, 128, "bf16", True, -0.5),
    (2, 130, 3, 128, 128, "bf16", True, -0.01),
    (1, 129, 2, 64, 64, "bf16", False, -0.5),
    (1, 100, 1, 128, 64, "bf16", True, -0.5),
    (1, 150, 2, 128, 128, "bf16", True, -2.0),   # in-chunk decay down to ~e^-64
    (1, 200, 2, 128, 128, "bf16", True, -4.0),   # beyond e^-80 inside a chunk
]


@pytest.mark.parametrize("B,T,H,Dk,Dv,dtype,s0,g_lo", FWD_CASES)
def test_fwd_small(kla, oracle_mod, B, T, H, Dk, Dv, dtype, s0, g_lo):
    inp = small_inputs(B, T, H, Dk, Dv, dtype, seed=T * 7 + H, s0=s0, g_lo=g_lo)
    eps = 1e-6
    o, ST = run_fwd(kla, inp, eps)
    ro, rST = oracle_mod.forward(*(np64(inp[k]) for k in ("q", "k", "v", "eta", "g")), eps, np64(inp["S0"]))
    assert rel_err(o, ro) <= TOL[dtype]
    assert rel_err(ST, rST) <= TOL[dtype]


def test_fwd_tiny_f32_workload(kla, oracle_mod):
    w = WORKLOADS["tiny_fwd_f32"]
    inp = make_inputs(w)
    o, ST = run_fwd(kla, inp, w.eps)
    ro, rST = oracle_mod.forward(*(np64(inp[k]) for k in ("q", "k", "v", "eta", "g")), w.eps, None)
    assert rel_err(o, ro) <= 1e-4
    assert rel_err(ST, rST) <= 1e-4


def test_fwd_prefill_b8_t2048_workload(kla, oracle_mod):
    w = WORKLOADS["prefill_b8_t2048_h8_d128"]
    inp = make_inputs(w)
    o, ST = run_fwd(kla, inp, w.eps)
    ro, rST = oracle_mod.forward(*(np64(inp[k]) for k in ("q", "k", "v", "eta", "g")), w.eps, None)
    assert rel_err(o, ro) <= 2e-2
    assert rel_err(ST, rST) <= 2e-2


def test_fwd_long_context_workload_sampled_heads(kla, oracle_mod):
    w = WORKLOADS["prefill_b1_t65536_h16_d128"]
    inp = make_inputs(w)
    o, ST = run_fwd(kla, inp, w.eps)
    pairs = [(0, 3), (0, 12)]
    args = [heads_slice(np64(inp[k]), pairs) for k in ("q", "k", "v", "eta", "g")]
    ro, rST = oracle_mod.forward(*args, w.eps, heads_slice(np64(inp["S0"]), pairs, state=True))
    go = heads_slice(np64(o), pairs)
    gST = heads_slice(np64(ST), pairs, state=True)
    assert rel_err(go, ro) <= 2e-2
    assert rel_err(gST, rST) <= 2e-2


@pytest.mark.parametrize("T,H,s0", [(4096 + 100, 2, True), (3000, 3, False)])
def test_fwd_segmented_long_sequence(kla, oracle_mod, T, H, s0):
    """Long sequences over few heads run as parallel segments chained by a scan."""
    assert kla.lib().kla_chunk_fwd_workspace(1, T, H, 128, 128, 64, 1) > 0
    inp = small_inputs(1, T, H, 128, 128, "bf16", seed=T + H, s0=s0, g_lo=-0.05)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    o, ST, Sc = kla.chunk_fwd(d["q"], d["k"], d["v"], d["eta"], d["g"], 1e-6, d["S0"], save_chunk_states=True)
    o1, ST1, Sc1 = kla.chunk_fwd(d["q"], d["k"], d["v"], d["eta"], d["g"], 1e-6, d["S0"], save_chunk_states=True,
                                 fused=True)
    torch.cuda.synchronize()
    kla.check_device_error()
    ro, rST = oracle_mod.forward(*(np64(inp[k]) for k in ("q", "k", "v", "eta", "g")), 1e-6, np64(inp["S0"]))
    assert rel_err(o, ro) <= 2e-2
    assert rel_err(ST, rST) <= 2e-2
    assert rel_err(o, np64(o1)) <= 1e-2
    assert rel_err(Sc, np64(Sc1)) <= 1e-2


@pytest.mark.parametrize("B,T,H,s0,g_lo,out_bf16", [(1, 1, 1, True, -0.5, False), (1, 64, 2, False, -0.5, False),
                                                    (2, 191, 3, True, -0.05, True), (1, 700, 1, True, -3.0, False)])
def test_fwd_split_and_fused_paths_agree(kla, oracle_mod, B, T, H, s0, g_lo, out_bf16):
    """The split path (chunk-parallel preparation + state pass, with the workspace) and the
    fused one-kernel path both match the oracle, including the per-chunk states."""
    inp = small_inputs(B, T, H, 128, 128, "bf16", seed=T + 11 * H, s0=s0, g_lo=g_lo)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    odt = torch.bfloat16 if out_bf16 else torch.float32
    outs = {}
    for fused in (False, True):
        outs[fused] = kla.chunk_fwd(d["q"], d["k"], d["v"], d["eta"], d["g"], 1e-6, d["S0"], save_chunk_states=True,
                                    out_dtype=odt, fused=fused)
    torch.cuda.synchronize()
    kla.check_device_error()
    ro, rST = oracle_mod.forward(*(np64(inp[k]) for k in ("q", "k", "v", "eta", "g")), 1e-6, np64(inp["S0"]))
    for fused, (o, ST, Sc) in outs.items():
        if out_bf16:  # a bf16 store is the fp32 result rounded once
            o32 = kla.chunk_fwd(d["q"], d["k"], d["v"], d["eta"], d["g"], 1e-6, d["S0"], fused=fused)[0]
            torch.testing.assert_close(o, o32.to(torch.bfloat16), rtol=0, atol=0)
            o = o32
        assert rel_err(o, ro) <= 2e-2, fused
        assert rel_err(ST, rST) <= 2e-2, fused
    assert rel_err(outs[False][2], np64(outs[True][2])) <= 1e-2  # chunk-start states
    if s0:
        torch.testing.assert_close(outs[False][2][:, :, 0], d["S0"])  # chunk 0 starts from S0


@pytest.mark.parametrize("B,T,H,launches", [(2, 300, 3, 2), (1, 4096 + 100, 2, 4), (8, 1024, 8, 4)])
def test_fwd_prep_and_state_stages_equal_one_call(kla, B, T, H, launches):
    """kla_chunk_fwd_prep then kla_chunk_fwd_state is kla_chunk_fwd with the same workspace,
    bit for bit.  The second shape takes the segmented state pass; the third runs kla_chunk_fwd
    as two slabs (the first slab's state pass concurrent with the second slab's preparation),
    against one state-pass run over the whole sequence here."""
    inp = small_inputs(B, T, H, 128, 128, "bf16", seed=T + H, g_lo=-0.05)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    assert kla.fwd_kernel_launches(d["k"], d["v"]) == launches
    ws = kla.fwd_workspace(d["k"], d["v"])
    o, ST, Sc = kla.chunk_fwd(d["q"], d["k"], d["v"], d["eta"], d["g"], 1e-6, d["S0"], save_chunk_states=True,
                              workspace=ws)
    ws2 = kla.fwd_workspace(d["k"], d["v"])
    Sc2 = torch.empty_like(Sc)
    kla.chunk_fwd_prep(d["q"], d["k"], d["v"], d["eta"], d["g"], 1e-6, ws2)
    o2, ST2 = kla.chunk_fwd_state(d["q"], d["v"], d["g"], d["S0"], ws2, S_chunks=Sc2)
    torch.cuda.synchronize()
    kla.check_device_error()
    assert torch.equal(o, o2) and torch.equal(ST, ST2) and torch.equal(Sc, Sc2)
    # the state pass's parts one by one (transition pass, segment scan, output pass)
    nseg = kla.fwd_state_segments(d["k"], d["v"])
    assert (nseg > 1) == (launches == 4 and B * H < 16)
    ws3 = kla.fwd_workspace(d["k"], d["v"])
    o3, ST3, Sc3 = torch.zeros_like(o), torch.zeros_like(ST), torch.zeros_like(Sc)
    kla.chunk_fwd_prep(d["q"], d["k"], d["v"], d["eta"], d["g"], 1e-6, ws3)
    for stage in (1, 2):
        kla.chunk_fwd_state(d["q"], d["v"], d["g"], d["S0"], ws3, o=o3, S_T=ST3, S_chunks=Sc3, stage=stage)
    torch.cuda.synchronize()
    if nseg == 1:  # nothing launched yet
        assert not o3.any() and not ST3.any() and not Sc3.any()
    kla.chunk_fwd_state(d["q"], d["v"], d["g"], d["S0"], ws3, o=o3, S_T=ST3, S_chunks=Sc3, stage=3)
    torch.cuda.synchronize()
    kla.check_device_error()
    assert torch.equal(o, o3) and torch.equal(ST, ST3) and torch.equal(Sc, Sc3)


def test_fwd_split_more_heads_than_sms(kla, oracle_mod):
    """B*H = 200 heads: the state pass needs two waves of CTAs; sampled heads vs the oracle."""
    inp = small_inputs(2, 150, 100, 128, 128, "bf16", seed=77, g_lo=-0.2)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    o, ST = kla.chunk_fwd(d["q"], d["k"], d["v"], d["eta"], d["g"], 1e-6, d["S0"])
    torch.cuda.synchronize()
    kla.check_device_error()
    pairs = [(0, 0), (0, 99), (1, 37), (1, 99)]
    args = [heads_slice(np64(inp[k]), pairs) for k in ("q", "k", "v", "eta", "g")]
    ro, rST = oracle_mod.forward(*args, 1e-6, heads_slice(np64(inp["S0"]), pairs, state=True))
    assert rel_err(heads_slice(np64(o), pairs), ro) <= 2e-2
    assert rel_err(heads_slice(np64(ST), pairs, state=True), rST) <= 2e-2


def test_fwd_split_zero_norm_key_and_zero_eta(kla, oracle_mod):
    """Split path edge cases: a key of zero norm with eps = 0 skips its write, eta = 0 only
    decays, and a chunk of only masked-out writes leaves the state decayed."""
    inp = small_inputs(1, 200, 2, 128, 128, "bf16", seed=13, g_lo=-0.1)
    inp["k"][0, 3] = 0.0
    inp["k"][0, 100, 1] = 0.0
    inp["eta"][0, 64:128] = 0.0
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    o, ST = kla.chunk_fwd(d["q"], d["k"], d["v"], d["eta"], d["g"], 0.0, d["S0"])
    torch.cuda.synchronize()
    kla.check_device_error()
    ro, rST = oracle_mod.forward(*(np64(inp[k]) for k in ("q", "k", "v", "eta", "g")), 0.0, np64(inp["S0"]))
    assert rel_err(o, ro) <= 2e-2
    assert rel_err(ST, rST) <= 2e-2


def test_fwd_segmented_in_place_state_and_bf16_out(kla, oracle_mod):
    """Segmented state pass with S_T written over S0 and a bf16 readout."""
    T, H = 4096 + 37, 2
    inp = small_inputs(1, T, H, 128, 128, "bf16", seed=19, g_lo=-0.05)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    S = d["S0"].clone()
    o16, S_out = kla.chunk_fwd(d["q"], d["k"], d["v"], d["eta"], d["g"], 1e-6, S, S_T=S, out_dtype=torch.bfloat16)
    o32, ST32 = kla.chunk_fwd(d["q"], d["k"], d["v"], d["eta"], d["g"], 1e-6, d["S0"])
    torch.cuda.synchronize()
    kla.check_device_error()
    assert S_out.data_ptr() == S.data_ptr()
    torch.testing.assert_close(o16, o32.to(torch.bfloat16), rtol=0, atol=0)
    torch.testing.assert_close(S, ST32, rtol=0, atol=0)
    ro, rST = oracle_mod.forward(*(np64(inp[k]) for k in ("q", "k", "v", "eta", "g")), 1e-6, np64(inp["S0"]))
    assert rel_err(o32, ro) <= 2e-2
    assert rel_err(S, rST) <= 2e-2


def test_fwd_state_passing_equals_one_call(kla):
    """Checkpoint/resume: forward(T1) then forward(T2, S0=S_T1) == forward(T1+T2)."""
    inp = small_inputs(2, 320, 2, 128, 128, "f32", seed=5, g_lo=-0.05)
    eps = 1e-6
    o, ST = run_fwd(kla, inp, eps)
    cut = 192
    a = {k: (v[:, :cut].contiguous() if v is not None and k != "S0" else v) for k, v in inp.items()}
    b_ = {k: (v[:, cut:].contiguous() if v is not None and k != "S0" else v) for k, v in inp.items()}
    o1, S1 = run_fwd(kla, a, eps)
    b_["S0"] = S1.cpu()
    o2, S2 = run_fwd(kla, b_, eps)
    torch.testing.assert_close(torch.cat([o1, o2], 1), o, rtol=1e-4, atol=1e-4 * o.float().pow(2).mean().sqrt().item())
    torch.testing.assert_close(S2, ST, rtol=1e-4, atol=1e-5)


def test_fwd_zero_key_and_zero_eta(kla, oracle_mod):
    """Edge cases: a key of zero norm with eps=0 skips the write; eta=0 only decays."""
    inp = small_inputs(1, 70, 2, 64, 64, "f32", seed=11)
    inp["k"][0, 5] = 0.0
    inp["k"][0, 66, 1] = 0.0
    inp["eta"][0, 10:20] = 0.0
    o, ST = run_fwd(kla, inp, 0.0)
    ro, rST = oracle_mod.forward(*(np64(inp[k]) for k in ("q", "k", "v", "eta", "g")), 0.0, np64(inp["S0"]))
    assert rel_err(o, ro) <= 1e-4
    assert rel_err(ST, rST) <= 1e-4


def test_fwd_empty_sequence(kla):
    S0 = torch.randn(2, 3, 64, 64, device="cuda")
    z = torch.zeros(2, 0, 3, 64, device="cuda")
    gz = torch.zeros(2, 0, 3, device="cuda")
    o, ST = kla.chunk_fwd(z, z, z, gz, gz, 1e-6, S0)
    torch.cuda.synchronize()
    assert o.shape == (2, 0, 3, 64)
    torch.testing.assert_close(ST, S0, rtol=0, atol=0)
    _, ST0 = kla.chunk_fwd(z, z, z, gz, gz, 1e-6, None)
    torch.cuda.synchronize()
    assert torch.count_nonzero(ST0) == 0


def test_fwd_state_out_may_alias_initial_state(kla):
    inp = small_inputs(1, 100, 2, 64, 64, "f32", seed=3)
    d = {k: v.cuda() for k, v in inp.items()}
    o_ref, S_ref = kla.chunk_fwd(d["q"], d["k"], d["v"], d["eta"], d["g"], 1e-6, d["S0"])
    S = d["S0"].clone()
    o, _ = kla.chunk_fwd(d["q"], d["k"], d["v"], d["eta"], d["g"], 1e-6, S, S_T=S)
    torch.cuda.synchronize()
    torch.testing.assert_close(o, o_ref, rtol=0, atol=0)
    torch.testing.assert_close(S, S_ref, rtol=0, atol=0)


# ---------------------------------------------------------------------------------------
# decode
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("Dk,Dv,dtype", [(128, 128, "bf16"), (64, 128, "f32"), (128, 64, "f32"), (64, 64, "bf16")])
def test_decode_small(kla, oracle_mod, Dk, Dv, dtype):
    w = Workload("dec", "decode", B=3, T=20, H=5, Dk=Dk, Dv=Dv, dtype=dtype, key_mode="scaled",
                 gate_mode="uniform", s0="normal", seed=Dk + Dv)
    inp = make_inputs(w)
    S = inp["S0"].cuda().clone()
    Sref = np64(inp["S0"])
    for t in range(w.T):
        o = kla.decode_step(inp["q"][t].cuda(), inp["k"][t].cuda(), inp["v"][t].cuda(),
                            inp["eta"][t].cuda(), inp["g"][t].cuda(), S, w.eps)
        ro, Sref = oracle_mod.decode_step(np64(inp["q"][t]), np64(inp["k"][t]), np64(inp["v"][t]),
                                          np64(inp["eta"][t]), np64(inp["g"][t]), w.eps, Sref)
        assert rel_err(o, ro) <= TOL[dtype]
    assert rel_err(S, Sref) <= TOL[dtype]


def test_decode_workload_1024_steps_sampled_heads(kla, oracle_mod):
    w = WORKLOADS["decode_b64_h16_d128_x1024"]
    inp = make_inputs(w)
    pairs = [(0, 0), (17, 5), (63, 15)]
    S = inp["S0"].cuda().clone()
    qd, kd, vd = inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda()
    ed, gd = inp["eta"].cuda(), inp["g"].cuda()
    outs = torch.empty(w.T, w.B, w.H, w.Dv, dtype=torch.float32, device="cuda")
    for t in range(w.T):
        kla.decode_step(qd[t], kd[t], vd[t], ed[t], gd[t], S, w.eps, o=outs[t])
    torch.cuda.synchronize()
    sel = lambda x: np.ascontiguousarray(np.stack([x[:, b, h] for b, h in pairs], axis=1)[:, :, None])
    q, k, v, eta, g = (sel(np64(inp[n])) for n in ("q", "k", "v", "eta", "g"))
    Sref = np.stack([np64(inp["S0"])[b, h] for b, h in pairs])[:, None]
    got = sel(np64(outs))
    ref = np.empty_like(got)
    for t in range(w.T):
        ref[t], Sref = oracle_mod.decode_step(q[t], k[t], v[t], eta[t], g[t], w.eps, Sref)
    assert rel_err(got, ref) <= 2e-2
    gS = np.stack([np64(S)[b, h] for b, h in pairs])[:, None]
    assert rel_err(gS, Sref) <= 2e-2


@pytest.mark.parametrize("dtype,tol", [("f32", 1e-5), ("bf16", 2e-2)])
def test_decode_equals_forward_T1(kla, dtype, tol):
    inp = small_inputs(2, 1, 3, 128, 128, dtype, seed=21)
    d = {k: v.cuda() for k, v in inp.items()}
    o, ST = kla.chunk_fwd(d["q"], d["k"], d["v"], d["eta"], d["g"], 1e-6, d["S0"])
    S = d["S0"].clone()
    c = lambda x: x[:, 0].contiguous()
    od = kla.decode_step(c(d["q"]), c(d["k"]), c(d["v"]), c(d["eta"]), c(d["g"]), S, 1e-6)
    torch.cuda.synchronize()
    assert rel_err(od, np64(o[:, 0])) <= tol
    assert rel_err(S, np64(ST)) <= tol


# ---------------------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------------------
GRADS = ("dq", "dk", "dv", "deta", "dg", "dS0")

BWD_CASES = [
    # B, T, H, Dk, Dv, dtype, s0, with dS_T
    (1, 64, 1, 64, 64, "f32", True, True),
    (1, 150, 2, 64, 64, "f32", True, False),
    (2, 97, 2, 128, 128, "f32", True, True),
    (1, 70, 1, 128, 64, "f32", False, True),
    (1, 130, 2, 64, 128, "f32", True, True),
    (2, 200, 2, 128, 128, "bf16", True, True),
    (1, 65, 3, 128, 128, "bf16", False, False),
]


@pytest.mark.parametrize("B,T,H,Dk,Dv,dtype,s0,with_dST", BWD_CASES)
def test_bwd_small(kla, oracle_mod, B, T, H, Dk, Dv, dtype, s0, with_dST):
    inp = small_inputs(B, T, H, Dk, Dv, dtype, seed=T + 3 * H, s0=s0, g_lo=-0.2)
    gen = torch.Generator().manual_seed(T)
    dO = torch.randn(B, T, H, Dv, generator=gen).to(inp["q"].dtype)
    dST = torch.randn(B, H, Dk, Dv, generator=gen) if with_dST else None
    eps = 1e-6
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    gr = kla.chunk_bwd(d["q"], d["k"], d["v"], d["eta"], d["g"], dO.cuda(), eps, d["S0"],
                       dST.cuda() if dST is not None else None)
    torch.cuda.synchronize()
    ref = oracle_mod.backward(*(np64(inp[k]) for k in ("q", "k", "v", "eta", "g")), eps, np64(inp["S0"]),
                              np64(dO), np64(dST))
    for name in GRADS:
        assert rel_err(gr[name], ref[name]) <= TOL[dtype], name


BWD_TC_CASES = [
    # B, T, H, s0, g_lo, with dS_T
    (1, 64, 1, True, -0.5, True),
    (2, 130, 3, True, -0.01, True),   # long memory: the state gradient crosses every chunk
    (1, 333, 2, False, -0.5, False),
    (1, 150, 2, True, -2.0, True),    # in-chunk decay down to ~e^-64
    (1, 200, 2, True, -4.0, False),   # beyond e^-80 inside a chunk
]


@pytest.mark.parametrize("B,T,H,s0,g_lo,with_dST", BWD_TC_CASES)
def test_bwd_tensor_core_and_cuda_core_paths_match_oracle(kla, oracle_mod, B, T, H, s0, g_lo, with_dST):
    """bf16, d = 128: the tensor-core backward (default workspace) and the CUDA-core backward
    (minimum workspace) both against the fp64 oracle."""
    inp = small_inputs(B, T, H, 128, 128, "bf16", seed=T + 7 * H, s0=s0, g_lo=g_lo)
    gen = torch.Generator().manual_seed(T + 1)
    dO = torch.randn(B, T, H, 128, generator=gen).to(torch.bfloat16)
    dST = torch.randn(B, H, 128, 128, generator=gen) if with_dST else None
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    args = (d["q"], d["k"], d["v"], d["eta"], d["g"], dO.cuda(), 1e-6, d["S0"],
            dST.cuda() if dST is not None else None)
    g_tc = kla.chunk_bwd(*args)
    g_cc = kla.chunk_bwd(*args, cuda_cores=True)
    torch.cuda.synchronize()
    kla.check_device_error()
    ref = oracle_mod.backward(*(np64(inp[k]) for k in ("q", "k", "v", "eta", "g")), 1e-6, np64(inp["S0"]),
                              np64(dO), np64(dST))
    for name in GRADS:
        assert rel_err(g_tc[name], ref[name]) <= 2e-2, ("tensor cores", name)
        assert rel_err(g_cc[name], ref[name]) <= 2e-2, ("cuda cores", name)


# (b, t, h) of the keys set to zero: one alone in its chunk, two in one chunk, and the last
# token of the sequence (inside a partial chunk)
ZERO_KEYS = ((0, 5, 0), (0, 70, 1), (0, 71, 1), (0, 139, 0))


@pytest.mark.parametrize("Dk,Dv,dtype,beta,eps,cuda_cores", [
    (128, 128, "bf16", "kaczmarz", 1e-6, False),  # tensor cores
    (128, 128, "bf16", "kaczmarz", 1e-6, True),   # CUDA cores
    (128, 128, "bf16", "direct", 1e-6, False),
    (128, 128, "bf16", "direct", 1e-6, True),
    (128, 128, "bf16", "kaczmarz", 0.0, False),   # ||k||^2 + eps == 0: no write, dk = 0
    (64, 64, "f32", "kaczmarz", 1e-6, False),
    (64, 128, "f32", "direct", 1e-6, False),
])
def test_bwd_zero_norm_keys_exact(kla, oracle_mod, Dk, Dv, dtype, beta, eps, cuda_cores):
    """At a key of zero norm the write vanishes and the exact gradient is
    dk_t = beta_t Gbar_t v_t (beta_t = eta_t / eps, or eta_t in the direct mode).  Those rows
    are compared on their own scale (with eps = 1e-6 they are ~1e6 times the others), the rest
    of every gradient as usual, all against the unmodified oracle."""
    inp = small_inputs(1, 140, 2, Dk, Dv, dtype, seed=41)
    for b, t, h in ZERO_KEYS:
        inp["k"][b, t, h] = 0
    inp["eta"][0, 9, :] = 0
    inp["eta"][0, 100, 0] = 0
    if beta == "direct":
        inp["eta"] = direct_eta(inp)
    gen = torch.Generator().manual_seed(5)
    dO = torch.randn(1, 140, 2, Dv, generator=gen).to(inp["q"].dtype)
    dST = torch.randn(1, 2, Dk, Dv, generator=gen)
    d = {k: v.cuda() for k, v in inp.items()}
    gr = kla.chunk_bwd(d["q"], d["k"], d["v"], d["eta"], d["g"], dO.cuda(), eps, d["S0"], dST.cuda(),
                       cuda_cores=cuda_cores, beta=beta)
    torch.cuda.synchronize()
    kla.check_device_error()
    ref = oracle_mod.backward(*(np64(inp[k]) for k in ("q", "k", "v", "eta", "g")), eps, np64(inp["S0"]),
                              np64(dO), np64(dST), beta=beta)
    tol = TOL[dtype]
    zmask = np.zeros((1, 140, 2), dtype=bool)
    for b, t, h in ZERO_KEYS:
        zmask[b, t, h] = True
    for name in GRADS:
        if name != "dk":
            assert rel_err(gr[name], ref[name]) <= tol, name
            continue
        got, want = np64(gr["dk"]), np.asarray(ref["dk"])
        assert rel_err(got[~zmask], want[~zmask]) <= tol, "dk, nonzero keys"
        if beta == "kaczmarz" and eps == 0.0:
            assert np.all(want[zmask] == 0) and np.all(got[zmask] == 0)
        else:
            assert np.abs(want[zmask]).max() > 0
            assert rel_err(got[zmask], want[zmask]) <= tol, "dk, zero-norm keys"


@pytest.mark.parametrize("T,H,s0,with_dST", [(4100, 2, True, True), (3000, 3, False, False)])
def test_bwd_segmented_reverse_pass(kla, oracle_mod, T, H, s0, with_dST):
    """Long sequences over few heads run the reverse state pass in segments: each segment's map
    of the state gradient (from lambda = I without dO) and offset (from lambda = 0 with dO) in
    parallel, a scan newest segment first, then each segment from its true end gradient.  Every
    gradient against the oracle (a ragged tail chunk in the first shape)."""
    nseg = kla.lib().kla_chunk_bwd_reverse_segments(1, T, H, 128, 128, 64, 1)
    assert nseg > 1
    inp = small_inputs(1, T, H, 128, 128, "bf16", seed=T + H, s0=s0, g_lo=-0.05)
    gen = torch.Generator().manual_seed(T)
    dO = torch.randn(1, T, H, 128, generator=gen).to(torch.bfloat16)
    dST = torch.randn(1, H, 128, 128, generator=gen) if with_dST else None
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    gr = kla.chunk_bwd(d["q"], d["k"], d["v"], d["eta"], d["g"], dO.cuda(), 1e-6, d["S0"],
                       dST.cuda() if dST is not None else None)
    torch.cuda.synchronize()
    kla.check_device_error()
    ref = oracle_mod.backward(*(np64(inp[k]) for k in ("q", "k", "v", "eta", "g")), 1e-6, np64(inp["S0"]),
                              np64(dO), np64(dST))
    for name in GRADS:
        assert rel_err(gr[name], ref[name]) <= 2e-2, name


def test_bwd_tensor_cores_more_heads_than_sms(kla, oracle_mod):
    B, T, H = 10, 70, 16  # 160 reverse-pass CTAs: more than one wave
    inp = small_inputs(B, T, H, 128, 128, "bf16", seed=77)
    dO = torch.randn(B, T, H, 128, generator=torch.Generator().manual_seed(6)).to(torch.bfloat16)
    d = {k: v.cuda() for k, v in inp.items()}
    gr = kla.chunk_bwd(d["q"], d["k"], d["v"], d["eta"], d["g"], dO.cuda(), 1e-6, d["S0"])
    torch.cuda.synchronize()
    pairs = [(0, 0), (9, 15), (4, 7)]
    args = [heads_slice(np64(inp[k]), pairs) for k in ("q", "k", "v", "eta", "g")]
    ref = oracle_mod.backward(*args, 1e-6, heads_slice(np64(inp["S0"]), pairs, state=True),
                              heads_slice(np64(dO), pairs), None)
    for name in GRADS:
        got = heads_slice(np64(gr[name]), pairs, state=(name == "dS0"))
        assert rel_err(got, ref[name]) <= 2e-2, name


@pytest.mark.parametrize("B,T,H,D,dtype,small_ws", [
    (2, 150, 3, 128, "bf16", False),   # tensor-core layout: records and tiles shared
    (2, 150, 3, 128, "bf16", True),    # minimum workspace: chunk states shared, CUDA-core backward
    (1, 130, 2, 64, "f32", False),
])
def test_train_pair_equals_separate_calls(kla, B, T, H, D, dtype, small_ws):
    """chunk_fwd_train + chunk_bwd_after_train give what chunk_fwd and chunk_bwd give."""
    inp = small_inputs(B, T, H, D, D, dtype, seed=T + H, g_lo=-0.1)
    d = {k: v.cuda() for k, v in inp.items()}
    gen = torch.Generator().manual_seed(3)
    dO = torch.randn(B, T, H, D, generator=gen).to(d["q"].dtype).cuda()
    dST = torch.randn(B, H, D, D, generator=gen).cuda()
    L = kla.lib()
    size = L.kla_chunk_bwd_workspace_min if small_ws else L.kla_chunk_bwd_workspace
    ws = torch.empty(size(B, T, H, D, D, 64, 1 if dtype == "bf16" else 0, 0), dtype=torch.uint8, device="cuda")
    o1, S1, _ = kla.chunk_fwd_train(d["q"], d["k"], d["v"], d["eta"], d["g"], 1e-6, d["S0"], workspace=ws)
    g1 = kla.chunk_bwd_after_train(d["q"], d["k"], d["v"], d["eta"], d["g"], dO, ws, 1e-6, dST)
    # the minimum workspace runs the one-kernel forward, as chunk_fwd does without a workspace
    o2, S2 = kla.chunk_fwd(d["q"], d["k"], d["v"], d["eta"], d["g"], 1e-6, d["S0"], fused=small_ws)
    g2 = kla.chunk_bwd(d["q"], d["k"], d["v"], d["eta"], d["g"], dO, 1e-6, d["S0"], dST, cuda_cores=small_ws)
    torch.cuda.synchronize()
    kla.check_device_error()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    for name in GRADS:
        if dtype == "bf16" and not small_ws:
            assert torch.equal(g1[name], g2[name]), name  # same kernels on the same tiles
        else:  # fp32 atomics may add in another order
            a, b = g1[name].double(), g2[name].double()
            assert (a - b).abs().max().item() <= 1e-5 * (b.pow(2).mean().sqrt().item() + 1e-30), name


def test_bwd_with_saved_chunk_states_matches_recompute(kla):
    inp = small_inputs(1, 190, 2, 128, 128, "bf16", seed=8)
    d = {k: v.cuda() for k, v in inp.items()}
    dO = torch.randn(1, 190, 2, 128, device="cuda").to(torch.bfloat16)
    _, _, Sc = kla.chunk_fwd(d["q"], d["k"], d["v"], d["eta"], d["g"], 1e-6, d["S0"], save_chunk_states=True)
    g1 = kla.chunk_bwd(d["q"], d["k"], d["v"], d["eta"], d["g"], dO, 1e-6, d["S0"], None, Sc)
    g2 = kla.chunk_bwd(d["q"], d["k"], d["v"], d["eta"], d["g"], dO, 1e-6, d["S0"], None, None)
    torch.cuda.synchronize()
    for name in GRADS:
        a, b = g1[name].float(), g2[name].float()
        scale = b.pow(2).mean().sqrt().item() + 1e-30
        assert (a - b).abs().max().item() / scale <= 2e-2, name


def test_bwd_training_workload_sampled_heads(kla, oracle_mod):
    w = WORKLOADS["train_b4_t4096_h16_d128"]
    inp = make_inputs(w)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    dO = d["dO"].to(d["q"].dtype)
    gr = kla.chunk_bwd(d["q"], d["k"], d["v"], d["eta"], d["g"], dO, w.eps, d["S0"])
    torch.cuda.synchronize()
    pairs = [(0, 0), (3, 9)]
    args = [heads_slice(np64(inp[k]), pairs) for k in ("q", "k", "v", "eta", "g")]
    ref = oracle_mod.backward(*args, w.eps, None, heads_slice(np64(dO), pairs), None)
    for name in GRADS:
        got = heads_slice(np64(gr[name]), pairs, state=(name == "dS0"))
        assert rel_err(got, ref[name]) <= 2e-2, name


def test_bwd_two_slab_reverse_pass_sampled_heads(kla, oracle_mod):
    """B=4 T=2048 H=16 (32 chunks per head): the reverse pass runs the newest chunks as a slab of
    its own while the gradient kernel takes them on the other SMs, then goes on over the older
    chunks from the state gradient it left.  Long memory (g >= -0.05), an initial state and a
    dS_T, so that the gradient crosses the slab boundary; sampled heads against the oracle."""
    B, T, H = 4, 2048, 16
    assert kla.lib().kla_chunk_bwd_reverse_slab_chunks(B, T, H, 128, 128, 64, 1) > 0
    inp = small_inputs(B, T, H, 128, 128, "bf16", seed=91, g_lo=-0.05)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    gen = torch.Generator().manual_seed(92)
    dO = torch.randn(B, T, H, 128, generator=gen).to(torch.bfloat16)
    dST = torch.randn(B, H, 128, 128, generator=gen) * 0.1
    gr = kla.chunk_bwd(d["q"], d["k"], d["v"], d["eta"], d["g"], dO.cuda(), 1e-6, d["S0"], dST.cuda())
    torch.cuda.synchronize()
    kla.check_device_error()
    pairs = [(0, 1), (3, 14)]
    args = [heads_slice(np64(inp[k]), pairs) for k in ("q", "k", "v", "eta", "g")]
    ref = oracle_mod.backward(*args, 1e-6, heads_slice(np64(inp["S0"]), pairs, state=True),
                              heads_slice(np64(dO), pairs), heads_slice(np64(dST), pairs, state=True))
    for name in GRADS:
        got = heads_slice(np64(gr[name]), pairs, state=(name == "dS0"))
        assert rel_err(got, ref[name]) <= 2e-2, name


def test_bwd_long_context_sampled_heads(kla, oracle_mod):
    """The tensor-core backward at the long-context shape (B=1, T=65536, H=16: 1024 chunks per
    head through the reverse pass, the segmented forward recomputed inside), sampled heads
    against the fp64 oracle."""
    w = WORKLOADS["prefill_b1_t65536_h16_d128"]
    inp = make_inputs(w)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    dO = torch.randn(w.B, w.T, w.H, w.Dv, generator=torch.Generator().manual_seed(65)).to(torch.bfloat16)
    gr = kla.chunk_bwd(d["q"], d["k"], d["v"], d["eta"], d["g"], dO.cuda(), w.eps, d["S0"])
    torch.cuda.synchronize()
    kla.check_device_error()
    pairs = [(0, 5)]
    args = [heads_slice(np64(inp[k]), pairs) for k in ("q", "k", "v", "eta", "g")]
    ref = oracle_mod.backward(*args, w.eps, heads_slice(np64(inp["S0"]), pairs, state=True),
                              heads_slice(np64(dO), pairs), None)
    for name in GRADS:
        got = heads_slice(np64(gr[name]), pairs, state=(name == "dS0"))
        assert rel_err(got, ref[name]) <= 2e-2, name


def test_bf16_outputs_are_rounded_fp32_outputs(kla):
    """out_dtype=bf16 stores round the same fp32 results once (forward, decode, backward)."""
    for Dk in (128, 64):
        inp = small_inputs(2, 150, 2, Dk, Dk, "bf16", seed=Dk)
        d = {k: v.cuda() for k, v in inp.items()}
        o32, _ = kla.chunk_fwd(d["q"], d["k"], d["v"], d["eta"], d["g"], 1e-6, d["S0"])
        o16, _ = kla.chunk_fwd(d["q"], d["k"], d["v"], d["eta"], d["g"], 1e-6, d["S0"], out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        assert o16.dtype == torch.bfloat16
        assert torch.equal(o16, o32.to(torch.bfloat16))
        S1, S2 = d["S0"].clone(), d["S0"].clone()
        c = lambda x: x[:, 0].contiguous()
        a32 = kla.decode_step(c(d["q"]), c(d["k"]), c(d["v"]), c(d["eta"]), c(d["g"]), S1, 1e-6)
        a16 = kla.decode_step(c(d["q"]), c(d["k"]), c(d["v"]), c(d["eta"]), c(d["g"]), S2, 1e-6,
                              out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        assert torch.equal(a16, a32.to(torch.bfloat16))
        dO = torch.randn(2, 150, 2, Dk, device="cuda").to(torch.bfloat16)
        g32 = kla.chunk_bwd(d["q"], d["k"], d["v"], d["eta"], d["g"], dO, 1e-6, d["S0"])
        g16 = kla.chunk_bwd(d["q"], d["k"], d["v"], d["eta"], d["g"], dO, 1e-6, d["S0"], out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        for n in ("dq", "dk", "dv"):
            # fp32 atomics may sum in a different order between the two calls: allow one bf16 ulp
            ref = g32[n].to(torch.bfloat16).float()
            assert torch.all((g16[n].float() - ref).abs() <= ref.abs() * 2.0 ** -7 + 1e-30), n


def test_no_device_timeouts_recorded(kla):
    inp = small_inputs(1, 300, 2, 128, 128, "bf16", seed=99)
    d = {k: v.cuda() for k, v in inp.items()}
    kla.chunk_fwd(d["q"], d["k"], d["v"], d["eta"], d["g"], 1e-6, d["S0"])
    kla.check_device_error()


def test_expired_device_wait_is_reported_and_context_survives(kla, oracle_mod):
    """Failure detection without a fault: the injected decode launch waits on a barrier that
    nothing completes; the bounded wait gives up after ~20 ms, the kernel stores nothing and
    records the expiry, and kla_check_device_error reports KLA_ERR_TIMEOUT.  The next call on
    the same context runs normally."""
    w = Workload("dec", "decode", B=4, T=2, H=8, Dk=128, Dv=128, dtype="bf16", key_mode="scaled",
                 gate_mode="uniform", s0="normal", seed=17)
    inp = make_inputs(w)
    d = {k: v.cuda() for k, v in inp.items()}
    S = d["S0"].clone()
    kla.check_device_error()  # start clean
    kla.debug_inject_wait_timeout()
    kla.decode_step(d["q"][0], d["k"][0], d["v"][0], d["eta"][0], d["g"][0], S, w.eps)
    with pytest.raises(kla.KLAError) as err:
        kla.check_device_error()
    assert err.value.status == 5  # KLA_ERR_TIMEOUT
    assert torch.equal(S, d["S0"])  # the aborted step stored nothing
    kla.check_device_error()  # the error word was cleared by the check
    o = kla.decode_step(d["q"][0], d["k"][0], d["v"][0], d["eta"][0], d["g"][0], S, w.eps)
    kla.check_device_error()
    ro, rS = oracle_mod.decode_step(np64(inp["q"][0]), np64(inp["k"][0]), np64(inp["v"][0]), np64(inp["eta"][0]),
                                    np64(inp["g"][0]), w.eps, np64(inp["S0"]))
    assert rel_err(o, ro) <= 2e-2
    assert rel_err(S, rS) <= 2e-2


def test_bwd_empty_sequence(kla):
    dST = torch.randn(1, 2, 64, 64, device="cuda")
    z = torch.zeros(1, 0, 2, 64, device="cuda")
    gz = torch.zeros(1, 0, 2, device="cuda")
    gr = kla.chunk_bwd(z, z, z, gz, gz, z, 1e-6, None, dST)
    torch.cuda.synchronize()
    torch.testing.assert_close(gr["dS0"], dST, rtol=0, atol=0)


# ---------------------------------------------------------------------------------------
# direct write strength: beta_t = eta_t as given (the Gated DeltaNet update), selected by
# KLA_BETA_DIRECT in the dtype argument (beta="direct" in the binding)
# ---------------------------------------------------------------------------------------
def direct_eta(inp):
    """A direct write strength that keeps every write a contraction for these keys:
    beta_t = eta_t / (||k_t||^2 + 1), computed on the CPU from the rounded keys."""
    k = inp["k"].double()
    return (inp["eta"].double() / ((k * k).sum(-1) + 1.0)).float()


@pytest.mark.parametrize("B,T,H,Dk,Dv,dtype,fused", [
    (1, 150, 2, 128, 128, "bf16", False),   # split path (preparation + state pass)
    (2, 130, 3, 128, 128, "bf16", True),    # fused one-kernel-per-head path
    (8, 1024, 8, 128, 128, "bf16", False),  # two slabs
    (1, 100, 2, 64, 128, "f32", False),     # CUDA-core path
])
def test_fwd_direct_beta_matches_oracle(kla, oracle_mod, B, T, H, Dk, Dv, dtype, fused):
    inp = small_inputs(B, T, H, Dk, Dv, dtype, seed=T + 5 * H, g_lo=-0.2)
    inp["eta"] = direct_eta(inp)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    o, ST = kla.chunk_fwd(d["q"], d["k"], d["v"], d["eta"], d["g"], 1e-6, d["S0"], fused=fused, beta="direct")
    torch.cuda.synchronize()
    kla.check_device_error()
    ro, rST = oracle_mod.forward(*(np64(inp[k]) for k in ("q", "k", "v", "eta", "g")), 1e-6, np64(inp["S0"]),
                                 beta="direct")
    assert rel_err(o, ro) <= TOL[dtype]
    assert rel_err(ST, rST) <= TOL[dtype]


def test_direct_beta_with_kaczmarz_eta_equals_kaczmarz(kla):
    """beta="direct" fed eta / (||k||^2 + eps) is the Kaczmarz forward (split path, bf16)."""
    inp = small_inputs(2, 300, 3, 128, 128, "bf16", seed=77)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    eps = 1e-3
    kk = d["k"].float()
    eta_d = (d["eta"] / ((kk * kk).sum(-1) + eps)).contiguous()
    o1, S1 = kla.chunk_fwd(d["q"], d["k"], d["v"], d["eta"], d["g"], eps, d["S0"])
    o2, S2 = kla.chunk_fwd(d["q"], d["k"], d["v"], eta_d, d["g"], eps, d["S0"], beta="direct")
    torch.cuda.synchronize()
    assert rel_err(o2, np64(o1)) <= 1e-3
    assert rel_err(S2, np64(S1)) <= 1e-3


@pytest.mark.parametrize("B,T,H,Dk,Dv,dtype", [(1, 150, 2, 128, 128, "bf16"), (1, 97, 2, 64, 64, "f32")])
def test_bwd_direct_beta_matches_oracle(kla, oracle_mod, B, T, H, Dk, Dv, dtype):
    """Both backward paths (tensor cores with the default workspace for bf16 d = 128, CUDA
    cores otherwise or with the minimum workspace) in the direct mode."""
    inp = small_inputs(B, T, H, Dk, Dv, dtype, seed=T + 9 * H, g_lo=-0.2)
    inp["eta"] = direct_eta(inp)
    gen = torch.Generator().manual_seed(T + 2)
    dO = torch.randn(B, T, H, Dv, generator=gen).to(inp["q"].dtype)
    dST = torch.randn(B, H, Dk, Dv, generator=gen)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    args = (d["q"], d["k"], d["v"], d["eta"], d["g"], dO.cuda(), 1e-6, d["S0"], dST.cuda())
    runs = {"default": kla.chunk_bwd(*args, beta="direct"),
            "cuda cores": kla.chunk_bwd(*args, cuda_cores=True, beta="direct")}
    torch.cuda.synchronize()
    kla.check_device_error()
    ref = oracle_mod.backward(*(np64(inp[k]) for k in ("q", "k", "v", "eta", "g")), 1e-6, np64(inp["S0"]),
                              np64(dO), np64(dST), beta="direct")
    for path, gr in runs.items():
        for name in GRADS:
            assert rel_err(gr[name], ref[name]) <= TOL[dtype], (path, name)


@pytest.mark.parametrize("Dk,Dv,dtype", [(128, 128, "bf16"), (64, 128, "f32")])
def test_decode_direct_beta_matches_oracle(kla, oracle_mod, Dk, Dv, dtype):
    w = Workload("dec", "decode", B=3, T=12, H=5, Dk=Dk, Dv=Dv, dtype=dtype, key_mode="scaled",
                 gate_mode="uniform", s0="normal", seed=Dk + 2 * Dv)
    inp = make_inputs(w)
    kk = inp["k"].double()
    eta = (inp["eta"].double() / ((kk * kk).sum(-1) + 1.0)).float()
    S = inp["S0"].cuda().clone()
    Sref = np64(inp["S0"])
    for t in range(w.T):
        o = kla.decode_step(inp["q"][t].cuda(), inp["k"][t].cuda(), inp["v"][t].cuda(), eta[t].cuda(),
                            inp["g"][t].cuda(), S, w.eps, beta="direct")
        ro, Sref = oracle_mod.decode_step(np64(inp["q"][t]), np64(inp["k"][t]), np64(inp["v"][t]), np64(eta[t]),
                                          np64(inp["g"][t]), w.eps, Sref, beta="direct")
        assert rel_err(o, ro) <= TOL[dtype]
    assert rel_err(S, Sref) <= TOL[dtype]
