"""kla_chunk_bwd_noalloc: the backward for callers that cannot allocate device memory.

Callers such as CUDA-graph captures that must not allocate, plugins whose host framework owns
all device memory, or latency-critical paths cannot hand kla_chunk_bwd a workspace.  For them
the library offers kla_chunk_bwd_noalloc, which uses a fixed scratch array compiled into
libkla.so.  These tests call it through the C ABI and check that it returns what
kla_chunk_bwd returns, on several calls in a row with different shapes, dtypes and backward
paths (the tensor-core path twice on the same shape), so leftovers of an earlier call in the
shared scratch would show up in a later one.  The file name makes
pytest collect it last.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from gated_delta_rule_kla_b200.workloads import Workload, make_inputs

KLA_F32, KLA_BF16 = 0, 1
TOL = {"f32": 1e-4, "bf16": 2e-2}
FAKE = ctypes.c_void_p(0x10000)


def _lib():
    from gated_delta_rule_kla_b200 import build
    build.build()
    import gated_delta_rule_kla_b200 as kla
    L = kla.lib()
    vp, fp, i, f = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    L.kla_chunk_bwd_noalloc.argtypes = [vp, vp, vp, fp, fp, f, fp, vp, fp, fp, vp, vp, vp, fp, fp, fp,
                                        i, i, i, i, i, i, i, i, vp]
    L.kla_chunk_bwd_noalloc.restype = i
    L.kla_chunk_bwd_noalloc_scratch_bytes.argtypes = []
    L.kla_chunk_bwd_noalloc_scratch_bytes.restype = ctypes.c_size_t
    return kla, L


def test_noalloc_rejects_problems_larger_than_its_scratch():
    _, L = _lib()
    cap = L.kla_chunk_bwd_noalloc_scratch_bytes()
    assert cap == 32 << 20
    B, T, H, D = 4, 4096, 16, 128
    assert L.kla_chunk_bwd_workspace(B, T, H, D, D, 64, KLA_BF16, 0) > cap
    st = L.kla_chunk_bwd_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, 1e-6, None, FAKE, None, None, FAKE, FAKE,
                                 FAKE, FAKE, FAKE, FAKE, B, T, H, D, D, 64, KLA_BF16, KLA_F32, None)
    assert st == 3  # KLA_ERR_WORKSPACE, rejected before anything is launched
    assert b"static scratch" in L.kla_last_error()


def test_noalloc_limit_is_the_cuda_core_size():
    """The call is accepted when the CUDA-core layout fits the scratch; the tensor-core layout
    decides only which backward runs.  At bf16 B=1 T=8192 H=1 d=128 the two straddle the
    scratch size (so that call runs the CUDA-core backward); at T=130 H=2 both fit."""
    _, L = _lib()
    cap = L.kla_chunk_bwd_noalloc_scratch_bytes()
    assert L.kla_chunk_bwd_workspace_min(1, 8192, 1, 128, 128, 64, KLA_BF16, 0) <= cap
    assert L.kla_chunk_bwd_workspace(1, 8192, 1, 128, 128, 64, KLA_BF16, 0) > cap
    assert L.kla_chunk_bwd_workspace(1, 130, 2, 128, 128, 64, KLA_BF16, 0) <= cap
    assert L.kla_chunk_bwd_workspace_min(1, 16384, 1, 128, 128, 64, KLA_BF16, 0) > cap


def _rel_err(got, ref):
    got = got.detach().double().cpu()
    ref = ref.detach().double().cpu()
    rms = math.sqrt(float((ref * ref).mean()))
    return float((got - ref).abs().max()) / rms if rms > 0 else float((got - ref).abs().max())


@pytest.mark.gpu
def test_noalloc_backward_matches_workspace_backward_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kla, L = _lib()
    dev = torch.device("cuda", 0)
    # In order: CUDA-core shapes (fp32, then bf16 d = 64); the tensor-core backward (bf16
    # d = 128, both layouts fit) right after a different shape and then again, so stale bytes
    # from an earlier call would show; a shape whose tensor-core layout does not fit (the
    # CUDA-core backward on the scratch).
    cases = [(2, 200, 2, 128, "f32", 31), (1, 130, 3, 64, "bf16", 32), (1, 130, 2, 128, "bf16", 33),
             (1, 130, 2, 128, "bf16", 34), (1, 8192, 1, 128, "bf16", 35)]
    for B, T, H, D, dtype, seed in cases:
        tensor_cores = dtype == "bf16" and D == 128 and \
            L.kla_chunk_bwd_workspace(B, T, H, D, D, 64, KLA_BF16, 0) <= L.kla_chunk_bwd_noalloc_scratch_bytes()
        w = Workload("noalloc", "train", B=B, T=T, H=H, Dk=D, Dv=D, dtype=dtype, key_mode="scaled",
                     gate_mode="uniform", s0="normal", seed=seed)
        inp = make_inputs(w)
        d = {k: v.to(dev) for k, v in inp.items()}
        dO = d["dO"].to(d["q"].dtype).contiguous()
        dST = torch.randn(B, H, D, D, generator=torch.Generator().manual_seed(seed)).to(dev)
        ref = kla.chunk_bwd(d["q"], d["k"], d["v"], d["eta"], d["g"], dO, w.eps, d["S0"], dST)
        out = dict(dq=torch.empty(B, T, H, D, device=dev), dk=torch.empty(B, T, H, D, device=dev),
                   dv=torch.empty(B, T, H, D, device=dev), deta=torch.empty(B, T, H, device=dev),
                   dg=torch.empty(B, T, H, device=dev), dS0=torch.empty(B, H, D, D, device=dev))
        p = lambda t: ctypes.c_void_p(t.data_ptr())
        stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
        st = L.kla_chunk_bwd_noalloc(p(d["q"]), p(d["k"]), p(d["v"]), p(d["eta"]), p(d["g"]), w.eps,
                                     p(d["S0"]), p(dO), p(dST), None, p(out["dq"]), p(out["dk"]),
                                     p(out["dv"]), p(out["deta"]), p(out["dg"]), p(out["dS0"]), B, T, H, D,
                                     D, 64, KLA_BF16 if dtype == "bf16" else KLA_F32, KLA_F32, stream)
        assert st == 0, L.kla_last_error()
        torch.cuda.synchronize()
        for name in ("dq", "dk", "dv", "deta", "dg", "dS0"):
            assert torch.isfinite(out[name]).all(), name
            assert _rel_err(out[name], ref[name]) <= TOL[dtype], name
            if tensor_cores:  # the tensor-core backward is deterministic: same bits as with a workspace
                assert torch.equal(out[name], ref[name]), name
