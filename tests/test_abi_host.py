"""Host-only checks of the C ABI (no GPU): the library loads, exports every entry point
include/kla.h declares, and rejects invalid calls before touching the device."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kla.h")

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3
FAKE = ctypes.c_void_p(0x10000)  # aligned, never dereferenced: validation fails first
MISALIGNED = ctypes.c_void_p(0x10004)


@pytest.fixture(scope="module")
def L():
    from gated_delta_rule_kla_b200 import build
    build.build()
    import gated_delta_rule_kla_b200 as kla
    return kla.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kla_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert {"kla_chunk_fwd", "kla_chunk_bwd", "kla_decode_step"} <= set(names)
    for n in names:
        assert hasattr(L, n), f"libkla.so does not export {n}"


def test_status_strings(L):
    for code, name in [(0, b"KLA_OK"), (1, b"KLA_ERR_INVALID_ARG"), (2, b"KLA_ERR_UNSUPPORTED"),
                       (3, b"KLA_ERR_WORKSPACE"), (4, b"KLA_ERR_CUDA"), (5, b"KLA_ERR_TIMEOUT")]:
        assert L.kla_status_string(code) == name
    assert L.kla_status_string(99) == b"KLA_ERR_UNKNOWN"
    assert L.kla_version() >= 100


def _fwd(L, B=1, T=64, H=1, Dk=128, Dv=128, chunk=64, dtype=1, out_dtype=0, eps=1e-6, q=FAKE, ws=None):
    return L.kla_chunk_fwd(q, FAKE, FAKE, FAKE, FAKE, eps, None, FAKE, FAKE, None, B, T, H, Dk, Dv,
                           chunk, dtype, out_dtype, ws, 0, None)


@pytest.mark.parametrize("kw,code", [
    (dict(Dk=96), UNSUPPORTED), (dict(Dv=32), UNSUPPORTED), (dict(chunk=32), UNSUPPORTED),
    (dict(dtype=7), UNSUPPORTED), (dict(out_dtype=3), UNSUPPORTED), (dict(eps=-1.0), INVALID), (dict(eps=float("nan")), INVALID),
    (dict(B=0), INVALID), (dict(H=0), INVALID), (dict(T=-1), INVALID),
    (dict(q=None), INVALID), (dict(q=MISALIGNED), INVALID),
])
def test_fwd_rejects_before_launch(L, kw, code):
    assert _fwd(L, **kw) == code
    assert len(L.kla_last_error()) > 0


def test_fwd_stages_reject_before_launch(L):
    need = L.kla_chunk_fwd_workspace(2, 300, 3, 128, 128, 64, 1)
    assert need >= 2 * 3 * 5 * 82432  # one record of ~80.5 KiB per chunk and head
    prep = lambda dtype=1, Dk=128, T=300, ws=FAKE, n=need: L.kla_chunk_fwd_prep(
        FAKE, FAKE, FAKE, FAKE, FAKE, 1e-6, 2, T, 3, Dk, 128, 64, dtype, ws, n, None)
    state = lambda dtype=1, ws=FAKE, n=need, q=FAKE, v=FAKE: L.kla_chunk_fwd_state(
        q, v, FAKE, None, FAKE, None, None, 2, 300, 3, 128, 128, 64, dtype, 0, ws, n, None)
    assert prep(dtype=0) == UNSUPPORTED and prep(Dk=64) == UNSUPPORTED
    assert prep(T=0) == INVALID
    assert prep(ws=None) == WORKSPACE and prep(n=need - 1) == WORKSPACE
    assert state(dtype=0) == UNSUPPORTED and state(ws=None) == WORKSPACE
    assert state(q=None) == INVALID and state(v=None) == INVALID and state(ws=MISALIGNED) == INVALID
    assert b"aligned" in L.kla_last_error()
    assert state(ws=None) == WORKSPACE and b"kla_chunk_fwd_state" in L.kla_last_error()
    stage = lambda k: L.kla_chunk_fwd_state_stage(k, FAKE, FAKE, FAKE, None, FAKE, None, None, 2, 300, 3, 128, 128,
                                                  64, 1, 0, FAKE, need, None)
    assert stage(-1) == INVALID and stage(4) == INVALID and b"stage" in L.kla_last_error()


def test_fwd_state_segments_query(L):
    # many heads or short sequences: one run per head; few heads over a long sequence: parallel
    # segments (with the 148 SMs assumed when no device answers)
    assert L.kla_chunk_fwd_state_segments(8, 2048, 8, 128, 128, 64, 1) == 1
    assert L.kla_chunk_fwd_state_segments(1, 65536, 16, 128, 128, 64, 1) > 1
    assert L.kla_chunk_fwd_state_segments(1, 4100, 1, 128, 128, 64, 1) > 1
    assert L.kla_chunk_fwd_state_segments(8, 2048, 8, 64, 128, 64, 1) == 0
    assert L.kla_chunk_fwd_state_segments(8, 2048, 8, 128, 128, 64, 0) == 0
    assert L.kla_chunk_fwd_state_segments(0, 2048, 8, 128, 128, 64, 1) == 0


def test_bwd_workspace_checked(L):
    need = L.kla_chunk_bwd_workspace(2, 100, 3, 64, 128, 64, 1, 0)
    ntok = 2 * 100 * 3
    r256 = lambda x: (x + 255) // 256 * 256
    assert need == r256(2 * 3 * 2 * 64 * 128 * 4) + 2 * r256(ntok * 64 * 4) + r256(3 * ntok * 4)
    assert L.kla_chunk_bwd_workspace(2, 100, 3, 64, 128, 64, 1, 1) == need - r256(2 * 3 * 2 * 64 * 128 * 4)
    st = L.kla_chunk_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, 1e-6, None, FAKE, None, None, FAKE, FAKE, FAKE,
                         FAKE, FAKE, FAKE, 2, 100, 3, 64, 128, 64, 1, 0, None, 0, None)
    assert st == WORKSPACE
    assert b"workspace" in L.kla_last_error()
    st = L.kla_chunk_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, 1e-6, None, FAKE, None, None, FAKE, FAKE, FAKE,
                         FAKE, FAKE, FAKE, 2, 100, 3, 64, 128, 64, 1, 0, FAKE, need - 1, None)
    assert st == WORKSPACE


def test_bwd_requires_outputs(L):
    st = L.kla_chunk_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, 1e-6, None, FAKE, None, None, None, FAKE, FAKE,
                         FAKE, FAKE, FAKE, 1, 64, 1, 64, 64, 64, 1, 0, FAKE, 1 << 30, None)
    assert st == INVALID


def test_decode_rejects_before_launch(L):
    st = L.kla_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, 1e-6, FAKE, None, 4, 2, 128, 96, 1, 0, None)
    assert st == UNSUPPORTED
    st = L.kla_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, 1e-6, None, None, 4, 2, 128, 128, 1, 0, None)
    assert st == INVALID
    st = L.kla_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, -0.5, FAKE, None, 4, 2, 128, 128, 1, 0, None)
    assert st == INVALID


def test_binding_has_no_cpu_fallback(L):
    import gated_delta_rule_kla_b200 as kla
    x = torch.zeros(1, 64, 1, 64)
    gates = torch.zeros(1, 64, 1)
    with pytest.raises(TypeError):
        kla.chunk_fwd(x, x, x, gates, gates)
    with pytest.raises(TypeError):
        kla.decode_step(x[:, 0], x[:, 0], x[:, 0], gates[:, 0], gates[:, 0], torch.zeros(1, 1, 64, 64))


def test_product_and_oracle_share_no_code():
    pkg = os.path.join(ROOT, "gated_delta_rule_kla_b200")
    imp = re.compile(r"^\s*(from\s+oracle\b|import\s+oracle\b|#\s*include\s*[<\"].*oracle)", re.M)
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert not imp.search(text), f"{f} imports the oracle"
                assert "kla_oracle" not in text, f"{f} names the oracle library"
    for f in os.listdir(os.path.join(ROOT, "oracle")):
        if f.endswith((".py", ".c", ".h")):
            text = open(os.path.join(ROOT, "oracle", f)).read()
            assert "gated_delta_rule_kla_b200" not in text
            assert "kla.h" not in text


def test_train_pair_rejects_before_launch(L):
    need = L.kla_chunk_bwd_workspace(2, 100, 3, 128, 128, 64, 1, 0)
    small = L.kla_chunk_bwd_workspace_min(2, 100, 3, 128, 128, 64, 1, 0)
    assert need > small  # bf16, d = 128: the tensor-core backward's layout
    fwd = lambda ws=FAKE, n=need, q=FAKE, Dk=128: L.kla_chunk_fwd_train(
        q, FAKE, FAKE, FAKE, FAKE, 1e-6, None, FAKE, None, 2, 100, 3, Dk, 128, 64, 1, 0, ws, n, None)
    bwd = lambda ws=FAKE, n=need, dO=FAKE: L.kla_chunk_bwd_after_train(
        FAKE, FAKE, FAKE, FAKE, FAKE, 1e-6, dO, None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 100, 3, 128, 128,
        64, 1, 0, ws, n, None)
    assert fwd(ws=None) == WORKSPACE and b"kla_chunk_fwd_train" in L.kla_last_error()
    assert fwd(n=small - 1) == WORKSPACE
    assert fwd(q=None) == INVALID and fwd(ws=MISALIGNED) == INVALID and fwd(Dk=96) == UNSUPPORTED
    assert bwd(ws=None) == WORKSPACE and b"kla_chunk_bwd_after_train" in L.kla_last_error()
    assert bwd(dO=None) == INVALID and bwd(n=small - 1) == WORKSPACE


DIRECT = 0x100  # KLA_BETA_DIRECT


def test_direct_beta_flag_is_stripped_and_still_validated(L):
    """KLA_BETA_DIRECT rides in dtype: the queries ignore it, the entry points accept it with
    a valid element type, and validation (element type, eps >= 0) still applies."""
    for B, T, H in [(8, 2048, 8), (2, 300, 3), (1, 65536, 16)]:
        assert L.kla_chunk_fwd_workspace(B, T, H, 128, 128, 64, 1 | DIRECT) == \
            L.kla_chunk_fwd_workspace(B, T, H, 128, 128, 64, 1)
        assert L.kla_chunk_fwd_kernel_launches(B, T, H, 128, 128, 64, 1 | DIRECT) == \
            L.kla_chunk_fwd_kernel_launches(B, T, H, 128, 128, 64, 1)
        assert L.kla_chunk_bwd_workspace(B, T, H, 128, 128, 64, 1 | DIRECT, 0) == \
            L.kla_chunk_bwd_workspace(B, T, H, 128, 128, 64, 1, 0)
    assert _fwd(L, dtype=7 | DIRECT) == UNSUPPORTED      # not an element type even without the flag
    assert _fwd(L, dtype=1 | 0x200) == UNSUPPORTED       # an unknown flag bit
    assert _fwd(L, dtype=1 | DIRECT, eps=-1.0) == INVALID  # eps is unused in the direct mode, still >= 0
    assert _fwd(L, dtype=1 | DIRECT, q=None) == INVALID
    st = L.kla_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, -0.5, FAKE, None, 4, 2, 128, 128, 1 | DIRECT, 0, None)
    assert st == INVALID


def test_forward_launch_plan(L):
    """Kernels per kla_chunk_fwd call with a full workspace: two slabs (preparation and state pass
    each twice) when the heads fill at most half the SMs and there are enough chunks; the
    segmented pass (preparation, transition pass, scan, output pass) for long sequences over
    few heads; one preparation and one state pass otherwise; the fused kernel (1) for shapes
    that take no workspace.  (Without a GPU the library plans for 148 SMs.)"""
    cases = [((8, 2048, 8), 4), ((4, 4096, 16), 4), ((8, 1024, 8), 4),   # two slabs
             ((1, 65536, 16), 4),                                       # segmented
             ((2, 300, 3), 2), ((16, 2048, 16), 2), ((1, 256, 2), 2)]   # one run
    for (B, T, H), n in cases:
        assert L.kla_chunk_fwd_kernel_launches(B, T, H, 128, 128, 64, 1) == n, (B, T, H)
    assert L.kla_chunk_fwd_kernel_launches(1, 300, 2, 64, 64, 64, 0) == 1  # fp32 d = 64: one kernel
    assert L.kla_chunk_fwd_kernel_launches(0, 300, 2, 128, 128, 64, 1) == 0  # invalid shape


def test_backward_reverse_segments(L):
    """The reverse state pass is segmented exactly where the forward's cost model segments the
    forward state pass: long sequences over few heads; one run for the workloads' other shapes."""
    assert L.kla_chunk_bwd_reverse_segments(8, 2048, 8, 128, 128, 64, 1) == 1
    assert L.kla_chunk_bwd_reverse_segments(4, 4096, 16, 128, 128, 64, 1) == 1
    assert L.kla_chunk_bwd_reverse_segments(1, 65536, 16, 128, 128, 64, 1) > 1
    assert L.kla_chunk_bwd_reverse_segments(1, 4100, 2, 128, 128, 64, 1) > 1
    assert L.kla_chunk_bwd_reverse_segments(1, 4100, 2, 64, 64, 64, 1) == 0  # no tensor-core backward
    assert L.kla_chunk_bwd_reverse_segments(1, 4100, 2, 128, 128, 64, 0) == 0
    # one reverse run per head: the newest chunks as a slab of their own when the gradient
    # kernel has enough work to fill the other SMs meanwhile (148 SMs assumed without a device)
    assert 0 < L.kla_chunk_bwd_reverse_slab_chunks(4, 4096, 16, 128, 128, 64, 1) < 64
    assert 0 < L.kla_chunk_bwd_reverse_slab_chunks(4, 2048, 16, 128, 128, 64, 1) < 32
    assert L.kla_chunk_bwd_reverse_slab_chunks(2, 150, 3, 128, 128, 64, 1) == 0
    assert L.kla_chunk_bwd_reverse_slab_chunks(1, 65536, 16, 128, 128, 64, 1) == 0  # segmented instead
    assert L.kla_chunk_bwd_reverse_slab_chunks(4, 4096, 16, 64, 64, 64, 1) == 0


def test_diag_forward_workspace_by_path(L):
    """bf16 at Dk = Dv = 128 takes the tensor-core split path: one record of 97 KiB per 64-token
    chunk and head; other shapes the CUDA-core split path over 16-token chunks."""
    tc = L.kla_chunk_fwd_diag_workspace(2, 300, 3, 128, 128, 64, 1)
    assert tc >= 2 * 3 * 5 * 99328
    assert L.kla_chunk_fwd_diag_kernel_launches(2, 300, 3, 128, 128, 64, 1) >= 2
    simt = L.kla_chunk_fwd_diag_workspace(2, 300, 3, 128, 128, 64, 0)
    assert simt >= 2 * 3 * 19 * 4 * (3 * 16 * 128 + 16 * 16 + 128)
    assert L.kla_chunk_fwd_diag_kernel_launches(2, 300, 3, 128, 128, 64, 0) == 2
    assert L.kla_chunk_fwd_diag_kernel_launches(2, 300, 3, 96, 128, 64, 1) == 0
    # 32 heads over 10 chunks run as two slabs (148 SMs); one head over 65 chunks as segments
    assert L.kla_chunk_fwd_diag_kernel_launches(2, 640, 16, 128, 128, 64, 1) == 4
    assert L.kla_chunk_fwd_diag_kernel_launches(1, 4100, 1, 128, 128, 64, 1) == 4
