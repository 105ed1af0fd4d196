"""Python binding of libkla.so -- Kaczmarz Linear Attention on NVIDIA B200 (sm_100a).

Thin argument marshalling over the C ABI declared in ``include/kla.h``: every step of the
computation runs in the library's CUDA kernels.  PyTorch is used only to allocate device
memory and to name the current CUDA stream.  There is no CPU fallback: if the library is
missing, or a tensor is not on a CUDA device, the call raises.

    chunk_fwd(q, k, v, eta, g, eps, S0)          -> (o, S_T[, S_chunks])   prefill
    chunk_bwd(q, k, v, eta, g, dO, eps, S0, ...) -> dict of gradients      training
    decode_step(q, k, v, eta, g, S, eps)         -> o  (S updated in place)

The method ("Kaczmarz Linear Attention", section 3.1 Eq. (3); section 3.3 Algorithm 1):
beta_t = eta_t/(||k_t||^2+eps), alpha_t = exp(g_t), Sbar = alpha_t S_{t-1},
S_t = Sbar + beta_t k_t (v_t - Sbar^T k_t)^T, o_t = S_t^T q_t.
"""
import ctypes
import os

import torch

__all__ = ["lib", "chunk_fwd", "chunk_fwd_prep", "chunk_fwd_state", "fwd_state_segments", "fwd_workspace",
           "fwd_kernel_launches",
           "chunk_bwd", "chunk_fwd_train", "chunk_bwd_after_train", "train_workspace",
           "decode_step", "check_device_error", "debug_inject_wait_timeout",
           "chunk_fwd_diag", "chunk_bwd_diag", "decode_step_diag", "gate_prologue", "gate_prologue_bwd", "KLAError", "CHUNK", "KLA_BETA_DIRECT",
           "library_path"]

CHUNK = 64
KLA_F32, KLA_BF16 = 0, 1
KLA_BETA_DIRECT = 0x100  # OR-ed into the input dtype code: beta_t = eta_t as given
_PKG = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_PKG, "libkla.so")
_lib = None


class KLAError(RuntimeError):
    """A non-OK status returned by libkla."""

    def __init__(self, status, name, detail):
        super().__init__(f"{name}: {detail}")
        self.status = status


def lib():
    """The loaded libkla.so (ctypes).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(library_path):
            raise RuntimeError(f"libkla.so not found at {library_path}; build it with "
                               "`python -m gated_delta_rule_kla_b200.build`")
        L = ctypes.CDLL(library_path)
        vp, fp, i, f, sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.kla_status_string.argtypes = [i]
        L.kla_status_string.restype = ctypes.c_char_p
        L.kla_last_error.argtypes = []
        L.kla_last_error.restype = ctypes.c_char_p
        L.kla_version.argtypes = []
        L.kla_version.restype = i
        L.kla_chunk_fwd_workspace.argtypes = [i, i, i, i, i, i, i]
        L.kla_chunk_fwd_workspace.restype = sz
        L.kla_chunk_fwd_kernel_launches.argtypes = [i, i, i, i, i, i, i]
        L.kla_chunk_fwd_kernel_launches.restype = i
        L.kla_chunk_fwd.argtypes = [vp, vp, vp, fp, fp, f, fp, vp, fp, fp, i, i, i, i, i, i, i, i, vp, sz, vp]
        L.kla_chunk_fwd.restype = i
        L.kla_chunk_fwd_prep.argtypes = [vp, vp, vp, fp, fp, f, i, i, i, i, i, i, i, vp, sz, vp]
        L.kla_chunk_fwd_prep.restype = i
        L.kla_chunk_fwd_state.argtypes = [vp, vp, fp, fp, vp, fp, fp, i, i, i, i, i, i, i, i, vp, sz, vp]
        L.kla_chunk_fwd_state.restype = i
        L.kla_chunk_fwd_state_stage.argtypes = [i, vp, vp, fp, fp, vp, fp, fp, i, i, i, i, i, i, i, i, vp, sz, vp]
        L.kla_chunk_fwd_state_stage.restype = i
        L.kla_chunk_fwd_state_segments.argtypes = [i, i, i, i, i, i, i]
        L.kla_chunk_fwd_state_segments.restype = i
        L.kla_chunk_bwd_reverse_slab_chunks.argtypes = [i, i, i, i, i, i, i]
        L.kla_chunk_bwd_reverse_slab_chunks.restype = i
        L.kla_chunk_bwd_workspace.argtypes = [i, i, i, i, i, i, i, i]
        L.kla_chunk_bwd_workspace.restype = sz
        L.kla_chunk_bwd_workspace_min.argtypes = [i, i, i, i, i, i, i, i]
        L.kla_chunk_bwd_workspace_min.restype = sz
        L.kla_chunk_bwd_reverse_segments.argtypes = [i, i, i, i, i, i, i]
        L.kla_chunk_bwd_reverse_segments.restype = i
        L.kla_chunk_fwd_train.argtypes = [vp, vp, vp, fp, fp, f, fp, vp, fp, i, i, i, i, i, i, i, i, vp, sz, vp]
        L.kla_chunk_fwd_train.restype = i
        L.kla_chunk_bwd_after_train.argtypes = [vp, vp, vp, fp, fp, f, vp, fp, vp, vp, vp, fp, fp, fp,
                                                i, i, i, i, i, i, i, i, vp, sz, vp]
        L.kla_chunk_bwd_after_train.restype = i
        L.kla_chunk_bwd.argtypes = [vp, vp, vp, fp, fp, f, fp, vp, fp, fp, vp, vp, vp, fp, fp, fp,
                                    i, i, i, i, i, i, i, i, vp, sz, vp]
        L.kla_chunk_bwd.restype = i
        L.kla_decode_step.argtypes = [vp, vp, vp, fp, fp, f, fp, vp, i, i, i, i, i, i, vp]
        L.kla_decode_step.restype = i
        L.kla_check_device_error.argtypes = [vp]
        L.kla_check_device_error.restype = i
        L.kla_debug_inject_wait_timeout.argtypes = []
        L.kla_debug_inject_wait_timeout.restype = None
        L.kla_chunk_fwd_diag_workspace.argtypes = [i, i, i, i, i, i, i]
        L.kla_chunk_fwd_diag_workspace.restype = sz
        L.kla_chunk_fwd_diag_kernel_launches.argtypes = [i, i, i, i, i, i, i]
        L.kla_chunk_fwd_diag_kernel_launches.restype = i
        L.kla_chunk_fwd_diag.argtypes = [vp, vp, vp, fp, fp, f, fp, vp, fp, i, i, i, i, i, i, i, i, vp, sz, vp]
        L.kla_chunk_fwd_diag.restype = i
        L.kla_chunk_bwd_diag_workspace.argtypes = [i, i, i, i, i, i, i]
        L.kla_chunk_bwd_diag_workspace.restype = sz
        L.kla_chunk_bwd_diag.argtypes = [vp, vp, vp, fp, fp, f, fp, vp, fp, vp, vp, vp, fp, fp, fp,
                                         i, i, i, i, i, i, i, i, vp, sz, vp]
        L.kla_chunk_bwd_diag.restype = i
        L.kla_decode_step_diag.argtypes = [vp, vp, vp, fp, fp, f, fp, vp, i, i, i, i, i, i, vp]
        L.kla_decode_step_diag.restype = i
        L.kla_gate_prologue.argtypes = [vp, vp, fp, vp, fp, fp, vp, i, i, i, i, i, vp]
        L.kla_gate_prologue.restype = i
        L.kla_gate_prologue_bwd_workspace.argtypes = [i, i, i]
        L.kla_gate_prologue_bwd_workspace.restype = sz
        L.kla_gate_prologue_bwd.argtypes = [vp, vp, fp, fp, vp, fp, fp, fp, fp, fp, fp, fp, i, i, i, i, i, vp, sz,
                                            vp]
        L.kla_gate_prologue_bwd.restype = i
        _lib = L
    return _lib


def _check(status, name):
    if status != 0:
        L = lib()
        raise KLAError(status, name, f"{L.kla_status_string(status).decode()}: "
                                     f"{L.kla_last_error().decode()}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(t):
    dt = t if isinstance(t, torch.dtype) else t.dtype
    if dt == torch.bfloat16:
        return KLA_BF16
    if dt == torch.float32:
        return KLA_F32
    raise TypeError(f"expected bfloat16 or float32, got {dt}")


def _in_code(t, beta):
    """Input dtype code with the write-strength mode: "kaczmarz" (beta_t = eta_t / (||k_t||^2 +
    eps), Eq. 3) or "direct" (beta_t = eta_t as given: the Gated DeltaNet update)."""
    if beta not in ("kaczmarz", "direct"):
        raise ValueError(f"beta must be 'kaczmarz' or 'direct', got {beta!r}")
    return _dtype_code(t) | (KLA_BETA_DIRECT if beta == "direct" else 0)


def _need(t, name, device, dtype=None, shape=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _stream(device, stream):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def chunk_fwd(q, k, v, eta, g, eps=1e-6, S0=None, *, o=None, S_T=None, save_chunk_states=False,
              output_final_state=True, out_dtype=torch.float32, stream=None, fused=False,
              workspace=None, beta="kaczmarz"):
    """Chunkwise prefill (section 4, Propositions 3-4).

    q, k: [B,T,H,Dk]; v: [B,T,H,Dv] (bf16 or fp32, same dtype); eta, g: [B,T,H] fp32;
    S0: [B,H,Dk,Dv] fp32 or None.  o is written in `out_dtype` (fp32 by default; a bf16
    store rounds each output once).  Returns (o, S_T) or (o, S_T, S_chunks) when
    save_chunk_states (S_chunks: [B,H,ceil(T/64),Dk,Dv], the state at each chunk start).
    bf16 inputs with Dk == Dv == 128 take the split path: a chunk-parallel preparation kernel
    stores every chunk's state-independent operands in the workspace kla_chunk_fwd_workspace()
    reports (allocated here unless `workspace` is given), then a sequential state pass (split
    into parallel segments for long sequences over few heads).  fused=True passes no workspace,
    which selects the one-kernel-per-head path.  beta="direct" takes eta as the write strength
    itself (beta_t = eta_t, the Gated DeltaNet update) instead of the Kaczmarz step; the other
    entry points take the same keyword.
    """
    dev = k.device
    B, T, H, Dk = k.shape
    Dv = v.shape[-1]
    dt = k.dtype
    _need(q, "q", dev, dt, (B, T, H, Dk)); _need(k, "k", dev, dt); _need(v, "v", dev, dt, (B, T, H, Dv))
    _need(eta, "eta", dev, torch.float32, (B, T, H)); _need(g, "g", dev, torch.float32, (B, T, H))
    _need(S0, "S0", dev, torch.float32, (B, H, Dk, Dv))
    if o is None:
        o = torch.empty(B, T, H, Dv, device=dev, dtype=out_dtype)
    _need(o, "o", dev, None, (B, T, H, Dv))
    if S_T is None and output_final_state:
        S_T = torch.empty(B, H, Dk, Dv, device=dev, dtype=torch.float32)
    _need(S_T, "S_T", dev, torch.float32, (B, H, Dk, Dv))
    Sc = None
    if save_chunk_states:
        Sc = torch.empty(B, H, (T + CHUNK - 1) // CHUNK, Dk, Dv, device=dev, dtype=torch.float32)
    L = lib()
    need = 0 if fused else L.kla_chunk_fwd_workspace(B, T, H, Dk, Dv, CHUNK, _dtype_code(k))
    if need > 0 and (workspace is None or workspace.numel() < need):
        workspace = torch.empty(need, device=dev, dtype=torch.uint8)
    ws_ptr, ws_n = (_ptr(workspace), workspace.numel()) if need > 0 else (None, 0)
    st = L.kla_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(eta), _ptr(g), float(eps), _ptr(S0),
                         _ptr(o), _ptr(S_T), _ptr(Sc), B, T, H, Dk, Dv, CHUNK, _in_code(k, beta),
                         _dtype_code(o), ws_ptr, ws_n, _stream(dev, stream))
    _check(st, "kla_chunk_fwd")
    return (o, S_T, Sc) if save_chunk_states else (o, S_T)


def fwd_workspace(k, v):
    """A workspace for kla_chunk_fwd / its two stages, sized for k [B,T,H,Dk] and v (None when
    the shapes take no workspace)."""
    B, T, H, Dk = k.shape
    need = lib().kla_chunk_fwd_workspace(B, T, H, Dk, v.shape[-1], CHUNK, _dtype_code(k))
    return torch.empty(need, device=k.device, dtype=torch.uint8) if need > 0 else None


def fwd_kernel_launches(k, v):
    """Kernels one chunk_fwd call with a workspace from fwd_workspace launches for k, v."""
    B, T, H, Dk = k.shape
    return lib().kla_chunk_fwd_kernel_launches(B, T, H, Dk, v.shape[-1], CHUNK, _dtype_code(k))


def chunk_fwd_prep(q, k, v, eta, g, eps, workspace, *, stream=None, beta="kaczmarz"):
    """First stage of the split forward: every chunk's state-independent operands into
    `workspace` (from fwd_workspace).  bf16 inputs with Dk == Dv == 128."""
    dev = k.device
    B, T, H, Dk = k.shape
    Dv = v.shape[-1]
    _need(q, "q", dev, k.dtype, (B, T, H, Dk)); _need(v, "v", dev, k.dtype, (B, T, H, Dv))
    _need(eta, "eta", dev, torch.float32, (B, T, H)); _need(g, "g", dev, torch.float32, (B, T, H))
    _need(workspace, "workspace", dev, torch.uint8)
    L = lib()
    st = L.kla_chunk_fwd_prep(_ptr(q), _ptr(k), _ptr(v), _ptr(eta), _ptr(g), float(eps), B, T, H, Dk, Dv,
                              CHUNK, _in_code(k, beta), _ptr(workspace), workspace.numel(), _stream(dev, stream))
    _check(st, "kla_chunk_fwd_prep")


def chunk_fwd_state(q, v, g, S0, workspace, *, o=None, S_T=None, S_chunks=None,
                    out_dtype=torch.float32, stream=None, stage=0):
    """Second stage of the split forward: the state pass over the records that chunk_fwd_prep
    left in `workspace` (it also reads q and v).  Writes o, S_T, S_chunks when given (allocates o
    and S_T when None).  `stage` 1, 2, 3 run the transition pass, segment scan and output pass
    of a segmented state pass alone (see fwd_state_segments); 0 runs all of it."""
    dev = q.device
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    _need(v, "v", dev, q.dtype, (B, T, H, Dv))
    _need(g, "g", dev, torch.float32, (B, T, H)); _need(S0, "S0", dev, torch.float32, (B, H, Dk, Dv))
    if o is None:
        o = torch.empty(B, T, H, Dv, device=dev, dtype=out_dtype)
    if S_T is None:
        S_T = torch.empty(B, H, Dk, Dv, device=dev, dtype=torch.float32)
    _need(o, "o", dev, None, (B, T, H, Dv)); _need(S_T, "S_T", dev, torch.float32, (B, H, Dk, Dv))
    _need(S_chunks, "S_chunks", dev, torch.float32, (B, H, (T + CHUNK - 1) // CHUNK, Dk, Dv))
    _need(workspace, "workspace", dev, torch.uint8)
    L = lib()
    st = L.kla_chunk_fwd_state_stage(int(stage), _ptr(q), _ptr(v), _ptr(g), _ptr(S0), _ptr(o), _ptr(S_T),
                                     _ptr(S_chunks), B, T, H, Dk, Dv, CHUNK, _dtype_code(q), _dtype_code(o),
                                     _ptr(workspace), workspace.numel(), _stream(dev, stream))
    _check(st, "kla_chunk_fwd_state")
    return o, S_T


def fwd_state_segments(k, v):
    """Parallel segments per head of the split forward's state pass for k, v (1: one run per
    head; 0: shapes the split path does not take)."""
    B, T, H, Dk = k.shape
    return lib().kla_chunk_fwd_state_segments(B, T, H, Dk, v.shape[-1], CHUNK, _dtype_code(k))


def chunk_bwd(q, k, v, eta, g, dO, eps=1e-6, S0=None, dS_T=None, S_chunks=None, *, stream=None,
              workspace=None, out_dtype=torch.float32, cuda_cores=False, beta="kaczmarz"):
    """Gradients of the chunkwise forward w.r.t. q, k, v, eta, g and S0.

    dO: [B,T,H,Dv] (same dtype as q); dS_T: [B,H,Dk,Dv] fp32 or None; S_chunks: the
    array chunk_fwd(save_chunk_states=True) returned for the same inputs, or None.
    dq, dk, dv are written in `out_dtype` (fp32 by default).  bf16 inputs with
    Dk == Dv == 128 run on the tensor cores unless `cuda_cores` is set (the workspace is then
    sized for the CUDA-core backward, which the library runs with a smaller workspace).
    Returns dict(dq, dk, dv, deta, dg, dS0).
    """
    dev = k.device
    B, T, H, Dk = k.shape
    Dv = v.shape[-1]
    dt = k.dtype
    _need(q, "q", dev, dt, (B, T, H, Dk)); _need(k, "k", dev, dt); _need(v, "v", dev, dt, (B, T, H, Dv))
    _need(eta, "eta", dev, torch.float32, (B, T, H)); _need(g, "g", dev, torch.float32, (B, T, H))
    _need(S0, "S0", dev, torch.float32, (B, H, Dk, Dv)); _need(dO, "dO", dev, dt, (B, T, H, Dv))
    _need(dS_T, "dS_T", dev, torch.float32, (B, H, Dk, Dv))
    NC = (T + CHUNK - 1) // CHUNK
    _need(S_chunks, "S_chunks", dev, torch.float32, (B, H, NC, Dk, Dv))
    out = dict(dq=torch.empty(q.shape, device=dev, dtype=out_dtype),
               dk=torch.empty(k.shape, device=dev, dtype=out_dtype),
               dv=torch.empty(v.shape, device=dev, dtype=out_dtype),
               deta=torch.empty_like(eta), dg=torch.empty_like(g),
               dS0=torch.empty(B, H, Dk, Dv, device=dev, dtype=torch.float32))
    L = lib()
    size = L.kla_chunk_bwd_workspace_min if cuda_cores else L.kla_chunk_bwd_workspace
    need = size(B, T, H, Dk, Dv, CHUNK, _dtype_code(k), int(S_chunks is not None))
    if workspace is None or workspace.numel() < need or (cuda_cores and workspace.numel() > need):
        workspace = torch.empty(max(need, 16), device=dev, dtype=torch.uint8)
    st = L.kla_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(eta), _ptr(g), float(eps), _ptr(S0), _ptr(dO),
                         _ptr(dS_T), _ptr(S_chunks), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                         _ptr(out["deta"]), _ptr(out["dg"]), _ptr(out["dS0"]), B, T, H, Dk, Dv, CHUNK,
                         _in_code(k, beta), _dtype_code(out_dtype), _ptr(workspace), workspace.numel(),
                         _stream(dev, stream))
    _check(st, "kla_chunk_bwd")
    return out


def train_workspace(k, v):
    """A workspace for chunk_fwd_train / chunk_bwd_after_train on these shapes (reusable)."""
    B, T, H, Dk = k.shape
    n = lib().kla_chunk_bwd_workspace(B, T, H, Dk, v.shape[-1], CHUNK, _dtype_code(k), 0)
    return torch.empty(max(n, 16), device=k.device, dtype=torch.uint8)


def chunk_fwd_train(q, k, v, eta, g, eps=1e-6, S0=None, *, workspace=None, o=None, S_T=None,
                    out_dtype=torch.float32, stream=None, beta="kaczmarz"):
    """Training forward: (o, S_T, workspace), the workspace holding what chunk_bwd_after_train
    needs for these inputs (kla_chunk_fwd_train)."""
    dev = k.device
    B, T, H, Dk = k.shape
    Dv = v.shape[-1]
    dt = k.dtype
    _need(q, "q", dev, dt, (B, T, H, Dk)); _need(k, "k", dev, dt); _need(v, "v", dev, dt, (B, T, H, Dv))
    _need(eta, "eta", dev, torch.float32, (B, T, H)); _need(g, "g", dev, torch.float32, (B, T, H))
    _need(S0, "S0", dev, torch.float32, (B, H, Dk, Dv))
    if o is None:
        o = torch.empty(B, T, H, Dv, device=dev, dtype=out_dtype)
    if S_T is None:
        S_T = torch.empty(B, H, Dk, Dv, device=dev, dtype=torch.float32)
    _need(o, "o", dev, None, (B, T, H, Dv)); _need(S_T, "S_T", dev, torch.float32, (B, H, Dk, Dv))
    if workspace is None:
        workspace = train_workspace(k, v)
    st = lib().kla_chunk_fwd_train(_ptr(q), _ptr(k), _ptr(v), _ptr(eta), _ptr(g), float(eps), _ptr(S0), _ptr(o),
                                   _ptr(S_T), B, T, H, Dk, Dv, CHUNK, _in_code(k, beta), _dtype_code(o),
                                   _ptr(workspace), workspace.numel(), _stream(dev, stream))
    _check(st, "kla_chunk_fwd_train")
    return o, S_T, workspace


def chunk_bwd_after_train(q, k, v, eta, g, dO, workspace, eps=1e-6, dS_T=None, *, out_dtype=torch.float32,
                          stream=None, beta="kaczmarz"):
    """Backward after chunk_fwd_train on the same inputs and workspace (kla_chunk_bwd_after_train).
    Returns dict(dq, dk, dv, deta, dg, dS0)."""
    dev = k.device
    B, T, H, Dk = k.shape
    Dv = v.shape[-1]
    dt = k.dtype
    _need(dO, "dO", dev, dt, (B, T, H, Dv)); _need(dS_T, "dS_T", dev, torch.float32, (B, H, Dk, Dv))
    out = dict(dq=torch.empty(q.shape, device=dev, dtype=out_dtype),
               dk=torch.empty(k.shape, device=dev, dtype=out_dtype),
               dv=torch.empty(v.shape, device=dev, dtype=out_dtype),
               deta=torch.empty_like(eta), dg=torch.empty_like(g),
               dS0=torch.empty(B, H, Dk, Dv, device=dev, dtype=torch.float32))
    st = lib().kla_chunk_bwd_after_train(_ptr(q), _ptr(k), _ptr(v), _ptr(eta), _ptr(g), float(eps), _ptr(dO),
                                         _ptr(dS_T), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                                         _ptr(out["deta"]), _ptr(out["dg"]), _ptr(out["dS0"]), B, T, H, Dk, Dv,
                                         CHUNK, _in_code(k, beta), _dtype_code(out_dtype), _ptr(workspace),
                                         workspace.numel(), _stream(dev, stream))
    _check(st, "kla_chunk_bwd_after_train")
    return out


def decode_step(q, k, v, eta, g, S, eps=1e-6, *, o=None, out_dtype=torch.float32, stream=None,
                beta="kaczmarz"):
    """One decode token for every (b, h): q, k [B,H,Dk]; v [B,H,Dv]; eta, g [B,H] fp32;
    S [B,H,Dk,Dv] fp32 updated in place.  Returns o [B,H,Dv]."""
    dev = S.device
    B, H, Dk, Dv = S.shape
    dt = k.dtype
    _need(q, "q", dev, dt, (B, H, Dk)); _need(k, "k", dev, dt, (B, H, Dk)); _need(v, "v", dev, dt, (B, H, Dv))
    _need(eta, "eta", dev, torch.float32, (B, H)); _need(g, "g", dev, torch.float32, (B, H))
    _need(S, "S", dev, torch.float32, (B, H, Dk, Dv))
    if o is None:
        o = torch.empty(B, H, Dv, device=dev, dtype=out_dtype)
    _need(o, "o", dev, None, (B, H, Dv))
    st = lib().kla_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(eta), _ptr(g), float(eps), _ptr(S), _ptr(o),
                               B, H, Dk, Dv, _in_code(k, beta), _dtype_code(o), _stream(dev, stream))
    _check(st, "kla_decode_step")
    return o


def chunk_fwd_diag(q, k, v, eta, g, eps=1e-6, S0=None, *, o=None, S_T=None, out_dtype=torch.float32,
                   stream=None, beta="kaczmarz", workspace=None, fused=False):
    """Prefill with diagonal (per-key-channel) gating (Appendix A.5, B.5): g is [B,T,H,Dk] fp32,
    the decay of token t is Diag(exp(g_t)).  Other arguments as chunk_fwd.  The split path's
    workspace (kla_chunk_fwd_diag_workspace) is allocated here unless given; fused=True passes
    none (the one-kernel path).  Returns (o, S_T)."""
    dev = k.device
    B, T, H, Dk = k.shape
    Dv = v.shape[-1]
    dt = k.dtype
    _need(q, "q", dev, dt, (B, T, H, Dk)); _need(k, "k", dev, dt); _need(v, "v", dev, dt, (B, T, H, Dv))
    _need(eta, "eta", dev, torch.float32, (B, T, H)); _need(g, "g", dev, torch.float32, (B, T, H, Dk))
    _need(S0, "S0", dev, torch.float32, (B, H, Dk, Dv))
    if o is None:
        o = torch.empty(B, T, H, Dv, device=dev, dtype=out_dtype)
    _need(o, "o", dev, None, (B, T, H, Dv))
    if S_T is None:
        S_T = torch.empty(B, H, Dk, Dv, device=dev, dtype=torch.float32)
    _need(S_T, "S_T", dev, torch.float32, (B, H, Dk, Dv))
    L = lib()
    need = 0 if fused else L.kla_chunk_fwd_diag_workspace(B, T, H, Dk, Dv, CHUNK, _dtype_code(k))
    if need > 0 and (workspace is None or workspace.numel() < need):
        workspace = torch.empty(need, device=dev, dtype=torch.uint8)
    ws_ptr, ws_n = (_ptr(workspace), workspace.numel()) if need > 0 else (None, 0)
    st = L.kla_chunk_fwd_diag(_ptr(q), _ptr(k), _ptr(v), _ptr(eta), _ptr(g), float(eps), _ptr(S0), _ptr(o),
                              _ptr(S_T), B, T, H, Dk, Dv, CHUNK, _in_code(k, beta), _dtype_code(o), ws_ptr, ws_n,
                              _stream(dev, stream))
    _check(st, "kla_chunk_fwd_diag")
    return o, S_T


def chunk_bwd_diag(q, k, v, eta, g, dO, eps=1e-6, S0=None, dS_T=None, *, workspace=None,
                   out_dtype=torch.float32, stream=None, beta="kaczmarz"):
    """Gradients of chunk_fwd_diag (dg is [B,T,H,Dk]).  Returns dict(dq, dk, dv, deta, dg, dS0)."""
    dev = k.device
    B, T, H, Dk = k.shape
    Dv = v.shape[-1]
    dt = k.dtype
    _need(q, "q", dev, dt, (B, T, H, Dk)); _need(k, "k", dev, dt); _need(v, "v", dev, dt, (B, T, H, Dv))
    _need(eta, "eta", dev, torch.float32, (B, T, H)); _need(g, "g", dev, torch.float32, (B, T, H, Dk))
    _need(S0, "S0", dev, torch.float32, (B, H, Dk, Dv)); _need(dO, "dO", dev, dt, (B, T, H, Dv))
    _need(dS_T, "dS_T", dev, torch.float32, (B, H, Dk, Dv))
    out = dict(dq=torch.empty(q.shape, device=dev, dtype=out_dtype),
               dk=torch.empty(k.shape, device=dev, dtype=out_dtype),
               dv=torch.empty(v.shape, device=dev, dtype=out_dtype),
               deta=torch.empty_like(eta), dg=torch.empty_like(g),
               dS0=torch.empty(B, H, Dk, Dv, device=dev, dtype=torch.float32))
    L = lib()
    need = L.kla_chunk_bwd_diag_workspace(B, T, H, Dk, Dv, CHUNK, _dtype_code(k))
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 16), device=dev, dtype=torch.uint8)
    st = L.kla_chunk_bwd_diag(_ptr(q), _ptr(k), _ptr(v), _ptr(eta), _ptr(g), float(eps), _ptr(S0), _ptr(dO),
                              _ptr(dS_T), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["deta"]),
                              _ptr(out["dg"]), _ptr(out["dS0"]), B, T, H, Dk, Dv, CHUNK, _in_code(k, beta),
                              _dtype_code(out_dtype), _ptr(workspace), workspace.numel(), _stream(dev, stream))
    _check(st, "kla_chunk_bwd_diag")
    return out


def decode_step_diag(q, k, v, eta, g, S, eps=1e-6, *, o=None, out_dtype=torch.float32, stream=None,
                     beta="kaczmarz"):
    """One decode token with diagonal gating: g is [B,H,Dk] fp32; otherwise as decode_step."""
    dev = S.device
    B, H, Dk, Dv = S.shape
    dt = k.dtype
    _need(q, "q", dev, dt, (B, H, Dk)); _need(k, "k", dev, dt, (B, H, Dk)); _need(v, "v", dev, dt, (B, H, Dv))
    _need(eta, "eta", dev, torch.float32, (B, H)); _need(g, "g", dev, torch.float32, (B, H, Dk))
    _need(S, "S", dev, torch.float32, (B, H, Dk, Dv))
    if o is None:
        o = torch.empty(B, H, Dv, device=dev, dtype=out_dtype)
    _need(o, "o", dev, None, (B, H, Dv))
    st = lib().kla_decode_step_diag(_ptr(q), _ptr(k), _ptr(v), _ptr(eta), _ptr(g), float(eps), _ptr(S), _ptr(o),
                                    B, H, Dk, Dv, _in_code(k, beta), _dtype_code(o), _stream(dev, stream))
    _check(st, "kla_decode_step_diag")
    return o


def gate_prologue(x, W, bias, q=None, *, stream=None):
    """Gates of every head from the token vectors (section 3.3): x [..., D], W [2H, D] (same
    dtype, bf16 or fp32), bias [2H] fp32 -> eta = sigmoid(x W_eta^T + b_eta), g = -softplus(x W_g^T
    + b_g), both [..., H] fp32; with q [..., H, Dk] also qhat = q / ||q|| (Algorithm 1's readout).
    Returns (eta, g) or (eta, g, qhat)."""
    dev = x.device
    D = x.shape[-1]
    lead = tuple(x.shape[:-1])
    N = int(torch.tensor(lead).prod().item()) if lead else 1
    H = W.shape[0] // 2
    dt = x.dtype
    _need(x, "x", dev, dt); _need(W, "W", dev, dt, (2 * H, D)); _need(bias, "bias", dev, torch.float32, (2 * H,))
    Dk = 0
    qhat = None
    if q is not None:
        Dk = q.shape[-1]
        _need(q, "q", dev, dt, lead + (H, Dk))
        qhat = torch.empty_like(q)
    eta = torch.empty(lead + (H,), device=dev, dtype=torch.float32)
    g = torch.empty(lead + (H,), device=dev, dtype=torch.float32)
    st = lib().kla_gate_prologue(_ptr(x), _ptr(W), _ptr(bias), _ptr(q), _ptr(eta), _ptr(g), _ptr(qhat), N, D, H,
                                 Dk, _dtype_code(x), _stream(dev, stream))
    _check(st, "kla_gate_prologue")
    return (eta, g) if q is None else (eta, g, qhat)


def gate_prologue_bwd(x, W, eta, g, deta, dg, q=None, dqhat=None, *, stream=None):
    """Backward of gate_prologue from its outputs (eta, g) and the upstream gradients.
    Returns dict(dx, dW, dbias) (+ dq when q is given), all fp32."""
    dev = x.device
    D = x.shape[-1]
    lead = tuple(x.shape[:-1])
    N = int(torch.tensor(lead).prod().item()) if lead else 1
    H = W.shape[0] // 2
    dt = x.dtype
    _need(x, "x", dev, dt); _need(W, "W", dev, dt, (2 * H, D))
    for t, n in ((eta, "eta"), (g, "g"), (deta, "deta"), (dg, "dg")):
        _need(t, n, dev, torch.float32, lead + (H,))
    Dk = 0
    out = dict(dx=torch.empty(lead + (D,), device=dev, dtype=torch.float32),
               dW=torch.empty(2 * H, D, device=dev, dtype=torch.float32),
               dbias=torch.empty(2 * H, device=dev, dtype=torch.float32))
    if q is not None:
        Dk = q.shape[-1]
        _need(q, "q", dev, dt, lead + (H, Dk)); _need(dqhat, "dqhat", dev, torch.float32, lead + (H, Dk))
        out["dq"] = torch.empty(lead + (H, Dk), device=dev, dtype=torch.float32)
    L = lib()
    ws = torch.empty(max(L.kla_gate_prologue_bwd_workspace(N, D, H), 16), device=dev, dtype=torch.uint8)
    st = L.kla_gate_prologue_bwd(_ptr(x), _ptr(W), _ptr(eta), _ptr(g), _ptr(q), _ptr(deta), _ptr(dg), _ptr(dqhat),
                                 _ptr(out["dx"]), _ptr(out["dW"]), _ptr(out["dbias"]), _ptr(out.get("dq")), N, D,
                                 H, Dk, _dtype_code(x), _ptr(ws), ws.numel(), _stream(dev, stream))
    _check(st, "kla_gate_prologue_bwd")
    return out


def debug_inject_wait_timeout():
    """Failure injection for tests: the next decode_step's kernel lets its first bounded wait
    expire (nothing is stored), so check_device_error then raises KLAError(KLA_ERR_TIMEOUT)."""
    lib().kla_debug_inject_wait_timeout()


def check_device_error(stream=None, device=None):
    """Synchronise the stream and raise KLAError if a kernel gave up on a bounded wait."""
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    _check(lib().kla_check_device_error(_stream(dev, stream)), "kla_check_device_error")
