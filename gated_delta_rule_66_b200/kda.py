"""Thin Python binding of libkda.so (include/kda.h).

Argument marshalling only: every step of the recurrence runs in the CUDA
kernels behind the C ABI.  Tensors must be CUDA, contiguous and of the
documented dtypes; outputs are allocated here with torch (device memory is
torch's job) and the call is enqueued on torch's current stream.  There is no
CPU fallback: if the compiled library is missing the import fails.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libkda.so")

KDA_DTYPE_FP32 = 0
KDA_DTYPE_BF16 = 1
KDA_BWD_STATES_FROM_FWD = 1
CHUNK = 32  # chunk length of the library's chunked kernels (workspace layout)

SYMBOLS = ("kda_last_error", "kda_device_status", "kda_fwd_workspace_bytes", "kda_fwd_scratch_bytes",
           "kda_bwd_workspace_bytes", "kda_fwd", "kda_fwd_varlen_workspace_bytes", "kda_fwd_varlen",
           "kda_bwd_varlen_workspace_bytes", "kda_bwd_varlen", "kda_decode_step", "kda_bwd",
           "kda_fwd_prep_workspace_bytes", "kda_fwd_prep", "kda_short_conv", "kda_decode_token",
           "kda_fwd_erase", "kda_fwd_erase_workspace_bytes", "kda_set_wait_polls")


class KdaError(RuntimeError):
    """A non-zero status from the KDA library, with its message."""

    def __init__(self, fn, code, msg):
        super().__init__(f"{fn} failed with status {code}: {msg}")
        self.code = code


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"{_LIB_PATH} is missing: build it with `python -m gated_delta_rule_66_b200.build` "
            "(the KDA library has no CPU fallback)")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, f, i, sz = ctypes.c_void_p, ctypes.c_float, ctypes.c_int, ctypes.c_size_t
    lib.kda_last_error.restype = ctypes.c_char_p
    lib.kda_last_error.argtypes = []
    lib.kda_device_status.restype = i
    lib.kda_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint)]
    lib.kda_set_wait_polls.restype = i
    lib.kda_set_wait_polls.argtypes = [ctypes.c_uint]
    lib.kda_fwd_workspace_bytes.restype = sz
    lib.kda_fwd_workspace_bytes.argtypes = [i, i, i, i, i]
    lib.kda_fwd_scratch_bytes.restype = sz
    lib.kda_fwd_scratch_bytes.argtypes = [i, i, i, i, i]
    lib.kda_bwd_workspace_bytes.restype = sz
    lib.kda_bwd_workspace_bytes.argtypes = [i, i, i, i, i, i]
    lib.kda_fwd.restype = i
    lib.kda_fwd.argtypes = [vp, vp, vp, vp, vp, vp, f, i, i, i, i, i, i, i, vp, vp, vp, sz, vp]
    lib.kda_fwd_varlen_workspace_bytes.restype = sz
    lib.kda_fwd_varlen_workspace_bytes.argtypes = [ctypes.POINTER(ctypes.c_int), i, i, i, i]
    lib.kda_fwd_varlen.restype = i
    lib.kda_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, f, ctypes.POINTER(ctypes.c_int), i, i, i, i, i, i,
                                   vp, vp, vp, sz, vp]
    lib.kda_bwd_varlen_workspace_bytes.restype = sz
    lib.kda_bwd_varlen_workspace_bytes.argtypes = [ctypes.POINTER(ctypes.c_int), i, i, i, i, i]
    lib.kda_bwd_varlen.restype = i
    lib.kda_bwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, f, ctypes.POINTER(ctypes.c_int), i, i, i, i, i,
                                   i, vp, vp, vp, vp, vp, vp, vp, sz, i, vp]
    lib.kda_decode_step.restype = i
    lib.kda_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, f, i, i, i, i, i, i, vp, vp]
    lib.kda_bwd.restype = i
    lib.kda_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, f, i, i, i, i, i, i, i,
                            vp, vp, vp, vp, vp, vp, vp, sz, i, vp]
    lib.kda_fwd_prep_workspace_bytes.restype = sz
    lib.kda_fwd_prep_workspace_bytes.argtypes = [i, i, i, i, i, i, i]
    lib.kda_fwd_prep.restype = i
    lib.kda_fwd_prep.argtypes = [vp, vp, vp, vp, vp, vp, f, vp, vp, f, vp, f, i, i, i, i, i, i, i, vp, vp, vp, sz,
                                 vp]
    lib.kda_short_conv.restype = i
    lib.kda_short_conv.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, vp, vp, vp, vp]
    lib.kda_decode_token.restype = i
    lib.kda_decode_token.argtypes = [vp, vp, vp, vp, vp, vp, i, vp, vp, vp, f, vp, vp, f, vp, f, i, i, i, i, i, i,
                                     vp, vp]
    lib.kda_fwd_erase.restype = i
    lib.kda_fwd_erase.argtypes = [vp, vp, vp, vp, vp, vp, f, i, i, i, i, i, i, i, vp, vp, vp, sz, vp]
    lib.kda_fwd_erase_workspace_bytes.restype = sz
    lib.kda_fwd_erase_workspace_bytes.argtypes = [i, i, i, i, i, i]
    return lib


_lib = _load()


def library():
    """The loaded ctypes handle of libkda.so (raw C-ABI access)."""
    return _lib


def _check(fn, rc):
    if rc != 0:
        raise KdaError(fn, rc, _lib.kda_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(t):
    if t.dtype == torch.float32:
        return KDA_DTYPE_FP32
    if t.dtype == torch.bfloat16:
        return KDA_DTYPE_BF16
    raise TypeError(f"q/k/v must be float32 or bfloat16, got {t.dtype}")


def _req(name, t, dtype=None, ndim=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.get_device() != torch.cuda.current_device():
        # the library launches on the calling thread's current device and on
        # its stream; a buffer of another GPU would be read across devices
        raise ValueError(f"{name} is on cuda:{t.get_device()} but the current CUDA device is "
                         f"cuda:{torch.cuda.current_device()} (use torch.cuda.device / set_device)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def device_status():
    """Reads and clears the kernels' device-side error bits on the current
    device (synchronises it); 0 means no kernel gave up on a bounded wait."""
    flags = ctypes.c_uint(0)
    _check("kda_device_status", _lib.kda_device_status(ctypes.byref(flags)))
    return int(flags.value)


def set_wait_polls(polls):
    """Test hook: probes of every bounded wait of the chunked tensor-core
    forward on the current device (0 restores the default).  A kernel whose
    wait runs out drains its own issued work, frees its tensor memory and sets
    bit 0 of device_status()."""
    _check("kda_set_wait_polls", _lib.kda_set_wait_polls(int(polls)))


def workspace_bytes(kind, B, T, H, HV, K, V):
    """Workspace bytes of ``kind`` = "fwd" (training forward: chunk states and
    records), "scratch" (forward scratch, no states) or "bwd"."""
    if kind == "fwd":
        return int(_lib.kda_fwd_workspace_bytes(B, T, HV, K, V))
    if kind == "scratch":
        return int(_lib.kda_fwd_scratch_bytes(B, T, HV, K, V))
    return int(_lib.kda_bwd_workspace_bytes(B, T, H, HV, K, V))


def fwd(q, k, v, g, beta, scale=None, initial_state=None, output_final_state=True,
        workspace=None, out=None, scratch=True):
    """Prefill forward.  Returns (o [B,T,HV,V] in v's dtype, S_T or None).

    q, k [B,T,H,K]; v [B,T,HV,V] (same dtype); g [B,T,HV,K], beta [B,T,HV] and
    initial_state [B,HV,K,V] float32.  ``workspace`` (a uint8 CUDA tensor of
    at least workspace_bytes("fwd", ...)) receives the chunk states for a
    later ``bwd(..., workspace=..., states_from_fwd=True)``.  Without one,
    ``scratch`` lets the library use a fresh scratch allocation of
    workspace_bytes("scratch", ...) (bf16 shapes that have a two-kernel
    forward); ``scratch=False`` passes no workspace at all.
    """
    B, T, H, K = q.shape
    HV, V = v.shape[2], v.shape[3]
    scale = 1.0 / math.sqrt(K) if scale is None else float(scale)
    dt = q.dtype
    for n, t in (("q", q), ("k", k), ("v", v)):
        _req(n, t, dt, 4)
    _req("g", g, torch.float32, 4)
    _req("beta", beta, torch.float32, 3)
    _req("initial_state", initial_state, torch.float32, 4)
    _req("workspace", workspace)
    o = torch.empty(B, T, HV, V, dtype=dt, device=q.device) if out is None else out
    _req("out", o, dt, 4)
    S_T = torch.empty(B, HV, K, V, dtype=torch.float32, device=q.device) if output_final_state else None
    if workspace is None and scratch:
        need = int(_lib.kda_fwd_scratch_bytes(B, T, HV, K, V))
        if need:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = _lib.kda_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(initial_state), scale,
                      B, T, H, HV, K, V, _dtype_code(q), _ptr(o), _ptr(S_T), _ptr(workspace),
                      ws_bytes, _stream())
    _check("kda_fwd", rc)
    return o, S_T


def _cu_array(cu_seqlens):
    cu = [int(x) for x in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
    return (ctypes.c_int * len(cu))(*cu), len(cu) - 1


def fwd_varlen(q, k, v, g, beta, cu_seqlens, scale=None, initial_state=None, output_final_state=True,
               workspace=None, out=None):
    """Packed variable-length prefill.  q, k [T,H,K], v [T,HV,V] bf16, g [T,HV,K]
    and beta [T,HV] float32 hold N sequences back to back; ``cu_seqlens`` (a
    host list or CPU tensor of N + 1 offsets) marks them.  initial_state
    [N,HV,K,V] float32.  Returns (o [T,HV,V], S_T [N,HV,K,V] or None).
    ``workspace`` defaults to a fresh allocation of kda_fwd_varlen_workspace_bytes.
    """
    T, H, K = q.shape
    HV, V = v.shape[1], v.shape[2]
    cu, N = _cu_array(cu_seqlens)
    scale = 1.0 / math.sqrt(K) if scale is None else float(scale)
    dt = q.dtype
    for n, t in (("q", q), ("k", k), ("v", v)):
        _req(n, t, dt, 3)
    _req("g", g, torch.float32, 3)
    _req("beta", beta, torch.float32, 2)
    _req("initial_state", initial_state, torch.float32, 4)
    if workspace is None:
        need = int(_lib.kda_fwd_varlen_workspace_bytes(cu, N, HV, K, V))
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _req("workspace", workspace)
    o = torch.empty(T, HV, V, dtype=dt, device=q.device) if out is None else out
    _req("out", o, dt, 3)
    S_T = torch.empty(N, HV, K, V, dtype=torch.float32, device=q.device) if output_final_state else None
    rc = _lib.kda_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(initial_state), scale, cu, N,
                             H, HV, K, V, _dtype_code(q), _ptr(o), _ptr(S_T), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream())
    _check("kda_fwd_varlen", rc)
    return o, S_T


def varlen_workspace_bytes(kind, cu_seqlens, H, HV, K, V):
    """Workspace bytes for packed sequences: "fwd" (two-kernel forward scratch)
    or "bwd" (the training workspace shared by fwd_varlen and bwd_varlen)."""
    cu, N = _cu_array(cu_seqlens)
    if kind == "fwd":
        return int(_lib.kda_fwd_varlen_workspace_bytes(cu, N, HV, K, V))
    return int(_lib.kda_bwd_varlen_workspace_bytes(cu, N, H, HV, K, V))


def bwd_varlen(q, k, v, g, beta, dO, cu_seqlens, scale=None, initial_state=None, dS_T=None, workspace=None,
               states_from_fwd=False):
    """Backward of fwd_varlen.  Returns (dq, dk, dv, dg, dbeta, dS0 [N,HV,K,V]).
    With ``states_from_fwd`` the ``workspace`` (of varlen_workspace_bytes("bwd"))
    must have gone through fwd_varlen on the same inputs."""
    T, H, K = q.shape
    HV, V = v.shape[1], v.shape[2]
    cu, N = _cu_array(cu_seqlens)
    scale = 1.0 / math.sqrt(K) if scale is None else float(scale)
    dt = q.dtype
    for n, t in (("q", q), ("k", k), ("v", v), ("dO", dO)):
        _req(n, t, dt, 3)
    _req("g", g, torch.float32, 3)
    _req("beta", beta, torch.float32, 2)
    _req("initial_state", initial_state, torch.float32, 4)
    _req("dS_T", dS_T, torch.float32, 4)
    need = int(_lib.kda_bwd_varlen_workspace_bytes(cu, N, H, HV, K, V))
    if workspace is None:
        if states_from_fwd:
            raise ValueError("states_from_fwd needs the workspace given to fwd_varlen")
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _req("workspace", workspace)
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    dg = torch.empty_like(g)
    dbeta = torch.empty_like(beta)
    dS0 = torch.empty(N, HV, K, V, dtype=torch.float32, device=q.device)
    rc = _lib.kda_bwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(initial_state), _ptr(dO),
                             _ptr(dS_T), scale, cu, N, H, HV, K, V, _dtype_code(q), _ptr(dq), _ptr(dk), _ptr(dv),
                             _ptr(dg), _ptr(dbeta), _ptr(dS0), _ptr(workspace),
                             workspace.numel() * workspace.element_size(),
                             KDA_BWD_STATES_FROM_FWD if states_from_fwd else 0, _stream())
    _check("kda_bwd_varlen", rc)
    return dq, dk, dv, dg, dbeta, dS0


def decode_step(q, k, v, g, beta, state, scale=None, out=None):
    """One decode token; ``state`` [B,HV,K,V] float32 is updated in place.

    q, k [B,H,K]; v [B,HV,V] (same dtype); g [B,HV,K], beta [B,HV] float32.
    Returns o [B,HV,V] in v's dtype.
    """
    B, H, K = q.shape
    HV, V = v.shape[1], v.shape[2]
    scale = 1.0 / math.sqrt(K) if scale is None else float(scale)
    dt = q.dtype
    for n, t in (("q", q), ("k", k), ("v", v)):
        _req(n, t, dt, 3)
    _req("g", g, torch.float32, 3)
    _req("beta", beta, torch.float32, 2)
    _req("state", state, torch.float32, 4)
    o = torch.empty(B, HV, V, dtype=dt, device=q.device) if out is None else out
    _req("out", o, dt, 3)
    rc = _lib.kda_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state), scale,
                              B, H, HV, K, V, _dtype_code(q), _ptr(o), _stream())
    _check("kda_decode_step", rc)
    return o


def bwd(q, k, v, g, beta, dO, scale=None, initial_state=None, dS_T=None, workspace=None,
        states_from_fwd=False, want_dS0=True):
    """Backward.  Returns (dq, dk, dv, dg, dbeta, dS0 or None).

    dq, dk [B,T,H,K] and dv [B,T,HV,V] in the input dtype; dg, dbeta, dS0
    float32.  ``workspace`` defaults to a fresh allocation of
    workspace_bytes("bwd", ...); pass the tensor given to ``fwd`` together
    with ``states_from_fwd=True`` to reuse its chunk states.
    """
    B, T, H, K = q.shape
    HV, V = v.shape[2], v.shape[3]
    scale = 1.0 / math.sqrt(K) if scale is None else float(scale)
    dt = q.dtype
    for n, t in (("q", q), ("k", k), ("v", v), ("dO", dO)):
        _req(n, t, dt, 4)
    _req("g", g, torch.float32, 4)
    _req("beta", beta, torch.float32, 3)
    _req("initial_state", initial_state, torch.float32, 4)
    _req("dS_T", dS_T, torch.float32, 4)
    need = workspace_bytes("bwd", B, T, H, HV, K, V)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _req("workspace", workspace)
    dev = q.device
    dq = torch.empty(B, T, H, K, dtype=dt, device=dev)
    dk = torch.empty(B, T, H, K, dtype=dt, device=dev)
    dv = torch.empty(B, T, HV, V, dtype=dt, device=dev)
    dg = torch.empty(B, T, HV, K, dtype=torch.float32, device=dev)
    dbeta = torch.empty(B, T, HV, dtype=torch.float32, device=dev)
    dS0 = torch.empty(B, HV, K, V, dtype=torch.float32, device=dev) if want_dS0 else None
    rc = _lib.kda_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(initial_state),
                      _ptr(dO), _ptr(dS_T), scale, B, T, H, HV, K, V, _dtype_code(q),
                      _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg), _ptr(dbeta), _ptr(dS0),
                      _ptr(workspace), workspace.numel() * workspace.element_size(),
                      KDA_BWD_STATES_FROM_FWD if states_from_fwd else 0, _stream())
    _check("kda_bwd", rc)
    return dq, dk, dv, dg, dbeta, dS0


# ----------------------------------------------------------------------------- preparation
L2_EPS = 1e-6  # KDA_L2_EPS: q/k row normalisation


def prep_workspace_bytes(B, T, H, HV, K, V, dtype=torch.bfloat16):
    """Scratch bytes with which ``fwd_prep`` runs its fastest path for every shape."""
    code = KDA_DTYPE_BF16 if dtype == torch.bfloat16 else KDA_DTYPE_FP32
    return int(_lib.kda_fwd_prep_workspace_bytes(B, T, H, HV, K, V, code))


def fwd_prep(q, k, v, z, A_log, dt_bias, beta_logit, gate_lower_bound=-5.0, scale=None, initial_state=None,
             out_gate=None, out_eps=L2_EPS, output_final_state=True, workspace=True):
    """Prefill from the raw projections (the preparation fused into the forward).

    q, k [B,T,H,K] (before L2 normalisation), v [B,T,HV,V], z [B,T,HV,K] (gate
    pre-activation) and out_gate [B,T,HV,V] (or None) share one dtype;
    A_log [HV], dt_bias [HV,K], beta_logit [B,T,HV] float32.
    ``gate_lower_bound`` < 0 selects the bounded gate, 0 the softplus form.
    ``workspace``: True allocates the scratch, None runs without, or a
    uint8 tensor.  Returns (o [B,T,HV,V], S_T or None).
    """
    B, T, H, K = q.shape
    HV, V = v.shape[2], v.shape[3]
    scale = 1.0 / math.sqrt(K) if scale is None else float(scale)
    dt = q.dtype
    for n, t in (("q", q), ("k", k), ("v", v), ("z", z)):
        _req(n, t, dt, 4)
    _req("out_gate", out_gate, dt, 4)
    _req("A_log", A_log, torch.float32, 1)
    _req("dt_bias", dt_bias, torch.float32, 2)
    _req("beta_logit", beta_logit, torch.float32, 3)
    _req("initial_state", initial_state, torch.float32, 4)
    o = torch.empty(B, T, HV, V, dtype=dt, device=q.device)
    S_T = torch.empty(B, HV, K, V, dtype=torch.float32, device=q.device) if output_final_state else None
    if workspace is True:
        n = prep_workspace_bytes(B, T, H, HV, K, V, dt)
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device) if n else None
    rc = _lib.kda_fwd_prep(_ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(A_log), _ptr(dt_bias), float(gate_lower_bound),
                           _ptr(beta_logit), _ptr(out_gate), float(out_eps), _ptr(initial_state), scale,
                           B, T, H, HV, K, V, _dtype_code(q), _ptr(o), _ptr(S_T), _ptr(workspace),
                           0 if workspace is None else workspace.numel(), _stream())
    _check("kda_fwd_prep", rc)
    return o, S_T


def short_conv(xq, xk, xv, w, state_in=None, output_state=True):
    """The short causal convolution with SiLU over whole sequences.

    xq, xk [B,T,H,K], xv [B,T,HV,V] (one dtype); w [2HK + HV V, W] float32;
    state_in [B, 2HK + HV V, W] float32 or None.  Returns (q, k, v, state_out
    or None).
    """
    B, T, H, K = xq.shape
    HV, V = xv.shape[2], xv.shape[3]
    W = w.shape[1]
    dt = xq.dtype
    for n, t in (("xq", xq), ("xk", xk), ("xv", xv)):
        _req(n, t, dt, 4)
    _req("w", w, torch.float32, 2)
    _req("state_in", state_in, torch.float32, 3)
    q, k, v = torch.empty_like(xq), torch.empty_like(xk), torch.empty_like(xv)
    st = torch.empty(B, w.shape[0], W, dtype=torch.float32, device=xq.device) if output_state else None
    rc = _lib.kda_short_conv(_ptr(xq), _ptr(xk), _ptr(xv), _ptr(w), _ptr(state_in), _ptr(st), B, T, H, HV, K, V,
                             W, _dtype_code(xq), _ptr(q), _ptr(k), _ptr(v), _stream())
    _check("kda_short_conv", rc)
    return q, k, v, st


def decode_token(xq, xk, xv, conv_w, conv_state, z, A_log, dt_bias, beta_logit, state, gate_lower_bound=-5.0,
                 scale=None, out_gate=None, out_eps=L2_EPS, conv_out=None):
    """One decode token from the raw projections; ``state`` [B,HV,K,V] and
    (unless ``conv_out`` is given) ``conv_state`` [B, 2HK + HV V, W] are
    updated in place (in place needs H == HV; pass ``conv_out`` otherwise).

    xq, xk [B,H,K], xv [B,HV,V], z [B,HV,K], out_gate [B,HV,V] or None (one
    dtype); conv_w [2HK + HV V, W], A_log [HV], dt_bias [HV,K], beta_logit
    [B,HV] float32.  Returns o [B,HV,V].
    """
    B, H, K = xq.shape
    HV, V = xv.shape[1], xv.shape[2]
    scale = 1.0 / math.sqrt(K) if scale is None else float(scale)
    dt = xq.dtype
    for n, t in (("xq", xq), ("xk", xk), ("xv", xv), ("z", z)):
        _req(n, t, dt, 3)
    _req("out_gate", out_gate, dt, 3)
    _req("conv_w", conv_w, torch.float32, 2)
    _req("conv_state", conv_state, torch.float32, 3)
    _req("conv_out", conv_out, torch.float32, 3)
    _req("A_log", A_log, torch.float32, 1)
    _req("dt_bias", dt_bias, torch.float32, 2)
    _req("beta_logit", beta_logit, torch.float32, 2)
    _req("state", state, torch.float32, 4)
    o = torch.empty(B, HV, V, dtype=dt, device=xq.device)
    out_win = conv_state if conv_out is None else conv_out
    rc = _lib.kda_decode_token(_ptr(xq), _ptr(xk), _ptr(xv), _ptr(conv_w), _ptr(conv_state), _ptr(out_win),
                               conv_w.shape[1], _ptr(z), _ptr(A_log), _ptr(dt_bias), float(gate_lower_bound),
                               _ptr(beta_logit), _ptr(out_gate), float(out_eps), _ptr(state), scale, B, H, HV, K, V,
                               _dtype_code(xq), _ptr(o), _stream())
    _check("kda_decode_token", rc)
    return o


# ----------------------------------------------------------------------------- erase/write variant
def fwd_erase(q, k, e, z, g, scale=None, initial_state=None, output_final_state=True, scratch=True):
    """Prefill of the asymmetric erase/write delta recurrence.

    q [B,T,HQ,K]; k (write), e (erase) [B,T,HV,K]; z [B,T,HV,V] (one dtype);
    g [B,T,HV,K] float32; HQ a multiple of HV (query head hq reads state head
    hq // (HQ // HV)).  Returns (o [B,T,HQ,V], S_T [B,HV,K,V] or None).
    ``scratch`` gives the library a fresh workspace of
    kda_fwd_erase_workspace_bytes (the two-kernel path); ``scratch=False``
    runs the single-kernel path.
    """
    B, T, HQ, K = q.shape
    HV, V = k.shape[2], z.shape[3]
    scale = 1.0 / math.sqrt(K) if scale is None else float(scale)
    dt = q.dtype
    for n, t in (("q", q), ("k", k), ("e", e), ("z", z)):
        _req(n, t, dt, 4)
    _req("g", g, torch.float32, 4)
    _req("initial_state", initial_state, torch.float32, 4)
    o = torch.empty(B, T, HQ, V, dtype=dt, device=q.device)
    S_T = torch.empty(B, HV, K, V, dtype=torch.float32, device=q.device) if output_final_state else None
    ws = None
    if scratch:
        need = int(_lib.kda_fwd_erase_workspace_bytes(B, T, HQ, HV, K, V))
        if need:
            ws = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if ws is None else ws.numel()
    rc = _lib.kda_fwd_erase(_ptr(q), _ptr(k), _ptr(e), _ptr(z), _ptr(g), _ptr(initial_state), scale, B, T, HQ, HV,
                            K, V, _dtype_code(q), _ptr(o), _ptr(S_T), _ptr(ws), ws_bytes, _stream())
    _check("kda_fwd_erase", rc)
    return o, S_T
