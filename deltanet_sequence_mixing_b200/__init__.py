"""B200 (sm_100a) delta-rule sequence mixing: Python binding of the C ABI.

The functions below carry the names of the C entry points in
``include/deltanet.h`` and only marshal arguments: torch supplies device
memory and the current stream, and every step of the computation runs in the
library's CUDA kernels.  There is no CPU fallback.

    o, S = deltanet_chunk_fwd(q, k, v, beta, alpha=None, S0=None, C=64, prestep=False)
    o    = deltanet_decode_step(q, k, v, beta, S, alpha=None, prestep=False)  # S in place
    o, S, z = linear_attn_fwd(q, k, v, S0=None, z0=None, C=64)
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import DeltaNetError, check, lib, status_string  # noqa: F401

__all__ = [
    "deltanet_chunk_fwd", "deltanet_chunk_fwd_host", "deltanet_decode_step", "linear_attn_fwd",
    "deltanet_chunk_bwd", "seq_segments",
    "workspace_for", "host_workspace_for",
    "deltanet_get_device_status", "deltanet_selftest_wait_timeout", "DeltaNetError",
]

_DT = {torch.float32: _lib.DN_F32, torch.bfloat16: _lib.DN_BF16}
_workspaces: dict = {}


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t, name, dtype=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    return t


def workspace_for(device, nbytes: int = 256) -> torch.Tensor:
    """A cleared device workspace of at least ``nbytes``, cached per device."""
    device = torch.device(device)
    ws = _workspaces.get(device)
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        check("deltanet_workspace_init",
              lib().deltanet_workspace_init(_ptr(ws), ws.numel(), _stream(device)))
        _workspaces[device] = ws
    return ws


def _ws_bytes(B, H, T, Dk, Dv, C, dt):
    n = lib().deltanet_workspace_bytes(B, H, T, Dk, Dv, C, dt)
    if n == 0:
        raise DeltaNetError("deltanet_workspace_bytes", _lib.DN_ERR_UNSUPPORTED)
    return n


def _options(prestep, alpha, per_dim_rank):
    opts = _lib.DN_OPT_PRESTEP if prestep else 0
    if alpha is not None and alpha.dim() == per_dim_rank:
        opts |= _lib.DN_OPT_GATE_PER_DIM
    return opts


def deltanet_chunk_fwd(q, k, v, beta, alpha=None, S0=None, C: int = 64, o=None, S_out=None,
                       workspace=None, prestep: bool = False, seq_split: bool = False):
    """Chunkwise DeltaNet forward.  q, k: (B,H,T,Dk); v: (B,H,T,Dv) (bf16 or f32);
    beta: (B,H,T) f32; alpha: (B,H,T) f32 (one decay per token) or (B,H,T,Dk)
    (one per key dimension); S0: (B,H,Dk,Dv) f32.  ``prestep``: q, k are raw
    projections and beta logits (silu + L2 normalise and sigmoid run inside).
    ``seq_split``: permission to run each sequence as segments side by side
    (DN_OPT_SEQ_SPLIT; see seq_segments).  Returns (o, S_out)."""
    _need(q, "q")
    dev, dtype = q.device, q.dtype
    if dtype not in _DT:
        raise TypeError(f"unsupported dtype {dtype}")
    for t, n in ((k, "k"), (v, "v")):
        _need(t, n, dtype, dev)
    _need(beta, "beta", torch.float32, dev)
    if alpha is not None:
        _need(alpha, "alpha", torch.float32, dev)
    if S0 is not None:
        _need(S0, "S0", torch.float32, dev)
    B, H, T, Dk = q.shape
    Dv = v.shape[-1]
    if o is None:
        o = torch.empty(B, H, T, Dv, dtype=dtype, device=dev)
    if S_out is None:
        S_out = torch.empty(B, H, Dk, Dv, dtype=torch.float32, device=dev)
    _need(o, "o", dtype, dev)
    _need(S_out, "S_out", torch.float32, dev)
    dt = _DT[dtype]
    opts = _options(prestep, alpha, 4) | (_lib.DN_OPT_SEQ_SPLIT if seq_split else 0)
    nb = lib().deltanet_workspace_bytes_ex(B, H, T, Dk, Dv, C, dt, opts)
    if nb == 0:
        raise DeltaNetError("deltanet_workspace_bytes_ex", _lib.DN_ERR_UNSUPPORTED)
    ws = workspace if workspace is not None else workspace_for(dev, nb)
    if opts == 0:
        check("deltanet_chunk_fwd", lib().deltanet_chunk_fwd(
            _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(alpha), _ptr(S0), _ptr(o), _ptr(S_out),
            B, H, T, Dk, Dv, C, dt, _ptr(ws), ws.numel(), _stream(dev)))
    else:
        check("deltanet_chunk_fwd_ex", lib().deltanet_chunk_fwd_ex(
            _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(alpha), _ptr(S0), _ptr(o), _ptr(S_out),
            B, H, T, Dk, Dv, C, dt, opts, _ptr(ws), ws.numel(), _stream(dev)))
    return o, S_out


def seq_segments(B, H, T, Dk, Dv, C=64, dtype=torch.bfloat16, prestep=False, per_dim=False,
                 seq_split=True) -> int:
    """Segments a deltanet_chunk_fwd call with these arguments runs on the
    current device (1: the sequence is not split)."""
    opts = (_lib.DN_OPT_PRESTEP if prestep else 0) | (_lib.DN_OPT_GATE_PER_DIM if per_dim else 0) | (
        _lib.DN_OPT_SEQ_SPLIT if seq_split else 0)
    return int(lib().deltanet_seq_segments(B, H, T, Dk, Dv, C, _DT[dtype], opts))


def deltanet_chunk_bwd(q, k, v, beta, dO, alpha=None, S0=None, dS_T=None, workspace=None):
    """Gradient of deltanet_chunk_fwd for the loss sum(dO * o) + sum(dS_T * S_T).
    Returns dict(dq, dk, dv, dbeta, dlog_alpha, dS0), float32 tensors
    (dlog_alpha is None when ungated)."""
    _need(q, "q")
    dev, dtype = q.device, q.dtype
    if dtype not in _DT:
        raise TypeError(f"unsupported dtype {dtype}")
    for t, n in ((k, "k"), (v, "v"), (dO, "dO")):
        _need(t, n, dtype, dev)
    _need(beta, "beta", torch.float32, dev)
    for t, n in ((alpha, "alpha"), (S0, "S0"), (dS_T, "dS_T")):
        if t is not None:
            _need(t, n, torch.float32, dev)
    B, H, T, Dk = q.shape
    Dv = v.shape[-1]
    f = dict(dtype=torch.float32, device=dev)
    out = dict(dq=torch.empty(B, H, T, Dk, **f), dk=torch.empty(B, H, T, Dk, **f),
               dv=torch.empty(B, H, T, Dv, **f), dbeta=torch.empty(B, H, T, **f),
               dlog_alpha=None if alpha is None else torch.empty(B, H, T, **f),
               dS0=torch.empty(B, H, Dk, Dv, **f))
    nb = lib().deltanet_chunk_bwd_workspace_bytes(B, H, T, Dk, Dv, _DT[dtype])
    if nb == 0:
        raise DeltaNetError("deltanet_chunk_bwd_workspace_bytes", _lib.DN_ERR_UNSUPPORTED)
    ws = workspace if workspace is not None else torch.empty(nb, dtype=torch.uint8, device=dev)
    check("deltanet_chunk_bwd", lib().deltanet_chunk_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(alpha), _ptr(S0), _ptr(dO), _ptr(dS_T),
        _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dbeta"]),
        _ptr(out["dlog_alpha"]), _ptr(out["dS0"]), B, H, T, Dk, Dv, _DT[dtype], _ptr(ws), ws.numel(),
        _stream(dev)))
    return out


def _need_host(t, name, dtype=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.is_cuda:
        raise ValueError(f"{name} must be a host tensor for the host-buffer call")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t


def host_workspace_for(device, B, H, T, Dk, Dv, C, dtype) -> torch.Tensor:
    """A device workspace for deltanet_chunk_fwd_host (cleared, not cached)."""
    device = torch.device(device)
    nb = lib().deltanet_host_workspace_bytes(B, H, T, Dk, Dv, C, _DT[dtype])
    if nb == 0:
        raise DeltaNetError("deltanet_host_workspace_bytes", _lib.DN_ERR_UNSUPPORTED)
    ws = torch.empty(nb, dtype=torch.uint8, device=device)
    check("deltanet_workspace_init", lib().deltanet_workspace_init(_ptr(ws), ws.numel(), _stream(device)))
    return ws


def deltanet_chunk_fwd_host(q, k, v, beta, alpha=None, S0=None, C: int = 64, o=None, S_out=None,
                            workspace=None, device=None):
    """deltanet_chunk_fwd on host tensors (page-locked for overlapped copies):
    the heads stream through the device in groups, copies overlapping the
    compute.  Asynchronous on the device's current stream: synchronize it
    before reading (o, S_out)."""
    _need_host(q, "q")
    dtype = q.dtype
    if dtype not in _DT:
        raise TypeError(f"unsupported dtype {dtype}")
    for t, n in ((k, "k"), (v, "v")):
        _need_host(t, n, dtype)
    _need_host(beta, "beta", torch.float32)
    for t, n in ((alpha, "alpha"), (S0, "S0")):
        if t is not None:
            _need_host(t, n, torch.float32)
    B, H, T, Dk = q.shape
    Dv = v.shape[-1]
    if o is None:
        o = torch.empty(B, H, T, Dv, dtype=dtype).pin_memory()
    if S_out is None:
        S_out = torch.empty(B, H, Dk, Dv, dtype=torch.float32).pin_memory()
    _need_host(o, "o", dtype)
    _need_host(S_out, "S_out", torch.float32)
    device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    if workspace is None:
        workspace = host_workspace_for(device, B, H, T, Dk, Dv, C, dtype)
    _need(workspace, "workspace", torch.uint8, device)
    with torch.cuda.device(device):
        check("deltanet_chunk_fwd_host", lib().deltanet_chunk_fwd_host(
            _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(alpha), _ptr(S0), _ptr(o), _ptr(S_out),
            B, H, T, Dk, Dv, C, _DT[dtype], _ptr(workspace), workspace.numel(), _stream(device)))
    return o, S_out


def linear_attn_fwd(q, k, v, S0=None, z0=None, C: int = 64, o=None, S_out=None, z_out=None,
                    workspace=None):
    """Chunkwise ELU+1 causal linear attention.  Returns (o, S_out, z_out)."""
    _need(q, "q")
    dev, dtype = q.device, q.dtype
    if dtype not in _DT:
        raise TypeError(f"unsupported dtype {dtype}")
    for t, n in ((k, "k"), (v, "v")):
        _need(t, n, dtype, dev)
    for t, n in ((S0, "S0"), (z0, "z0")):
        if t is not None:
            _need(t, n, torch.float32, dev)
    B, H, T, Dk = q.shape
    Dv = v.shape[-1]
    if o is None:
        o = torch.empty(B, H, T, Dv, dtype=dtype, device=dev)
    if S_out is None:
        S_out = torch.empty(B, H, Dk, Dv, dtype=torch.float32, device=dev)
    if z_out is None:
        z_out = torch.empty(B, H, Dk, dtype=torch.float32, device=dev)
    dt = _DT[dtype]
    nb = _ws_bytes(B, H, T, Dk, Dv, C, dt)
    ws = workspace if workspace is not None else workspace_for(dev, nb)
    check("linear_attn_fwd", lib().linear_attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(S0), _ptr(z0), _ptr(o), _ptr(S_out), _ptr(z_out),
        B, H, T, Dk, Dv, C, dt, _ptr(ws), ws.numel(), _stream(dev)))
    return o, S_out, z_out


def deltanet_decode_step(q, k, v, beta, S, alpha=None, o=None, prestep: bool = False):
    """One decode step.  q, k: (B,H,Dk); v: (B,H,Dv); beta: (B,H) f32; alpha:
    (B,H) f32 or (B,H,Dk) (one decay per key dimension); S: (B,H,Dk,Dv) f32,
    updated in place.  ``prestep``: q, k raw and beta logits.  Returns o (B,H,Dv)."""
    _need(q, "q")
    dev, dtype = q.device, q.dtype
    if dtype not in _DT:
        raise TypeError(f"unsupported dtype {dtype}")
    for t, n in ((k, "k"), (v, "v")):
        _need(t, n, dtype, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(S, "S", torch.float32, dev)
    if alpha is not None:
        _need(alpha, "alpha", torch.float32, dev)
    B, H, Dk = q.shape
    Dv = v.shape[-1]
    if o is None:
        o = torch.empty(B, H, Dv, dtype=dtype, device=dev)
    opts = _options(prestep, alpha, 3)
    if opts == 0:
        check("deltanet_decode_step", lib().deltanet_decode_step(
            _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(alpha), _ptr(S), _ptr(o),
            B, H, Dk, Dv, _DT[dtype], _stream(dev)))
    else:
        check("deltanet_decode_step_ex", lib().deltanet_decode_step_ex(
            _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(alpha), _ptr(S), _ptr(o),
            B, H, Dk, Dv, _DT[dtype], opts, _stream(dev)))
    return o


def deltanet_get_device_status(device=None, workspace=None) -> int:
    """Synchronise and return the sticky device status of ``workspace`` (or of the
    cached workspace of ``device``)."""
    device = torch.device(device if device is not None else "cuda")
    ws = workspace if workspace is not None else workspace_for(device)
    return lib().deltanet_get_device_status(_ptr(ws), _stream(device))


def deltanet_selftest_wait_timeout(wait_ns: int, workspace, device=None) -> int:
    """Launch the bounded-wait self test on ``workspace``; returns the launch status."""
    device = torch.device(device if device is not None else workspace.device)
    return lib().deltanet_selftest_wait_timeout(_ptr(workspace), workspace.numel(), int(wait_ns),
                                                _stream(device))


def reset_device_status(device=None, workspace=None) -> None:
    device = torch.device(device if device is not None else "cuda")
    ws = workspace if workspace is not None else workspace_for(device)
    check("deltanet_workspace_init",
          lib().deltanet_workspace_init(_ptr(ws), ws.numel(), _stream(device)))
