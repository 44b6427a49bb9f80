"""Float64 CPU oracle for the delta-rule sequence mixer (test infrastructure).

TEST INFRASTRUCTURE ONLY: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference arm of ``bench.py`` may import this package.  The
product library never loads it, and it never loads the product library.

* ``deltanet``     - the per-token delta rule (optionally gated, per-dimension
                     gated, or behind the layer's silu / L2 / sigmoid pre-step),
                     ``oracle.c``.
* ``deltanet_bwd`` - its gradient, the reverse sweep of the per-token loop, ``oracle.c``.
* ``linear_attn``  - ELU+1 causal linear attention, ``oracle.c``.
* ``chunk_form``   - the chunkwise WY form in numpy (see ``chunk_form.py``).

Inputs may be numpy arrays or CPU torch tensors; bfloat16 tensors are passed as
their bit patterns and widened exactly inside the C code.  Results are float64
numpy arrays.  Parity: pinned (``tests/test_oracle_pins.py``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import time

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

F32, BF16, F64 = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` next to it (plain gcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm", "-lpthread"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        vp, fp, dp, L, I = (ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                            ctypes.c_long, ctypes.c_int)
        lib.oracle_deltanet.argtypes = [vp, vp, vp, I, fp, fp, dp, dp, dp, L, L, L, L, L, I]
        lib.oracle_deltanet.restype = I
        lib.oracle_linear_attn.argtypes = [vp, vp, vp, I, dp, dp, dp, dp, dp, L, L, L, L, L, I]
        lib.oracle_linear_attn.restype = I
        lib.oracle_deltanet_ex.argtypes = [vp, vp, vp, I, fp, fp, dp, dp, dp, L, L, L, L, L, I, I]
        lib.oracle_deltanet_ex.restype = I
        lib.oracle_deltanet_bwd.argtypes = [vp, vp, vp, I, fp, fp, dp, dp, dp,
                                            dp, dp, dp, dp, dp, dp, L, L, L, L, L, I]
        lib.oracle_deltanet_bwd.restype = I
        _lib = lib
    return _lib


def _as_stored(x):
    """Return (contiguous numpy array of the stored bits, dtype code)."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), BF16
            if x.dtype == torch.float32:
                return x.numpy(), F32
            if x.dtype == torch.float64:
                return x.numpy(), F64
            raise TypeError(f"oracle inputs must be float32 or bfloat16, got {x.dtype}")
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.float64:
        return x, F64
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.uint16:
        return x, BF16
    raise TypeError(f"oracle inputs must be float32 or bfloat16 bits, got {x.dtype}")


def _f32(x):
    if x is None:
        return None
    try:
        import torch

        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().float().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(x, dtype=np.float32)


def _f64(x):
    if x is None:
        return None
    try:
        import torch

        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().double().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


PRESTEP, ALPHA_PER_DIM = 1, 2


def deltanet(q, k, v, beta, alpha=None, S0=None, nthreads: int = 0, prestep: bool = False):
    """Delta rule over (B,H,T,D) sequences; returns ``(o, S_out)`` in float64.

    Follows the direct per-token loop of "GPT-2 から Kimi K3 まで" (news.ainew.jp),
    section "DeltaNet (Parallelizing linear transformers with delta rule)", with
    the gate of the Gated DeltaNet paragraph of "How a Baseten Engineer Traced 7
    Years of Attention Mechanism Evolution" (decay first, then the delta write).

    ``alpha`` of shape (B,H,T) is the scalar gate; of shape (B,H,T,Dk) it is the
    per-dimension gate of the same page's KDA paragraph (row i of the state
    decays by alpha_t[i]).  ``prestep``: q and k are raw projections and beta
    holds logits; each token first takes the DeltaNet layer's maps of the
    section "DeltaNet (Fast weight programmers)": q, k <- normalize(silu(.)),
    beta <- sigmoid(beta).
    """
    qa, dt = _as_stored(q)
    ka, dtk = _as_stored(k)
    va, dtv = _as_stored(v)
    if not (dt == dtk == dtv):
        raise TypeError("q, k, v must share one dtype")
    B, H, T, Dk = qa.shape
    Dv = va.shape[-1]
    if ka.shape != (B, H, T, Dk) or va.shape != (B, H, T, Dv):
        raise ValueError("shape mismatch")
    b = _f32(beta).reshape(B, H, T)
    flags = PRESTEP if prestep else 0
    a = None
    if alpha is not None:
        a = _f32(alpha)
        if a.size == B * H * T * Dk and a.ndim == 4:
            flags |= ALPHA_PER_DIM
            a = a.reshape(B, H, T, Dk)
        else:
            a = a.reshape(B, H, T)
    s0 = None if S0 is None else _f64(S0).reshape(B, H, Dk, Dv)
    o = np.zeros((B, H, T, Dv), np.float64)
    S = np.zeros((B, H, Dk, Dv), np.float64)
    rc = _load().oracle_deltanet_ex(_ptr(qa), _ptr(ka), _ptr(va), dt, _ptr(b), _ptr(a), _ptr(s0),
                                    _ptr(o), _ptr(S), B, H, T, Dk, Dv, flags, nthreads)
    if rc != 0:
        raise RuntimeError(f"oracle_deltanet failed ({rc})")
    return o, S


def deltanet_bwd(q, k, v, beta, dO, alpha=None, S0=None, dS_T=None, nthreads: int = 0):
    """Gradient of the delta rule: the reverse sweep of the per-token loop (see
    ``oracle_deltanet_bwd`` in ``oracle.c``), in float64.

    The loss is ``sum(dO * o) + sum(dS_T * S_T)``.  Returns a dict with dq, dk
    (B,H,T,Dk), dv (B,H,T,Dv), dbeta (B,H,T), dalpha (B,H,T, or None when
    ungated) and dS0 (B,H,Dk,Dv).  q, k, v may be float64, float32 or bfloat16.
    """
    qa, dt = _as_stored(q)
    ka, dtk = _as_stored(k)
    va, dtv = _as_stored(v)
    if not (dt == dtk == dtv):
        raise TypeError("q, k, v must share one dtype")
    B, H, T, Dk = qa.shape
    Dv = va.shape[-1]
    b = _f32(beta).reshape(B, H, T)
    a = None if alpha is None else _f32(alpha).reshape(B, H, T)
    s0 = None if S0 is None else _f64(S0).reshape(B, H, Dk, Dv)
    do = _f64(dO).reshape(B, H, T, Dv)
    dst = None if dS_T is None else _f64(dS_T).reshape(B, H, Dk, Dv)
    out = dict(dq=np.zeros((B, H, T, Dk)), dk=np.zeros((B, H, T, Dk)), dv=np.zeros((B, H, T, Dv)),
               dbeta=np.zeros((B, H, T)), dalpha=None if a is None else np.zeros((B, H, T)),
               dS0=np.zeros((B, H, Dk, Dv)))
    rc = _load().oracle_deltanet_bwd(_ptr(qa), _ptr(ka), _ptr(va), dt, _ptr(b), _ptr(a), _ptr(s0),
                                     _ptr(do), _ptr(dst), _ptr(out["dq"]), _ptr(out["dk"]),
                                     _ptr(out["dv"]), _ptr(out["dbeta"]), _ptr(out["dalpha"]),
                                     _ptr(out["dS0"]), B, H, T, Dk, Dv, nthreads)
    if rc != 0:
        raise RuntimeError(f"oracle_deltanet_bwd failed ({rc})")
    return out


def linear_attn(q, k, v, S0=None, z0=None, nthreads: int = 0):
    """ELU+1 causal linear attention; returns ``(o, S_out, z_out)`` in float64.

    Follows the cached forward of "GPT-2 から Kimi K3 まで" (news.ainew.jp),
    section "Linear attention", one token at a time.
    """
    qa, dt = _as_stored(q)
    ka, _ = _as_stored(k)
    va, _ = _as_stored(v)
    B, H, T, Dk = qa.shape
    Dv = va.shape[-1]
    s0 = None if S0 is None else _f64(S0).reshape(B, H, Dk, Dv)
    z0_ = None if z0 is None else _f64(z0).reshape(B, H, Dk)
    o = np.zeros((B, H, T, Dv), np.float64)
    S = np.zeros((B, H, Dk, Dv), np.float64)
    z = np.zeros((B, H, Dk), np.float64)
    rc = _load().oracle_linear_attn(_ptr(qa), _ptr(ka), _ptr(va), dt, _ptr(s0), _ptr(z0_),
                                    _ptr(o), _ptr(S), _ptr(z), B, H, T, Dk, Dv, nthreads)
    if rc != 0:
        raise RuntimeError(f"oracle_linear_attn failed ({rc})")
    return o, S, z


def timed(fn, *args, **kw):
    """Run ``fn`` once and return (result, wall seconds)."""
    t0 = time.perf_counter()
    r = fn(*args, **kw)
    return r, time.perf_counter() - t0
