"""ctypes loader for ``libdeltanet_b200.so`` (the C ABI of include/deltanet.h).

Argument marshalling only: every step of the computation runs in the CUDA
library.  There is no CPU fallback; if the library is missing or cannot be
loaded, the first call raises.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdeltanet_b200.so")

DN_OK = 0
DN_ERR_INVALID_ARG = -1
DN_ERR_UNSUPPORTED = -2
DN_ERR_ALIGNMENT = -3
DN_ERR_CUDA = -4
DN_ERR_DEVICE_TIMEOUT = -5
DN_ERR_WORKSPACE = -6
DN_F32, DN_BF16 = 0, 1
DN_OPT_PRESTEP, DN_OPT_GATE_PER_DIM, DN_OPT_SEQ_SPLIT = 1, 2, 4

# Every symbol include/deltanet.h declares, with (restype, argtypes).
_vp, _sz, _i, _ll, _u = (ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_longlong,
                         ctypes.c_uint)
SIGNATURES = {
    "deltanet_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "deltanet_workspace_init": (_i, [_vp, _sz, _vp]),
    "deltanet_chunk_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "deltanet_decode_step": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]),
    "deltanet_decode_step_ex": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _u,
                                     _vp]),
    "deltanet_workspace_bytes_ex": (_sz, [_i, _i, _i, _i, _i, _i, _i, _u]),
    "deltanet_seq_segments": (_i, [_i, _i, _i, _i, _i, _i, _i, _u]),
    "deltanet_seq_segments_sm": (_i, [_i, _i, _i, _i, _i, _i, _i, _u, _i]),
    "deltanet_chunk_fwd_ex": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                   _i, _i, _i, _i, _i, _i, _i, _u, _vp, _sz, _vp]),
    "linear_attn_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                             _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "deltanet_chunk_fwd_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                        _i, _i, _i, _i, _i, _i, _i, _vp]),
    "deltanet_host_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "deltanet_chunk_fwd_host": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                     _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "deltanet_chunk_bwd_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "deltanet_chunk_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                _vp, _vp, _vp, _vp, _vp, _vp,
                                _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "deltanet_get_device_status": (_i, [_vp, _vp]),
    "deltanet_selftest_wait_timeout": (_i, [_vp, _sz, _ll, _vp]),
    "deltanet_status_string": (ctypes.c_char_p, [_i]),
    "deltanet_version": (_i, []),
}

_lib = None


class DeltaNetError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {code} ({status_string(code)})")


def lib():
    """Load the shared library once; raise if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m deltanet_sequence_mixing_b200.build` (there is no fallback)")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(h, name)
            f.restype, f.argtypes = res, args
        _lib = h
    return _lib


def status_string(code: int) -> str:
    try:
        return lib().deltanet_status_string(code).decode()
    except Exception:  # pragma: no cover - only while loading fails
        return "?"


def check(fn: str, code: int) -> None:
    if code != DN_OK:
        raise DeltaNetError(fn, code)
