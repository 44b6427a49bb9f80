"""Host-side checks of the C ABI (no GPU needed).

The library loads, exports every function that include/deltanet.h declares,
and rejects bad arguments with the documented status codes before making any
CUDA call (so these run on a machine without a GPU).
"""
import ctypes
import os
import re

import pytest

from deltanet_sequence_mixing_b200 import _lib
from deltanet_sequence_mixing_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "include")


@pytest.fixture(scope="module")
def L():
    build()
    return _lib.lib()


def _declared_functions():
    names = set()
    for fn in os.listdir(HEADER_DIR):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(HEADER_DIR, fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M):
            if not m.group(0).lstrip().startswith(("typedef", "#")):
                names.add(m.group(1))
    return names


def test_header_declares_expected_entry_points():
    names = _declared_functions()
    for n in ("deltanet_chunk_fwd", "deltanet_decode_step", "linear_attn_fwd",
              "deltanet_workspace_bytes", "deltanet_get_device_status", "deltanet_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    names = _declared_functions()
    assert names, "no declarations parsed"
    for n in sorted(names):
        assert hasattr(L, n), f"{n} declared in include/ but not exported"
        assert n in _lib.SIGNATURES, f"{n} has no binding signature"


def test_status_strings(L):
    for code in range(0, -7, -1):
        s = _lib.status_string(code)
        assert s and s != "unknown status"
    assert _lib.status_string(-99) == "unknown status"
    assert L.deltanet_version() >= 100


def test_workspace_bytes(L):
    assert L.deltanet_workspace_bytes(4, 16, 4096, 128, 128, 64, 1) >= 256
    assert L.deltanet_workspace_bytes(4, 16, 4096, 96, 128, 64, 1) == 0
    assert L.deltanet_workspace_bytes(4, 16, 4096, 128, 128, 32, 1) == 0
    assert L.deltanet_workspace_bytes(-1, 16, 4096, 128, 128, 64, 1) == 0
    assert L.deltanet_workspace_bytes(4, 16, 4096, 128, 128, 64, 7) == 0
    # bf16: status word + per (b, h, chunk) the bf16 C x C factors Tb, Tbg and C floats of g
    for C, T in ((64, 4096), (64, 100), (128, 65536), (128, 300)):
        nch = -(-T // C)
        want = 256 + 4 * 16 * nch * (2 * C * C * 2 + C * 4)
        assert L.deltanet_workspace_bytes(4, 16, T, 128, 128, C, 1) == want
    assert L.deltanet_workspace_bytes(4, 16, 4096, 128, 128, 64, 0) == 256  # f32: status only
    assert L.deltanet_workspace_bytes(4, 16, 4096, 128, 128, 128, 0) == 0  # C = 128 is bf16 only
    # one pre-pass CTA per (b, h, chunk) on a one-dimensional grid: at most INT_MAX of them
    assert L.deltanet_workspace_bytes(1, 65536, 64 * 32768, 64, 64, 64, 1) == 0
    assert L.deltanet_workspace_bytes(1, 65536, 64 * 32767, 64, 64, 64, 1) > 0


# Fake, never dereferenced device addresses: every call below must be rejected
# on the host before any CUDA call.
A = 1 << 32
MB = 1 << 20


def _chunk(L, q=A, k=A + 64 * MB, v=A + 128 * MB, beta=A + 192 * MB, alpha=None, S0=None,
           o=A + 256 * MB, S_out=A + 320 * MB, B=2, H=2, T=100, Dk=64, Dv=64, C=64, dt=1,
           ws=A + 400 * MB, ws_bytes=None):
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    if ws_bytes is None:
        ws_bytes = max(256, L.deltanet_workspace_bytes(max(B, 0), max(H, 0), max(T, 0), 64, 64, 64, 1))
    return L.deltanet_chunk_fwd(vp(q), vp(k), vp(v), vp(beta), vp(alpha), vp(S0), vp(o),
                                vp(S_out), B, H, T, Dk, Dv, C, dt, vp(ws), ws_bytes, None)


def test_chunk_rejects_bad_arguments(L):
    E = _lib
    assert _chunk(L, q=None) == E.DN_ERR_INVALID_ARG
    assert _chunk(L, beta=None) == E.DN_ERR_INVALID_ARG
    assert _chunk(L, o=None) == E.DN_ERR_INVALID_ARG
    assert _chunk(L, B=-1) == E.DN_ERR_INVALID_ARG
    assert _chunk(L, T=-5) == E.DN_ERR_INVALID_ARG
    assert _chunk(L, Dk=96) == E.DN_ERR_UNSUPPORTED
    assert _chunk(L, Dv=32) == E.DN_ERR_UNSUPPORTED
    assert _chunk(L, C=32) == E.DN_ERR_UNSUPPORTED
    assert _chunk(L, dt=5) == E.DN_ERR_UNSUPPORTED
    assert _chunk(L, ws=None) == E.DN_ERR_WORKSPACE
    assert _chunk(L, ws_bytes=16) == E.DN_ERR_WORKSPACE
    assert _chunk(L, q=A + 8) == E.DN_ERR_ALIGNMENT
    assert _chunk(L, o=A + 256 * MB + 2) == E.DN_ERR_ALIGNMENT
    assert _chunk(L, S0=A + 500 * MB + 4) == E.DN_ERR_ALIGNMENT
    assert _chunk(L, C=128, dt=0) == E.DN_ERR_UNSUPPORTED  # C = 128 is built for bf16 only
    assert _chunk(L, C=128, dt=0, T=0) == E.DN_ERR_UNSUPPORTED


def test_chunk_rejects_grids_past_int_max(L):
    """B * H * ceil(T / C) pre-pass CTAs must fit one grid dimension (INT_MAX):
    one chunk past it is rejected before launch, not at launch."""
    E = _lib
    big = 1 << 40
    assert _chunk(L, B=1, H=65536, T=64 * 32768, q=big, k=2 * big, v=3 * big, beta=4 * big,
                  o=5 * big, S_out=None, ws=6 * big, ws_bytes=1 << 62) == E.DN_ERR_UNSUPPORTED


def test_chunk_rejects_overlaps(L):
    E = _lib
    assert _chunk(L, o=A + 4096) == E.DN_ERR_INVALID_ARG  # o inside q
    assert _chunk(L, S_out=A + 64 * MB) == E.DN_ERR_INVALID_ARG  # S_out inside k
    S0 = A + 500 * MB
    assert _chunk(L, S0=S0, S_out=S0 + 256) == E.DN_ERR_INVALID_ARG  # partial overlap
    assert _chunk(L, ws=A + 256 * MB) == E.DN_ERR_INVALID_ARG  # workspace inside o


def test_host_workspace_bytes(L):
    """Status word + two staging slots of ceil(B*H/4) heads, every region on a
    256-byte boundary: q, k, v, o, beta, alpha, S0, S_out and the group's
    pre-pass factors (4 C^2 + 4 C bytes per chunk for bf16)."""
    r = lambda x: (x + 255) // 256 * 256
    for (B, H, T, Dk, Dv, C, dt) in [(4, 16, 4096, 128, 128, 64, 1), (3, 5, 333, 128, 64, 64, 0),
                                     (1, 1, 200, 64, 128, 128, 1), (2, 3, 0, 64, 64, 64, 1)]:
        Hg = (B * H + 3) // 4
        es = 2 if dt == 1 else 4
        tok = Hg * T
        wy = Hg * ((T + C - 1) // C) * (4 * C * C + 4 * C) if (dt == 1 and T > 0) else 0
        slot = (2 * r(tok * Dk * es) + 2 * r(tok * Dv * es) + 2 * r(tok * 4)
                + 2 * r(Hg * Dk * Dv * 4) + r(wy))
        assert L.deltanet_host_workspace_bytes(B, H, T, Dk, Dv, C, dt) == 256 + 2 * slot
    assert L.deltanet_host_workspace_bytes(4, 16, 4096, 96, 128, 64, 1) == 0
    assert L.deltanet_host_workspace_bytes(4, 16, 4096, 128, 128, 64, 7) == 0
    assert L.deltanet_host_workspace_bytes(-1, 16, 4096, 128, 128, 64, 1) == 0


def _chunk_host(L, q=A, k=A + 64 * MB, v=A + 128 * MB, beta=A + 192 * MB, alpha=None, S0=None,
                o=A + 256 * MB, S_out=A + 320 * MB, B=2, H=2, T=100, Dk=64, Dv=64, C=64, dt=1,
                ws=A + 400 * MB, ws_bytes=None):
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    if ws_bytes is None:
        ws_bytes = max(256, L.deltanet_host_workspace_bytes(max(B, 0), max(H, 0), max(T, 0), 64, 64, 64, 1))
    return L.deltanet_chunk_fwd_host(vp(q), vp(k), vp(v), vp(beta), vp(alpha), vp(S0), vp(o),
                                     vp(S_out), B, H, T, Dk, Dv, C, dt, vp(ws), ws_bytes, None)


def test_chunk_host_rejects_bad_arguments(L):
    """The host-buffer call validates like the device call, before any CUDA
    call; its host pointers need no alignment, its workspace does."""
    E = _lib
    assert _chunk_host(L, q=None) == E.DN_ERR_INVALID_ARG
    assert _chunk_host(L, beta=None) == E.DN_ERR_INVALID_ARG
    assert _chunk_host(L, B=-1) == E.DN_ERR_INVALID_ARG
    assert _chunk_host(L, Dk=96) == E.DN_ERR_UNSUPPORTED
    assert _chunk_host(L, C=32) == E.DN_ERR_UNSUPPORTED
    assert _chunk_host(L, ws=None) == E.DN_ERR_WORKSPACE
    assert _chunk_host(L, ws_bytes=1024) == E.DN_ERR_WORKSPACE
    assert _chunk_host(L, ws=A + 400 * MB + 8) == E.DN_ERR_ALIGNMENT
    assert _chunk_host(L, o=A + 4096) == E.DN_ERR_INVALID_ARG  # o inside q
    S0 = A + 500 * MB
    assert _chunk_host(L, S0=S0, S_out=S0 + 256) == E.DN_ERR_INVALID_ARG  # partial overlap


def test_decode_rejects_bad_arguments(L):
    E = _lib
    vp = ctypes.c_void_p

    def dec(q=A, k=A + MB, v=A + 2 * MB, beta=A + 3 * MB, alpha=None, S=A + 8 * MB,
            o=A + 4 * MB, B=4, H=2, Dk=128, Dv=128, dt=1):
        f = lambda x: None if x is None else vp(x)
        return L.deltanet_decode_step(f(q), f(k), f(v), f(beta), f(alpha), f(S), f(o), B, H, Dk,
                                      Dv, dt, None)

    assert dec(S=None) == E.DN_ERR_INVALID_ARG
    assert dec(beta=None) == E.DN_ERR_INVALID_ARG
    assert dec(Dk=48) == E.DN_ERR_UNSUPPORTED
    assert dec(S=A + 8 * MB + 4) == E.DN_ERR_ALIGNMENT
    assert dec(o=A + 8 * MB) == E.DN_ERR_INVALID_ARG  # o inside S
    assert dec(B=-2) == E.DN_ERR_INVALID_ARG


def test_linear_rejects_bad_arguments(L):
    E = _lib
    vp = ctypes.c_void_p

    def lin(q=A, k=A + 64 * MB, v=A + 128 * MB, S0=None, z0=None, o=A + 256 * MB,
            S_out=None, z_out=None, Dk=64, C=64):
        f = lambda x: None if x is None else vp(x)
        return L.linear_attn_fwd(f(q), f(k), f(v), f(S0), f(z0), f(o), f(S_out), f(z_out),
                                 2, 2, 100, Dk, 64, C, 1, vp(A + 400 * MB), 1 << 24, None)

    assert lin(v=None) == E.DN_ERR_INVALID_ARG
    assert lin(Dk=80) == E.DN_ERR_UNSUPPORTED
    assert lin(C=96) == E.DN_ERR_UNSUPPORTED
    assert lin(C=128) == E.DN_ERR_UNSUPPORTED  # linear attention is built for C = 64 only
    assert lin(z0=A + 300 * MB, z_out=A + 300 * MB + 4) == E.DN_ERR_ALIGNMENT
    assert lin(z0=A + 300 * MB, z_out=A + 300 * MB + 16) == E.DN_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors():
    import torch

    import deltanet_sequence_mixing_b200 as dn

    x = torch.zeros(1, 1, 4, 64)
    with pytest.raises(ValueError, match="CUDA"):
        dn.deltanet_chunk_fwd(x, x, x, torch.zeros(1, 1, 4))


def test_option_flags_are_validated_on_the_host(L):
    """The *_ex calls: unknown option bits, a per-dimension gate without alpha,
    and the options with C = 128 are rejected before any CUDA call."""
    E = _lib
    vp = lambda x: None if x is None else ctypes.c_void_p(x)

    def ex(opts, alpha=None, C=64, T=100):
        return L.deltanet_chunk_fwd_ex(vp(A), vp(A + 64 * MB), vp(A + 128 * MB), vp(A + 192 * MB),
                                       vp(alpha), None, vp(A + 256 * MB), vp(A + 320 * MB),
                                       2, 2, T, 64, 64, C, 1, opts, vp(A + 400 * MB), 1 << 20, None)

    assert ex(8) == E.DN_ERR_INVALID_ARG
    assert ex(E.DN_OPT_GATE_PER_DIM) == E.DN_ERR_INVALID_ARG  # per-dimension gate needs alpha
    assert ex(E.DN_OPT_PRESTEP, C=128) == E.DN_ERR_UNSUPPORTED
    assert ex(E.DN_OPT_GATE_PER_DIM, alpha=A + 500 * MB, C=128) == E.DN_ERR_UNSUPPORTED
    # the per-dimension alpha covers B*H*T*Dk floats: an alpha that ends inside o overlaps it
    assert ex(E.DN_OPT_GATE_PER_DIM, alpha=A + 256 * MB - 2 * 2 * 100 * 64 * 4 + 64) == E.DN_ERR_INVALID_ARG
    # the pre-step alone on bf16 runs on the tcgen05 path: the pre-pass factors,
    # then (each from a 256-byte boundary) the mapped keys and queries, B*H*T*Dk bf16 each
    base = L.deltanet_workspace_bytes(2, 2, 100, 64, 64, 64, 1)
    r256 = lambda x: (x + 255) // 256 * 256
    assert L.deltanet_workspace_bytes_ex(2, 2, 100, 64, 64, 64, 1, 1) == \
        256 + r256(base - 256) + 2 * r256(2 * 2 * 100 * 64 * 2)
    assert L.deltanet_workspace_bytes_ex(2, 2, 100, 64, 64, 64, 0, 1) == 256
    assert L.deltanet_workspace_bytes_ex(2, 2, 100, 64, 64, 64, 1, 2) == 256
    assert L.deltanet_workspace_bytes_ex(2, 2, 100, 64, 64, 64, 1, 3) == 256
    assert L.deltanet_workspace_bytes_ex(2, 2, 100, 64, 64, 128, 1, 1) == 0
    assert L.deltanet_workspace_bytes_ex(2, 2, 100, 64, 64, 64, 1, 8) == 0
    # the sequence split is a permission: where it does not apply (here: no GPU to
    # size it against, float32, C = 128, other options) the call runs unsplit
    plain = L.deltanet_workspace_bytes(2, 2, 4096, 64, 64, 64, 1)
    assert L.deltanet_workspace_bytes_ex(2, 2, 4096, 64, 64, 64, 1, 4) == plain
    assert L.deltanet_workspace_bytes_ex(2, 2, 4096, 64, 64, 128, 1, 4) == \
        L.deltanet_workspace_bytes(2, 2, 4096, 64, 64, 128, 1)
    assert L.deltanet_workspace_bytes_ex(2, 2, 4096, 64, 64, 64, 0, 4) == 256
    assert L.deltanet_workspace_bytes_ex(2, 2, 100, 64, 64, 64, 1, 5) == \
        L.deltanet_workspace_bytes_ex(2, 2, 100, 64, 64, 64, 1, 1)
    for opts in (4, 5, 6):
        assert L.deltanet_seq_segments(2, 2, 4096, 64, 64, 64, 1, opts) == 1
    assert L.deltanet_workspace_bytes_ex(2, 2, 100, 64, 64, 64, 1, 0) == \
        L.deltanet_workspace_bytes(2, 2, 100, 64, 64, 64, 1)

    def dec(opts, alpha=None):
        return L.deltanet_decode_step_ex(vp(A), vp(A + MB), vp(A + 2 * MB), vp(A + 3 * MB), vp(alpha),
                                         vp(A + 8 * MB), vp(A + 4 * MB), 4, 2, 128, 128, 1, opts, None)

    assert dec(8) == E.DN_ERR_INVALID_ARG
    assert dec(E.DN_OPT_GATE_PER_DIM) == E.DN_ERR_INVALID_ARG
    # a (B,H,Dk) alpha of 4*2*128 floats starting 1 KB before S overlaps S
    assert dec(E.DN_OPT_GATE_PER_DIM, alpha=A + 8 * MB - 1024) == E.DN_ERR_INVALID_ARG


def test_sequence_split_segment_rule(L):
    """The segment count the split takes, for a 148-SM B200 and other SM
    counts (host logic, no GPU): a divisor G <= 16 of T with at least 8 chunks
    per segment and B*H*G*(Dk + Dv)/64 <= SMs, minimising T/(64 G) + 2 (G - 1)
    + 8 chunk periods, and 1 when nothing beats the plain call's T/64."""
    seg = lambda B, H, T, Dk=128, Dv=128, opts=4, sms=148, C=64, dt=1: \
        L.deltanet_seq_segments_sm(B, H, T, Dk, Dv, C, dt, opts, sms)
    assert seg(1, 16, 4096) == 2        # as many heads as two segments allow
    assert seg(1, 2, 4096) == 4
    assert seg(1, 3, 3000, 128, 64) == 4
    assert seg(2, 2, 2200, 64, 64) == 4
    assert seg(1, 1, 9100) == 7         # odd counts when T's divisors call for them
    assert seg(1, 1, 32768) == 16
    assert seg(1, 8, 65536) == 4
    assert seg(1, 4, 65536) == 8
    assert seg(1, 32, 65536) == 1       # the plain chain already fills the SMs
    assert seg(4, 16, 1024) == 1
    assert seg(1, 1, 1000) == 1         # too short for two 8-chunk segments to pay
    # fewer SMs: both chains of every segment must fit one wave
    assert seg(1, 8, 65536, sms=64) == 2
    assert seg(1, 8, 65536, sms=63) == 1
    # only bf16, C = 64, and no option besides the pre-step
    assert seg(1, 2, 4096, opts=5) == 4
    assert seg(1, 2, 4096, opts=0) == 1
    assert seg(1, 2, 4096, opts=6) == 1
    assert seg(1, 2, 4096, opts=7) == 1
    assert seg(1, 2, 4096, dt=0) == 1
    assert seg(1, 2, 4096, C=128) == 1
    assert seg(1, 2, 4096, Dk=96) == 1
    assert seg(1, 2, 4096, sms=0) == 1
