"""deltanet_chunk_fwd_noalloc, the workspace-free entry point, against deltanet_chunk_fwd.

The variant exists for callers that cannot allocate device memory where they
call the library (allocator hooks, pre-budgeted embedded runtimes, paths that
must not synchronise through cudaMalloc); it keeps its scratch in a static
device array.  This file is named to be collected last, so that a run that
stops at the first failure has run every other test before it; it passes both
alone in a fresh process and after the rest of the suite.
"""
import ctypes

import pytest
import torch

from deltanet_sequence_mixing_b200 import inputs as gen

pytestmark = pytest.mark.gpu

LIMIT = 1 << 20  # bytes of the library's static scratch


@pytest.fixture(scope="module")
def dn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import deltanet_sequence_mixing_b200 as m

    m.lib()
    return m


def _noalloc(L, x, o, S_out, C=64):
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    B, H, T, Dk = x["q"].shape
    Dv = x["v"].shape[-1]
    dt = 1 if x["q"].dtype == torch.bfloat16 else 0
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.deltanet_chunk_fwd_noalloc(p(x["q"]), p(x["k"]), p(x["v"]), p(x["beta"]),
                                        p(x["alpha"]), None, p(o), p(S_out), B, H, T, Dk, Dv, C,
                                        dt, stream)


def _inputs(B, H, T, dtype, gated, seed):
    return {k: (None if v is None else v.to("cuda"))
            for k, v in gen.make_inputs(B, H, T, 128, 128, dtype, gated, seed).items()}


def _longest_T(L, B, H, C):
    """Largest multiple of C whose bf16 problem still fits the static scratch."""
    T = C
    while L.deltanet_workspace_bytes(B, H, T + C, 128, 128, C, 1) <= LIMIT:
        T += C
    return T


def _cases(L):
    # (B, H, T, dtype, gated, C): bf16 at both chunk sizes, the C = 128 case at
    # the longest sequence the scratch holds, and float32 (status word only)
    return [(2, 3, 300, torch.bfloat16, False, 64), (2, 3, 300, torch.bfloat16, True, 64),
            (1, 1, _longest_T(L, 1, 1, 128), torch.bfloat16, True, 128),
            (2, 2, 333, torch.float32, True, 64)]


@pytest.mark.parametrize("case", range(4))
def test_noalloc_matches_workspace_entry_point(dn, case):
    """Two calls in a row (sharing the static scratch) each give results bit for
    bit equal to deltanet_chunk_fwd's: the same kernels on the same inputs, only
    the scratch differs."""
    L = dn.lib()
    B, H, T, dtype, gated, C = _cases(L)[case]
    assert dn.lib().deltanet_workspace_bytes(B, H, T, 128, 128, C, 1 if dtype == torch.bfloat16 else 0) <= LIMIT
    for call, seed in enumerate((21, 22)):
        x = _inputs(B, H, T, dtype, gated, seed)
        o_ref, S_ref = dn.deltanet_chunk_fwd(x["q"], x["k"], x["v"], x["beta"], x["alpha"], C=C)
        o = torch.full_like(o_ref, float("nan"))
        S = torch.full_like(S_ref, float("nan"))
        rc = _noalloc(L, x, o, S, C)
        assert rc == 0, f"call {call}: {dn.status_string(rc)}"
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref), f"call {call}: o differs"
        assert torch.equal(S, S_ref), f"call {call}: S differs"


def test_noalloc_rejects_a_problem_past_the_scratch(dn):
    """One chunk more than the scratch holds: DN_ERR_WORKSPACE, nothing launched
    (the outputs keep their contents)."""
    L = dn.lib()
    C = 128
    T = _longest_T(L, 1, 1, C) + C
    assert L.deltanet_workspace_bytes(1, 1, T, 128, 128, C, 1) > LIMIT
    x = _inputs(1, 1, T, torch.bfloat16, True, 23)
    o = torch.full((1, 1, T, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    S = torch.full((1, 1, 128, 128), 7.0, device="cuda")
    assert _noalloc(L, x, o, S, C) == -6
    torch.cuda.synchronize()
    assert bool((o == 7.0).all()) and bool((S == 7.0).all())


def test_noalloc_rejects_like_the_workspace_entry_point(dn):
    L = dn.lib()
    vp = ctypes.c_void_p
    # unsupported head size and negative length are rejected on the host
    assert L.deltanet_chunk_fwd_noalloc(vp(256), vp(512), vp(768), vp(1024), None, None, vp(2048),
                                        None, 1, 1, 64, 96, 64, 64, 1, None) == -2
    assert L.deltanet_chunk_fwd_noalloc(vp(256), vp(512), vp(768), vp(1024), None, None, vp(2048),
                                        None, 1, 1, -4, 64, 64, 64, 1, None) == -1
