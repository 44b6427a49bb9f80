"""deltanet_chunk_fwd_noalloc, the workspace-free entry point, against deltanet_chunk_fwd.

The variant exists for callers that cannot allocate device memory where they
call the library (allocator hooks, pre-budgeted embedded runtimes, paths that
must not synchronise through cudaMalloc); it keeps its scratch in a static
device array.  This file is named to be collected last, so that a run that
stops at the first failure has run every other test before it; it passes both
alone in a fresh process and after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

from deltanet_sequence_mixing_b200 import inputs as gen

pytestmark = pytest.mark.gpu

TOL = 2e-2  # the bf16 parity tolerance used by the GPU parity tests


def _rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


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
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.deltanet_chunk_fwd_noalloc(p(x["q"]), p(x["k"]), p(x["v"]), p(x["beta"]),
                                        p(x["alpha"]), None, p(o), p(S_out), B, H, T, Dk, Dv, C,
                                        1, stream)


@pytest.mark.parametrize("gated", [False, True])
def test_noalloc_matches_workspace_entry_point(dn, gated):
    dev = torch.device("cuda")
    L = dn.lib()
    for call, seed in enumerate((21, 22)):  # two calls in a row share the static scratch
        x = {k: (None if v is None else v.to(dev))
             for k, v in gen.make_inputs(2, 3, 300, 128, 128, torch.bfloat16, gated, seed).items()}
        o_ref, S_ref = dn.deltanet_chunk_fwd(x["q"], x["k"], x["v"], x["beta"], x["alpha"])
        o = torch.empty_like(o_ref)
        S = torch.empty_like(S_ref)
        rc = _noalloc(L, x, o, S)
        assert rc == 0, f"call {call}: {dn.status_string(rc)}"
        torch.cuda.synchronize()
        assert _rel(o.float().cpu(), o_ref.float().cpu()) <= TOL
        assert _rel(S.cpu(), S_ref.cpu()) <= TOL
        assert torch.isfinite(o.float()).all()


def test_noalloc_rejects_like_the_workspace_entry_point(dn):
    L = dn.lib()
    vp = ctypes.c_void_p
    # unsupported head size and negative length are rejected on the host
    assert L.deltanet_chunk_fwd_noalloc(vp(256), vp(512), vp(768), vp(1024), None, None, vp(2048),
                                        None, 1, 1, 64, 96, 64, 64, 1, None) == -2
    assert L.deltanet_chunk_fwd_noalloc(vp(256), vp(512), vp(768), vp(1024), None, None, vp(2048),
                                        None, 1, 1, -4, 64, 64, 64, 1, None) == -1
