"""The host-buffer chunked forward (deltanet_chunk_fwd_host) against the
device-buffer call on the same inputs.  The host call runs the same kernels on
groups of heads, so its results must be bit-identical; every group boundary
case is covered (one group, a short last group, T == 0, in-place state carry).
"""
import numpy as np
import pytest
import torch

from deltanet_sequence_mixing_b200 import inputs as gen

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import deltanet_sequence_mixing_b200 as m

    m.lib()
    return m


def _pin(t):
    return None if t is None else t.contiguous().pin_memory()


def _device_call(dn, x, S0, C):
    dev = torch.device("cuda")
    g = {k: (None if v is None else v.to(dev)) for k, v in x.items()}
    o, S = dn.deltanet_chunk_fwd(g["q"], g["k"], g["v"], g["beta"], g["alpha"],
                                 None if S0 is None else S0.to(dev), C=C)
    torch.cuda.synchronize()
    return o.cpu(), S.cpu()


def _host_call(dn, x, S0, C, in_place=False):
    h = {k: _pin(v) for k, v in x.items()}
    hS0 = _pin(S0)
    S_out = hS0 if in_place else None
    B, H, T, Dk = x["q"].shape
    ws = dn.host_workspace_for("cuda", B, H, T, Dk, x["v"].shape[-1], C, x["q"].dtype)
    o, S = dn.deltanet_chunk_fwd_host(h["q"], h["k"], h["v"], h["beta"], h["alpha"], hS0, C=C,
                                      S_out=S_out, workspace=ws)
    torch.cuda.synchronize()
    assert dn.deltanet_get_device_status(workspace=ws) == 0
    return o, S


@pytest.mark.parametrize("B,H,T,Dk,Dv,dtype,gated,C", [
    (1, 1, 200, 128, 128, torch.bfloat16, False, 64),   # one group of one head
    (3, 5, 333, 128, 64, torch.bfloat16, True, 64),     # 15 heads: groups of 4, last one short
    (2, 8, 256, 128, 128, torch.bfloat16, False, 128),  # C = 128
    (2, 3, 150, 64, 64, torch.float32, True, 64),       # the float32 path
])
def test_host_call_matches_device_call(dn, B, H, T, Dk, Dv, dtype, gated, C):
    x = gen.make_inputs(B, H, T, Dk, Dv, dtype, gated=gated, seed=B * 100 + H + T)
    S0 = torch.randn(B, H, Dk, Dv, generator=torch.Generator().manual_seed(T)) * 0.1
    o_d, S_d = _device_call(dn, x, S0, C)
    o_h, S_h = _host_call(dn, x, S0, C)
    assert torch.equal(o_h.float(), o_d.float())
    assert torch.equal(S_h, S_d)


def test_host_call_in_place_state_and_no_initial_state(dn):
    x = gen.make_inputs(2, 5, 190, 128, 128, torch.bfloat16, gated=True, seed=3)
    S0 = torch.randn(2, 5, 128, 128, generator=torch.Generator().manual_seed(9)) * 0.1
    o_d, S_d = _device_call(dn, x, S0, 64)
    o_h, S_h = _host_call(dn, x, S0.clone(), 64, in_place=True)
    assert torch.equal(o_h.float(), o_d.float()) and torch.equal(S_h, S_d)
    o_d0, S_d0 = _device_call(dn, x, None, 64)
    o_h0, S_h0 = _host_call(dn, x, None, 64)
    assert torch.equal(o_h0.float(), o_d0.float()) and torch.equal(S_h0, S_d0)


def test_host_call_empty_sequence_copies_state(dn):
    S0 = torch.randn(2, 3, 64, 64, generator=torch.Generator().manual_seed(1))
    e = torch.empty(2, 3, 0, 64, dtype=torch.bfloat16)
    be = torch.empty(2, 3, 0, dtype=torch.float32)
    o, S = dn.deltanet_chunk_fwd_host(_pin(e), _pin(e), _pin(e), _pin(be), None, _pin(S0))
    torch.cuda.synchronize()
    assert o.shape == (2, 3, 0, 64)
    assert np.array_equal(S.numpy(), S0.numpy())
