"""GPU parity of the gradient (deltanet_chunk_bwd) against the float64 oracle's
reverse sweep of the per-token loop (itself pinned by finite differences).

The loss is sum(dO * o) + sum(dS_T * S_T).  Gates, per gradient: rel-L2 <= 1e-4
for float32 inputs and <= 2e-2 for bfloat16 inputs (the same values reach both
sides; the GPU computes in float32).  The log-decay gradient is compared with
alpha * dL/dalpha of the oracle.
"""
import numpy as np
import pytest
import torch

from deltanet_sequence_mixing_b200 import inputs as gen

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def rel_l2(x, ref):
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-300))


@pytest.fixture(scope="module")
def dn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import deltanet_sequence_mixing_b200 as m

    m.lib()
    return m


def _case(B, H, T, Dk, Dv, dtype, gated, seed, with_state=True):
    x = gen.make_inputs(B, H, T, Dk, Dv, dtype, gated=gated, seed=seed)
    g = torch.Generator().manual_seed(seed + 1)
    dO = torch.randn(B, H, T, Dv, generator=g).to(dtype)
    S0 = torch.randn(B, H, Dk, Dv, generator=g) * 0.2 if with_state else None
    dST = torch.randn(B, H, Dk, Dv, generator=g) if with_state else None
    return x, dO, S0, dST


def _check(dn, oracle_mod, x, dO, S0, dST, dtype):
    cu = lambda t: None if t is None else t.cuda()
    got = dn.deltanet_chunk_bwd(cu(x["q"]), cu(x["k"]), cu(x["v"]), cu(x["beta"]), cu(dO),
                                cu(x["alpha"]), cu(S0), cu(dST))
    torch.cuda.synchronize()
    ref = oracle_mod.deltanet_bwd(x["q"], x["k"], x["v"], x["beta"], dO.double(), x["alpha"],
                                  None if S0 is None else S0.double(),
                                  None if dST is None else dST.double())
    errs = {n: rel_l2(got[n].cpu(), ref[n]) for n in ("dq", "dk", "dv", "dbeta", "dS0")}
    if x["alpha"] is not None:
        errs["dlog_alpha"] = rel_l2(got["dlog_alpha"].cpu(), x["alpha"].double().numpy() * ref["dalpha"])
    bad = {n: e for n, e in errs.items() if not e <= TOL[dtype]}
    assert not bad, f"rel-L2 above {TOL[dtype]}: {bad} (all: {errs})"
    return got


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("gated", [False, True])
@pytest.mark.parametrize("Dk,Dv", [(64, 64), (128, 128), (128, 64), (64, 128)])
@pytest.mark.parametrize("T", [1, 31, 33, 100])
def test_backward_shapes(dn, oracle_mod, dtype, gated, Dk, Dv, T):
    x, dO, S0, dST = _case(2, 2, T, Dk, Dv, dtype, gated, seed=600 + T + Dk + Dv)
    _check(dn, oracle_mod, x, dO, S0, dST, dtype)


@pytest.mark.parametrize("gated", [False, True])
def test_backward_longer_sequence_without_states(dn, oracle_mod, gated):
    x, dO, _, _ = _case(1, 3, 300, 128, 128, torch.float32, gated, seed=610, with_state=False)
    _check(dn, oracle_mod, x, dO, None, None, torch.float32)


def test_backward_gate_zero_and_one(dn, oracle_mod):
    """alpha = 1 on a run of tokens and a hard wipe (alpha = 0 enters as
    e^-87, whose log-gradient the oracle gives as alpha * dL/dalpha = 0)."""
    x, dO, S0, dST = _case(1, 2, 130, 64, 64, torch.float32, True, seed=611)
    x["alpha"][:, :, 40:70] = 1.0
    x["alpha"][:, :, 90] = 0.0
    _check(dn, oracle_mod, x, dO, S0, dST, torch.float32)


def test_backward_deterministic_and_empty(dn):
    x, dO, S0, dST = _case(2, 2, 77, 128, 128, torch.bfloat16, True, seed=612)
    cu = lambda t: None if t is None else t.cuda()
    a = dn.deltanet_chunk_bwd(cu(x["q"]), cu(x["k"]), cu(x["v"]), cu(x["beta"]), cu(dO),
                              cu(x["alpha"]), cu(S0), cu(dST))
    b = dn.deltanet_chunk_bwd(cu(x["q"]), cu(x["k"]), cu(x["v"]), cu(x["beta"]), cu(dO),
                              cu(x["alpha"]), cu(S0), cu(dST))
    torch.cuda.synchronize()
    for n in a:
        if a[n] is not None:
            assert torch.equal(a[n], b[n]), n
    e = torch.zeros(2, 2, 0, 64, dtype=torch.bfloat16, device="cuda")
    dS = torch.randn(2, 2, 64, 64, device="cuda")
    g = dn.deltanet_chunk_bwd(e, e, e, torch.zeros(2, 2, 0, device="cuda"), e, dS_T=dS)
    torch.cuda.synchronize()
    assert torch.equal(g["dS0"], dS)
