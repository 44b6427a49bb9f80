"""GPU parity of the optional forms against the float64 oracle.

* the layer's pre-step inside the calls (q, k <- normalize(silu(.)),
  beta <- sigmoid(.)): "GPT-2 から Kimi K3 まで" (news.ainew.jp), section
  "DeltaNet (Fast weight programmers)", the layer's forward;
* per-dimension decay (alpha (B,H,T,Dk)): "How a Baseten Engineer Traced 7
  Years of Attention Mechanism Evolution", the KDA paragraph.

Gates as the other parity tests: rel-L2 <= 1e-4 (float32 inputs), <= 2e-2
(bfloat16 inputs, float32 state).
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


def _gpu(d):
    return {k: (None if v is None else v.to("cuda")) for k, v in d.items()}


def _inputs(B, H, T, Dk, Dv, dtype, gate, prestep, seed):
    return gen.make_inputs(B, H, T, Dk, Dv, dtype, gated=gate != "none", seed=seed, raw=prestep,
                           gate_per_dim=gate == "per_dim")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("gate", ["none", "scalar", "per_dim"])
@pytest.mark.parametrize("prestep", [False, True])
@pytest.mark.parametrize("Dk,Dv", [(128, 128), (64, 128)])
@pytest.mark.parametrize("T", [1, 63, 200])
def test_chunk_options(dn, oracle_mod, dtype, gate, prestep, Dk, Dv, T):
    if gate != "per_dim" and not prestep:
        pytest.skip("the plain forms are covered by test_gpu_parity")
    x = _inputs(2, 2, T, Dk, Dv, dtype, gate, prestep, seed=500 + T + Dk)
    S0 = torch.randn(2, 2, Dk, Dv, generator=torch.Generator().manual_seed(3)) * 0.1
    g = _gpu(x)
    o, S = dn.deltanet_chunk_fwd(g["q"], g["k"], g["v"], g["beta"], g["alpha"], S0.cuda(),
                                 prestep=prestep)
    torch.cuda.synchronize()
    assert dn.deltanet_get_device_status() == 0
    o_ref, S_ref = oracle_mod.deltanet(x["q"], x["k"], x["v"], x["beta"], x["alpha"], S0.double(),
                                       prestep=prestep)
    eo, es = rel_l2(o.float().cpu(), o_ref), rel_l2(S.cpu(), S_ref)
    assert eo <= TOL[dtype] and es <= TOL[dtype], f"rel-L2 o={eo:.3e} S={es:.3e}"


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_chunk_per_dim_steep_and_zero_decays(dn, oracle_mod, dtype):
    """Per-dimension decays near zero (log-decay spans of hundreds within a
    chunk) and exactly zero on some dimensions (a wipe of those rows)."""
    x = _inputs(1, 2, 300, 128, 128, dtype, "per_dim", False, seed=510)
    x["alpha"][:, 0, :, :16] = float(np.exp(-6.0))
    x["alpha"][:, 1, 100, 5:9] = 0.0
    g = _gpu(x)
    o, S = dn.deltanet_chunk_fwd(g["q"], g["k"], g["v"], g["beta"], g["alpha"])
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_mod.deltanet(x["q"], x["k"], x["v"], x["beta"], x["alpha"])
    assert rel_l2(o.float().cpu(), o_ref) <= TOL[dtype]
    assert rel_l2(S.cpu(), S_ref) <= TOL[dtype]


def test_chunk_per_dim_uniform_matches_scalar_gate(dn):
    """A per-dimension decay that is the same on every dimension gives the
    scalar-gated result (bf16 inputs: the two run on different kernels, so
    they agree to the bf16 gate)."""
    x = _inputs(2, 2, 257, 128, 128, torch.bfloat16, "scalar", False, seed=511)
    g = _gpu(x)
    o1, S1 = dn.deltanet_chunk_fwd(g["q"], g["k"], g["v"], g["beta"], g["alpha"])
    a4 = g["alpha"][..., None].expand(-1, -1, -1, 128).contiguous()
    o2, S2 = dn.deltanet_chunk_fwd(g["q"], g["k"], g["v"], g["beta"], a4)
    torch.cuda.synchronize()
    assert rel_l2(o2.float().cpu(), o1.float().cpu()) <= 2e-2
    assert rel_l2(S2.cpu(), S1.cpu()) <= 2e-2


def test_chunk_options_reject_chunk_128(dn):
    x = _gpu(_inputs(1, 1, 64, 128, 128, torch.bfloat16, "none", True, seed=512))
    with pytest.raises(dn.DeltaNetError):
        dn.deltanet_chunk_fwd(x["q"], x["k"], x["v"], x["beta"], C=128, prestep=True)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("gate", ["none", "scalar", "per_dim"])
@pytest.mark.parametrize("prestep", [False, True])
@pytest.mark.parametrize("Dk,Dv", [(128, 128), (64, 64), (128, 64)])
def test_decode_options(dn, oracle_mod, dtype, gate, prestep, Dk, Dv):
    if gate != "per_dim" and not prestep:
        pytest.skip("the plain forms are covered by test_gpu_parity")
    B, H, steps = 3, 4, 5
    S0 = torch.randn(B, H, Dk, Dv, generator=torch.Generator().manual_seed(4)) * 0.2
    S = S0.cuda()
    seq = _inputs(B, H, steps, Dk, Dv, dtype, gate, prestep, seed=520 + Dk + Dv)
    outs = []
    for t in range(steps):
        st = {k: (None if v is None else v[:, :, t].contiguous().cuda()) for k, v in seq.items()}
        outs.append(dn.deltanet_decode_step(st["q"], st["k"], st["v"], st["beta"], S,
                                            alpha=st["alpha"], prestep=prestep).float().cpu())
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_mod.deltanet(seq["q"], seq["k"], seq["v"], seq["beta"], seq["alpha"],
                                       S0.double(), prestep=prestep)
    eo, es = rel_l2(torch.stack(outs, 2), o_ref), rel_l2(S.cpu(), S_ref)
    assert eo <= TOL[dtype] and es <= TOL[dtype], f"rel-L2 o={eo:.3e} S={es:.3e}"


def test_prestep_decode_continues_prestep_prefill(dn, oracle_mod):
    """Decode with the pre-step continues the chunked call with the pre-step."""
    B, H, T, steps = 2, 3, 130, 4
    x = _inputs(B, H, T + steps, 128, 128, torch.bfloat16, "per_dim", True, seed=530)
    pre = {k: v[:, :, :T].contiguous().cuda() for k, v in x.items()}
    _, S = dn.deltanet_chunk_fwd(pre["q"], pre["k"], pre["v"], pre["beta"], pre["alpha"],
                                 prestep=True)
    outs = []
    for t in range(T, T + steps):
        st = {k: v[:, :, t].contiguous().cuda() for k, v in x.items()}
        outs.append(dn.deltanet_decode_step(st["q"], st["k"], st["v"], st["beta"], S,
                                            alpha=st["alpha"], prestep=True).float().cpu())
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_mod.deltanet(x["q"], x["k"], x["v"], x["beta"], x["alpha"], prestep=True)
    assert rel_l2(torch.stack(outs, 2), o_ref[:, :, T:]) <= 2e-2
    assert rel_l2(S.cpu(), S_ref) <= 2e-2
