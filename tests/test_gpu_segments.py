"""The sequence split (DN_OPT_SEQ_SPLIT): segments of each sequence run side by
side and are joined afterwards, using the affine chunk transition of "GPT-2 から
Kimi K3 まで" (news.ainew.jp), section "DeltaNet (Parallelizing linear
transformers with delta rule)".  The result is the recurrence itself, so the
check is the float64 oracle of that recurrence, at the bf16 bar, on problems
where the library does split (few heads, long enough sequences), with gating,
an initial state, ragged segment ends and in-place state carry."""
import numpy as np
import pytest
import torch

from deltanet_sequence_mixing_b200 import inputs as gen

pytestmark = pytest.mark.gpu

TOL = 2e-2  # bf16 inputs, float32 state


@pytest.fixture(scope="module")
def dn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import deltanet_sequence_mixing_b200 as m

    m.lib()  # fail loudly if the library is missing
    return m


def rel_l2(x, ref):
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-300))


def _run(dn, x, S0, seq_split, S_out=None):
    g = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    o, S = dn.deltanet_chunk_fwd(g["q"], g["k"], g["v"], g["beta"], g["alpha"],
                                 None if S0 is None else S0.cuda(), C=64, S_out=S_out,
                                 seq_split=seq_split)
    torch.cuda.synchronize()
    assert dn.deltanet_get_device_status() == 0
    return o.float().cpu().numpy(), S.cpu().numpy()


# (B, H, T, Dk, Dv, gated, with S0, segments the B200's 148 SMs give)
CASES = [
    (1, 16, 4096, 128, 128, False, False, 2),  # as many heads as two segments allow
    (1, 2, 4096, 128, 128, True, True, 4),
    (1, 3, 3000, 128, 64, True, True, 4),    # 750-token segments: a ragged last chunk in each
    (2, 2, 2200, 64, 64, True, False, 4),    # 550-token segments
    (1, 1, 2048, 64, 128, False, True, 4),
    (1, 1, 9100, 128, 128, True, True, 7),   # 1300-token segments, an odd count
    (1, 1, 32768, 128, 128, False, True, 16),
]
@pytest.mark.parametrize("B,H,T,Dk,Dv,gated,with_s0,G", CASES)
def test_split_matches_oracle(dn, oracle_mod, B, H, T, Dk, Dv, gated, with_s0, G):
    assert dn.seq_segments(B, H, T, Dk, Dv) == G
    x = gen.make_inputs(B, H, T, Dk, Dv, torch.bfloat16, gated=gated, seed=T + H + Dk)
    S0 = torch.randn(B, H, Dk, Dv, generator=torch.Generator().manual_seed(T)) * 0.1 if with_s0 else None
    o, S = _run(dn, x, S0, True)
    o_ref, S_ref = oracle_mod.deltanet(x["q"], x["k"], x["v"], x["beta"], x["alpha"],
                                       None if S0 is None else S0.double())
    eo, es = rel_l2(o, o_ref), rel_l2(S, S_ref)
    assert eo <= TOL and es <= TOL, f"rel-L2 o={eo:.3e} S={es:.3e}"
    # and close to the unsplit call (the two differ only in rounding)
    o1, S1 = _run(dn, x, S0, False)
    assert rel_l2(o, o1) <= 1e-2 and rel_l2(S, S1) <= 1e-2


def test_split_with_the_layer_prestep(dn, oracle_mod):
    """The split with the layer's pre-step inside (raw q, k projections and
    beta logits; the pre-pass maps them once for both chains)."""
    B, H, T = 1, 2, 4096
    assert dn.seq_segments(B, H, T, 128, 128, prestep=True) == 4
    x = gen.make_inputs(B, H, T, 128, 128, torch.bfloat16, gated=True, seed=31, raw=True)
    S0 = torch.randn(B, H, 128, 128, generator=torch.Generator().manual_seed(31)) * 0.1
    g = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    o, S = dn.deltanet_chunk_fwd(g["q"], g["k"], g["v"], g["beta"], g["alpha"], S0.cuda(), C=64, prestep=True,
                                 seq_split=True)
    torch.cuda.synchronize()
    assert dn.deltanet_get_device_status() == 0
    o_ref, S_ref = oracle_mod.deltanet(x["q"], x["k"], x["v"], x["beta"], x["alpha"], S0.double(), prestep=True)
    eo, es = rel_l2(o.float().cpu().numpy(), o_ref), rel_l2(S.cpu().numpy(), S_ref)
    assert eo <= TOL and es <= TOL, f"rel-L2 o={eo:.3e} S={es:.3e}"
    o1, S1 = dn.deltanet_chunk_fwd(g["q"], g["k"], g["v"], g["beta"], g["alpha"], S0.cuda(), C=64, prestep=True)
    torch.cuda.synchronize()
    assert rel_l2(o.float().cpu().numpy(), o1.float().cpu().numpy()) <= 1e-2
    assert rel_l2(S.cpu().numpy(), S1.cpu().numpy()) <= 1e-2


def test_split_workspace_sizes(dn):
    """With G > 1 the workspace grows by the split's arrays; the pre-step adds
    the mapped k and q (B*H*T*Dk bf16 each, from 256-byte boundaries)."""
    L = dn.lib()
    B, H, T, D = 1, 2, 4096, 128
    r256 = lambda x: (x + 255) // 256 * 256
    plain = L.deltanet_workspace_bytes_ex(B, H, T, D, D, 64, 1, 0)
    split = L.deltanet_workspace_bytes_ex(B, H, T, D, D, 64, 1, 4)
    split_pre = L.deltanet_workspace_bytes_ex(B, H, T, D, D, 64, 1, 5)
    # R (B*H*T*Dk bf16) and four (B*H*G, Dk, Dv) float32 states at least
    assert split >= plain + B * H * T * D * 2 + 4 * B * H * 4 * D * D * 4
    assert split_pre - split == 2 * r256(B * H * T * D * 2)


def test_split_in_place_state(dn, oracle_mod):
    """S_out may be S0 itself: the split reads S0 before it writes S_out."""
    B, H, T = 1, 2, 4096
    x = gen.make_inputs(B, H, T, 128, 128, torch.bfloat16, gated=True, seed=5)
    S0 = torch.randn(B, H, 128, 128, generator=torch.Generator().manual_seed(9)) * 0.1
    S_dev = S0.cuda()
    g = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    o, S = dn.deltanet_chunk_fwd(g["q"], g["k"], g["v"], g["beta"], g["alpha"], S_dev, C=64, S_out=S_dev,
                                 seq_split=True)
    torch.cuda.synchronize()
    assert S.data_ptr() == S_dev.data_ptr()
    o_ref, S_ref = oracle_mod.deltanet(x["q"], x["k"], x["v"], x["beta"], x["alpha"], S0.double())
    assert rel_l2(o.float().cpu().numpy(), o_ref) <= TOL
    assert rel_l2(S.cpu().numpy(), S_ref) <= TOL


def test_split_not_taken_gives_the_plain_call(dn):
    """Where the split does not apply (here: too many heads for the SMs) the
    permission changes nothing: the results are the plain call's, bit for bit."""
    B, H, T = 4, 16, 1024
    assert dn.seq_segments(B, H, T, 128, 128) == 1
    x = gen.make_inputs(B, H, T, 128, 128, torch.bfloat16, gated=True, seed=3)
    o, S = _run(dn, x, None, True)
    o1, S1 = _run(dn, x, None, False)
    assert np.array_equal(o, o1) and np.array_equal(S, S1)
