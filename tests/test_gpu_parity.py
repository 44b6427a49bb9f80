"""GPU parity: the CUDA path through the C ABI against the float64 oracle.

Gates (relative L2 error, ||x - x_ref|| / ||x_ref||, on o and on the final
state): 1e-4 for float32 inputs (float32 arithmetic throughout), 2e-2 for
bfloat16 inputs (bf16 tensor-core operands, float32 state and accumulation,
bf16 output rounding).  Inputs come from the seeded generator module; the
oracle sees the identical stored values.
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

    m.lib()  # fail loudly if the library is missing
    return m


def _cpu(t):
    return None if t is None else t.detach().cpu()


def _to(d, dev):
    return {k: (None if v is None else v.to(dev)) for k, v in d.items()}


def _run_delta(dn, x, C=64, S0=None):
    dev = torch.device("cuda")
    g = _to(x, dev)
    o, S = dn.deltanet_chunk_fwd(g["q"], g["k"], g["v"], g["beta"], g["alpha"],
                                 None if S0 is None else S0.to(dev), C=C)
    torch.cuda.synchronize()
    assert dn.deltanet_get_device_status() == 0
    return o.float().cpu().numpy(), S.cpu().numpy()


def _check_delta(dn, oracle_mod, x, C=64, S0=None):
    o, S = _run_delta(dn, x, C, S0)
    o_ref, S_ref = oracle_mod.deltanet(x["q"], x["k"], x["v"], x["beta"], x["alpha"],
                                       None if S0 is None else S0.double())
    tol = TOL[x["q"].dtype]
    eo, es = rel_l2(o, o_ref), rel_l2(S, S_ref)
    assert eo <= tol and es <= tol, f"rel-L2 o={eo:.3e} S={es:.3e} (tol {tol})"
    return eo, es


def test_tiny_fp32_config(dn, oracle_mod):
    """The tiny configuration exactly: B1 H2 T256 D64 fp32, C64, seed 0."""
    w = gen.TINY
    x = gen.make_workload(w, seed=0)
    _check_delta(dn, oracle_mod, x, C=w.C)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("Dk,Dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("T", [1, 63, 64, 200, 333])
def test_delta_shapes_ragged(dn, oracle_mod, dtype, Dk, Dv, T):
    x = gen.make_inputs(2, 3, T, Dk, Dv, dtype, gated=False, seed=T + Dk)
    _check_delta(dn, oracle_mod, x)


@pytest.mark.parametrize("gated", [False, True])
def test_slice_width_wide_and_narrow_grids(dn, oracle_mod, gated):
    """The bf16 C = 64 kernel splits Dv into 64-column slices, or into 32-column
    ones when the problem has so few heads that twice the CTAs still fit one wave
    on the B200's 148 SMs.  80 heads (320 32-column slices) take the 64-column
    grid and one of its heads alone the 32-column grid: both match the oracle
    (ragged T, initial state, decay) and give the same bits for the same head."""
    B, H, T = 10, 8, 200
    x = gen.make_inputs(B, H, T, 128, 128, torch.bfloat16, gated=gated, seed=91 + gated)
    S0 = torch.randn(B, H, 128, 128, generator=torch.Generator().manual_seed(5)) * 0.05
    o, S = _run_delta(dn, x, 64, S0)
    o_ref, S_ref = oracle_mod.deltanet(x["q"], x["k"], x["v"], x["beta"], x["alpha"], S0.double())
    tol = TOL[torch.bfloat16]
    assert rel_l2(o, o_ref) <= tol and rel_l2(S, S_ref) <= tol
    one = {k: (None if v is None else v[2:3, 5:6].contiguous()) for k, v in x.items()}
    o1, S1 = _run_delta(dn, one, 64, S0[2:3, 5:6].contiguous())
    assert np.array_equal(o1, o[2:3, 5:6]) and np.array_equal(S1, S[2:3, 5:6])


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("T", [64, 257])
def test_gated(dn, oracle_mod, dtype, T):
    x = gen.make_inputs(2, 2, T, 128, 128, dtype, gated=True, seed=7)
    _check_delta(dn, oracle_mod, x)


@pytest.mark.parametrize("gated", [False, True])
@pytest.mark.parametrize("Dk,Dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("T", [1, 127, 128, 129, 300, 700])
def test_chunk128_bf16(dn, oracle_mod, gated, Dk, Dv, T):
    """Chunk size 128 (bf16): one state application per 128 tokens."""
    x = gen.make_inputs(2, 2, T, Dk, Dv, torch.bfloat16, gated=gated, seed=300 + T + Dk + Dv)
    _check_delta(dn, oracle_mod, x, C=128)


@pytest.mark.parametrize("gated", [False, True])
def test_chunk128_initial_state_and_gate_zero(dn, oracle_mod, gated):
    x = gen.make_inputs(1, 3, 333, 128, 128, torch.bfloat16, gated=gated, seed=41)
    if gated:
        x["alpha"][:, :, 150] = 0.0
    S0 = torch.randn(1, 3, 128, 128, generator=torch.Generator().manual_seed(5)) * 0.2
    _check_delta(dn, oracle_mod, x, C=128, S0=S0)


def test_chunk_size_invariance_bf16(dn):
    """C = 64 and C = 128 compute the same recurrence: the two results agree to
    within the bf16 gate (each is within it of the oracle)."""
    x = gen.make_inputs(2, 2, 1000, 128, 128, torch.bfloat16, gated=True, seed=42)
    o1, S1 = _run_delta(dn, x, C=64)
    o2, S2 = _run_delta(dn, x, C=128)
    assert rel_l2(o2, o1) <= 2 * TOL[torch.bfloat16] and rel_l2(S2, S1) <= 2 * TOL[torch.bfloat16]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_gated_strong_decay_both_sides_of_the_factor_range(dn, oracle_mod, dtype):
    """Steep gates: per 64-token chunk the log-decay spans about 145 in head 0
    (the decay factors split about the chunk's midpoint) and about 170 in
    head 1 (one exponential per element); head 2 mixes steep and mild gates."""
    x = gen.make_inputs(1, 3, 300, 128, 128, dtype, gated=True, seed=13)
    x["alpha"][:, 0] = float(np.exp(-2.3))
    x["alpha"][:, 1] = float(np.exp(-2.7))
    x["alpha"][:, 2, ::3] = float(np.exp(-6.0))
    _check_delta(dn, oracle_mod, x)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_gate_zero_and_one(dn, oracle_mod, dtype):
    x = gen.make_inputs(1, 2, 190, 128, 128, dtype, gated=True, seed=8)
    x["alpha"][:, :, 70] = 0.0
    x["alpha"][:, :, 100:140] = 1.0
    _check_delta(dn, oracle_mod, x)
    # alpha == 1 everywhere equals the ungated call
    ones = dict(x, alpha=torch.ones_like(x["alpha"]))
    o1, S1 = _run_delta(dn, ones)
    o2, S2 = _run_delta(dn, dict(x, alpha=None))
    assert rel_l2(o1, o2) <= TOL[dtype] * 0.1 and rel_l2(S1, S2) <= TOL[dtype] * 0.1


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_initial_state_and_resume(dn, oracle_mod, dtype):
    """Two calls with S carried equal one call (the cache contract)."""
    x = gen.make_inputs(2, 2, 300, 128, 128, dtype, gated=True, seed=9)
    S0 = torch.randn(2, 2, 128, 128, generator=torch.Generator().manual_seed(1)) * 0.1
    _check_delta(dn, oracle_mod, x, S0=S0)
    a = {k: (None if v is None else v[:, :, :130].contiguous()) for k, v in x.items()}
    b = {k: (None if v is None else v[:, :, 130:].contiguous()) for k, v in x.items()}
    oa, Sa = _run_delta(dn, a, S0=S0)
    ob, Sb = _run_delta(dn, b, S0=torch.from_numpy(Sa))
    o_ref, S_ref = oracle_mod.deltanet(x["q"], x["k"], x["v"], x["beta"], x["alpha"], S0.double())
    tol = TOL[dtype]
    assert rel_l2(np.concatenate([oa, ob], 2), o_ref) <= tol
    assert rel_l2(Sb, S_ref) <= tol


def test_in_place_state_carry(dn, oracle_mod):
    x = gen.make_inputs(1, 2, 150, 128, 128, torch.bfloat16, seed=10)
    dev = torch.device("cuda")
    g = _to(x, dev)
    S = (torch.randn(1, 2, 128, 128, generator=torch.Generator().manual_seed(2)) * 0.1)
    S_ref0 = S.double().clone()
    Sg = S.to(dev)
    dn.deltanet_chunk_fwd(g["q"], g["k"], g["v"], g["beta"], None, Sg, S_out=Sg)
    torch.cuda.synchronize()
    _, S_ref = oracle_mod.deltanet(x["q"], x["k"], x["v"], x["beta"], None, S_ref0)
    assert rel_l2(Sg.cpu().numpy(), S_ref) <= 2e-2


def test_empty_sequence_copies_state(dn):
    dev = torch.device("cuda")
    q = torch.zeros(2, 2, 0, 64, dtype=torch.bfloat16, device=dev)
    S0 = torch.randn(2, 2, 64, 64, device=dev)
    o, S = dn.deltanet_chunk_fwd(q, q, q, torch.zeros(2, 2, 0, device=dev), None, S0)
    torch.cuda.synchronize()
    assert o.shape == (2, 2, 0, 64)
    assert torch.equal(S, S0)


@pytest.mark.parametrize("dtype,C", [(torch.bfloat16, 64), (torch.bfloat16, 128), (torch.float32, 64)])
@pytest.mark.parametrize("with_S0", [True, False])
def test_empty_sequence_every_chunk_size(dn, dtype, C, with_S0):
    """T = 0 copies S0 (or zeros) to S_out for every built chunk size and dtype,
    on the device call and on the host-buffer call."""
    dev = torch.device("cuda")
    q = torch.zeros(2, 3, 0, 128, dtype=dtype, device=dev)
    S0 = torch.randn(2, 3, 128, 128, device=dev) if with_S0 else None
    S_out = torch.full((2, 3, 128, 128), float("nan"), device=dev)
    o, S = dn.deltanet_chunk_fwd(q, q, q, torch.zeros(2, 3, 0, device=dev), None, S0, C=C,
                                 S_out=S_out)
    torch.cuda.synchronize()
    assert o.shape == (2, 3, 0, 128)
    assert torch.equal(S, S0 if with_S0 else torch.zeros_like(S))
    qh = torch.zeros(2, 3, 0, 128, dtype=dtype)
    oh, Sh = dn.deltanet_chunk_fwd_host(qh, qh, qh, torch.zeros(2, 3, 0), None,
                                        None if S0 is None else S0.cpu(), C=C)
    torch.cuda.synchronize()
    assert torch.equal(Sh, S.cpu())


def test_linear_attn_empty_sequence_copies_state(dn):
    dev = torch.device("cuda")
    q = torch.zeros(1, 2, 0, 64, dtype=torch.bfloat16, device=dev)
    S0 = torch.rand(1, 2, 64, 64, device=dev)
    z0 = torch.rand(1, 2, 64, device=dev) + 1
    _, S, z = dn.linear_attn_fwd(q, q, q, S0, z0)
    _, S2, z2 = dn.linear_attn_fwd(q, q, q)
    torch.cuda.synchronize()
    assert torch.equal(S, S0) and torch.equal(z, z0)
    assert not S2.any() and not z2.any()


def test_more_heads_than_one_grid_row(dn, oracle_mod):
    """B * H = 70,000 sequences (past the 65,535 limit of a grid's second
    dimension), three tokens each: every head is computed; sampled heads match
    the oracle and all heads are finite."""
    dev = torch.device("cuda")
    x = gen.make_inputs(1, 70000, 3, 64, 64, torch.bfloat16, gated=True, seed=17)
    g = _to(x, dev)
    o, S = dn.deltanet_chunk_fwd(g["q"], g["k"], g["v"], g["beta"], g["alpha"])
    torch.cuda.synchronize()
    assert dn.deltanet_get_device_status() == 0
    assert torch.isfinite(o.float()).all() and torch.isfinite(S).all()
    o_ref, S_ref = oracle_mod.deltanet(x["q"], x["k"], x["v"], x["beta"], x["alpha"])
    assert rel_l2(o.float().cpu(), o_ref) <= TOL[torch.bfloat16]
    assert rel_l2(S.cpu(), S_ref) <= TOL[torch.bfloat16]
    for h in (0, 65535, 65536, 69999):
        assert rel_l2(S[0, h].cpu(), S_ref[0, h]) <= TOL[torch.bfloat16]


def test_deterministic(dn):
    x = _to(gen.make_inputs(2, 4, 500, 128, 128, torch.bfloat16, gated=True, seed=11), "cuda")
    o1, S1 = dn.deltanet_chunk_fwd(x["q"], x["k"], x["v"], x["beta"], x["alpha"])
    o2, S2 = dn.deltanet_chunk_fwd(x["q"], x["k"], x["v"], x["beta"], x["alpha"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


# -- linear attention ------------------------------------------------------------

def _check_linear(dn, oracle_mod, x, S0=None, z0=None):
    dev = torch.device("cuda")
    o, S, z = dn.linear_attn_fwd(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev),
                                 None if S0 is None else S0.to(dev),
                                 None if z0 is None else z0.to(dev))
    torch.cuda.synchronize()
    o_ref, S_ref, z_ref = oracle_mod.linear_attn(x["q"], x["k"], x["v"],
                                                 None if S0 is None else S0.double(),
                                                 None if z0 is None else z0.double())
    tol = TOL[x["q"].dtype]
    e = (rel_l2(o.float().cpu(), o_ref), rel_l2(S.cpu(), S_ref), rel_l2(z.cpu(), z_ref))
    assert max(e) <= tol, f"rel-L2 o,S,z = {e}"


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("Dk,Dv", [(64, 64), (128, 128), (128, 64)])
@pytest.mark.parametrize("T", [1, 64, 200])
def test_linear_attn(dn, oracle_mod, dtype, Dk, Dv, T):
    x = gen.make_inputs(2, 2, T, Dk, Dv, dtype, seed=12 + T)
    _check_linear(dn, oracle_mod, x)


def test_linear_attn_carry(dn, oracle_mod):
    x = gen.make_inputs(1, 3, 150, 128, 128, torch.bfloat16, seed=13)
    g = torch.Generator().manual_seed(3)
    S0 = torch.rand(1, 3, 128, 128, generator=g)
    z0 = torch.rand(1, 3, 128, generator=g) + 1
    _check_linear(dn, oracle_mod, x, S0, z0)


# -- decode ------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("Dk,Dv", [(128, 128), (64, 64), (64, 128), (128, 64)])
@pytest.mark.parametrize("gated", [False, True])
def test_decode_steps(dn, oracle_mod, dtype, Dk, Dv, gated):
    """Several decode steps from a random state equal the oracle recurrence."""
    B, H, steps = 3, 5, 6
    dev = torch.device("cuda")
    S0 = torch.randn(B, H, Dk, Dv, generator=torch.Generator().manual_seed(4)) * 0.2
    S = S0.to(dev)
    seq = gen.make_inputs(B, H, steps, Dk, Dv, dtype, gated=gated, seed=14)
    outs = []
    for t in range(steps):
        st = {k: (None if v is None else v[:, :, t].contiguous().to(dev)) for k, v in seq.items()}
        outs.append(dn.deltanet_decode_step(st["q"], st["k"], st["v"], st["beta"], S,
                                            alpha=st["alpha"]).float().cpu())
    torch.cuda.synchronize()
    o = torch.stack(outs, 2).numpy()
    o_ref, S_ref = oracle_mod.deltanet(seq["q"], seq["k"], seq["v"], seq["beta"], seq["alpha"],
                                       S0.double())
    tol = TOL[dtype]
    assert rel_l2(o, o_ref) <= tol and rel_l2(S.cpu(), S_ref) <= tol


def test_decode_after_prefill(dn, oracle_mod):
    """Decode continues from the chunked prefill's final state."""
    dev = torch.device("cuda")
    B, H, T, steps = 2, 4, 130, 5
    x = gen.make_inputs(B, H, T + steps, 128, 128, torch.bfloat16, seed=15)
    pre = {k: (None if v is None else v[:, :, :T].contiguous().to(dev)) for k, v in x.items()}
    _, S = dn.deltanet_chunk_fwd(pre["q"], pre["k"], pre["v"], pre["beta"])
    outs = []
    for t in range(T, T + steps):
        st = {k: (None if v is None else v[:, :, t].contiguous().to(dev)) for k, v in x.items()}
        outs.append(dn.deltanet_decode_step(st["q"], st["k"], st["v"], st["beta"], S).float().cpu())
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_mod.deltanet(x["q"], x["k"], x["v"], x["beta"])
    assert rel_l2(torch.stack(outs, 2).numpy(), o_ref[:, :, T:]) <= 2e-2
    assert rel_l2(S.cpu(), S_ref) <= 2e-2


# -- bounded waits -------------------------------------------------------------------

def test_bounded_wait_times_out_cleanly(dn):
    """A wait nothing satisfies ends in DN_ERR_DEVICE_TIMEOUT read by the host, and the
    context keeps working afterwards."""
    dev = torch.device("cuda")
    ws = torch.zeros(dn.lib().deltanet_workspace_bytes(1, 1, 64, 64, 64, 64, 1), dtype=torch.uint8,
                     device=dev)
    assert dn.deltanet_selftest_wait_timeout(20_000_000, ws) == 0
    assert dn.deltanet_get_device_status(workspace=ws) == dn._lib.DN_ERR_DEVICE_TIMEOUT
    dn.reset_device_status(workspace=ws)
    assert dn.deltanet_get_device_status(workspace=ws) == 0
    x = _to(gen.make_inputs(1, 1, 64, 64, 64, torch.bfloat16, seed=16), dev)
    dn.deltanet_chunk_fwd(x["q"], x["k"], x["v"], x["beta"], workspace=ws)
    assert dn.deltanet_get_device_status(workspace=ws) == 0
