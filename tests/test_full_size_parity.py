"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times (caller-sized workspace, preallocated outputs, one call over
the whole batch).

The CUDA path runs on every head of the workload; the float64 oracle then
recomputes a few sampled heads in full (whole sequences, from the identical
stored inputs) and the sampled outputs and final states are compared with
the bf16 gate, rel-L2 <= 2e-2 per head.  Sizes:
  prefill         B4 H16 T4096 D128 bf16 C64
  prefill-linear  the same shape, ELU+1 linear attention
  long            B1 H32 T65536 D128 bf16 C64
  forget          B8 H16 T8192 D128 bf16 gated C64
  decode          256 sequences x 32 heads, D128, fp32 states from a 512-token
                  prefill, then 1024 single-token steps with fresh inputs
"""
import numpy as np
import pytest
import torch

from deltanet_sequence_mixing_b200 import inputs as gen

pytestmark = pytest.mark.gpu

TOL = 2e-2


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


def _sample_heads(B, H):
    """First, last and two interior (b, h) pairs."""
    cand = [(0, 0), (B - 1, H - 1), (B // 2, H // 3), ((B - 1) // 3, (2 * H) // 3)]
    out = []
    for bh in cand:
        if bh not in out:
            out.append(bh)
    return out


def _heads(t, heads):
    """(B, H, ...) device tensor -> (1, n, ...) CPU tensor of the sampled heads."""
    if t is None:
        return None
    return torch.stack([t[b, h] for b, h in heads]).unsqueeze(0).cpu()


def _run_chunk_like_bench(dn, w, x):
    dev = x["q"].device
    o = torch.empty_like(x["v"])
    S = torch.empty(w.B, w.H, w.Dk, w.Dv, device=dev)
    nb = dn.lib().deltanet_workspace_bytes(w.B, w.H, w.T, w.Dk, w.Dv, w.C, 1)
    ws = torch.zeros(nb, dtype=torch.uint8, device=dev)
    dn.deltanet_chunk_fwd(x["q"], x["k"], x["v"], x["beta"], x["alpha"], None, C=w.C, o=o,
                          S_out=S, workspace=ws)
    torch.cuda.synchronize()
    assert dn.deltanet_get_device_status(workspace=ws) == 0
    return o, S


@pytest.mark.parametrize("w", [gen.PREFILL, gen.FORGET, gen.LONG64, gen.LONG128], ids=lambda w: w.name)
def test_full_size_chunk_forward_sampled_heads(dn, oracle_mod, w):
    dev = torch.device("cuda")
    x = gen.make_workload(w, seed=11, device=dev)
    o, S = _run_chunk_like_bench(dn, w, x)
    heads = _sample_heads(w.B, w.H)
    sx = {k: _heads(v, heads) for k, v in x.items()}
    o_ref, S_ref = oracle_mod.deltanet(sx["q"], sx["k"], sx["v"], sx["beta"], sx["alpha"])
    o_s = _heads(o, heads).float().numpy()
    S_s = _heads(S, heads).numpy()
    assert np.isfinite(o.float().sum().item()) and np.isfinite(S.sum().item())
    for i, bh in enumerate(heads):
        eo, es = rel_l2(o_s[0, i], o_ref[0, i]), rel_l2(S_s[0, i], S_ref[0, i])
        assert eo <= TOL and es <= TOL, f"{w.name} head {bh}: rel-L2 o={eo:.3e} S={es:.3e}"


def test_full_size_linear_attention_sampled_heads(dn, oracle_mod):
    w = gen.PREFILL_LINEAR
    dev = torch.device("cuda")
    x = gen.make_workload(w, seed=12, device=dev)
    o = torch.empty_like(x["v"])
    S = torch.empty(w.B, w.H, w.Dk, w.Dv, device=dev)
    z = torch.empty(w.B, w.H, w.Dk, device=dev)
    dn.linear_attn_fwd(x["q"], x["k"], x["v"], C=w.C, o=o, S_out=S, z_out=z)
    torch.cuda.synchronize()
    heads = _sample_heads(w.B, w.H)
    sx = {k: _heads(v, heads) for k, v in x.items()}
    o_ref, S_ref, z_ref = oracle_mod.linear_attn(sx["q"], sx["k"], sx["v"])
    o_s, S_s, z_s = (_heads(t, heads).float().numpy() for t in (o, S, z))
    for i, bh in enumerate(heads):
        errs = [rel_l2(o_s[0, i], o_ref[0, i]), rel_l2(S_s[0, i], S_ref[0, i]),
                rel_l2(z_s[0, i], z_ref[0, i])]
        assert max(errs) <= TOL, f"head {bh}: rel-L2 o, S, z = {errs}"


def test_full_size_decode_sampled_states(dn, oracle_mod):
    B, H, D = gen.DECODE_SEQS, gen.DECODE_HEADS, 128
    n_pre, n_steps = gen.DECODE_PREFILL, gen.DECODE_STEPS
    dev = torch.device("cuda")
    pre = gen.make_inputs(B, H, n_pre, D, D, torch.bfloat16, seed=4, device=dev)
    _, S = dn.deltanet_chunk_fwd(pre["q"], pre["k"], pre["v"], pre["beta"])
    steps = gen.make_inputs(B, H, n_steps, D, D, torch.bfloat16, seed=5, device=dev)
    qs, ks, vs = (steps[n].permute(2, 0, 1, 3).contiguous() for n in ("q", "k", "v"))
    bs = steps["beta"].permute(2, 0, 1).contiguous()
    heads = _sample_heads(B, H)
    bi = torch.tensor([b for b, _ in heads], device=dev)
    hi = torch.tensor([h for _, h in heads], device=dev)
    o = torch.empty(B, H, D, dtype=torch.bfloat16, device=dev)
    o_hist = torch.empty(n_steps, len(heads), D, dtype=torch.bfloat16, device=dev)
    for t in range(n_steps):
        dn.deltanet_decode_step(qs[t], ks[t], vs[t], bs[t], S, o=o)
        o_hist[t] = o[bi, hi]
    torch.cuda.synchronize()
    # the oracle runs the plain recurrence over prefill + decode tokens
    sx = {n: torch.cat([_heads(pre[n], heads), _heads(steps[n], heads)], dim=2)
          for n in ("q", "k", "v", "beta")}
    o_ref, S_ref = oracle_mod.deltanet(sx["q"], sx["k"], sx["v"], sx["beta"])
    o_dec = o_hist.permute(1, 0, 2).float().cpu().numpy()
    S_s = _heads(S, heads).numpy()
    for i, bh in enumerate(heads):
        eo = rel_l2(o_dec[i], o_ref[0, i, n_pre:])
        es = rel_l2(S_s[0, i], S_ref[0, i])
        assert eo <= TOL and es <= TOL, f"state {bh}: rel-L2 o={eo:.3e} S={es:.3e}"
