"""The chunkwise WY form (oracle/chunk_form.py) equals the per-token oracle.

The pages give the chunked loop for additive attention and say the delta updates
of a chunk can be computed at once by a Householder reparameterisation, but the
reparameterised formula itself is missing; this pins the derived form (the one
the CUDA chunk kernels implement) against the per-token definition for every
chunk size, including C = 1 (regular recurrence) and C = T (one chunk).
"""
import numpy as np
import pytest

from oracle import chunk_form


def _inputs(seed, B, H, T, Dk, Dv, gated, zero_alpha=False):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, T, Dk)).astype(np.float32)
    k = rng.standard_normal((B, H, T, Dk))
    k = (k / np.linalg.norm(k, axis=-1, keepdims=True)).astype(np.float32)
    v = rng.standard_normal((B, H, T, Dv)).astype(np.float32)
    beta = (1 / (1 + np.exp(-rng.standard_normal((B, H, T))))).astype(np.float32)
    alpha = None
    if gated:
        alpha = np.exp(-np.log1p(np.exp(rng.standard_normal((B, H, T))))).astype(np.float32)
        if zero_alpha:
            alpha[..., T // 3] = 0.0
    S0 = rng.standard_normal((B, H, Dk, Dv))
    return q, k, v, beta, alpha, S0


@pytest.mark.parametrize("gated", [False, True])
@pytest.mark.parametrize("C", [1, 2, 7, 16, 64, 128, 200])
def test_chunk_form_matches_recurrence(oracle_mod, gated, C):
    q, k, v, beta, alpha, S0 = _inputs(C, 1, 2, 200, 16, 12, gated)
    o_ref, S_ref = oracle_mod.deltanet(q, k, v, beta, alpha=alpha, S0=S0)
    o, S = chunk_form.deltanet_chunked(q, k, v, beta, alpha, S0, C=C)
    np.testing.assert_allclose(o, o_ref, atol=1e-10, rtol=1e-10)
    np.testing.assert_allclose(S, S_ref, atol=1e-10, rtol=1e-10)


def test_chunk_form_gate_zero_exact(oracle_mod):
    q, k, v, beta, alpha, S0 = _inputs(5, 1, 1, 130, 8, 8, True, zero_alpha=True)
    o_ref, S_ref = oracle_mod.deltanet(q, k, v, beta, alpha=alpha, S0=S0)
    o, S = chunk_form.deltanet_chunked(q, k, v, beta, alpha, S0, C=64)
    np.testing.assert_allclose(o, o_ref, atol=1e-10)
    np.testing.assert_allclose(S, S_ref, atol=1e-10)


@pytest.mark.parametrize("C", [1, 5, 64, 97])
def test_linear_chunk_form_matches_recurrence(oracle_mod, C):
    rng = np.random.default_rng(C)
    q, k, v = (rng.standard_normal((1, 2, 97, 8)).astype(np.float32) for _ in range(3))
    S0 = rng.uniform(0, 1, (1, 2, 8, 8))
    z0 = rng.uniform(0.5, 1, (1, 2, 8))
    o_ref, S_ref, z_ref = oracle_mod.linear_attn(q, k, v, S0=S0, z0=z0)
    o, S, z = chunk_form.linear_attn_chunked(q, k, v, S0, z0, C=C)
    np.testing.assert_allclose(o, o_ref, rtol=1e-11)
    np.testing.assert_allclose(S, S_ref, rtol=1e-11)
    np.testing.assert_allclose(z, z_ref, rtol=1e-11)


@pytest.mark.parametrize("gated", [False, True])
@pytest.mark.parametrize("C", [1, 5, 16, 64])
def test_chunked_gradient_equals_reverse_sweep(oracle_mod, gated, C):
    """The chunk-form gradient equals the oracle's per-token reverse sweep for
    every chunk size (alpha * dL/dalpha for the log-decay gradient)."""
    from oracle import chunk_form

    rng = np.random.default_rng(70 + C + gated)
    B, H, T, Dk, Dv = 1, 2, 37, 6, 5
    q = rng.standard_normal((B, H, T, Dk))
    k = rng.standard_normal((B, H, T, Dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, H, T, Dv))
    beta = rng.uniform(0.1, 0.9, (B, H, T)).astype(np.float32)
    alpha = rng.uniform(0.4, 1.0, (B, H, T)).astype(np.float32) if gated else None
    S0 = rng.standard_normal((B, H, Dk, Dv)) * 0.3
    dO = rng.standard_normal((B, H, T, Dv))
    dST = rng.standard_normal((B, H, Dk, Dv))
    ref = oracle_mod.deltanet_bwd(q, k, v, beta, dO, alpha, S0, dST)
    got = chunk_form.deltanet_chunked_bwd(q, k, v, beta, dO, alpha, S0, dST, C=C)
    for name in ("dq", "dk", "dv", "dbeta", "dS0"):
        np.testing.assert_allclose(got[name], ref[name], rtol=1e-9, atol=1e-10, err_msg=name)
    if gated:
        np.testing.assert_allclose(got["dlogalpha"], alpha.astype(np.float64) * ref["dalpha"],
                                   rtol=1e-9, atol=1e-10)
