"""Pins of the float64 oracle against what the pages and the mathematics fix.

None of these re-types the oracle's loop: each checks a property the pages
state, a closed form, an independent expansion, or a hand-worked fixture.
"""
import json
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, rng):
    return rng.standard_normal(shape).astype(np.float32)


def _unit_rows(x):
    return (x / np.linalg.norm(x, axis=-1, keepdims=True)).astype(np.float32)


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _seq(a, D=None):
    """(T, D) list -> (1, 1, T, D) float32 array."""
    a = np.asarray(a, np.float32)
    return a.reshape((1, 1) + a.shape)


# -- hand-worked fixtures -------------------------------------------------------

def test_golden_delta_rule(oracle_mod):
    g = _golden("delta_rule_worked.json")
    o, S = oracle_mod.deltanet(_seq(g["q"]), _seq(g["k"]), _seq(g["v"]),
                               np.asarray(g["beta"], np.float32).reshape(1, 1, -1))
    np.testing.assert_allclose(o[0, 0], g["o"], atol=2e-6)
    np.testing.assert_allclose(S[0, 0], g["S"], atol=2e-6)


def test_golden_gated_scalar(oracle_mod):
    g = _golden("gated_scalar_worked.json")
    o, S = oracle_mod.deltanet(_seq(g["q"]), _seq(g["k"]), _seq(g["v"]),
                               np.asarray(g["beta"], np.float32).reshape(1, 1, -1),
                               alpha=np.asarray(g["alpha"], np.float32).reshape(1, 1, -1))
    np.testing.assert_allclose(o[0, 0], g["o"], atol=1e-12)
    np.testing.assert_allclose(S[0, 0], g["S"], atol=1e-12)


def test_golden_linear_attn(oracle_mod):
    g = _golden("linear_attn_worked.json")
    o, S, z = oracle_mod.linear_attn(_seq(g["q"]), _seq(g["k"]), _seq(g["v"]))
    np.testing.assert_allclose(o[0, 0], g["o"], rtol=1e-6)
    np.testing.assert_allclose(S[0, 0], g["S"], rtol=1e-6)
    np.testing.assert_allclose(z[0, 0], g["z"], rtol=1e-6)


# -- properties the pages state ---------------------------------------------------

def test_zero_write_strength_keeps_state(oracle_mod):
    """beta = 0: nothing is written, so S stays S0 and o_t = q_t S0."""
    rng = np.random.default_rng(1)
    B, H, T, Dk, Dv = 2, 3, 17, 8, 5
    q, k, v = _rand((B, H, T, Dk), rng), _unit_rows(_rand((B, H, T, Dk), rng)), _rand((B, H, T, Dv), rng)
    S0 = rng.standard_normal((B, H, Dk, Dv))
    o, S = oracle_mod.deltanet(q, k, v, np.zeros((B, H, T), np.float32), S0=S0)
    np.testing.assert_allclose(S, S0, rtol=0, atol=0)
    np.testing.assert_allclose(o, np.einsum("bhti,bhij->bhtj", q.astype(np.float64), S0), atol=1e-12)


def test_zero_delta_when_value_already_stored(oracle_mod):
    """v_t equal to what k_t reads from the state: the delta is zero, S is unchanged."""
    rng = np.random.default_rng(2)
    B, H, T, Dk, Dv = 1, 2, 23, 6, 7
    q, k = _rand((B, H, T, Dk), rng), _unit_rows(_rand((B, H, T, Dk), rng))
    beta = rng.uniform(0.1, 1.0, (B, H, T)).astype(np.float32)
    S0 = rng.standard_normal((B, H, Dk, Dv)).astype(np.float32).astype(np.float64)
    v32 = np.einsum("bhti,bhij->bhtj", k.astype(np.float64), S0).astype(np.float32)
    o, S = oracle_mod.deltanet(q, k, v32, beta, S0=S0)
    # the only residual is v32's float32 rounding of k S0
    resid = np.abs(v32.astype(np.float64) - np.einsum("bhti,bhij->bhtj", k.astype(np.float64), S0)).max()
    assert np.abs(S - S0).max() <= 4 * T * resid + 1e-12
    np.testing.assert_allclose(o, np.einsum("bhti,bhij->bhtj", q.astype(np.float64), S0),
                               atol=4 * T * resid * np.sqrt(Dk) + 1e-12)


def test_unit_key_full_strength_overwrites(oracle_mod):
    """beta = 1 and |k| = 1: after the write, k_t reads back exactly v_t (q_t = k_t)."""
    rng = np.random.default_rng(3)
    B, H, T, Dk, Dv = 2, 2, 40, 16, 9
    k = _unit_rows(_rand((B, H, T, Dk), rng))
    v = _rand((B, H, T, Dv), rng)
    S0 = rng.standard_normal((B, H, Dk, Dv))
    o, _ = oracle_mod.deltanet(k, k, v, np.ones((B, H, T), np.float32), S0=S0)
    # |k|^2 differs from 1 only by float32 rounding of the normalised key
    n2 = (k.astype(np.float64) ** 2).sum(-1, keepdims=True)
    assert np.abs(n2 - 1).max() < 1e-6
    np.testing.assert_allclose(o, v, atol=2e-5)


def test_orthonormal_keys_closed_form(oracle_mod):
    """Orthonormal keys (T <= Dk), S0 = 0: no read interference, so the deltas are
    beta_t v_t and O = tril(Q K^T) diag(beta) V, S_T = K^T diag(beta) V."""
    rng = np.random.default_rng(4)
    Dk, Dv, T = 12, 6, 10
    Kf = np.linalg.qr(rng.standard_normal((Dk, Dk)))[0][:T]  # orthonormal rows
    k = Kf.astype(np.float32)
    k64 = k.astype(np.float64)
    q, v = _rand((T, Dk), rng), _rand((T, Dv), rng)
    beta = rng.uniform(0, 1, T).astype(np.float32)
    o, S = oracle_mod.deltanet(_seq(q), _seq(k), _seq(v), beta.reshape(1, 1, T))
    # float32 rounding leaves k_s . k_t ~ 1e-7 off zero; the closed form holds to that order
    G = k64 @ k64.T
    off = np.abs(G - np.diag(np.diag(G))).max()
    bv = beta[:, None].astype(np.float64) * v
    S_ref = (k64 * 1.0).T @ (bv * 1.0)
    O_ref = np.tril(q.astype(np.float64) @ k64.T) @ bv
    np.testing.assert_allclose(S[0, 0], S_ref, atol=50 * off + 1e-6)
    np.testing.assert_allclose(o[0, 0], O_ref, atol=50 * off * np.abs(q).max() * Dk + 1e-6)


def test_householder_transition(oracle_mod):
    """One token: S_1 = (I - beta k^T k) S0 + beta k^T v (generalised Householder form)."""
    rng = np.random.default_rng(5)
    Dk, Dv = 9, 4
    k = _unit_rows(_rand((1, Dk), rng))
    v, q = _rand((1, Dv), rng), _rand((1, Dk), rng)
    S0 = rng.standard_normal((Dk, Dv))
    beta = np.float32(0.37)
    _, S = oracle_mod.deltanet(_seq(q), _seq(k), _seq(v), np.full((1, 1, 1), beta),
                               S0=S0.reshape(1, 1, Dk, Dv))
    k64, b = k.astype(np.float64), float(beta)
    Hh = np.eye(Dk) - b * k64.T @ k64
    np.testing.assert_allclose(S[0, 0], Hh @ S0 + b * k64.T @ v.astype(np.float64), atol=1e-12)


def test_unrolled_transition_product(oracle_mod):
    """Brute force on tiny inputs: S_T = sum_t (M_T ... M_{t+1}) N_t + (M_T ... M_1) S0 with
    M_t = alpha_t (I - beta_t k_t^T k_t), N_t = beta_t k_t^T v_t; o_t = q_t S_t."""
    rng = np.random.default_rng(6)
    T, Dk, Dv = 7, 5, 3
    q, k, v = _rand((T, Dk), rng), _unit_rows(_rand((T, Dk), rng)), _rand((T, Dv), rng)
    beta = rng.uniform(0, 1, T).astype(np.float32)
    alpha = rng.uniform(0.2, 1, T).astype(np.float32)
    S0 = rng.standard_normal((Dk, Dv))
    o, S = oracle_mod.deltanet(_seq(q), _seq(k), _seq(v), beta.reshape(1, 1, T),
                               alpha=alpha.reshape(1, 1, T), S0=S0.reshape(1, 1, Dk, Dv))
    K, V, Q = k.astype(np.float64), v.astype(np.float64), q.astype(np.float64)
    Ms = [float(alpha[t]) * (np.eye(Dk) - float(beta[t]) * np.outer(K[t], K[t])) for t in range(T)]
    Ns = [float(beta[t]) * np.outer(K[t], V[t]) for t in range(T)]
    for t in range(T):
        # expansion: S_t = (M_t...M_0) S0 + sum_{s<=t} (M_t...M_{s+1}) N_s
        prod = np.eye(Dk)
        acc = np.zeros((Dk, Dv))
        for s in range(t, -1, -1):
            acc += prod @ Ns[s]
            prod = prod @ Ms[s]
        St = prod @ S0 + acc
        np.testing.assert_allclose(o[0, 0, t], Q[t] @ St, atol=1e-11)
    np.testing.assert_allclose(S[0, 0], St, atol=1e-11)


def test_gate_one_is_plain_deltanet(oracle_mod):
    rng = np.random.default_rng(7)
    B, H, T, D = 1, 2, 33, 8
    q, k, v = _rand((B, H, T, D), rng), _unit_rows(_rand((B, H, T, D), rng)), _rand((B, H, T, D), rng)
    beta = rng.uniform(0, 1, (B, H, T)).astype(np.float32)
    o1, S1 = oracle_mod.deltanet(q, k, v, beta)
    o2, S2 = oracle_mod.deltanet(q, k, v, beta, alpha=np.ones((B, H, T), np.float32))
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(S1, S2)


def test_gate_zero_wipes_then_writes(oracle_mod):
    """alpha_t = 0: the state is wiped before the write, so S_t = beta_t k_t^T v_t."""
    rng = np.random.default_rng(8)
    T, Dk, Dv = 12, 6, 5
    q, k, v = _rand((T, Dk), rng), _unit_rows(_rand((T, Dk), rng)), _rand((T, Dv), rng)
    beta = rng.uniform(0, 1, T).astype(np.float32)
    alpha = rng.uniform(0.3, 1, T).astype(np.float32)
    alpha[-1] = 0.0
    S0 = rng.standard_normal((1, 1, Dk, Dv))
    _, S = oracle_mod.deltanet(_seq(q), _seq(k), _seq(v), beta.reshape(1, 1, T),
                               alpha=alpha.reshape(1, 1, T), S0=S0)
    np.testing.assert_allclose(S[0, 0], float(beta[-1]) * np.outer(k[-1], v[-1]).astype(np.float64),
                               atol=1e-12)


def test_resume_equals_one_shot(oracle_mod):
    """Carrying S across two calls equals one call over the concatenated sequence
    (the cache contract of the pages' forward(x, cache))."""
    rng = np.random.default_rng(9)
    B, H, T1, T2, D = 2, 2, 19, 13, 8
    T = T1 + T2
    q, k, v = _rand((B, H, T, D), rng), _unit_rows(_rand((B, H, T, D), rng)), _rand((B, H, T, D), rng)
    beta = rng.uniform(0, 1, (B, H, T)).astype(np.float32)
    alpha = rng.uniform(0.5, 1, (B, H, T)).astype(np.float32)
    o, S = oracle_mod.deltanet(q, k, v, beta, alpha=alpha)
    s1, s2 = slice(0, T1), slice(T1, T)
    oa, Sa = oracle_mod.deltanet(q[:, :, s1].copy(), k[:, :, s1].copy(), v[:, :, s1].copy(),
                                 beta[:, :, s1].copy(), alpha=alpha[:, :, s1].copy())
    ob, Sb = oracle_mod.deltanet(q[:, :, s2].copy(), k[:, :, s2].copy(), v[:, :, s2].copy(),
                                 beta[:, :, s2].copy(), alpha=alpha[:, :, s2].copy(), S0=Sa)
    np.testing.assert_allclose(np.concatenate([oa, ob], 2), o, atol=1e-12)
    np.testing.assert_allclose(Sb, S, atol=1e-12)
    # linear attention carries (S, z) the same way
    lo, lS, lz = oracle_mod.linear_attn(q, k, v)
    la, lSa, lza = oracle_mod.linear_attn(q[:, :, s1].copy(), k[:, :, s1].copy(), v[:, :, s1].copy())
    lb, lSb, lzb = oracle_mod.linear_attn(q[:, :, s2].copy(), k[:, :, s2].copy(), v[:, :, s2].copy(),
                                          S0=lSa, z0=lza)
    np.testing.assert_allclose(np.concatenate([la, lb], 2), lo, rtol=1e-12)
    np.testing.assert_allclose(lSb, lS, rtol=1e-12)
    np.testing.assert_allclose(lzb, lz, rtol=1e-12)


def test_linear_attn_matmul_closed_form(oracle_mod):
    """Causal ELU+1 linear attention equals its matmul (C = N) form:
    O = tril(Q' K'^T) V / tril(Q' K'^T) 1, S_T = K'^T V, z_T = K'^T 1, with the feature
    map taken from torch's ELU."""
    rng = np.random.default_rng(10)
    B, H, T, Dk, Dv = 2, 2, 37, 8, 6
    q, k, v = _rand((B, H, T, Dk), rng), _rand((B, H, T, Dk), rng), _rand((B, H, T, Dv), rng)
    o, S, z = oracle_mod.linear_attn(q, k, v)
    elu1 = lambda x: torch.nn.functional.elu(torch.from_numpy(x).double()) + 1
    Qp, Kp, V = elu1(q), elu1(k), torch.from_numpy(v).double()
    P = torch.tril(Qp @ Kp.transpose(-1, -2))
    O_ref = (P @ V) / P.sum(-1, keepdim=True)
    np.testing.assert_allclose(o, O_ref.numpy(), rtol=1e-11)
    np.testing.assert_allclose(S, (Kp.transpose(-1, -2) @ V).numpy(), rtol=1e-11)
    np.testing.assert_allclose(z, Kp.sum(-2).numpy(), rtol=1e-11)


def _elu1(x):
    """ELU(x) + 1 in float64 (x + 1 above zero, e^x at or below)."""
    x = np.asarray(x, np.float64)
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def test_delta_rule_without_read_is_elu1_linear_attention(oracle_mod):
    """The delta update with its read term dropped and beta = 1 is the additive
    update S += k^T v ("GPT-2 から Kimi K3 まで", section "DeltaNet (Fast weight
    programmers)" against section "Linear attention").  With the ELU+1 maps on
    q and k and a ones column appended to V, the additive state's last column
    is the normaliser z and q'S's last entry is q'.z, so the ratio of the other
    columns to it is ELU+1 linear attention.

    Two independent routes to that reduction, both against oracle.linear_attn:
    (1) an additive numpy loop (the delta write with the read removed);
    (2) the delta-rule oracle itself, with the read made to vanish: key t is
        placed in its own block of a T*Dk-dimensional key space (so every key
        is orthogonal to all earlier ones and k_t S_{t-1} = 0 exactly) and the
        query repeats q'_t in every block (so q S_t still sums q'_t . k'_s over
        s <= t)."""
    rng = np.random.default_rng(31)
    T, Dk, Dv = 7, 4, 3
    q = _rand((1, 1, T, Dk), rng)
    k = _rand((1, 1, T, Dk), rng)
    v = _rand((1, 1, T, Dv), rng)
    o_ref, S_ref, z_ref = oracle_mod.linear_attn(q, k, v)
    qp, kp = _elu1(q[0, 0]), _elu1(k[0, 0])
    va = np.concatenate([v[0, 0].astype(np.float64), np.ones((T, 1))], axis=1)

    # (1) additive loop on the augmented values
    S = np.zeros((Dk, Dv + 1))
    o1 = np.zeros((T, Dv))
    for t in range(T):
        S = S + np.outer(kp[t], va[t])  # write; no read term, beta = 1
        r = qp[t] @ S
        o1[t] = r[:Dv] / r[Dv]
    np.testing.assert_allclose(o1, o_ref[0, 0], rtol=1e-12)
    np.testing.assert_allclose(S[:, :Dv], S_ref[0, 0], rtol=1e-12)
    np.testing.assert_allclose(S[:, Dv], z_ref[0, 0], rtol=1e-12)

    # (2) the delta-rule oracle with block-orthogonal keys (float32 inputs)
    kb = np.zeros((1, 1, T, T * Dk), np.float32)
    qb = np.zeros((1, 1, T, T * Dk), np.float32)
    for t in range(T):
        kb[0, 0, t, t * Dk:(t + 1) * Dk] = kp[t]
        qb[0, 0, t] = np.tile(qp[t], T)
    beta = np.ones((1, 1, T), np.float32)
    o2, S2 = oracle_mod.deltanet(qb, kb, va.astype(np.float32).reshape(1, 1, T, Dv + 1), beta)
    ratio = o2[0, 0, :, :Dv] / o2[0, 0, :, Dv:]
    # the ELU+1 values were rounded to float32 once (relative 6e-8 per entry)
    np.testing.assert_allclose(ratio, o_ref[0, 0], rtol=1e-6, atol=1e-6)
    S_fold = S2[0, 0].reshape(T, Dk, Dv + 1).sum(axis=0)  # sum the key blocks back up
    np.testing.assert_allclose(S_fold[:, :Dv], S_ref[0, 0], rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(S_fold[:, Dv], z_ref[0, 0], rtol=1e-6, atol=1e-6)


def test_bf16_inputs_widen_exactly(oracle_mod):
    """bfloat16 inputs give the same result as their exact float32 values."""
    g = torch.Generator().manual_seed(11)
    B, H, T, D = 1, 2, 29, 16
    q, k, v = (torch.randn(B, H, T, D, generator=g).bfloat16() for _ in range(3))
    beta = torch.rand(B, H, T, generator=g)
    o1, S1 = oracle_mod.deltanet(q, k, v, beta)
    o2, S2 = oracle_mod.deltanet(q.float(), k.float(), v.float(), beta)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(S1, S2)
    l1 = oracle_mod.linear_attn(q, k, v)
    l2 = oracle_mod.linear_attn(q.float(), k.float(), v.float())
    for a, b in zip(l1, l2):
        np.testing.assert_array_equal(a, b)


def test_empty_sequence(oracle_mod):
    """T = 0: no outputs, S_out = S0."""
    rng = np.random.default_rng(12)
    S0 = rng.standard_normal((1, 2, 4, 3))
    z = np.zeros((1, 2, 0, 4), np.float32)
    o, S = oracle_mod.deltanet(z, z, np.zeros((1, 2, 0, 3), np.float32),
                               np.zeros((1, 2, 0), np.float32), S0=S0)
    assert o.shape == (1, 2, 0, 3)
    np.testing.assert_array_equal(S, S0)


def test_planted_mistakes_fail_pins(oracle_mod):
    """A wrong oracle must fail the pins above: plant a read from the undecayed state
    and an output taken before the write, in a numpy copy of the recurrence, and check
    the golden fixtures reject both."""
    g = _golden("gated_scalar_worked.json")

    def wrong(read_undecayed, out_before_write):
        S, out = 0.0, []
        for t in range(3):
            a, b, v = g["alpha"][t], g["beta"][t], g["v"][t][0]
            Sd = a * S
            r = S if read_undecayed else Sd
            if out_before_write:
                out.append(Sd)
            S = Sd + b * (v - r)
            if not out_before_write:
                out.append(S)
        return out

    ref = [x[0] for x in g["o"]]
    assert wrong(False, False) == pytest.approx(ref)
    assert wrong(True, False) != pytest.approx(ref)
    assert wrong(False, True) != pytest.approx(ref)


# -- per-dimension decay (KDA) -------------------------------------------------

def test_golden_kda_per_dim(oracle_mod):
    g = _golden("kda_per_dim_worked.json")
    a = np.asarray(g["alpha"], np.float32).reshape(1, 1, 3, 2)
    o, S = oracle_mod.deltanet(_seq(g["q"]), _seq(g["k"]), _seq(g["v"]),
                               np.asarray(g["beta"], np.float32).reshape(1, 1, -1), alpha=a)
    np.testing.assert_allclose(o[0, 0], g["o"], atol=1e-6)
    np.testing.assert_allclose(S[0, 0], g["S"], atol=1e-6)


def test_kda_uniform_decay_is_scalar_gating(oracle_mod):
    """alpha_t[i] = a_t for every key dimension reduces to the scalar gate."""
    rng = np.random.default_rng(41)
    B, H, T, Dk, Dv = 1, 2, 19, 6, 5
    q, v = _rand((B, H, T, Dk), rng), _rand((B, H, T, Dv), rng)
    k = _unit_rows(_rand((B, H, T, Dk), rng))
    beta = rng.uniform(0.1, 0.9, (B, H, T)).astype(np.float32)
    a = rng.uniform(0.3, 1.0, (B, H, T)).astype(np.float32)
    o1, S1 = oracle_mod.deltanet(q, k, v, beta, alpha=a)
    o2, S2 = oracle_mod.deltanet(q, k, v, beta, alpha=np.repeat(a[..., None], Dk, axis=-1))
    np.testing.assert_allclose(o2, o1, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(S2, S1, rtol=1e-13, atol=1e-13)


def test_kda_transition_is_decayed_householder(oracle_mod):
    """Each token maps S to (I - beta k^T k) diag(alpha) S + beta k^T v (the
    generalised Householder transition after the per-dimension decay), and a
    zero decay on dimension i wipes row i before the write."""
    rng = np.random.default_rng(42)
    Dk, Dv, T = 5, 4, 6
    q, v = _rand((1, 1, T, Dk), rng), _rand((1, 1, T, Dv), rng)
    k = _unit_rows(_rand((1, 1, T, Dk), rng))
    beta = rng.uniform(0.2, 1.0, (1, 1, T)).astype(np.float32)
    a = rng.uniform(0.0, 1.0, (1, 1, T, Dk)).astype(np.float32)
    a[0, 0, 2, 1] = 0.0
    S0 = rng.standard_normal((1, 1, Dk, Dv))
    o, S_T = oracle_mod.deltanet(q, k, v, beta, alpha=a, S0=S0)
    S = S0[0, 0].copy()
    for t in range(T):
        kt = k[0, 0, t].astype(np.float64)
        P = np.eye(Dk) - beta[0, 0, t] * np.outer(kt, kt)
        S = P @ np.diag(a[0, 0, t].astype(np.float64)) @ S + beta[0, 0, t] * np.outer(kt, v[0, 0, t])
        np.testing.assert_allclose(o[0, 0, t], q[0, 0, t].astype(np.float64) @ S, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S_T[0, 0], S, rtol=1e-11, atol=1e-12)


# -- the layer's pre-step (silu, L2 normalise, sigmoid) ------------------------------

def test_prestep_is_the_layer_feature_maps(oracle_mod):
    """With the pre-step, q and k pass through F.normalize(F.silu(.)) and beta
    through sigmoid ("GPT-2 から Kimi K3 まで", section "DeltaNet (Fast weight
    programmers)", the layer's forward) before the delta rule: equal to the plain
    oracle on inputs mapped by torch's own silu / normalize / sigmoid (rounded to
    float32 once), gated and not."""
    rng = np.random.default_rng(43)
    B, H, T, Dk, Dv = 2, 2, 23, 8, 6
    q, k, v = _rand((B, H, T, Dk), rng), _rand((B, H, T, Dk), rng), _rand((B, H, T, Dv), rng)
    logit = _rand((B, H, T), rng)
    a = rng.uniform(0.5, 1.0, (B, H, T)).astype(np.float32)
    fmap = lambda x: torch.nn.functional.normalize(torch.nn.functional.silu(torch.from_numpy(x).double()),
                                                   dim=-1).float().numpy()
    b = torch.sigmoid(torch.from_numpy(logit).double()).float().numpy()
    for alpha in (None, a):
        o1, S1 = oracle_mod.deltanet(q, k, v, logit, alpha=alpha, prestep=True)
        o2, S2 = oracle_mod.deltanet(fmap(q), fmap(k), v, b, alpha=alpha)
        np.testing.assert_allclose(o1, o2, rtol=2e-6, atol=2e-6)
        np.testing.assert_allclose(S1, S2, rtol=2e-6, atol=2e-6)


def test_prestep_zero_key_writes_nothing(oracle_mod):
    """silu(0) = 0 and the normaliser's floor keep a zero raw key at zero: that
    token neither reads nor writes (S unchanged, o = q S)."""
    rng = np.random.default_rng(44)
    Dk, Dv = 4, 3
    q, v = _rand((1, 1, 1, Dk), rng), _rand((1, 1, 1, Dv), rng)
    k = np.zeros((1, 1, 1, Dk), np.float32)
    S0 = rng.standard_normal((1, 1, Dk, Dv))
    o, S = oracle_mod.deltanet(q, k, v, np.zeros((1, 1, 1), np.float32), S0=S0, prestep=True)
    np.testing.assert_allclose(S, S0, rtol=0, atol=0)
    qn = torch.nn.functional.normalize(torch.nn.functional.silu(torch.from_numpy(q[0, 0, 0]).double()),
                                       dim=-1).numpy()
    np.testing.assert_allclose(o[0, 0, 0], qn @ S0[0, 0], rtol=1e-12)


# -- the gradient (reverse sweep) ------------------------------------------------------

def _fd_check(oracle_mod, gated):
    """Every gradient entry of oracle.deltanet_bwd against a central finite
    difference of the forward oracle's loss sum(dO * o) + sum(dS_T * S_T),
    Richardson-extrapolated (error O(h^4)).  q, k, v, S0 are perturbed in
    float64; beta and alpha (float32 inputs of the oracle) sit on a 2^-14 grid
    and are perturbed by 2^-9 and 2^-8, which float32 holds exactly."""
    rng = np.random.default_rng(61 + gated)
    B, H, T, Dk, Dv = 1, 2, 6, 3, 2
    q = rng.standard_normal((B, H, T, Dk))
    k = rng.standard_normal((B, H, T, Dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, H, T, Dv))
    grid = lambda x: (np.round(x * 2 ** 14) / 2 ** 14).astype(np.float32)
    beta = grid(rng.uniform(0.2, 0.8, (B, H, T)))
    alpha = grid(rng.uniform(0.5, 0.95, (B, H, T))) if gated else None
    S0 = rng.standard_normal((B, H, Dk, Dv)) * 0.5
    dO = rng.standard_normal((B, H, T, Dv))
    dST = rng.standard_normal((B, H, Dk, Dv))
    g = oracle_mod.deltanet_bwd(q, k, v, beta, dO, alpha, S0, dST)

    def loss(q_, k_, v_, b_, a_, s_):
        o, S = oracle_mod.deltanet(q_, k_, v_, b_, a_, s_)
        return float((o * dO).sum() + (S * dST).sum())

    def fd(name, x, h, cast=lambda y: y):
        grad = np.zeros(x.shape)
        for idx in np.ndindex(x.shape):
            def at(step):
                y = x.astype(np.float64).copy()
                y[idx] += step
                args = dict(q_=q, k_=k, v_=v, b_=beta, a_=alpha, s_=S0)
                args[name] = cast(y)
                return loss(**args)
            d1 = (at(h) - at(-h)) / (2 * h)
            d2 = (at(2 * h) - at(-2 * h)) / (4 * h)
            grad[idx] = (4 * d1 - d2) / 3
        return grad

    f32 = lambda y: y.astype(np.float32)
    checks = [("dq", fd("q_", q, 1e-4)), ("dk", fd("k_", k, 1e-4)), ("dv", fd("v_", v, 1e-4)),
              ("dS0", fd("s_", S0, 1e-4)), ("dbeta", fd("b_", beta, 2.0 ** -9, f32))]
    if gated:
        checks.append(("dalpha", fd("a_", alpha, 2.0 ** -9, f32)))
    for name, ref in checks:
        np.testing.assert_allclose(g[name], ref, rtol=1e-7, atol=1e-8, err_msg=name)
    if not gated:
        assert g["dalpha"] is None


def test_gradient_matches_finite_differences(oracle_mod):
    _fd_check(oracle_mod, gated=False)


def test_gradient_matches_finite_differences_gated(oracle_mod):
    _fd_check(oracle_mod, gated=True)


def test_gradient_of_a_single_write(oracle_mod):
    """One token from S0 = 0 (worked by hand): S = b k^T v, o = b (q.k) v, so
    dL/dv = b (q.k) dO + b dS^T k, dL/db = (q.k) (v.dO) + k dS v^T,
    dL/dq = b (v.dO) k, dL/dS0 = q^T dO + dS - b k^T (k (q^T dO + dS))."""
    q = np.array([[[[1.0, 2.0]]]])
    k = np.array([[[[0.6, 0.8]]]])
    v = np.array([[[[3.0, -1.0]]]])
    b = np.array([[[0.5]]], np.float32)
    dO = np.array([[[[1.0, 2.0]]]])
    dS = np.array([[[[0.5, 0.0], [0.0, -1.0]]]])
    g = oracle_mod.deltanet_bwd(q, k, v, b, dO, dS_T=dS)
    qk, vdo = 0.6 + 1.6, 3.0 - 2.0
    kdSv = k[0, 0, 0] @ dS[0, 0] @ v[0, 0, 0]
    np.testing.assert_allclose(g["dv"][0, 0, 0], 0.5 * qk * dO[0, 0, 0] + 0.5 * dS[0, 0].T @ k[0, 0, 0])
    np.testing.assert_allclose(g["dbeta"][0, 0, 0], qk * vdo + kdSv)
    np.testing.assert_allclose(g["dq"][0, 0, 0], 0.5 * vdo * k[0, 0, 0])
    Gt = np.outer(q[0, 0, 0], dO[0, 0, 0]) + dS[0, 0]
    np.testing.assert_allclose(g["dS0"][0, 0], Gt - 0.5 * np.outer(k[0, 0, 0], k[0, 0, 0] @ Gt))


# -- the affine chunk transition behind the sequence split ------------------------

@pytest.mark.parametrize("gated", [False, True])
def test_segments_joined_by_their_affine_maps_give_the_whole_sequence(oracle_mod, gated):
    """The transition over any run of tokens is affine in the entry state ("GPT-2
    から Kimi K3 まで", section "DeltaNet (Parallelizing linear transformers with
    delta rule)": a product of generalised Householder factors, each decayed by
    its gate, plus the writes).  So, on the oracle alone: run each segment from a
    zero state (outputs O', end state S_end) and its homogeneous chain (v = 0
    from S0 = I: outputs R, end state A = the product of its transitions); then
    S_in of the next segment = A S_in + S_end and the segment's outputs are
    O' + R S_in.  Joined over unequal, ragged segments this must reproduce the
    whole sequence from S0, outputs and final state."""
    rng = np.random.default_rng(17 + gated)
    B, H, T, Dk, Dv = 1, 2, 300, 8, 6
    q = torch.from_numpy(_rand((B, H, T, Dk), rng))
    k = torch.from_numpy(_unit_rows(_rand((B, H, T, Dk), rng)))
    v = torch.from_numpy(_rand((B, H, T, Dv), rng))
    beta = torch.from_numpy(rng.uniform(0.1, 1.0, (B, H, T)).astype(np.float32))
    alpha = torch.from_numpy(rng.uniform(0.85, 1.0, (B, H, T)).astype(np.float32)) if gated else None
    S0 = rng.standard_normal((B, H, Dk, Dv))
    o_whole, S_whole = oracle_mod.deltanet(q, k, v, beta, alpha, S0)

    eye = np.broadcast_to(np.eye(Dk), (B, H, Dk, Dk)).copy()
    S_in = S0
    o_join = np.zeros_like(o_whole)
    for a, b in ((0, 110), (110, 171), (171, 300)):
        sl = slice(a, b)
        part = lambda x: None if x is None else x[:, :, sl].contiguous()
        o_zero, S_end = oracle_mod.deltanet(part(q), part(k), part(v), part(beta), part(alpha))
        zeros = torch.zeros(B, H, b - a, Dk)
        R, A = oracle_mod.deltanet(part(q), part(k), zeros, part(beta), part(alpha), eye)
        o_join[:, :, sl] = o_zero + R @ S_in
        S_in = A @ S_in + S_end
    scale = np.abs(o_whole).max()
    assert np.abs(o_join - o_whole).max() <= 1e-11 * scale
    assert np.abs(S_in - S_whole).max() <= 1e-11 * np.abs(S_whole).max()
    # and the homogeneous chain's end state is the product of its transitions:
    # entered with any state X it carries X to A X
    X = rng.standard_normal((B, H, Dk, Dv))
    _, S_X = oracle_mod.deltanet(q[:, :, :50].contiguous(), k[:, :, :50].contiguous(), torch.zeros(B, H, 50, Dv),
                                 beta[:, :, :50].contiguous(), None if alpha is None else alpha[:, :, :50].contiguous(),
                                 X)
    _, A50 = oracle_mod.deltanet(q[:, :, :50].contiguous(), k[:, :, :50].contiguous(), torch.zeros(B, H, 50, Dk),
                                 beta[:, :, :50].contiguous(), None if alpha is None else alpha[:, :, :50].contiguous(),
                                 eye)
    assert np.abs(S_X - A50 @ X).max() <= 1e-12 * np.abs(S_X).max()
