"""Chunkwise (WY / Householder) form of the delta rule, numpy float64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The pages state that the delta updates of a chunk can all be computed at once
through a Householder reparameterisation ("GPT-2 から Kimi K3 まで", news.ainew.jp,
section "DeltaNet (Parallelizing linear transformers with delta rule)": a
first-order linear recurrence with generalised Householder transition matrices),
and give the additive chunk loop (same section: ``o = q_c S + tril(q_c k_c^T) v_c``,
``S += k_c^T v_c``).  The reparameterised formula itself is cut off on the page,
so the form below is derived from the per-token recurrence, for a chunk of rows
r = 1..C entered with state S0 (gates alpha, write strengths beta):

    Gamma[r, s] = alpha_{s+1} * ... * alpha_r   for s <= r, else 0
    gamma[r]    = alpha_1 * ... * alpha_r
    A = strictly_lower(diag(beta) (K K^T * Gamma)),   T = (I + A)^-1
    U = T diag(beta) (V - diag(gamma) K S0)           (the chunk's deltas)
    O = diag(gamma) Q S0 + (tril(Q K^T) * Gamma) U
    S_C = gamma_C S0 + (diag(gamma_C / gamma) K)^T U

Ungated: alpha = 1, so Gamma is the lower-triangular ones matrix, gamma = 1.
The gates enter as products, not as exp(log), so alpha = 0 is exact here.

Parity: pinned by tests/test_chunk_form.py (equals the per-token oracle for
every chunk size, including C = 1 and C = T).
"""
from __future__ import annotations

import numpy as np


def _decay_tables(a):
    """Gamma (C x C) and gamma (C,) for one chunk's gates ``a`` (products)."""
    C = a.shape[0]
    Gam = np.zeros((C, C))
    for r in range(C):
        Gam[r, r] = 1.0
        for s in range(r - 1, -1, -1):
            Gam[r, s] = Gam[r, s + 1] * a[s + 1]
    gam = np.cumprod(a)
    return Gam, gam


def deltanet_chunked(q, k, v, beta, alpha=None, S0=None, C: int = 64):
    """Chunkwise delta rule.  Arrays (B,H,T,D) float64-convertible; returns (o, S)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    beta = np.asarray(beta, np.float64)
    B, H, T, Dk = q.shape
    Dv = v.shape[-1]
    alpha = np.ones((B, H, T)) if alpha is None else np.asarray(alpha, np.float64)
    S_all = np.zeros((B, H, Dk, Dv)) if S0 is None else np.array(S0, np.float64)
    o = np.zeros((B, H, T, Dv))
    for b in range(B):
        for h in range(H):
            S = S_all[b, h].copy()
            for c0 in range(0, T, C):
                sl = slice(c0, min(c0 + C, T))
                Q, K, V = q[b, h, sl], k[b, h, sl], v[b, h, sl]
                bt, a = beta[b, h, sl], alpha[b, h, sl]
                n = Q.shape[0]
                Gam, gam = _decay_tables(a)
                A = np.tril(bt[:, None] * (K @ K.T) * Gam, -1)
                Tm = np.linalg.inv(np.eye(n) + A)
                U = Tm @ (bt[:, None] * (V - gam[:, None] * (K @ S)))
                o[b, h, sl] = gam[:, None] * (Q @ S) + (np.tril(Q @ K.T) * Gam) @ U
                tail = Gam[n - 1]  # gamma_C / gamma_s as products: Gamma[C-1, s]
                S = gam[n - 1] * S + (tail[:, None] * K).T @ U
            S_all[b, h] = S
    return o, S_all


def linear_attn_chunked(q, k, v, S0=None, z0=None, C: int = 64):
    """Chunkwise ELU+1 linear attention (the additive chunk loop plus normaliser).

    Additive chunk loop of "GPT-2 から Kimi K3 まで" (news.ainew.jp), section
    "DeltaNet (Parallelizing linear transformers with delta rule)", applied to
    the feature-mapped q', k' of section "Linear attention", with the
    normaliser z carried the same way as S.
    """
    def fmap(x):
        x = np.asarray(x, np.float64)
        return np.where(x > 0, x, np.expm1(np.minimum(x, 0.0))) + 1.0

    qp, kp = fmap(q), fmap(k)
    v = np.asarray(v, np.float64)
    B, H, T, Dk = qp.shape
    Dv = v.shape[-1]
    S_all = np.zeros((B, H, Dk, Dv)) if S0 is None else np.array(S0, np.float64)
    z_all = np.zeros((B, H, Dk)) if z0 is None else np.array(z0, np.float64)
    o = np.zeros((B, H, T, Dv))
    for b in range(B):
        for h in range(H):
            S, z = S_all[b, h].copy(), z_all[b, h].copy()
            for c0 in range(0, T, C):
                sl = slice(c0, min(c0 + C, T))
                Q, K, V = qp[b, h, sl], kp[b, h, sl], v[b, h, sl]
                P = np.tril(Q @ K.T)
                num = Q @ S + P @ V
                den = Q @ z + P.sum(axis=1)
                o[b, h, sl] = num / den[:, None]
                S = S + K.T @ V
                z = z + K.sum(axis=0)
            S_all[b, h], z_all[b, h] = S, z
    return o, S_all, z_all


def deltanet_chunked_bwd(q, k, v, beta, dO, alpha=None, S0=None, dS_T=None, C: int = 64):
    """Gradient of the chunk form above, chunk by chunk from the last (numpy
    float64, test-side math).  The loss is sum(dO * o) + sum(dS_T * S_T).
    Returns dict(dq, dk, dv, dbeta, dlogalpha, dS0); dlogalpha (the gradient with
    respect to log alpha, = alpha * dL/dalpha) is None when ungated.

    With g the within-chunk cumulative log decay, Gamma = exp(g_r - g_s) and
    gamma = exp(g), every quantity of the forward is a product of matrices, so
    the reverse pass runs the same products transposed:
      dU  = (tril(Q K^T) * Gamma)^T dO + K_out dS+          K_out = diag(gamma_n / gamma) K
      dS  = (diag(gamma) Q)^T dO + gamma_n dS+ - W^T dU     W = T diag(beta gamma) K
      dP  = tril(dO U^T)  (scores),  dT = dW (diag(beta gamma) K)^T + dU (diag(beta) V)^T
      dA  = -strict_lower(T^T dT T^T)
    and the chain rule through Gamma / gamma gives the gradient of g, whose
    reverse cumulative sum within the chunk is the gradient of log alpha.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    beta = np.asarray(beta, np.float64)
    dO = np.asarray(dO, np.float64)
    B, H, T, Dk = q.shape
    Dv = v.shape[-1]
    gated = alpha is not None
    la = np.zeros((B, H, T)) if alpha is None else np.log(np.asarray(alpha, np.float64))
    out = dict(dq=np.zeros((B, H, T, Dk)), dk=np.zeros((B, H, T, Dk)), dv=np.zeros((B, H, T, Dv)),
               dbeta=np.zeros((B, H, T)), dlogalpha=np.zeros((B, H, T)) if gated else None,
               dS0=np.zeros((B, H, Dk, Dv)))
    for b in range(B):
        for h in range(H):
            chunks = [slice(c0, min(c0 + C, T)) for c0 in range(0, T, C)]
            # forward: entry state of every chunk
            S = np.zeros((Dk, Dv)) if S0 is None else np.array(S0[b, h], np.float64)
            entry = []
            for sl in chunks:
                entry.append(S.copy())
                Q, K, V, bt = q[b, h, sl], k[b, h, sl], v[b, h, sl], beta[b, h, sl]
                n = Q.shape[0]
                g = np.cumsum(la[b, h, sl])
                Gam = np.tril(np.exp(g[:, None] - g[None, :]))
                gam = np.exp(g)
                Tm = np.linalg.inv(np.eye(n) + np.tril(bt[:, None] * (K @ K.T) * Gam, -1))
                U = Tm @ (bt[:, None] * (V - gam[:, None] * (K @ S)))
                S = gam[-1] * S + (np.exp(g[-1] - g)[:, None] * K).T @ U
            dSp = np.zeros((Dk, Dv)) if dS_T is None else np.array(dS_T[b, h], np.float64)
            for ci in range(len(chunks) - 1, -1, -1):
                sl, S = chunks[ci], entry[ci]
                Q, K, V, bt = q[b, h, sl], k[b, h, sl], v[b, h, sl], beta[b, h, sl]
                dOc = dO[b, h, sl]
                n = Q.shape[0]
                g = np.cumsum(la[b, h, sl])
                Gam = np.tril(np.exp(g[:, None] - g[None, :]))
                gam = np.exp(g)
                e_out = np.exp(g[-1] - g)
                MA = (K @ K.T) * Gam
                A = np.tril(bt[:, None] * MA, -1)
                Tm = np.linalg.inv(np.eye(n) + A)
                BK = (bt * gam)[:, None] * K
                BV = bt[:, None] * V
                W, Uh = Tm @ BK, Tm @ BV
                U = Uh - W @ S
                MP = np.tril((Q @ K.T) * Gam)
                Kout = e_out[:, None] * K
                # reverse
                dU = MP.T @ dOc + Kout @ dSp
                dS = (gam[:, None] * Q).T @ dOc + gam[-1] * dSp - W.T @ dU
                dMP = np.tril(dOc @ U.T)
                dQ = gam[:, None] * (dOc @ S.T) + (dMP * Gam) @ K
                dK = (dMP * Gam).T @ Q + e_out[:, None] * (U @ dSp.T)
                dg = gam * np.sum(dOc * (Q @ S), axis=1)
                EP = dMP * MP
                dg += EP.sum(1) - EP.sum(0)
                c_out = e_out * np.sum(K * (U @ dSp.T), axis=1)
                dg[-1] += gam[-1] * np.sum(dSp * S) + c_out.sum()
                dg -= c_out
                dW = -dU @ S.T
                dT = dW @ BK.T + dU @ BV.T
                dBK, dBV = Tm.T @ dW, Tm.T @ dU
                dV = bt[:, None] * dBV
                dK += (bt * gam)[:, None] * dBK
                dbt = gam * np.sum(dBK * K, axis=1) + np.sum(dBV * V, axis=1)
                dg += bt * gam * np.sum(dBK * K, axis=1)
                dA = -np.tril(Tm.T @ dT @ Tm.T, -1)
                dbt += np.sum(dA * MA, axis=1)
                dMA = bt[:, None] * dA
                dK += (dMA * Gam) @ K + (dMA * Gam).T @ K
                EA = dMA * MA
                dg += EA.sum(1) - EA.sum(0)
                out["dq"][b, h, sl] = dQ
                out["dk"][b, h, sl] = dK
                out["dv"][b, h, sl] = dV
                out["dbeta"][b, h, sl] = dbt
                if gated:
                    out["dlogalpha"][b, h, sl] = np.cumsum(dg[::-1])[::-1]
                dSp = dS
            out["dS0"][b, h] = dSp
    return out
