"""Float64 numpy routines of the KDA oracle, for small inputs.

TEST INFRASTRUCTURE ONLY (see the package docstring).

``recurrence_literal``: the KDA recurrence with every matrix formed explicitly,
    S_t = (I - beta_t k_t k_t^T) Diag(exp(g_t)) S_{t-1} + beta_t k_t v_t^T,
    o_t = S_t^T q_t
(miniKimiK3 model card, Architecture, "Kimi Delta Attention" bullet: a delta
rule write with per-channel gated decay).  It is the definition typed out with
numpy matrix products and serves as a second, independent statement of what
``kda_oracle.cpp`` computes.

``chunked``: the chunked parallel form of the same recurrence ("trains through a
chunked parallel form" in the same bullet; the "Inside Kimi" course outline,
DeltaNet lesson: sequential and chunkwise forms must agree).  The pages name the
form but print no equations; the equations below are derived from the
recurrence.  Inside one chunk of length L (positions r, i in [0, L)) with
initial state S0:
    Gamma_r = sum_{j<=r} g_j                      (per key channel)
    Kbar_r  = exp(Gamma_r) * k_r,   Qbar_r = exp(Gamma_r) * q_r
    Kend_i  = exp(Gamma_{L-1} - Gamma_i) * k_i
    A[r,i]  = sum_c k_rc k_ic exp(Gamma_rc - Gamma_ic)   for i < r, else 0
    Aqk[r,i]= sum_c q_rc k_ic exp(Gamma_rc - Gamma_ic)   for i <= r, else 0
    Tm      = (I + diag(beta) A)^-1
    W = Tm diag(beta) Kbar,   U = Tm diag(beta) V,   Delta = U - W S0
    O       = Qbar S0 + Aqk Delta
    S_next  = Diag(exp(Gamma_{L-1})) S0 + Kend^T Delta
Derivation: with S~_r = Diag(exp(-Gamma_r)) S_r the recurrence becomes the
undecayed delta rule S~_r = S~_{r-1} + khat_r delta_r^T, khat_r = exp(-Gamma_r) k_r,
delta_r = beta_r (v_r - S~_{r-1}^T Kbar_r); stacking the rows gives
(I + diag(beta) A) Delta = diag(beta) (V - Kbar S0).
The pairwise exponents exp(Gamma_r - Gamma_i) are evaluated directly, with no
factoring through a reference point.
"""
from __future__ import annotations

import numpy as np

__all__ = ["recurrence_literal", "chunked"]


def recurrence_literal(q, k, v, g, beta, h0=None):
    """One sequence, one head.  q,k,g [T,dk]; v [T,dv]; beta [T]; h0 [dk,dv].
    Returns (o [T,dv], S_T [dk,dv]) in float64."""
    q, k, v, g = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g))
    beta = np.asarray(beta, dtype=np.float64)
    T, dk = k.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv)) if h0 is None else np.array(h0, dtype=np.float64)
    eye = np.eye(dk)
    o = np.zeros((T, dv))
    for t in range(T):
        kt = k[t][:, None]
        S = (eye - beta[t] * (kt @ kt.T)) @ np.diag(np.exp(g[t])) @ S \
            + beta[t] * (kt @ v[t][None, :])
        o[t] = S.T @ q[t]
    return o, S


def chunked(q, k, v, g, beta, h0=None, C: int = 64):
    """One sequence, one head, chunk length C (the last chunk may be shorter).
    Same arguments and results as ``recurrence_literal``."""
    q, k, v, g = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g))
    beta = np.asarray(beta, dtype=np.float64)
    T, dk = k.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv)) if h0 is None else np.array(h0, dtype=np.float64)
    o = np.zeros((T, dv))
    for t0 in range(0, T, C):
        t1 = min(t0 + C, T)
        L = t1 - t0
        qc, kc, vc, bc = q[t0:t1], k[t0:t1], v[t0:t1], beta[t0:t1]
        gam = np.cumsum(g[t0:t1], axis=0)                      # [L, dk]
        kbar = np.exp(gam) * kc
        qbar = np.exp(gam) * qc
        kend = np.exp(gam[-1][None, :] - gam) * kc
        A = np.zeros((L, L))
        Aqk = np.zeros((L, L))
        for r in range(L):
            for i in range(r + 1):
                e = np.exp(gam[r] - gam[i])
                if i < r:
                    A[r, i] = np.sum(kc[r] * kc[i] * e)
                Aqk[r, i] = np.sum(qc[r] * kc[i] * e)
        Tm = np.linalg.inv(np.eye(L) + bc[:, None] * A)
        W = Tm @ (bc[:, None] * kbar)
        U = Tm @ (bc[:, None] * vc)
        delta = U - W @ S
        o[t0:t1] = qbar @ S + Aqk @ delta
        S = np.exp(gam[-1])[:, None] * S + kend.T @ delta
    return o, S
