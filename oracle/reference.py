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

``chunked_backward``: the gradients of L = sum(o * dout) + sum(S_T * dhT) taken
through the chunked form above, chunk by chunk in reverse (the form is what
trains, same bullet).  With dS the gradient of the state after a chunk, each
chunk's adjoint is the chain rule applied to the lines above, last line first:
    dDelta  = Aqk^T dO + Kend dS
    dS0     = Qbar^T dO + Diag(exp(Gamma_{L-1})) dS - W^T dDelta
    dU = dDelta,   dW = -dDelta S0^T
    dTm     = dU (diag(beta) V)^T + dW (diag(beta) Kbar)^T
    dM      = -Tm^T dTm Tm^T  (strictly lower part; M = I + diag(beta) A)
and from there to q, k, v, beta and Gamma through the definitions of Qbar, Kbar,
Kend, A and Aqk; dg is the reverse cumulative sum of dGamma inside the chunk.
dS0 is the state gradient at the chunk's start, which the previous chunk takes
as its dS.  It is pinned against the reverse-mode recurrence of the C++ oracle,
which finite differences and autograd pin in turn.
"""
from __future__ import annotations

import numpy as np

__all__ = ["recurrence_literal", "chunked", "chunked_backward"]


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


def _chunk_terms(qc, kc, vc, gc, bc, S0):
    """The chunk quantities of ``chunked`` for one chunk with initial state S0."""
    L = kc.shape[0]
    gam = np.cumsum(gc, axis=0)                                   # [L, dk]
    kbar = np.exp(gam) * kc
    qbar = np.exp(gam) * qc
    kend = np.exp(gam[-1][None, :] - gam) * kc
    # E[r, i, c] = exp(Gamma_rc - Gamma_ic) for i <= r, else exactly 0 (never formed
    # from a positive exponent, so strong decay cannot overflow it)
    lower = np.tril(np.ones((L, L), dtype=bool))[:, :, None]
    E = np.exp(np.where(lower, gam[:, None, :] - gam[None, :, :], -np.inf))
    A = np.tril(np.einsum("rc,ic,ric->ri", kc, kc, E), -1)
    Aqk = np.einsum("rc,ic,ric->ri", qc, kc, E)
    Tm = np.linalg.inv(np.eye(L) + bc[:, None] * A)
    W = Tm @ (bc[:, None] * kbar)
    U = Tm @ (bc[:, None] * vc)
    delta = U - W @ S0
    return dict(gam=gam, kbar=kbar, qbar=qbar, kend=kend, E=E, A=A, Aqk=Aqk, Tm=Tm, W=W,
                delta=delta)


def chunked_backward(q, k, v, g, beta, dout, h0=None, dhT=None, C: int = 64):
    """One sequence, one head: float64 gradients of sum(o * dout) + sum(S_T * dhT)
    through the chunked form with chunk length C.  Arguments as ``chunked``, plus
    dout [T, dv] and dhT [dk, dv] (None: zero).  Returns a dict of dq, dk, dv, dg
    [T, .], dbeta [T], dh0 [dk, dv], and dS_start [nchunks, dk, dv]: the gradient
    with respect to the state at the start of every chunk (dS_start[0] = dh0)."""
    q, k, v, g, dout = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, dout))
    beta = np.asarray(beta, dtype=np.float64)
    T, dk = k.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv)) if h0 is None else np.array(h0, dtype=np.float64)
    starts, terms = [], []
    for t0 in range(0, T, C):                                   # forward: keep each chunk
        t1 = min(t0 + C, T)
        c = _chunk_terms(q[t0:t1], k[t0:t1], v[t0:t1], g[t0:t1], beta[t0:t1], S)
        starts.append(S)
        terms.append(c)
        S = np.exp(c["gam"][-1])[:, None] * S + c["kend"].T @ c["delta"]
    res = {n: np.zeros_like(x) for n, x in (("dq", q), ("dk", k), ("dv", v), ("dg", g),
                                           ("dbeta", beta))}
    res["dS_start"] = np.zeros((len(terms), dk, dv))
    dS = np.zeros((dk, dv)) if dhT is None else np.array(dhT, dtype=np.float64)
    for ci in reversed(range(len(terms))):
        t0 = ci * C
        t1 = min(t0 + C, T)
        qc, kc, vc, bc, do = q[t0:t1], k[t0:t1], v[t0:t1], beta[t0:t1], dout[t0:t1]
        S0, c = starts[ci], terms[ci]
        gam, kbar, qbar, kend, E = c["gam"], c["kbar"], c["qbar"], c["kend"], c["E"]
        Tm, W, delta = c["Tm"], c["W"], c["delta"]
        last = np.exp(gam[-1])
        # O = Qbar S0 + Aqk Delta;  S_next = Diag(exp(Gamma_last)) S0 + Kend^T Delta
        d_delta = c["Aqk"].T @ do + kend @ dS
        d_qbar = do @ S0.T
        d_aqk = np.tril(do @ delta.T)
        d_kend = delta @ dS.T
        dS0 = qbar.T @ do + last[:, None] * dS - W.T @ d_delta
        # Delta = U - W S0;  U = Tm diag(beta) V;  W = Tm diag(beta) Kbar
        dU, dW = d_delta, -d_delta @ S0.T
        vb, kb = bc[:, None] * vc, bc[:, None] * kbar
        d_vb, d_kb = Tm.T @ dU, Tm.T @ dW
        dTm = dU @ vb.T + dW @ kb.T
        dv_c = bc[:, None] * d_vb
        dbeta_c = np.sum(d_vb * vc, axis=1) + np.sum(d_kb * kbar, axis=1)
        d_kbar = bc[:, None] * d_kb
        # Tm = M^-1 with M = I + diag(beta) A, A strictly lower
        dM = np.tril(-Tm.T @ dTm @ Tm.T, -1)
        dbeta_c += np.sum(dM * c["A"], axis=1)
        dA = bc[:, None] * dM
        # Qbar = exp(Gamma) q, Kbar = exp(Gamma) k, Kend = exp(Gamma_last - Gamma) k,
        # and the state decay exp(Gamma_last)
        dq_c = d_qbar * np.exp(gam)
        dk_c = d_kbar * np.exp(gam) + d_kend * np.exp(gam[-1][None, :] - gam)
        dgam = d_qbar * qbar + d_kbar * kbar - d_kend * kend
        dgam[-1] += np.sum(d_kend * kend, axis=0) + last * np.sum(S0 * dS, axis=1)
        # A[r,i] = sum_c k_rc k_ic E[r,i,c];  Aqk[r,i] = sum_c q_rc k_ic E[r,i,c]
        PA = dA[:, :, None] * E
        dk_c += np.einsum("ric,ic->rc", PA, kc) + np.einsum("ric,rc->ic", PA, kc)
        tA = PA * kc[:, None, :] * kc[None, :, :]
        PQ = d_aqk[:, :, None] * E
        dq_c += np.einsum("ric,ic->rc", PQ, kc)
        dk_c += np.einsum("ric,rc->ic", PQ, qc)
        tQ = PQ * qc[:, None, :] * kc[None, :, :]
        dgam += tA.sum(axis=1) - tA.sum(axis=0) + tQ.sum(axis=1) - tQ.sum(axis=0)
        # Gamma_r = sum_{j <= r} g_j
        res["dg"][t0:t1] = np.cumsum(dgam[::-1], axis=0)[::-1]
        res["dq"][t0:t1], res["dk"][t0:t1], res["dv"][t0:t1] = dq_c, dk_c, dv_c
        res["dbeta"][t0:t1] = dbeta_c
        res["dS_start"][ci] = dS0
        dS = dS0
    res["dh0"] = dS
    return res
