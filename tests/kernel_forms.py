"""Kernel-shaped restatements of quantities the float64 oracle defines: the
blocking and splitting a GPU kernel uses, written out in float64 numpy so that
each can be pinned, in test_oracle.py, against the oracle's plain form
(``oracle.reference.chunked_backward``).  They are not part of the oracle and no
GPU test uses them as its reference.

``pair_grads_blocked``: the gradient terms of A and Aqk (the pairwise-decay sums)
as products of two matrices per 16-token block pair.  For r in block a and i in
block b <= a, exp(Gamma_r - Gamma_i) = exp(Gamma_r - Gamma_ref) exp(Gamma_ref - Gamma_i)
with Gamma_ref the log-decay at block b's first token: the first factor is at
most 1 (Gamma does not increase when g <= 0), the second is bounded by the decay
inside one block, so neither overflows however long the chunk's total decay.
The Gamma terms follow from the row terms: sum_i dA_ri k_rc k_ic E_ric equals
k_rc times the pair term of dk_r, and likewise for the other three.

``aqk_diagonal_apart``: the same pair terms with Aqk's diagonal (i = r, decay factor
exp(0) = 1) taken out of the decay-weighted sums and added to dq and dk alone.  Its
two Gamma terms, q_rc k_rc dAqk_rr on the row side and its negative on the column
side, cancel exactly, so dgam is unchanged; the gradient kernel computes it this way
so that bf16 rounding of the two cancelling terms never reaches dg.

``reverse_state_segments``: chunked_backward's chunk-start state gradients without the
forward states.  Substituting dDelta into dS0 gives dS_n = Y_n dS_{n+1} + c_n
with Y_n = Diag(exp(Gamma_last)) - W^T Kend and c_n = (Qbar - Aqk W)^T dO_n,
neither of which depends on the state.  The reverse recurrence is affine, so
it splits into segments of G chunks: each segment is run from its end once
from zero (its local part) and once as the product of its Y_n (its
transition), and the segments are then chained from the last.
"""
from __future__ import annotations

import numpy as np

from oracle.reference import _chunk_terms

__all__ = ["pair_grads_blocked", "reverse_state_segments", "aqk_diagonal_apart"]


def reverse_state_segments(q, k, v, g, beta, dout, dhT=None, C: int = 64, G: int = 4):
    """One sequence, one head: the gradient with respect to the state at every chunk
    start ([nchunks, dk, dv], as ``chunked_backward``'s dS_start), computed from
    per-chunk affine maps dS_n = Y_n dS_{n+1} + c_n grouped in segments of G chunks."""
    q, k, v, g, dout = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, dout))
    beta = np.asarray(beta, dtype=np.float64)
    T, dk = k.shape
    dv = v.shape[1]
    Y, c = [], []
    zero = np.zeros((dk, dv))
    for t0 in range(0, T, C):                                   # per chunk, independent
        t1 = min(t0 + C, T)
        ct = _chunk_terms(q[t0:t1], k[t0:t1], v[t0:t1], g[t0:t1], beta[t0:t1], zero)
        Y.append(np.diag(np.exp(ct["gam"][-1])) - ct["W"].T @ ct["kend"])
        c.append((ct["qbar"] - ct["Aqk"] @ ct["W"]).T @ dout[t0:t1])
    n = len(Y)
    segs = [(a, min(a + G, n)) for a in range(0, n, G)]
    # per segment, from its end: local part (from zero) and transition (product of Y)
    loc, trans = [], []
    for a, b in segs:
        Lp, Xp = np.zeros((dk, dv)), np.eye(dk)
        for i in reversed(range(a, b)):
            Lp = Y[i] @ Lp + c[i]
            Xp = Y[i] @ Xp
        loc.append(Lp)
        trans.append(Xp)
    # chain the segments from the last: gradient entering each segment's end
    end = np.zeros((dk, dv)) if dhT is None else np.array(dhT, dtype=np.float64)
    seg_end = [None] * len(segs)
    for p in reversed(range(len(segs))):
        seg_end[p] = end
        end = trans[p] @ end + loc[p]
    # rerun each segment from its end gradient for the chunk starts inside it
    out = np.zeros((n, dk, dv))
    for p, (a, b) in enumerate(segs):
        d = seg_end[p]
        for i in reversed(range(a, b)):
            d = Y[i] @ d + c[i]
            out[i] = d
    return out


def pair_grads_blocked(dA, dAqk, q, k, gam, block: int = 16):
    """One chunk: the contributions of dA (strictly lower) and dAqk (lower) to dq, dk
    and dGamma, through A[r,i] = sum_c k_rc k_ic E[r,i,c] and Aqk[r,i] = sum_c q_rc
    k_ic E[r,i,c], E[r,i,c] = exp(Gamma_rc - Gamma_ic) (i <= r), computed by block
    pairs with the exponent split at each column block's first token."""
    dA, dAqk, q, k, gam = (np.asarray(x, dtype=np.float64) for x in (dA, dAqk, q, k, gam))
    L = k.shape[0]
    dq, dk, dgam = np.zeros_like(q), np.zeros_like(k), np.zeros_like(k)
    for b0 in range(0, L, block):                       # column block b: tokens i
        b1 = min(b0 + block, L)
        ref = gam[b0]
        kin = k[b0:b1] * np.exp(ref[None, :] - gam[b0:b1])          # >= |k|, bounded
        for a0 in range(b0, L, block):                  # row blocks a >= b: tokens r
            a1 = min(a0 + block, L)
            down = np.exp(gam[a0:a1] - ref[None, :])                  # <= 1
            PA = np.tril(dA[a0:a1, b0:b1], b0 - a0 - 1) if a0 == b0 else dA[a0:a1, b0:b1]
            PQ = np.tril(dAqk[a0:a1, b0:b1], b0 - a0) if a0 == b0 else dAqk[a0:a1, b0:b1]
            kr, qr = k[a0:a1] * down, q[a0:a1] * down
            row_k = down * (PA @ kin)                   # sum_i dA_ri k_i E_ri   (rows r)
            row_q = down * (PQ @ kin)                   # sum_i dAqk_ri k_i E_ri
            col_k = np.exp(ref[None, :] - gam[b0:b1]) * (PA.T @ kr + PQ.T @ qr)   # rows i
            dk[a0:a1] += row_k
            dq[a0:a1] += row_q
            dk[b0:b1] += col_k
            dgam[a0:a1] += k[a0:a1] * row_k + q[a0:a1] * row_q
            dgam[b0:b1] -= k[b0:b1] * col_k
    return dq, dk, dgam


def aqk_diagonal_apart(dA, dAqk, q, k, gam):
    """(dq, dk, dgam) of the pairwise-decay sums, Aqk's diagonal apart (module docstring):
    dA strictly lower, dAqk lower with its diagonal [L, L]; q, k, gam [L, dk]."""
    d = np.diag(dAqk).copy()
    off = np.tril(dAqk, -1)
    L = len(gam)
    lower = np.tril(np.ones((L, L), dtype=bool))[:, :, None]           # pairs i <= r
    E = np.exp(np.where(lower, gam[:, None, :] - gam[None, :, :], -np.inf))
    PA, PQ = dA[:, :, None] * E, off[:, :, None] * E
    dq = np.einsum("ric,ic->rc", PQ, k) + d[:, None] * k
    dk = (np.einsum("ric,ic->rc", PA, k) + np.einsum("ric,rc->ic", PA, k)
          + np.einsum("ric,rc->ic", PQ, q) + d[:, None] * q)
    tA, tQ = PA * k[:, None, :] * k[None, :, :], PQ * q[:, None, :] * k[None, :, :]
    dgam = tA.sum(1) - tA.sum(0) + tQ.sum(1) - tQ.sum(0)
    return dq, dk, dgam
