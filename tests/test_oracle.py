"""Pins for the float64 oracle, checked against what the pages and the mathematics fix.

Each test states the passage or the mathematical fact it pins.  None of them
re-types the oracle's formula to compare the oracle with itself: they use closed
forms, invariants, a hand-worked example (tests/golden/hand_tiny.txt), autograd,
brute force and mutation checks.
"""
from fractions import Fraction
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import reference as ref

import kernel_forms as kf

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_inputs(rng, T, H, dk, dv, B=1, beta=None, g_scale=0.3):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q /= np.linalg.norm(q, axis=-1, keepdims=True) * np.sqrt(dk)
    v = rng.standard_normal((B, T, H, dv))
    g = -g_scale * rng.random((B, T, H, dk)) * 2
    b = rng.random((B, T, H)) if beta is None else np.full((B, T, H), float(beta))
    return q, k, v, g, b


def _load_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *rest = line.split()
            vals[key] = [Fraction(x) for x in rest]
    return vals


def _hand_inputs():
    G = _load_golden("hand_tiny.txt")
    f = lambda key: np.array([float(x) for x in G[key]])
    q = np.stack([f("q1"), f("q2")])[None, :, None, :]
    k = np.stack([f("k1"), f("k2")])[None, :, None, :]
    v = np.stack([f("v1"), f("v2")])[None, :, None, :]
    g = np.log(np.stack([f("alpha1"), f("alpha2")]))[None, :, None, :]
    b = np.array([f("beta1")[0], f("beta2")[0]])[None, :, None]
    h0 = f("S0").reshape(1, 1, 2, 2)
    return G, q, k, v, g, b, h0


# ----------------------------------------------------------------------------
# Hand-worked example: pins orientation of S, the decay axis and the order of
# decay, write and read (miniKimiK3 card, "Kimi Delta Attention" bullet).
# ----------------------------------------------------------------------------
def test_hand_worked_example(oracle_lib):
    G, q, k, v, g, b, h0 = _hand_inputs()
    out, hT = oracle.prefill(q, k, v, g, b, h0)
    o1 = np.array([float(x) for x in G["o1"]])
    o2 = np.array([float(x) for x in G["o2"]])
    S2 = np.array([float(x) for x in G["S2"]]).reshape(2, 2)
    np.testing.assert_allclose(out[0, 0, 0], o1, rtol=0, atol=1e-14)
    np.testing.assert_allclose(out[0, 1, 0], o2, rtol=0, atol=1e-14)
    np.testing.assert_allclose(hT[0, 0], S2, rtol=0, atol=1e-14)
    # the numpy literal form agrees as well
    o_l, S_l = ref.recurrence_literal(q[0, :, 0], k[0, :, 0], v[0, :, 0], g[0, :, 0],
                                      b[0, :, 0], h0[0, 0])
    np.testing.assert_allclose(o_l, np.stack([o1, o2]), atol=1e-14)
    np.testing.assert_allclose(S_l, S2, atol=1e-14)


def test_hand_worked_example_fractions_consistent():
    """Re-derive the golden values with exact Fraction arithmetic, step by step
    as in the fixture's comments (decay rows, read k^T A, write, read q)."""
    G = _load_golden("hand_tiny.txt")
    S = [[G["S0"][0], G["S0"][1]], [G["S0"][2], G["S0"][3]]]
    outs = []
    for t in (1, 2):
        a, k, v, b, q = (G[f"{n}{t}"] for n in ("alpha", "k", "v", "beta", "q"))
        A = [[a[c] * S[c][j] for j in range(2)] for c in range(2)]
        kA = [k[0] * A[0][j] + k[1] * A[1][j] for j in range(2)]
        S = [[A[c][j] + b[0] * k[c] * (v[j] - kA[j]) for j in range(2)] for c in range(2)]
        outs.append([q[0] * S[0][j] + q[1] * S[1][j] for j in range(2)])
    assert outs[0] == G["o1"] and outs[1] == G["o2"]
    assert [S[0][0], S[0][1], S[1][0], S[1][1]] == G["S2"]


# Mutation check: plausible mistakes in the recurrence must fail the hand pin.
def _mutant(q, k, v, g, b, h0, mutation):
    S = np.array(h0, dtype=np.float64)
    outs = []
    for t in range(len(k)):
        a = np.exp(g[t])
        kt, vt = k[t], v[t]
        if mutation == "decay_after_write":
            S = S + b[t] * np.outer(kt, vt - kt @ S)
            S = a[:, None] * S
        elif mutation == "decay_on_value_axis":
            A = S * a[None, :]
            S = A + b[t] * np.outer(kt, vt - kt @ A)
        elif mutation == "read_before_write":
            A = a[:, None] * S
            outs.append(A.T @ q[t])
            S = A + b[t] * np.outer(kt, vt - kt @ A)
            continue
        elif mutation == "sign_flip":
            A = a[:, None] * S
            S = A + b[t] * np.outer(kt, vt + kt @ A)
        elif mutation == "transposed_read":
            # same write, but the output reads S q instead of S^T q (dk == dv here)
            A = a[:, None] * S
            S = A + b[t] * np.outer(kt, vt - kt @ A)
            outs.append(S @ q[t])
            continue
        elif mutation == "no_beta_on_v":
            A = a[:, None] * S
            S = A - b[t] * np.outer(kt, kt @ A) + np.outer(kt, vt)
        outs.append(S.T @ q[t])
    return np.array(outs), S


@pytest.mark.parametrize("mutation", ["decay_after_write", "decay_on_value_axis",
                                      "read_before_write", "sign_flip",
                                      "transposed_read", "no_beta_on_v"])
def test_hand_example_catches_mutations(mutation):
    G, q, k, v, g, b, h0 = _hand_inputs()
    o, S = _mutant(q[0, :, 0], k[0, :, 0], v[0, :, 0], g[0, :, 0], b[0, :, 0], h0[0, 0],
                   mutation)
    o_ref = np.array([[float(x) for x in G["o1"]], [float(x) for x in G["o2"]]])
    S_ref = np.array([float(x) for x in G["S2"]]).reshape(2, 2)
    assert not (np.allclose(o, o_ref, atol=1e-9) and np.allclose(S, S_ref, atol=1e-9))


# ----------------------------------------------------------------------------
# beta = 0: the write vanishes and the state only decays per channel
# (the KDA update with beta = 0; "Inside Kimi" outline, KDA gating lesson:
# channel-wise decay).  Closed form S_T = Diag(exp(sum_t g_t)) h0.
# ----------------------------------------------------------------------------
def test_beta_zero_pure_channel_decay(oracle_lib):
    rng = np.random.default_rng(1)
    B, T, H, dk, dv = 2, 37, 3, 8, 5
    q, k, v, g, b = _rand_inputs(rng, T, H, dk, dv, B=B, beta=0.0)
    h0 = rng.standard_normal((B, H, dk, dv))
    out, hT = oracle.prefill(q, k, v, g, b, h0)
    gam = np.cumsum(g, axis=1)                                       # [B,T,H,dk]
    for bi in range(B):
        for h in range(H):
            np.testing.assert_allclose(hT[bi, h], np.exp(gam[bi, -1, h])[:, None] * h0[bi, h],
                                       rtol=1e-13, atol=1e-15)
            for t in range(T):
                St = np.exp(gam[bi, t, h])[:, None] * h0[bi, h]
                np.testing.assert_allclose(out[bi, t, h], St.T @ q[bi, t, h],
                                           rtol=1e-12, atol=1e-15)


def test_beta_zero_no_decay_state_constant(oracle_lib):
    """g = 0 and beta = 0: S stays h0 and o_t = h0^T q_t."""
    rng = np.random.default_rng(2)
    q, k, v, g, b = _rand_inputs(rng, 20, 2, 6, 7, beta=0.0)
    g[:] = 0.0
    h0 = rng.standard_normal((1, 2, 6, 7))
    out, hT = oracle.prefill(q, k, v, g, b, h0)
    np.testing.assert_array_equal(hT, h0)
    for h in range(2):
        np.testing.assert_allclose(out[0, :, h], q[0, :, h] @ h0[0, h], rtol=1e-14, atol=1e-15)


# ----------------------------------------------------------------------------
# beta = 1 and |k| = 1: the write is error-correcting, S_t^T k_t = v_t exactly
# (miniKimiK3 card, KDA bullet: "error-correcting write").  Reading with q = k
# exposes S_t^T k_t as the output.
# ----------------------------------------------------------------------------
def test_error_correcting_write(oracle_lib):
    rng = np.random.default_rng(3)
    q, k, v, g, b = _rand_inputs(rng, 50, 2, 16, 12, B=2, beta=1.0)
    h0 = rng.standard_normal((2, 2, 16, 12))
    out, _ = oracle.prefill(k, k, v, g, b, h0)
    np.testing.assert_allclose(out, v, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------
# alpha = 1, beta = 1, orthonormal keys, S0 = 0: exact recall of every stored
# pair ("Inside Kimi" outline: adversarial recall / sequence recall).
# ----------------------------------------------------------------------------
def test_exact_recall_orthonormal_keys(oracle_lib):
    rng = np.random.default_rng(4)
    dk, dv, T = 16, 10, 12
    Q, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Q.T[:T]                                 # T orthonormal rows
    v = rng.standard_normal((T, dv))
    # query at step t reads back the value stored at step j(t) <= t
    j_of_t = np.array([rng.integers(0, t + 1) for t in range(T)])
    q = keys[j_of_t]
    g = np.zeros((T, dk))
    b = np.ones(T)
    out, hT = oracle.prefill(q[None, :, None], keys[None, :, None], v[None, :, None],
                             g[None, :, None], b[None, :, None])
    np.testing.assert_allclose(out[0, :, 0], v[j_of_t], atol=1e-13)
    np.testing.assert_allclose(hT[0, 0], keys.T @ v, atol=1e-13)


# ----------------------------------------------------------------------------
# One gradient-descent step: S_t = A - beta * grad_S (1/2 ||S^T k - v||^2) at
# S = A = Diag(alpha) S_{t-1} (miniKimiK3 card, KDA bullet).  The gradient comes
# from torch autograd, not from a hand-written formula.  With g = 0 this is the
# textbook delta rule (DeltaNet, "Inside Kimi" outline).
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("zero_decay", [True, False])
def test_one_gradient_step(oracle_lib, zero_decay):
    rng = np.random.default_rng(5)
    dk, dv = 9, 7
    for trial in range(5):
        S0 = rng.standard_normal((dk, dv))
        k = rng.standard_normal(dk)
        v = rng.standard_normal(dv)
        q = rng.standard_normal(dk)
        g = np.zeros(dk) if zero_decay else -rng.random(dk)
        beta = rng.random()
        A = torch.tensor(np.exp(g)[:, None] * S0, dtype=torch.float64, requires_grad=True)
        loss = 0.5 * ((A.T @ torch.tensor(k) - torch.tensor(v)) ** 2).sum()
        loss.backward()
        expect = (A - beta * A.grad).detach().numpy()
        out, hT = oracle.prefill(q[None, None, None], k[None, None, None], v[None, None, None],
                                 g[None, None, None], np.array([[[beta]]]),
                                 S0[None, None])
        np.testing.assert_allclose(hT[0, 0], expect, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(out[0, 0, 0], expect.T @ q, rtol=1e-13, atol=1e-14)


# ----------------------------------------------------------------------------
# The C++ oracle and the numpy literal form (dk x dk factor materialised) agree.
# ----------------------------------------------------------------------------
def test_cpp_matches_literal_form(oracle_lib):
    rng = np.random.default_rng(6)
    B, T, H, dk, dv = 2, 23, 3, 8, 6
    q, k, v, g, b = _rand_inputs(rng, T, H, dk, dv, B=B)
    h0 = rng.standard_normal((B, H, dk, dv))
    out, hT = oracle.prefill(q, k, v, g, b, h0)
    for bi in range(B):
        for h in range(H):
            o_l, S_l = ref.recurrence_literal(q[bi, :, h], k[bi, :, h], v[bi, :, h],
                                              g[bi, :, h], b[bi, :, h], h0[bi, h])
            np.testing.assert_allclose(out[bi, :, h], o_l, rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(hT[bi, h], S_l, rtol=1e-12, atol=1e-14)


# ----------------------------------------------------------------------------
# Chunked form == recurrence ("Inside Kimi" outline: sequential and chunkwise
# delta-style implementations agree on deterministic fixtures).  C = 1 is the
# recurrence itself; T not divisible by C exercises the ragged last chunk.
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("C", [1, 2, 4, 5, 64])
@pytest.mark.parametrize("T", [1, 7, 63, 64, 65, 130])
def test_chunked_form_equals_recurrence(oracle_lib, C, T):
    rng = np.random.default_rng(100 + 7 * C + T)
    dk, dv = 8, 6
    q, k, v, g, b = _rand_inputs(rng, T, 1, dk, dv, g_scale=1.5)
    h0 = rng.standard_normal((1, 1, dk, dv))
    out, hT = oracle.prefill(q, k, v, g, b, h0)
    o_c, S_c = ref.chunked(q[0, :, 0], k[0, :, 0], v[0, :, 0], g[0, :, 0], b[0, :, 0],
                           h0[0, 0], C=C)
    scale = max(np.abs(out).max(), 1e-30)
    assert np.abs(o_c - out[0, :, 0]).max() / scale < 1e-12
    assert np.abs(S_c - hT[0, 0]).max() / max(np.abs(hT).max(), 1e-30) < 1e-12


def test_chunked_form_strong_decay(oracle_lib):
    """Chunk-wide decay far beyond float32 range (Gamma down to about -300): the
    chunked algebra is still exact in float64 with pairwise exponents."""
    rng = np.random.default_rng(7)
    T, dk, dv = 150, 8, 8
    q, k, v, g, b = _rand_inputs(rng, T, 1, dk, dv, g_scale=2.5)
    out, hT = oracle.prefill(q, k, v, g, b)
    o_c, S_c = ref.chunked(q[0, :, 0], k[0, :, 0], v[0, :, 0], g[0, :, 0], b[0, :, 0], C=64)
    assert np.abs(o_c - out[0, :, 0]).max() <= 1e-12 * np.abs(out).max()


# ----------------------------------------------------------------------------
# The chunked form's backward (reference.chunked_backward: the adjoint of each
# chunk's WY step, chunks in reverse) gives the gradients of the recurrence: the
# C++ oracle's reverse-mode sweep, itself pinned by finite differences and
# autograd below.  Ragged last chunks, C = 1 (one token per chunk) and strong decay.
# ----------------------------------------------------------------------------
def _bwd_pair(rng, T, dk, dv, C, g_scale=1.5):
    q, k, v, g, b = _rand_inputs(rng, T, 1, dk, dv, g_scale=g_scale)
    h0 = rng.standard_normal((1, 1, dk, dv))
    dout = rng.standard_normal((1, T, 1, dv))
    dhT = rng.standard_normal((1, 1, dk, dv))
    rec = oracle.backward(q, k, v, g, b, dout, h0, dhT)
    chk = ref.chunked_backward(q[0, :, 0], k[0, :, 0], v[0, :, 0], g[0, :, 0], b[0, :, 0],
                               dout[0, :, 0], h0[0, 0], dhT[0, 0], C=C)
    return (q, k, v, g, b, h0, dout, dhT), rec, chk


def _assert_grads_equal(rec, chk, tol):
    for key in ("dq", "dk", "dv", "dg", "dbeta"):
        a = rec[key][0, :, 0]
        assert np.abs(chk[key] - a).max() <= tol * max(np.abs(a).max(), 1e-30), key
    a = rec["dh0"][0, 0]
    assert np.abs(chk["dh0"] - a).max() <= tol * max(np.abs(a).max(), 1e-30), "dh0"


@pytest.mark.parametrize("C", [1, 2, 4, 5, 64])
@pytest.mark.parametrize("T", [1, 7, 63, 64, 65, 130])
def test_chunked_backward_equals_recurrent_backward(oracle_lib, C, T):
    rng = np.random.default_rng(500 + 7 * C + T)
    _, rec, chk = _bwd_pair(rng, T, 8, 6, C)
    _assert_grads_equal(rec, chk, 1e-11)


def test_chunked_backward_strong_decay(oracle_lib):
    """Chunk-wide decay down to about exp(-300): the pairwise exponents keep every
    gradient term finite and exact in float64."""
    _, rec, chk = _bwd_pair(np.random.default_rng(8), 150, 8, 8, 64, g_scale=2.5)
    assert all(np.isfinite(chk[key]).all() for key in ("dq", "dk", "dv", "dg", "dbeta", "dh0"))
    _assert_grads_equal(rec, chk, 1e-11)


def test_chunked_backward_state_gradient_at_chunk_starts(oracle_lib):
    """dS_start[c] is the gradient of the loss with respect to the state entering
    chunk c: the recurrent backward of the suffix from chunk c, started from the
    forward state there, returns it as its dh0."""
    rng = np.random.default_rng(9)
    T, dk, dv, C = 150, 6, 5, 32
    (q, k, v, g, b, h0, dout, dhT), _, chk = _bwd_pair(rng, T, dk, dv, C)
    for c in range(chk["dS_start"].shape[0]):
        t0 = c * C
        S_c = h0
        if t0 > 0:
            _, S_c = oracle.prefill(q[:, :t0], k[:, :t0], v[:, :t0], g[:, :t0], b[:, :t0], h0)
        suf = oracle.backward(q[:, t0:], k[:, t0:], v[:, t0:], g[:, t0:], b[:, t0:],
                              dout[:, t0:], S_c, dhT)
        ref_ds = suf["dh0"][0, 0]
        assert np.abs(chk["dS_start"][c] - ref_ds).max() <= 1e-11 * np.abs(ref_ds).max(), c
    assert np.array_equal(chk["dS_start"][0], chk["dh0"])


def _pair_terms_einsum(dA, dAqk, q, k, gam):
    """The pairwise terms exactly as chunked_backward forms them (full E tensor)."""
    L = k.shape[0]
    lower = np.tril(np.ones((L, L), dtype=bool))[:, :, None]
    E = np.exp(np.where(lower, gam[:, None, :] - gam[None, :, :], -np.inf))
    PA, PQ = np.tril(dA, -1)[:, :, None] * E, np.tril(dAqk)[:, :, None] * E
    dk = np.einsum("ric,ic->rc", PA, k) + np.einsum("ric,rc->ic", PA, k) + \
        np.einsum("ric,rc->ic", PQ, q)
    dq = np.einsum("ric,ic->rc", PQ, k)
    tA, tQ = PA * k[:, None, :] * k[None, :, :], PQ * q[:, None, :] * k[None, :, :]
    dgam = tA.sum(1) - tA.sum(0) + tQ.sum(1) - tQ.sum(0)
    return dq, dk, dgam


@pytest.mark.parametrize("L,g_scale", [(64, 0.3), (64, 2.5), (45, 1.0), (16, 0.5), (7, 0.5)])
def test_pair_grads_blocked_equal_pairwise_terms(L, g_scale):
    """Splitting the exponents at 16-token reference points changes nothing but
    rounding; with strong decay (Gamma down to about -160 in one chunk) every
    factor stays finite."""
    rng = np.random.default_rng(L + int(10 * g_scale))
    q, k, _, g, _ = _rand_inputs(rng, L, 1, 8, 4, g_scale=g_scale)
    q, k, gam = q[0, :, 0], k[0, :, 0], np.cumsum(g[0, :, 0], axis=0)
    dA, dAqk = rng.standard_normal((L, L)), rng.standard_normal((L, L))
    want = _pair_terms_einsum(dA, dAqk, q, k, gam)
    got = kf.pair_grads_blocked(dA, dAqk, q, k, gam)
    for w, x, name in zip(want, got, ("dq", "dk", "dgam")):
        assert np.isfinite(x).all(), name
        assert np.abs(x - w).max() <= 1e-12 * max(np.abs(w).max(), 1e-30), name


@pytest.mark.parametrize("L,g_scale", [(64, 0.3), (64, 6.0), (23, 1.0)])
def test_aqk_diagonal_apart_equals_pairwise_terms(L, g_scale):
    """Aqk's diagonal (decay factor 1) contributes nothing to dGamma: its row-side and
    column-side terms cancel exactly, so taking it out of the decay-weighted sums and
    adding its dq, dk terms alone gives the plain pairwise terms, strong decay included."""
    rng = np.random.default_rng(L + int(10 * g_scale))
    q, k, _, g, _ = _rand_inputs(rng, L, 1, 8, 4, g_scale=g_scale)
    q, k, gam = q[0, :, 0], k[0, :, 0], np.cumsum(g[0, :, 0], axis=0)
    dA = np.tril(rng.standard_normal((L, L)), -1)
    dAqk = np.tril(rng.standard_normal((L, L)))
    want = _pair_terms_einsum(dA, dAqk, q, k, gam)
    got = kf.aqk_diagonal_apart(dA, dAqk, q, k, gam)
    for w, x, name in zip(want, got, ("dq", "dk", "dgam")):
        assert np.abs(x - w).max() <= 1e-12 * max(np.abs(w).max(), 1e-30), name
    # and the diagonal's own Gamma terms are the cancelling pair: with everything else
    # zero, the plain terms give dgam = 0 exactly up to rounding
    only = np.diag(np.diag(dAqk))
    _, _, dg0 = _pair_terms_einsum(np.zeros_like(dA), only, q, k, gam)
    assert np.abs(dg0).max() <= 1e-12 * np.abs(q * k).max() * np.abs(np.diag(dAqk)).max()


@pytest.mark.parametrize("T,C,G", [(150, 32, 2), (130, 64, 1), (400, 16, 7), (64, 64, 3)])
def test_reverse_state_segments_equal_chunk_start_gradients(oracle_lib, T, C, G):
    """The reverse state recurrence needs no forward state and splits into segments:
    its chunk-start gradients equal chunked_backward's, whose dS_start the suffix
    pin above ties to the recurrent backward."""
    rng = np.random.default_rng(T + C + G)
    (q, k, v, g, b, h0, dout, dhT), _, chk = _bwd_pair(rng, T, 6, 5, C)
    seg = kf.reverse_state_segments(q[0, :, 0], k[0, :, 0], v[0, :, 0], g[0, :, 0], b[0, :, 0],
                                     dout[0, :, 0], dhT[0, 0], C=C, G=G)
    assert seg.shape == chk["dS_start"].shape
    assert np.abs(seg - chk["dS_start"]).max() <= 1e-11 * np.abs(chk["dS_start"]).max()


# ----------------------------------------------------------------------------
# Packed documents are isolated (Mini-K3-1H-mamba2 card, packed-document
# paragraph: state flow resets at every boundary; a later document gets exactly
# nothing from earlier ones).  Forward analogue of the zero-gradient gate, over
# several boundaries and seeds.
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_document_isolation(oracle_lib, seed):
    rng = np.random.default_rng(seed)
    lens = [int(x) for x in rng.integers(1, 90, size=5)]
    T, H, dk, dv = sum(lens), 2, 8, 6
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q, k, v, g, b = _rand_inputs(rng, T, H, dk, dv)
    h0 = rng.standard_normal((len(lens), H, dk, dv))
    out, hT = oracle.prefill(q, k, v, g, b, h0, cu_seqlens=cu)
    for d, (s, e) in enumerate(zip(cu[:-1], cu[1:])):
        o_d, S_d = oracle.prefill(q[:, s:e], k[:, s:e], v[:, s:e], g[:, s:e], b[:, s:e],
                                  h0[d:d + 1])
        np.testing.assert_array_equal(out[:, s:e], o_d)     # bitwise
        np.testing.assert_array_equal(hT[d:d + 1], S_d)
    # perturb every input of document 1: documents 0, 2, 3, 4 are unchanged exactly
    s, e = cu[1], cu[2]
    q2, k2, v2, g2, b2 = (x.copy() for x in (q, k, v, g, b))
    for x in (q2, k2, v2):
        x[:, s:e] += rng.standard_normal(x[:, s:e].shape)
    g2[:, s:e] *= 0.5
    b2[:, s:e] = rng.random(b2[:, s:e].shape)
    h02 = h0.copy()
    h02[1] += 1.0
    out2, hT2 = oracle.prefill(q2, k2, v2, g2, b2, h02, cu_seqlens=cu)
    keep = np.ones(T, dtype=bool)
    keep[s:e] = False
    np.testing.assert_array_equal(out2[:, keep], out[:, keep])
    np.testing.assert_array_equal(np.delete(hT2, 1, axis=0), np.delete(hT, 1, axis=0))
    assert not np.array_equal(out2[:, s:e], out[:, s:e])


def test_empty_documents_pass_state_through(oracle_lib):
    """A zero-length document leaves its final state equal to its initial state."""
    rng = np.random.default_rng(9)
    lens = [5, 0, 7]
    cu = np.array([0, 5, 5, 12], dtype=np.int32)
    q, k, v, g, b = _rand_inputs(rng, 12, 1, 4, 4)
    h0 = rng.standard_normal((3, 1, 4, 4))
    _, hT = oracle.prefill(q, k, v, g, b, h0, cu_seqlens=cu)
    np.testing.assert_array_equal(hT[1], h0[1])


# ----------------------------------------------------------------------------
# The state is the only carry: prefill [0,T) == prefill [0,t) then [t,T) with
# hT -> h0; and decode steps == prefill of the same tokens (same recurrence in
# both modes, miniKimiK3 card: chunked form for training, recurrence for decode).
# ----------------------------------------------------------------------------
def test_split_sequence(oracle_lib):
    rng = np.random.default_rng(10)
    T, H, dk, dv = 90, 2, 8, 6
    q, k, v, g, b = _rand_inputs(rng, T, H, dk, dv)
    h0 = rng.standard_normal((1, H, dk, dv))
    out, hT = oracle.prefill(q, k, v, g, b, h0)
    t = 41
    o1, s1 = oracle.prefill(q[:, :t], k[:, :t], v[:, :t], g[:, :t], b[:, :t], h0)
    o2, s2 = oracle.prefill(q[:, t:], k[:, t:], v[:, t:], g[:, t:], b[:, t:], s1)
    np.testing.assert_array_equal(np.concatenate([o1, o2], axis=1), out)
    np.testing.assert_array_equal(s2, hT)


def test_decode_equals_prefill(oracle_lib):
    rng = np.random.default_rng(11)
    N, H, dk, dv, steps = 3, 2, 8, 6, 16
    q, k, v, g, b = _rand_inputs(rng, steps, H, dk, dv, B=N)
    S0 = rng.standard_normal((N, H, dk, dv))
    out, hT = oracle.prefill(q, k, v, g, b, S0)
    S = S0
    for t in range(steps):
        o, S = oracle.decode(q[:, t], k[:, t], v[:, t], g[:, t], b[:, t], S)
        np.testing.assert_array_equal(o, out[:, t])
    np.testing.assert_array_equal(S, hT)


# ----------------------------------------------------------------------------
# Stability: with beta in [0,1], |k| = 1, alpha <= 1 the map
# (I - beta k k^T) Diag(alpha) has spectral norm <= 1, hence
# ||S_t||_F <= ||S_{t-1}||_F + beta ||v_t|| ("Inside Kimi" outline: state
# corruption and unstable updates as failure modes).
# ----------------------------------------------------------------------------
def test_state_norm_bound(oracle_lib):
    rng = np.random.default_rng(12)
    T, dk, dv = 300, 16, 16
    q, k, v, g, b = _rand_inputs(rng, T, 1, dk, dv, g_scale=0.05)
    S = rng.standard_normal((1, 1, dk, dv)) * 3
    for t in range(T):
        prev = np.linalg.norm(S)
        _, S = oracle.decode(q[:, t], k[:, t], v[:, t], g[:, t], b[:, t], S)
        assert np.linalg.norm(S) <= prev + b[0, t, 0] * np.linalg.norm(v[0, t, 0]) + 1e-12


def test_oracle_rejects_bad_cu_seqlens(oracle_lib):
    rng = np.random.default_rng(13)
    q, k, v, g, b = _rand_inputs(rng, 10, 1, 4, 4)
    with pytest.raises(ValueError):
        oracle.prefill(q, k, v, g, b, cu_seqlens=np.array([0, 6, 4, 10], dtype=np.int32))
    with pytest.raises(ValueError):
        oracle.prefill(q, k, v, g, b, cu_seqlens=np.array([0, 6, 9], dtype=np.int32))


# ---- grouped decay (decay-granularity variant, "decay-g64" family card) -------
@pytest.mark.parametrize("G", [2, 4, 8])
def test_grouped_decay_beta_zero_closed_form(oracle_lib, G):
    """With beta = 0 only the decay acts: row c of the state decays by
    exp(sum_t g[t, c // G]) -- consecutive channels share one decay value."""
    rng = np.random.default_rng(40 + G)
    T, H, dk, dv = 9, 2, 8, 3
    q, k, v, _, b = _rand_inputs(rng, T, H, dk, dv, beta=0.0)
    gg = -0.5 * rng.random((1, T, H, dk // G))
    h0 = rng.standard_normal((1, H, dk, dv))
    out, hT = oracle.prefill(q, k, v, gg, b, h0)
    for h in range(H):
        for c in range(dk):
            grp = c // G
            np.testing.assert_allclose(hT[0, h, c], np.exp(gg[0, :, h, grp].sum()) * h0[0, h, c],
                                       rtol=1e-12)
        for t in range(T):
            decay = np.array([np.exp(gg[0, :t + 1, h, c // G].sum()) for c in range(dk)])
            np.testing.assert_allclose(out[0, t, h], (decay[:, None] * h0[0, h]).T @ q[0, t, h],
                                       rtol=1e-10, atol=1e-14)


def test_grouped_decay_single_group_is_scalar_gated_delta_rule(oracle_lib):
    """G = dk: one decay per head and token, i.e. the scalar-gated delta rule
    S_t = a_t (I - beta k k^T) S_{t-1} + beta k v^T (the scalar commutes with the
    rank-1 factor), written out here with a matrix product per step."""
    rng = np.random.default_rng(44)
    T, H, dk, dv = 7, 1, 4, 3
    q, k, v, _, b = _rand_inputs(rng, T, H, dk, dv)
    gg = -0.4 * rng.random((1, T, H, 1))
    h0 = rng.standard_normal((1, H, dk, dv))
    out, hT = oracle.prefill(q, k, v, gg, b, h0)
    S = h0[0, 0].copy()
    for t in range(T):
        kt, vt, bt = k[0, t, 0], v[0, t, 0], b[0, t, 0]
        S = np.exp(gg[0, t, 0, 0]) * (np.eye(dk) - bt * np.outer(kt, kt)) @ S + bt * np.outer(kt, vt)
        np.testing.assert_allclose(out[0, t, 0], S.T @ q[0, t, 0], rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(hT[0, 0], S, rtol=1e-11, atol=1e-14)


# ---- backward (the chunked form "trains through"; gradient checks by finite differences) ----
def _loss_fd(args, dout, dhT, cu=None):
    o, s = oracle.prefill(args["q"], args["k"], args["v"], args["g"], args["b"], args["h0"], cu)
    return (o * dout).sum() + (s * dhT).sum()


@pytest.mark.parametrize("packed", [False, True])
def test_backward_matches_finite_differences(oracle_lib, packed):
    """Central differences of L = <out, dout> + <hT, dhT> on the float64 forward
    (the course outline's finite-difference gradient checks)."""
    rng = np.random.default_rng(60 + packed)
    T, H, dk, dv = 7, 2, 4, 3
    q, k, v, g, b = _rand_inputs(rng, T, H, dk, dv)
    cu = np.array([0, 3, 7], dtype=np.int32) if packed else None
    nseq = 2 if packed else 1
    h0 = rng.standard_normal((nseq, H, dk, dv))
    dout = rng.standard_normal((1, T, H, dv))
    dhT = rng.standard_normal((nseq, H, dk, dv))
    r = oracle.backward(q, k, v, g, b, dout, h0, dhT, cu)
    args = dict(q=q, k=k, v=v, g=g, b=b, h0=h0)
    eps = 1e-6
    for name, key in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("g", "dg"), ("b", "dbeta"),
                      ("h0", "dh0")):
        x = args[name]
        num = np.zeros_like(x)
        for i in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[i] += eps
            xm[i] -= eps
            num[i] = (_loss_fd({**args, name: xp}, dout, dhT, cu) -
                      _loss_fd({**args, name: xm}, dout, dhT, cu)) / (2 * eps)
        np.testing.assert_allclose(r[key], num, rtol=1e-6, atol=1e-7, err_msg=name)


def test_backward_matches_autograd_of_literal_recurrence(oracle_lib):
    """torch autograd through a float64 restatement with the dk x dk factor
    (I - beta k k^T) Diag(exp g) materialised (recurrence_literal's form)."""
    rng = np.random.default_rng(70)
    T, H, dk, dv = 6, 1, 5, 4
    q, k, v, g, b = _rand_inputs(rng, T, H, dk, dv)
    h0 = rng.standard_normal((1, H, dk, dv))
    dout = rng.standard_normal((1, T, H, dv))
    dhT = rng.standard_normal((1, H, dk, dv))
    r = oracle.backward(q, k, v, g, b, dout, h0, dhT)
    tq, tk, tv, tg, tb, th = (torch.tensor(x, dtype=torch.float64, requires_grad=True)
                              for x in (q, k, v, g, b, h0))
    S = th[0, 0]
    loss = 0.0
    for t in range(T):
        kt, vt = tk[0, t, 0], tv[0, t, 0]
        M = (torch.eye(dk, dtype=torch.float64) - tb[0, t, 0] * torch.outer(kt, kt)) @ \
            torch.diag(torch.exp(tg[0, t, 0]))
        S = M @ S + tb[0, t, 0] * torch.outer(kt, vt)
        loss = loss + (S.T @ tq[0, t, 0] * torch.tensor(dout[0, t, 0])).sum()
    loss = loss + (S * torch.tensor(dhT[0, 0])).sum()
    loss.backward()
    for key, t in (("dq", tq), ("dk", tk), ("dv", tv), ("dg", tg), ("dbeta", tb), ("dh0", th)):
        np.testing.assert_allclose(r[key], t.grad.numpy(), rtol=1e-11, atol=1e-13, err_msg=key)


def test_backward_document_isolation_zero_gradient(oracle_lib):
    """A loss on document 2 only gives exactly zero gradient to every input of
    document 1 and to its initial state (the packed-document card's zero-gradient
    isolation gate: state flow resets at every boundary)."""
    rng = np.random.default_rng(71)
    T, H, dk, dv = 9, 2, 4, 3
    q, k, v, g, b = _rand_inputs(rng, T, H, dk, dv)
    cu = np.array([0, 4, 9], dtype=np.int32)
    h0 = rng.standard_normal((2, H, dk, dv))
    dout = rng.standard_normal((1, T, H, dv))
    dout[:, :4] = 0.0
    dhT = rng.standard_normal((2, H, dk, dv))
    dhT[0] = 0.0
    r = oracle.backward(q, k, v, g, b, dout, h0, dhT, cu)
    for key in ("dq", "dk", "dv", "dg", "dbeta"):
        assert np.all(r[key][:, :4] == 0.0), key
        assert np.any(r[key][:, 4:] != 0.0), key
    assert np.all(r["dh0"][0] == 0.0) and np.any(r["dh0"][1] != 0.0)


# ---- fused input prep and output gate (short convolution, L2 norm, sigmoid gate) ----

def test_short_conv_matches_numpy_convolve():
    """Per channel, the causal convolution of one document is numpy's full
    convolution with the taps reversed, cut to the document's length."""
    rng = np.random.default_rng(80)
    x = rng.standard_normal((2, 11, 3, 5))
    w = rng.standard_normal((3, 5, 4))
    y = oracle.short_conv(x, w)
    for b in range(2):
        for h in range(3):
            for c in range(5):
                ref = np.convolve(x[b, :, h, c], w[h, c, ::-1])[:11]
                np.testing.assert_allclose(y[b, :, h, c], ref, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("tap", [0, 1, 2, 3])
def test_short_conv_delta_taps_shift(tap):
    """A single unit tap j of a width-4 convolution delays the sequence by 3 - j
    tokens, with zeros shifted in at the document start."""
    rng = np.random.default_rng(81 + tap)
    x = rng.standard_normal((1, 9, 2, 3))
    w = np.zeros((2, 3, 4))
    w[..., tap] = 1.0
    y = oracle.short_conv(x, w)
    s = 3 - tap
    assert np.array_equal(y[0, s:], x[0, :9 - s])
    assert np.all(y[0, :s] == 0)


def test_short_conv_restarts_at_document_boundaries():
    """Packed documents: each document's convolution equals that document run
    alone, and perturbing one document leaves the others unchanged."""
    rng = np.random.default_rng(85)
    lens = [5, 1, 0, 7, 2]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    x = rng.standard_normal((1, T, 2, 3))
    w = rng.standard_normal((2, 3, 3))
    y = oracle.short_conv(x, w, cu)
    for d in range(len(lens)):
        a, b = cu[d], cu[d + 1]
        alone = oracle.short_conv(x[:, a:b], w)
        assert np.array_equal(y[:, a:b], alone)
    x2 = x.copy()
    x2[:, cu[3]:cu[4]] += 5.0
    y2 = oracle.short_conv(x2, w, cu)
    assert np.array_equal(np.delete(y2, np.s_[cu[3]:cu[4]], axis=1),
                          np.delete(y, np.s_[cu[3]:cu[4]], axis=1))


def test_l2_normalize_properties():
    rng = np.random.default_rng(86)
    x = rng.standard_normal((3, 4, 2, 16))
    n = oracle.l2_normalize(x)
    np.testing.assert_allclose(np.linalg.norm(n, axis=-1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(oracle.l2_normalize(7.5 * x), n, rtol=1e-14)   # scale-free
    z = np.zeros((1, 2, 1, 8))
    assert np.array_equal(oracle.l2_normalize(z), z)                        # no NaN at 0


def test_output_gate_special_values():
    rng = np.random.default_rng(87)
    o = rng.standard_normal((2, 5, 3, 4))
    z = rng.standard_normal((2, 5, 3, 4))
    assert np.array_equal(oracle.output_gate(o, np.zeros_like(o)), o / 2)    # sigmoid(0) = 1/2
    np.testing.assert_allclose(oracle.output_gate(o, z) + oracle.output_gate(o, -z), o,
                               rtol=1e-14, atol=1e-15)                        # s(z) + s(-z) = 1
    np.testing.assert_allclose(oracle.output_gate(o, np.full_like(o, 60.0)), o, rtol=1e-15)


def test_prefill_fused_identity_prep_reduces_to_prefill(oracle_lib):
    """A width-1 unit convolution on inputs that are already unit-norm leaves k
    unchanged and scales q by dk^-1/2: the fused prefill is then the plain one."""
    rng = np.random.default_rng(88)
    T, H, dk, dv = 40, 2, 8, 6
    qr = rng.standard_normal((1, T, H, dk))
    kr = rng.standard_normal((1, T, H, dk))
    qr /= np.linalg.norm(qr, axis=-1, keepdims=True)
    kr /= np.linalg.norm(kr, axis=-1, keepdims=True)
    v = rng.standard_normal((1, T, H, dv))
    g = -np.abs(rng.standard_normal((1, T, H, dk))) * 0.1
    b = 1 / (1 + np.exp(-rng.standard_normal((1, T, H))))
    w = np.ones((H, dk, 1))
    o1, s1 = oracle.prefill_fused(qr, kr, v, g, b, w, w)
    o2, s2 = oracle.prefill(qr / np.sqrt(dk), kr, v, g, b)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(s1, s2, rtol=1e-12, atol=1e-14)
    o3, _ = oracle.prefill_fused(qr, kr, v, g, b)                     # no prep: q, k as given
    o4, _ = oracle.prefill(qr, kr, v, g, b)
    assert np.array_equal(o3, o4)
