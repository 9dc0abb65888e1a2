"""The oracle's closed-form pins, run on the GPU kernels directly (no oracle involved):
pure channel decay at beta = 0, the error-correcting write at beta = 1, exact recall
with orthonormal keys, a constant state at g = beta = 0, and the hand-worked example
(miniKimiK3 model card, "Kimi Delta Attention" bullet).  Inputs are chosen so that
their storage values are exact (unit keys with four +-1/2 entries, Hadamard rows / 8),
so the closed forms hold for the values the kernels read.  Paths: the bf16
tensor-core prefill (split, including the segmented state pass), the fp32 CUDA-core
prefill and the multi-token decode."""
import os

import numpy as np
import pytest
import torch

import gated_delta_rule_74_b200 as kda

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
# (storage dtype, dk = dv): bf16 tensor-core prefill, fp32 CUDA-core prefill
PATHS = [("bf16", 128), ("bf16", 64), ("f32", 64)]
TOL = {"bf16": 1e-2, "f32": 1e-4}
DT = {"bf16": torch.bfloat16, "f32": torch.float32}


def _rel(x, ref):
    x = x.detach().double().cpu().numpy() if hasattr(x, "detach") else np.asarray(x)
    ref = np.asarray(ref, np.float64)
    return float(np.abs(x - ref).max() / max(np.abs(ref).max(), 1e-30))


def _prefill(q, k, v, g, b, h0, dtype):
    """q, k [T, H, d], v [T, H, dv], g [T, H, d], b [T, H], h0 [H, d, dv] (numpy) ->
    GPU out [T, H, dv], hT [H, d, dv] from one B = 1 kda_chunk_fwd call."""
    t = lambda a, dt: torch.tensor(np.ascontiguousarray(a)[None], dtype=dt).cuda()
    out, hT = kda.kda_chunk_fwd(t(q, DT[dtype]), t(k, DT[dtype]), t(v, DT[dtype]),
                                t(g, torch.float32), t(b, torch.float32), h0=t(h0, torch.float32))
    torch.cuda.synchronize()
    return out[0], hT[0]


def _decode(q, k, v, g, b, h0, dtype):
    """The same tokens as one kda_decode_tokens launch (N = 1)."""
    t = lambda a, dt: torch.tensor(np.ascontiguousarray(a)[None], dtype=dt).cuda()
    S = t(h0, torch.float32)
    out = kda.kda_decode_tokens(t(q, DT[dtype]), t(k, DT[dtype]), t(v, DT[dtype]),
                                t(g, torch.float32), t(b, torch.float32), S)
    torch.cuda.synchronize()
    return out[0], S[0]


def _stored(a, dtype):
    """The values the kernels read (storage rounding), as float64."""
    return torch.tensor(a).to(DT[dtype]).double().numpy()


def _unit_keys(rng, T, H, d):
    """Unit keys exact in bf16: four entries +-1/2 on random channels."""
    k = np.zeros((T, H, d))
    for t in range(T):
        for h in range(H):
            ch = rng.choice(d, 4, replace=False)
            k[t, h, ch] = rng.choice([-0.5, 0.5], 4)
    return k


def _decay(rng, T, H, d):
    return -np.exp(rng.uniform(-2, 0, (1, H, 1))) * np.log1p(np.exp(rng.standard_normal((T, H, d))))


def _runners():
    return [("prefill", _prefill), ("decode_tokens", _decode)]


@pytest.mark.parametrize("dtype,d", PATHS)
@pytest.mark.parametrize("T", [150, 1300])
def test_beta_zero_is_pure_channel_decay(dtype, d, T):
    """beta = 0: S_t = Diag(exp(Gamma_t)) h0 and o_t = S_t^T q_t (Gamma = cumsum g)."""
    rng = np.random.default_rng(T + d)
    H = 2
    q = _stored(rng.standard_normal((T, H, d)) / np.sqrt(d), dtype)
    k = _stored(_unit_keys(rng, T, H, d), dtype)
    v = _stored(rng.standard_normal((T, H, d)), dtype)
    g = _decay(rng, T, H, d) * 0.05
    b = np.zeros((T, H))
    h0 = rng.standard_normal((H, d, d))
    gam = np.cumsum(g.astype(np.float32).astype(np.float64), axis=0)
    S_ref = np.exp(gam[-1])[:, :, None] * h0
    o_ref = np.einsum("thc,hcj->thj", q * np.exp(gam), h0)
    for name, run in _runners():
        if name == "decode_tokens" and T > 200:
            continue
        out, hT = run(q, k, v, g, b, h0, dtype)
        assert _rel(hT, S_ref) <= TOL[dtype], name
        assert _rel(out, o_ref) <= TOL[dtype], name


@pytest.mark.parametrize("dtype,d", PATHS)
def test_error_correcting_write(dtype, d):
    """beta = 1 and |k| = 1: S_t^T k_t = v_t after every step, so reading with q = k
    returns v exactly, whatever the decay and the initial state."""
    rng = np.random.default_rng(7 + d)
    T, H = 200, 2
    k = _unit_keys(rng, T, H, d)
    v = _stored(rng.standard_normal((T, H, d)), dtype)
    g = _decay(rng, T, H, d)
    b = np.ones((T, H))
    h0 = rng.standard_normal((H, d, d)) * 0.1
    for name, run in _runners():
        out, _ = run(k, k, v, g, b, h0, dtype)
        assert _rel(out, v) <= TOL[dtype], name


def _hadamard(n):
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


@pytest.mark.parametrize("dtype,d", PATHS)
def test_exact_recall_orthonormal_keys(dtype, d):
    """alpha = 1, beta = 1, orthonormal keys, S_0 = 0: S_T = sum_t k_t v_t^T, and a
    query equal to an earlier key k_j returns v_j."""
    rng = np.random.default_rng(11 + d)
    T, H = 60, 2
    rows = _hadamard(64) / 8.0                         # orthonormal, exact in bf16
    k = np.zeros((T, H, d))
    j_of_t = np.zeros((T, H), dtype=int)
    for h in range(H):
        k[:, h, :64] = rows[rng.permutation(64)[:T]]
        j_of_t[:, h] = [rng.integers(0, t + 1) for t in range(T)]
    q = np.stack([k[j_of_t[:, h], h] for h in range(H)], axis=1)
    v = _stored(rng.standard_normal((T, H, d)), dtype)
    g = np.zeros((T, H, d))
    b = np.ones((T, H))
    h0 = np.zeros((H, d, d))
    o_ref = np.stack([v[j_of_t[:, h], h] for h in range(H)], axis=1)
    S_ref = np.einsum("thc,thj->hcj", k, v)
    for name, run in _runners():
        out, hT = run(q, k, v, g, b, h0, dtype)
        assert _rel(out, o_ref) <= TOL[dtype], name
        assert _rel(hT, S_ref) <= TOL[dtype], name


@pytest.mark.parametrize("dtype,d", PATHS)
def test_no_decay_no_write_keeps_the_state(dtype, d):
    """g = 0 and beta = 0: S stays h0 (bit for bit) and o_t = h0^T q_t."""
    rng = np.random.default_rng(13 + d)
    T, H = 130, 2
    q = _stored(rng.standard_normal((T, H, d)) / np.sqrt(d), dtype)
    k = _stored(_unit_keys(rng, T, H, d), dtype)
    v = _stored(rng.standard_normal((T, H, d)), dtype)
    g = np.zeros((T, H, d))
    b = np.zeros((T, H))
    h0 = rng.standard_normal((H, d, d)).astype(np.float32).astype(np.float64)
    o_ref = np.einsum("thc,hcj->thj", q, h0)
    for name, run in _runners():
        out, hT = run(q, k, v, g, b, h0, dtype)
        assert np.array_equal(hT.double().cpu().numpy(), h0), name
        assert _rel(out, o_ref) <= TOL[dtype], name


def _golden():
    from fractions import Fraction
    vals = {}
    with open(os.path.join(GOLDEN, "hand_tiny.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                key, *rest = line.split()
                vals[key] = np.array([float(Fraction(x)) for x in rest])
    return vals


@pytest.mark.parametrize("dtype,d", PATHS)
def test_hand_worked_example_embedded(dtype, d):
    """The dk = dv = 2 hand-worked example (tests/golden/hand_tiny.txt), embedded in the
    first two channels of a d-wide head: all other channels stay exactly zero."""
    G = _golden()
    T, H = 2, 1
    q, k, v, g = (np.zeros((T, H, d)) for _ in range(4))
    for t, s in ((0, "1"), (1, "2")):
        q[t, 0, :2], k[t, 0, :2], v[t, 0, :2] = G["q" + s], G["k" + s], G["v" + s]
        g[t, 0, :2] = np.log(G["alpha" + s])
    b = np.array([[G["beta1"][0]], [G["beta2"][0]]])
    h0 = np.zeros((H, d, d))
    h0[0, :2, :2] = G["S0"].reshape(2, 2)
    o_ref = np.zeros((T, H, d))
    o_ref[0, 0, :2], o_ref[1, 0, :2] = G["o1"], G["o2"]
    S_ref = np.zeros((H, d, d))
    S_ref[0, :2, :2] = G["S2"].reshape(2, 2)
    for name, run in _runners():
        out, hT = run(q, k, v, g, b, h0, dtype)
        assert _rel(out, o_ref) <= TOL[dtype], name
        assert _rel(hT, S_ref) <= TOL[dtype], name
        assert np.all(hT.double().cpu().numpy()[0, 2:, :] == 0), name
        assert np.all(hT.double().cpu().numpy()[0, :, 2:] == 0), name
