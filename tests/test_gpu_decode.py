"""GPU parity of kda_decode_step against the float64 oracle."""
import numpy as np
import pytest
import torch

import kda_inputs as ki
import oracle
from _helpers import TOL, rel_err

pytestmark = pytest.mark.gpu


def _run_steps(d, steps, sample=None):
    import gated_delta_rule_74_b200 as kda
    S = d["S0"].cuda()
    outs = []
    for t in range(steps):
        o = kda.kda_decode_step(d["q"][t].cuda(), d["k"][t].cuda(), d["v"][t].cuda(),
                                d["g"][t].cuda(), d["beta"][t].cuda(), S)
        outs.append(o if sample is None else o.reshape(-1, o.shape[-1])[sample])
    torch.cuda.synchronize()
    return outs, S


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
def test_decode_small(dtype, dk, dv):
    spec = ki.DecodeSpec("t", N=5, H=3, dk=dk, dv=dv, steps=4, dtype=dtype, decay="alog", seed=7)
    d = ki.make_decode(spec)
    outs, S = _run_steps(d, 4)
    S_ref = d["S0"]
    for t in range(4):
        o_ref, S_ref = oracle.decode(d["q"][t], d["k"][t], d["v"][t], d["g"][t], d["beta"][t], S_ref)
        assert rel_err(outs[t], o_ref) <= TOL[dtype], t
    assert rel_err(S, S_ref) <= TOL[dtype]


def test_decode_cfg4_sampled():
    """Full config-4 shape (N=256, H=96, d=128, 16 consecutive tokens, 1.61 GB of
    fp32 state) on the GPU; the oracle checks 96 sampled (n, h) pairs."""
    d = ki.make_decode("decode_n256_h96")
    N, H = d["N"], d["H"]
    rng = np.random.default_rng(0)
    pairs = np.sort(rng.choice(N * H, size=96, replace=False))
    outs, S = _run_steps(d, d["steps"], sample=torch.from_numpy(pairs).cuda())
    flat = lambda t: t.reshape(-1, *t.shape[2:])[pairs][:, None]   # [P, 1, ...]
    S_ref = d["S0"].reshape(N * H, 128, 128)[pairs][:, None]
    for t in range(d["steps"]):
        o_ref, S_ref = oracle.decode(flat(d["q"][t]), flat(d["k"][t]), flat(d["v"][t]),
                                     flat(d["g"][t]), d["beta"][t].reshape(-1)[pairs][:, None],
                                     S_ref)
        assert rel_err(outs[t], o_ref[:, 0]) <= TOL["bf16"], t
    S_got = S.reshape(N * H, 128, 128)[torch.from_numpy(pairs).cuda()]
    assert rel_err(S_got, S_ref[:, 0]) <= TOL["bf16"]


# ---- multi-token decode: L steps in one launch ------------------------------
def _tokens_inputs(d):
    """[steps, N, H, .] -> [N, L, H, .] on the GPU."""
    return {n: d[n].transpose(0, 1).contiguous().cuda() for n in ("q", "k", "v", "g", "beta")}


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("L", [1, 5, 8, 9, 17])
def test_decode_tokens_equals_single_steps_bitwise(dtype, dk, dv, L):
    """The fused launch takes each token with the single step's arithmetic in the
    same order: outputs and final state are bit-for-bit those of L steps."""
    import gated_delta_rule_74_b200 as kda
    spec = ki.DecodeSpec("t", N=3, H=5, dk=dk, dv=dv, steps=L, dtype=dtype, decay="alog",
                         seed=L + dk + dv)
    d = ki.make_decode(spec)
    outs, S_steps = _run_steps(d, L)
    x = _tokens_inputs(d)
    S = d["S0"].cuda()
    out = kda.kda_decode_tokens(x["q"], x["k"], x["v"], x["g"], x["beta"], S)
    torch.cuda.synchronize()
    assert torch.equal(out, torch.stack(outs, dim=1))
    assert torch.equal(S, S_steps)


@pytest.mark.parametrize("L", [16, 40])
def test_decode_tokens_matches_oracle(L):
    """L tokens per sequence from a nonzero state: the recurrence over those
    tokens (oracle prefill with h0 = S)."""
    import gated_delta_rule_74_b200 as kda
    spec = ki.DecodeSpec("t", N=4, H=6, dk=128, dv=128, steps=L, dtype="bf16", decay="alog",
                         seed=100 + L)
    d = ki.make_decode(spec)
    x = _tokens_inputs(d)
    S = d["S0"].cuda()
    out = kda.kda_decode_tokens(x["q"], x["k"], x["v"], x["g"], x["beta"], S)
    torch.cuda.synchronize()
    tr = lambda t: t.transpose(0, 1)
    o_ref, s_ref = oracle.prefill(tr(d["q"]), tr(d["k"]), tr(d["v"]), tr(d["g"]),
                                  tr(d["beta"]), d["S0"])
    assert rel_err(out, o_ref) <= TOL["bf16"]
    assert rel_err(S, s_ref) <= TOL["bf16"]


def test_decode_tokens_cfg4_sampled():
    """The config-4 workload (N=256, H=96, d=128, 16 tokens) as one launch; the
    oracle checks 64 sampled (n, h) pairs over all 16 tokens."""
    import gated_delta_rule_74_b200 as kda
    d = ki.make_decode("decode_n256_h96")
    N, H, L = d["N"], d["H"], d["steps"]
    x = _tokens_inputs(d)
    S = d["S0"].cuda()
    out = kda.kda_decode_tokens(x["q"], x["k"], x["v"], x["g"], x["beta"], S)
    torch.cuda.synchronize()
    rng = np.random.default_rng(1)
    pairs = np.sort(rng.choice(N * H, size=64, replace=False))
    n_idx, h_idx = pairs // H, pairs % H
    sel = lambda t: t[:, n_idx, h_idx][:, :, None]           # [L, P, 1, ...]
    o_ref, s_ref = oracle.prefill(sel(d["q"]).transpose(0, 1), sel(d["k"]).transpose(0, 1),
                                  sel(d["v"]).transpose(0, 1), sel(d["g"]).transpose(0, 1),
                                  d["beta"][:, n_idx, h_idx][:, :, None].transpose(0, 1),
                                  d["S0"].reshape(N * H, 128, 128)[pairs][:, None])
    got = out.cpu()[n_idx, :, h_idx]                          # [P, L, dv]
    assert rel_err(got, o_ref[:, :, 0]) <= TOL["bf16"]
    S_got = S.reshape(N * H, 128, 128)[torch.from_numpy(pairs).cuda()]
    assert rel_err(S_got, s_ref[:, 0]) <= TOL["bf16"]
