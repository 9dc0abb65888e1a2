"""kda_decode_chunk (L <= 16 tokens as one chunk on the tensor cores) against the
oracle's recurrence and against the bit-exact multi-token decode."""
import numpy as np
import pytest
import torch

import gated_delta_rule_74_b200 as kda
import kda_inputs as ki
import oracle
from _helpers import TOL, rel_err

pytestmark = pytest.mark.gpu


def _inputs(N, H, L, seed):
    d = ki.make_decode(ki.DecodeSpec("c", N=N, H=H, dk=128, dv=128, steps=L, dtype="bf16",
                                     decay="alog", seed=seed))
    x = {n: d[n].transpose(0, 1).contiguous() for n in ("q", "k", "v", "g", "beta")}
    return d, x


@pytest.mark.parametrize("L", [1, 2, 7, 16])
def test_decode_chunk_matches_oracle(L):
    d, x = _inputs(N=3, H=4, L=L, seed=L)
    S = d["S0"].cuda()
    out = kda.kda_decode_chunk(*(x[n].cuda() for n in ("q", "k", "v", "g", "beta")), S)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], d["S0"])
    assert rel_err(out, o_ref) <= TOL["bf16"]
    assert rel_err(S, s_ref) <= TOL["bf16"]


def test_decode_chunk_close_to_single_steps():
    d, x = _inputs(N=5, H=3, L=16, seed=31)
    S1, S2 = d["S0"].cuda(), d["S0"].cuda()
    xs = [x[n].cuda() for n in ("q", "k", "v", "g", "beta")]
    o1 = kda.kda_decode_chunk(*xs, S1)
    o2 = kda.kda_decode_tokens(*xs, S2)
    torch.cuda.synchronize()
    assert rel_err(o1, o2.double().cpu().numpy()) <= TOL["bf16"]
    assert rel_err(S1, S2.double().cpu().numpy()) <= TOL["bf16"]


def test_decode_chunk_cfg4_sampled():
    """The config-4 shape (N = 256, H = 96, 16 tokens), 200 sampled (n, h) pairs."""
    d = ki.make_decode("decode_n256_h96")
    x = {n: d[n].transpose(0, 1).contiguous() for n in ("q", "k", "v", "g", "beta")}
    S = d["S0"].cuda()
    out = kda.kda_decode_chunk(*(x[n].cuda() for n in ("q", "k", "v", "g", "beta")), S)
    torch.cuda.synchronize()
    rng = np.random.default_rng(7)
    ns = rng.choice(d["N"], 50, replace=False)
    for n in ns[:50]:
        hs = (int(rng.integers(0, d["H"] - 4)),)
        lo, hi = hs[0], hs[0] + 4
        sel = lambda t: t[n:n + 1, :, lo:hi]
        o_ref, s_ref = oracle.prefill(sel(x["q"]), sel(x["k"]), sel(x["v"]), sel(x["g"]),
                                      sel(x["beta"]), d["S0"][n:n + 1, lo:hi])
        assert rel_err(out[n:n + 1, :, lo:hi], o_ref) <= TOL["bf16"]
        assert rel_err(S[n:n + 1, lo:hi], s_ref) <= TOL["bf16"]
    assert kda.kda_device_status(reset=True) == kda.KDA_OK
