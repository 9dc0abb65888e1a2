"""Grouped decay (one log-decay per group of G consecutive key channels, the
decay-granularity variant of the "decay-g64" family card) on the GPU: bit-for-bit
the per-channel path fed with the expanded g, and the oracle's recurrence."""
import pytest
import torch

import gated_delta_rule_74_b200 as kda
import kda_inputs as ki
import oracle
from _helpers import TOL, rel_err, to_dev

pytestmark = pytest.mark.gpu


def _grouped(x, G):
    """One decay value per group: the first channel's draw of each group."""
    return x["g"][..., ::G].contiguous()


@pytest.mark.parametrize("dtype,dk,dv,G", [("bf16", 128, 128, 64), ("bf16", 128, 128, 2),
                                           ("bf16", 64, 64, 64), ("bf16", 128, 64, 128),
                                           ("f32", 64, 64, 16), ("f32", 128, 128, 64)])
def test_grouped_prefill_equals_expanded_bitwise(dtype, dk, dv, G):
    spec = ki.PrefillSpec("g", B=2, T=300, H=3, dk=dk, dv=dv, dtype=dtype, decay="alog", seed=G,
                          h0=True)
    x = ki.make_prefill(spec)
    d = to_dev(x)
    gg = _grouped(x, G).cuda()
    gx = torch.repeat_interleave(gg, G, dim=-1).contiguous()
    o1, s1 = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], gg, d["beta"], h0=d["h0"])
    o2, s2 = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], gx, d["beta"], h0=d["h0"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


@pytest.mark.parametrize("T", [640, 1300])
def test_grouped_prefill_matches_oracle(T):
    """decay-g64 at d = 128 over a split (segmented) sequence."""
    spec = ki.PrefillSpec("g64", B=1, T=T, H=2, dk=128, dv=128, dtype="bf16", decay="alog",
                          seed=T + 7, h0=True)
    x = ki.make_prefill(spec)
    d = to_dev(x)
    gg = _grouped(x, 64)
    out, hT = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], gg.cuda(), d["beta"], h0=d["h0"])
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.prefill(x["q"], x["k"], x["v"], gg, x["beta"], x["h0"])
    assert rel_err(out, o_ref) <= TOL["bf16"]
    assert rel_err(hT, s_ref) <= TOL["bf16"]


def test_grouped_prefill_packed_matches_oracle():
    spec = ki.PrefillSpec("varlen", B=0, T=0, H=2, dk=128, dv=128, dtype="bf16", decay="alog",
                          seed=21, h0=True, varlen=True)
    x = ki.make_prefill(spec, doc_lens=[700, 130, 1100])
    d = to_dev(x)
    gg = _grouped(x, 64)
    out, hT = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], gg.cuda(), d["beta"], h0=d["h0"],
                                cu_seqlens=d["cu_seqlens"])
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.prefill(x["q"], x["k"], x["v"], gg, x["beta"], x["h0"], x["cu_seqlens"])
    assert rel_err(out, o_ref) <= TOL["bf16"]
    assert rel_err(hT, s_ref) <= TOL["bf16"]


@pytest.mark.parametrize("G", [64, 4])
def test_grouped_decode_tokens(G):
    d = ki.make_decode(ki.DecodeSpec("t", N=4, H=3, dk=128, dv=128, steps=12, dtype="bf16",
                                     decay="alog", seed=G))
    x = {n: d[n].transpose(0, 1).contiguous().cuda() for n in ("q", "k", "v", "g", "beta")}
    gg = x["g"][..., ::G].contiguous()
    S1, S2 = d["S0"].cuda(), d["S0"].cuda()
    o1 = kda.kda_decode_tokens(x["q"], x["k"], x["v"], gg, x["beta"], S1)
    o2 = kda.kda_decode_tokens(x["q"], x["k"], x["v"],
                               torch.repeat_interleave(gg, G, dim=-1).contiguous(), x["beta"], S2)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    tr = lambda t: t.transpose(0, 1)
    o_ref, s_ref = oracle.prefill(tr(d["q"]), tr(d["k"]), tr(d["v"]), tr(d["g"])[..., ::G],
                                  tr(d["beta"]), d["S0"])
    assert rel_err(o1, o_ref) <= TOL["bf16"]
    assert rel_err(S1, s_ref) <= TOL["bf16"]
