"""The seeded input generators produce the documented shapes and distributions."""
import torch

import kda_inputs as ki


def test_prefill_shapes_and_ranges():
    x = ki.make_prefill("b16_t512_d64", T=64, B=2)
    assert x["q"].shape == (2, 64, 8, 64) and x["q"].dtype == torch.bfloat16
    assert x["g"].dtype == torch.float32 and (x["g"] <= 0).all()
    assert ((x["beta"] > 0) & (x["beta"] < 1)).all()
    kn = x["k"].float().norm(dim=-1)
    assert torch.allclose(kn, torch.ones_like(kn), atol=1e-2)
    qn = x["q"].float().norm(dim=-1)
    assert torch.allclose(qn, torch.full_like(qn, 64 ** -0.5), atol=1e-3)
    assert x["h0"] is None and x["cu_seqlens"] is None


def test_prefill_deterministic():
    a = ki.make_prefill("fp32_t256")
    b = ki.make_prefill("fp32_t256")
    for key in ("q", "k", "v", "g", "beta"):
        assert torch.equal(a[key], b[key])
    assert a["q"].dtype == torch.float32


def test_varlen_doc_lengths():
    x = ki.make_prefill("packed_16k")
    cu = x["cu_seqlens"]
    assert int(cu[0]) == 0 and int(cu[-1]) == 16384 == x["T"]
    lens = (cu[1:] - cu[:-1]).tolist()
    assert all(l <= 4096 for l in lens) and all(l >= 128 for l in lens[:-1])
    assert x["q"].shape[0] == 1 and x["B"] == len(lens)


def test_alog_decay_and_h0():
    x = ki.make_prefill("t32k_h96", T=128, H=4)
    assert x["h0"].shape == (1, 4, 128, 128)
    assert abs(float(x["h0"].std()) - 0.02) < 2e-3
    assert (x["g"] <= 0).all()


def test_decode_inputs():
    d = ki.make_decode("decode_n256_h96", N=4, H=3, steps=2)
    assert d["q"].shape == (2, 4, 3, 128) and d["S0"].shape == (4, 3, 128, 128)
    assert d["beta"].shape == (2, 4, 3)
