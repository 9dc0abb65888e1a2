"""Fused input prep and output gate (kda_chunk_fwd_fused) on the GPU against the
oracle's float64 definition: q = dk^-1/2 n(conv_q * q_raw), k = n(conv_k * k_raw)
(causal per-channel convolutions restarting at document starts, n = L2
normalisation), out = o * sigmoid(gate).  bf16 inputs: bound 1e-2."""
import pytest
import torch

import gated_delta_rule_74_b200 as kda
import kda_inputs as ki
import oracle
from _helpers import TOL, rel_err, to_dev

pytestmark = pytest.mark.gpu


def _run(x, conv=True, gate=True, with_h0=True):
    d = to_dev(x)
    out, hT = kda.kda_chunk_fwd_fused(
        d["q_raw"], d["k_raw"], d["v"], d["g"], d["beta"],
        conv_q=d["conv_q"] if conv else None, conv_k=d["conv_k"] if conv else None,
        gate=d["gate"] if gate else None, h0=d["h0"] if with_h0 else None,
        cu_seqlens=d["cu_seqlens"])
    torch.cuda.synchronize()
    return out, hT


def _ref(x, conv=True, gate=True, with_h0=True, heads=None):
    return oracle.prefill_fused(x["q_raw"], x["k_raw"], x["v"], x["g"], x["beta"],
                                x["conv_q"] if conv else None, x["conv_k"] if conv else None,
                                x["gate"] if gate else None, x["h0"] if with_h0 else None,
                                x["cu_seqlens"], heads=heads)


@pytest.mark.parametrize("dk,dv,W,T,gate", [(128, 128, 4, 200, True), (64, 64, 2, 130, False),
                                             (128, 64, 1, 64, True), (64, 128, 3, 1, True),
                                             (128, 128, 3, 97, False)])
def test_fused_matches_oracle(dk, dv, W, T, gate):
    spec = ki.PrefillSpec("fz", B=2, T=T, H=3, dk=dk, dv=dv, dtype="bf16", decay="alog",
                          seed=T + W, h0=True)
    x = ki.make_fused_prefill(spec, W=W, gate=gate)
    out, hT = _run(x, gate=gate)
    o_ref, s_ref = _ref(x, gate=gate)
    assert rel_err(out, o_ref) <= TOL["bf16"]
    assert rel_err(hT, s_ref) <= TOL["bf16"]


def test_fused_packed_documents_restart_the_convolution():
    """Documents shorter than the window, empty ones, chunk-crossing halos."""
    spec = ki.PrefillSpec("varlen", B=0, T=0, H=2, dk=128, dv=128, dtype="bf16", decay="alog",
                          seed=41, h0=True, varlen=True)
    x = ki.make_fused_prefill(spec, W=4, doc_lens=[130, 2, 0, 65, 300, 3])
    out, hT = _run(x)
    o_ref, s_ref = _ref(x)
    assert rel_err(out, o_ref) <= TOL["bf16"]
    assert rel_err(hT, s_ref) <= TOL["bf16"]
    # a document packed gives the same bits as the document alone (chunks and the
    # convolution restart at its first token)
    cu = x["cu_seqlens"].tolist()
    a, b = cu[4], cu[5]
    y = {n: (t[:, a:b].contiguous() if isinstance(t, torch.Tensor) and t.dim() >= 3
             and t.shape[1] == x["q_raw"].shape[1] else t) for n, t in x.items()}
    y["cu_seqlens"] = None
    y["h0"] = x["h0"][4:5].contiguous()
    o_alone, _ = _run(y)
    assert torch.equal(o_alone[0], out[0, a:b])


def test_fused_without_prep_or_gate_is_kda_chunk_fwd():
    spec = ki.PrefillSpec("fz", B=1, T=300, H=2, dk=128, dv=128, dtype="bf16", decay="alog",
                          seed=5, h0=True)
    x = ki.make_fused_prefill(spec)
    d = to_dev(x)
    o1, s1 = kda.kda_chunk_fwd_fused(d["q"], d["k"], d["v"], d["g"], d["beta"], h0=d["h0"])
    o2, s2 = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], h0=d["h0"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)
    # gate only: o * sigmoid(z) of the same KDA output
    o3, _ = kda.kda_chunk_fwd_fused(d["q"], d["k"], d["v"], d["g"], d["beta"], h0=d["h0"],
                                    gate=d["gate"])
    torch.cuda.synchronize()
    ref = oracle.output_gate(o2.float().cpu().numpy(), x["gate"])
    assert rel_err(o3, ref) <= 2 ** -7


def test_fused_long_sequence_sampled_heads():
    """The headline shape (T = 8192, 12 heads of 128, segmented state pass), two
    heads against the oracle."""
    x = ki.make_fused_prefill("t8k_h12", W=4)
    out, hT = _run(x)
    heads = (3, 5)
    o_ref, s_ref = _ref(x, heads=heads)
    assert rel_err(out[:, :, heads[0]:heads[1]], o_ref) <= TOL["bf16"]
    assert rel_err(hT[:, heads[0]:heads[1]], s_ref) <= TOL["bf16"]


def test_fused_rejects_f32_and_half_conv():
    x = ki.make_fused_prefill(ki.PrefillSpec("fz", B=1, T=8, H=1, dk=64, dv=64, dtype="f32",
                                             decay="alog", seed=1, h0=False))
    d = to_dev(x)
    with pytest.raises(kda.KdaError):
        kda.kda_chunk_fwd_fused(d["q_raw"], d["k_raw"], d["v"], d["g"], d["beta"],
                                conv_q=d["conv_q"], conv_k=d["conv_k"])
    with pytest.raises(ValueError):
        kda.kda_chunk_fwd_fused(d["q_raw"], d["k_raw"], d["v"], d["g"], d["beta"],
                                conv_q=d["conv_q"])


def test_fused_packed_long_documents_segmented():
    """Packed documents long enough for the segmented state pass (16-chunk segments):
    the gate applies in both passes, the convolution restarts per document."""
    spec = ki.PrefillSpec("varlen", B=0, T=0, H=2, dk=128, dv=128, dtype="bf16", decay="alog",
                          seed=43, h0=True, varlen=True)
    x = ki.make_fused_prefill(spec, W=4, doc_lens=[1500, 70, 1100, 700])
    out, hT = _run(x)
    o_ref, s_ref = _ref(x)
    assert rel_err(out, o_ref) <= TOL["bf16"]
    assert rel_err(hT, s_ref) <= TOL["bf16"]
