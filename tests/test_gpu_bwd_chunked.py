"""The chunked backward on the tensor cores (kda_chunk_bwd with bf16 inputs and
128-wide heads) against the oracle's float64 reverse-mode differentiation of the
recurrence, on the same seeded inputs.

The chunked form's matrix products take bf16 operands with fp32 accumulation, as
the forward's do, so the gradients are held to the forward's bf16 bound
max|d - d_ref| / max|d_ref| <= 1e-2 (miniKimiK3 model card, "Kimi Delta
Attention" bullet: KDA trains through the chunked form; the bound is the one the
bf16 path is held to throughout).  Cases: ragged and single-token sequences, the
optional states, packed documents (an empty one and ragged lengths), the
zero-gradient isolation of packed documents (Mini-K3-1H-mamba2 card,
packed-document paragraph: no state or gradient flow across a boundary), grouped
decay, the bench's long workload on sampled heads, and agreement with the fp32
recurrent sweep."""
import pytest
import torch

import gated_delta_rule_74_b200 as kda
import kda_inputs as ki
import oracle
from _helpers import TOL, rel_err, to_dev

pytestmark = pytest.mark.gpu

TOL_BF16 = TOL["bf16"]
NAMES = ("dq", "dk", "dv", "dg", "dbeta", "dh0")


def _cotangents(x, seed, nseq, with_dhT=True):
    gen = torch.Generator().manual_seed(seed)
    q, v = x["q"], x["v"]
    dout = torch.randn(v.shape, generator=gen).to(q.dtype)
    dhT = None
    if with_dhT:
        dhT = 0.1 * torch.randn((nseq, q.shape[2], q.shape[3], v.shape[3]), generator=gen)
    return dout, dhT


def _bwd(d, dout, dhT, h0=True, g=None, **kw):
    r = kda.kda_chunk_bwd(d["q"], d["k"], d["v"], d["g"] if g is None else g, d["beta"],
                          dout.cuda(), h0=d["h0"] if h0 else None,
                          dhT=None if dhT is None else dhT.cuda(), cu_seqlens=d["cu_seqlens"],
                          **kw)
    torch.cuda.synchronize()
    return r


def _assert_close(r, ref, tol=TOL_BF16, heads=None):
    errs = {}
    for n in NAMES:
        if r[n] is None or n not in ref:
            continue
        got = r[n]
        if heads is not None:
            got = got[:, heads[0]:heads[1]] if n == "dh0" else got[:, :, heads[0]:heads[1]]
        assert torch.isfinite(got).all(), n
        errs[n] = rel_err(got, ref[n])
    assert all(e <= tol for e in errs.values()), errs
    return errs


@pytest.mark.parametrize("T,decay", [(200, "alog"), (64, "logsigmoid"), (1, "alog"),
                                     (129, "logsigmoid"), (640, "alog")])
def test_matches_oracle(T, decay):
    spec = ki.PrefillSpec("bwdc", B=2, T=T, H=3, dk=128, dv=128, dtype="bf16", decay=decay,
                          seed=T + 5, h0=True)
    x = ki.make_prefill(spec)
    dout, dhT = _cotangents(x, 100 + T, 2)
    r = _bwd(to_dev(x), dout, dhT)
    ref = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], dout, x["h0"], dhT)
    _assert_close(r, ref)


@pytest.mark.parametrize("with_h0,with_dhT", [(False, False), (False, True), (True, False)])
def test_optional_states(with_h0, with_dhT):
    spec = ki.PrefillSpec("bwdc", B=1, T=97, H=2, dk=128, dv=128, dtype="bf16", decay="alog",
                          seed=11, h0=True)
    x = ki.make_prefill(spec)
    dout, dhT = _cotangents(x, 12, 1, with_dhT)
    r = _bwd(to_dev(x), dout, dhT, h0=with_h0)
    assert (r["dh0"] is None) == (not with_h0)
    ref = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], dout,
                          x["h0"] if with_h0 else None, dhT)
    _assert_close(r, ref)


def test_packed_documents_with_empty_and_ragged():
    spec = ki.PrefillSpec("varlen", B=0, T=0, H=2, dk=128, dv=128, dtype="bf16", decay="alog",
                          seed=31, h0=True, varlen=True)
    x = ki.make_prefill(spec, doc_lens=[130, 0, 64, 257, 1])
    nseq = x["cu_seqlens"].numel() - 1
    dout, dhT = _cotangents(x, 32, nseq)
    r = _bwd(to_dev(x), dout, dhT)
    ref = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], dout, x["h0"], dhT,
                          x["cu_seqlens"])
    _assert_close(r, ref)
    assert torch.equal(r["dh0"][1].cpu(), dhT[1])       # the empty document: dh0 = dhT


def test_packed_documents_are_isolated():
    """Changing one document's output gradient leaves the other documents' gradients
    unchanged: dq, dk, dv and dh0 bit for bit, dg and dbeta up to the summation order of
    their shared-memory atomics."""
    spec = ki.PrefillSpec("varlen", B=0, T=0, H=2, dk=128, dv=128, dtype="bf16", decay="alog",
                          seed=33, h0=True, varlen=True)
    x = ki.make_prefill(spec, doc_lens=[100, 70, 130])
    nseq = x["cu_seqlens"].numel() - 1
    dout, dhT = _cotangents(x, 34, nseq)
    d = to_dev(x)
    a = _bwd(d, dout, dhT)
    dout2 = dout.clone()
    dout2[:, 100:170] = torch.randn(dout2[:, 100:170].shape,
                                    generator=torch.Generator().manual_seed(35)).to(dout.dtype)
    b = _bwd(d, dout2, dhT)
    for n in ("dq", "dk", "dv", "dg", "dbeta"):
        for lo, hi in ((0, 100), (170, 300)):
            if n in ("dg", "dbeta"):
                assert rel_err(a[n][:, lo:hi], b[n][:, lo:hi].double().cpu().numpy()) <= 1e-6
            else:
                assert torch.equal(a[n][:, lo:hi], b[n][:, lo:hi]), (n, lo)
        assert not torch.equal(a[n][:, 100:170], b[n][:, 100:170]), n
    assert torch.equal(a["dh0"][0], b["dh0"][0]) and torch.equal(a["dh0"][2], b["dh0"][2])


def test_zero_tokens():
    spec = ki.PrefillSpec("bwdc", B=2, T=1, H=2, dk=128, dv=128, dtype="bf16", decay="alog",
                          seed=3, h0=True)
    x = ki.make_prefill(spec)
    x = {n: (t[:, :0].contiguous() if isinstance(t, torch.Tensor) and n != "h0"
             and t.dim() >= 3 else t) for n, t in x.items()}
    dout = torch.zeros((2, 0, 2, 128), dtype=torch.bfloat16)
    dhT = torch.randn((2, 2, 128, 128))
    r = _bwd(to_dev(x), dout, dhT)
    assert torch.equal(r["dh0"].cpu(), dhT)


@pytest.mark.parametrize("G", [64, 8, 128])
def test_grouped_decay(G):
    """One decay per group of G key channels: dg of a shared value is the sum of the
    per-channel gradients over its group."""
    spec = ki.PrefillSpec("bwdc", B=2, T=150, H=2, dk=128, dv=128, dtype="bf16", decay="alog",
                          seed=G + 7, h0=True)
    x = ki.make_prefill(spec)
    gg = x["g"][..., ::G].contiguous()
    dout, dhT = _cotangents(x, 61 + G, 2)
    r = _bwd(to_dev(x), dout, dhT, g=gg.cuda())
    assert tuple(r["dg"].shape) == tuple(gg.shape)
    ref = oracle.backward(x["q"], x["k"], x["v"], gg, x["beta"], dout, x["h0"], dhT)
    ref["dg"] = ref["dg"].reshape(*gg.shape, G).sum(-1)
    _assert_close(r, ref)


def test_long_sequence_sampled_heads():
    """The bench's backward workload (B=1, T=8192, H=12, d=128, bf16), two heads
    checked against the oracle."""
    spec = ki.PrefillSpec("bwdc", B=1, T=8192, H=12, dk=128, dv=128, dtype="bf16",
                          decay="alog", seed=8192, h0=False)
    x = ki.make_prefill(spec)
    dout, dhT = _cotangents(x, 8193, 1)
    r = _bwd(to_dev(x), dout, dhT, h0=False)
    heads = (0, 1)
    ref = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], dout, None, dhT,
                          heads=heads)
    _assert_close(r, ref, heads=heads)
    heads = (11, 12)
    ref = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], dout, None, dhT,
                          heads=heads)
    _assert_close(r, ref, heads=heads)


def test_long_many_heads_sampled():
    """B=1, T=32768, H=96 (the long-prefill shape): 512 chunks x 96 heads, so the chunk
    records and state images span more than 4 GB of scratch (byte offsets past 2^32); the
    last head, whose records sit at the end, against the oracle."""
    spec = ki.PrefillSpec("bwdc", B=1, T=32768, H=96, dk=128, dv=128, dtype="bf16",
                          decay="alog", seed=32768, h0=False)
    x = ki.make_prefill(spec)
    gen = torch.Generator().manual_seed(32769)
    dout = torch.randn(x["v"].shape, generator=gen).to(torch.bfloat16)
    r = _bwd(to_dev(x), dout, None, h0=False)
    heads = (95, 96)
    ref = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], dout, None, None,
                          heads=heads)
    _assert_close(r, ref, heads=heads)


def test_agrees_with_recurrent_sweep():
    spec = ki.PrefillSpec("bwdc", B=2, T=300, H=4, dk=128, dv=128, dtype="bf16",
                          decay="logsigmoid", seed=77, h0=True)
    x = ki.make_prefill(spec)
    dout, dhT = _cotangents(x, 78, 2)
    d = to_dev(x)
    a = _bwd(d, dout, dhT)
    b = _bwd(d, dout, dhT, recurrent=True)
    for n in NAMES:
        assert rel_err(a[n], b[n].double().cpu().numpy()) <= TOL_BF16, n


def test_repeatable():
    """dq, dk, dv and dh0 bit for bit across calls; dg and dbeta add per-chunk sums with
    shared-memory atomics (fp32 rounding only)."""
    spec = ki.PrefillSpec("bwdc", B=1, T=300, H=2, dk=128, dv=128, dtype="bf16", decay="alog",
                          seed=41, h0=True)
    x = ki.make_prefill(spec)
    dout, dhT = _cotangents(x, 42, 1)
    d = to_dev(x)
    a = _bwd(d, dout, dhT)
    b = _bwd(d, dout, dhT)
    for n in ("dq", "dk", "dv", "dh0"):
        assert torch.equal(a[n], b[n]), n
    for n in ("dg", "dbeta"):
        assert rel_err(a[n], b[n].double().cpu().numpy()) <= 1e-6, n
