"""The recurrent prefill backward on the GPU (kda_chunk_bwd_recurrent, and
kda_chunk_bwd for the inputs it sends there: fp32 or 64-wide heads) against the
oracle's float64 reverse-mode differentiation of the recurrence, on the same
seeded inputs.

The sweep computes in fp32 on the exact values of the (bf16 or fp32) inputs, so
every gradient is held to the fp32 bound max|d - d_ref| / max|d_ref| <= 1e-4,
whatever the storage dtype.  The chunked form (bf16, 128-wide heads) has its own
tests in test_gpu_bwd_chunked.py."""
import pytest
import torch

import gated_delta_rule_74_b200 as kda
import kda_inputs as ki
import oracle
from _helpers import rel_err, to_dev

pytestmark = pytest.mark.gpu

TOL_BWD = 1e-4
NAMES = ("dq", "dk", "dv", "dg", "dbeta", "dh0")


def _cotangents(x, seed, nseq, with_dhT=True):
    """Seeded dL/dout (in out's dtype) and dL/dhT (fp32)."""
    gen = torch.Generator().manual_seed(seed)
    q, v = x["q"], x["v"]
    dout = torch.randn(v.shape, generator=gen).to(q.dtype)
    dhT = None
    if with_dhT:
        dhT = 0.1 * torch.randn((nseq, q.shape[2], q.shape[3], v.shape[3]), generator=gen)
    return dout, dhT


def _run(x, dout, dhT, with_h0=True, heads=None):
    d = to_dev(x)
    h0 = d["h0"] if with_h0 else None
    r = kda.kda_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], dout.cuda(), h0=h0,
                          dhT=None if dhT is None else dhT.cuda(), cu_seqlens=d["cu_seqlens"],
                          recurrent=True)
    torch.cuda.synchronize()
    ref = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], dout,
                          x["h0"] if with_h0 else None, dhT, x["cu_seqlens"], heads=heads)
    return r, ref


def _assert_close(r, ref, heads=None):
    for n in NAMES:
        if r[n] is None:
            continue
        got = r[n] if heads is None else (r[n][:, heads[0]:heads[1]] if n == "dh0"
                                          else r[n][:, :, heads[0]:heads[1]])
        e = rel_err(got, ref[n])
        assert e <= TOL_BWD, f"{n}: {e:.3e}"


@pytest.mark.parametrize("dtype,dk,dv,T", [("f32", 64, 64, 150), ("bf16", 128, 128, 200),
                                           ("bf16", 64, 128, 64), ("f32", 128, 64, 129),
                                           ("bf16", 64, 64, 1)])
def test_bwd_matches_oracle(dtype, dk, dv, T):
    spec = ki.PrefillSpec("bwd", B=2, T=T, H=3, dk=dk, dv=dv, dtype=dtype, decay="logsigmoid",
                          seed=T + dk, h0=True)
    x = ki.make_prefill(spec)
    dout, dhT = _cotangents(x, 5 + T, 2)
    r, ref = _run(x, dout, dhT)
    _assert_close(r, ref)


@pytest.mark.parametrize("with_h0,with_dhT", [(False, False), (False, True), (True, False)])
def test_bwd_optional_states(with_h0, with_dhT):
    spec = ki.PrefillSpec("bwd", B=1, T=97, H=2, dk=128, dv=128, dtype="bf16", decay="alog",
                          seed=11, h0=True)
    x = ki.make_prefill(spec)
    dout, dhT = _cotangents(x, 12, 1, with_dhT)
    r, ref = _run(x, dout, dhT, with_h0=with_h0)
    assert (r["dh0"] is None) == (not with_h0)
    _assert_close(r, ref)


def test_bwd_packed_documents_with_empty_and_ragged():
    """Packed documents (one empty, lengths not multiples of 64): gradients stay
    inside their document."""
    spec = ki.PrefillSpec("varlen", B=0, T=0, H=2, dk=128, dv=128, dtype="bf16", decay="alog",
                          seed=31, h0=True, varlen=True)
    x = ki.make_prefill(spec, doc_lens=[130, 0, 64, 257, 1])
    nseq = x["cu_seqlens"].numel() - 1
    dout, dhT = _cotangents(x, 32, nseq)
    r, ref = _run(x, dout, dhT)
    _assert_close(r, ref)
    # the empty document passes dhT straight to dh0
    assert torch.equal(r["dh0"][1].cpu(), dhT[1])


def test_bwd_zero_tokens():
    spec = ki.PrefillSpec("bwd", B=2, T=1, H=2, dk=64, dv=64, dtype="f32", decay="alog", seed=3,
                          h0=True)
    x = ki.make_prefill(spec)
    x = {n: (t[:, :0].contiguous() if isinstance(t, torch.Tensor) and n not in ("h0",)
             and t.dim() >= 3 else t) for n, t in x.items()}
    dout = torch.zeros((2, 0, 2, 64))
    dhT = torch.randn((2, 2, 64, 64))
    d = to_dev(x)
    r = kda.kda_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], dout.cuda(), h0=d["h0"],
                          dhT=dhT.cuda(), recurrent=True)
    torch.cuda.synchronize()
    assert torch.equal(r["dh0"].cpu(), dhT)


def test_bwd_long_sequence_sampled_heads():
    """The bench's backward workload shape (T = 8192, d = 128, bf16), two heads
    checked against the oracle."""
    spec = ki.PrefillSpec("bwd", B=1, T=8192, H=12, dk=128, dv=128, dtype="bf16",
                          decay="alog", seed=8192, h0=False)
    x = ki.make_prefill(spec)
    dout, dhT = _cotangents(x, 8193, 1)
    d = to_dev(x)
    r = kda.kda_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], dout.cuda(), dhT=dhT.cuda(),
                          recurrent=True)
    torch.cuda.synchronize()
    heads = (5, 7)
    ref = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], dout, None, dhT,
                          heads=heads)
    for n in ("dq", "dk", "dv", "dg", "dbeta"):
        e = rel_err(r[n][:, :, heads[0]:heads[1]], ref[n])
        assert e <= TOL_BWD, f"{n}: {e:.3e}"


def test_bwd_repeatable():
    spec = ki.PrefillSpec("bwd", B=1, T=300, H=2, dk=128, dv=128, dtype="bf16", decay="alog",
                          seed=41, h0=True)
    x = ki.make_prefill(spec)
    dout, dhT = _cotangents(x, 42, 1)
    d = to_dev(x)
    a = kda.kda_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], dout.cuda(), h0=d["h0"],
                          dhT=dhT.cuda(), recurrent=True)
    b = kda.kda_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], dout.cuda(), h0=d["h0"],
                          dhT=dhT.cuda(), recurrent=True)
    torch.cuda.synchronize()
    # dv and dh0 are column-local: reproducible bit for bit; dq, dk, dg and dbeta
    # sum per-warp parts in arrival order: equal up to fp32 rounding
    for n in ("dv", "dh0"):
        assert torch.equal(a[n], b[n]), n
    for n in ("dq", "dk", "dg", "dbeta"):
        assert rel_err(a[n], b[n].double().cpu().numpy()) <= 1e-6, n


@pytest.mark.parametrize("dtype,dk,dv,G", [("bf16", 128, 128, 64), ("bf16", 128, 128, 2),
                                           ("f32", 64, 64, 16), ("bf16", 64, 128, 64),
                                           ("f32", 128, 64, 4)])
def test_bwd_grouped_decay_matches_oracle(dtype, dk, dv, G):
    """One decay per group of G key channels: dg of a shared value is the sum of
    the per-channel gradients over its group (chain rule of the expansion)."""
    spec = ki.PrefillSpec("bwd", B=2, T=150, H=2, dk=dk, dv=dv, dtype=dtype, decay="alog",
                          seed=G + dk, h0=True)
    x = ki.make_prefill(spec)
    gg = x["g"][..., ::G].contiguous()
    dout, dhT = _cotangents(x, 61 + G, 2)
    d = to_dev(x)
    r = kda.kda_chunk_bwd(d["q"], d["k"], d["v"], gg.cuda(), d["beta"], dout.cuda(),
                          h0=d["h0"], dhT=dhT.cuda(), recurrent=True)
    torch.cuda.synchronize()
    ref = oracle.backward(x["q"], x["k"], x["v"], gg, x["beta"], dout, x["h0"], dhT)
    assert tuple(r["dg"].shape) == tuple(gg.shape)
    ref["dg"] = ref["dg"].reshape(*gg.shape, G).sum(-1)
    _assert_close(r, ref)


def test_bwd_grouped_packed_documents():
    spec = ki.PrefillSpec("varlen", B=0, T=0, H=2, dk=128, dv=128, dtype="bf16", decay="alog",
                          seed=71, h0=True, varlen=True)
    x = ki.make_prefill(spec, doc_lens=[100, 0, 64, 33])
    G = 64
    gg = x["g"][..., ::G].contiguous()
    nseq = x["cu_seqlens"].numel() - 1
    dout, dhT = _cotangents(x, 72, nseq)
    d = to_dev(x)
    r = kda.kda_chunk_bwd(d["q"], d["k"], d["v"], gg.cuda(), d["beta"], dout.cuda(),
                          h0=d["h0"], dhT=dhT.cuda(), cu_seqlens=d["cu_seqlens"], recurrent=True)
    torch.cuda.synchronize()
    ref = oracle.backward(x["q"], x["k"], x["v"], gg, x["beta"], dout, x["h0"], dhT,
                          x["cu_seqlens"])
    ref["dg"] = ref["dg"].reshape(*gg.shape, G).sum(-1)
    _assert_close(r, ref)
