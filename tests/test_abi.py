"""The C-ABI library loads, exports every declared symbol and validates its
arguments on the host.  No test here launches GPU work: each call carries at
least one invalid argument, so the library returns before touching CUDA."""
import ctypes

import pytest

import gated_delta_rule_74_b200 as kda


@pytest.fixture(scope="module")
def L():
    from gated_delta_rule_74_b200 import build
    build.build()
    return kda.lib()


def test_exports_every_declared_symbol(L):
    names = kda.header_symbols()
    assert set(names) >= {"kda_chunk_fwd", "kda_decode_step", "kda_status_string", "kda_version"}
    for n in names:
        assert hasattr(L, n), f"libkda.so does not export {n}"


def test_status_strings_and_version(L):
    assert kda.kda_status_string(0) == "KDA_OK"
    assert kda.kda_status_string(-1) == "KDA_ERR_INVALID_ARG"
    assert kda.kda_status_string(-2) == "KDA_ERR_UNSUPPORTED"
    assert kda.kda_status_string(-3) == "KDA_ERR_CUDA"
    assert kda.kda_status_string(-4) == "KDA_ERR_TIMEOUT"
    assert kda.kda_status_string(12345) == "KDA_ERR_UNKNOWN"
    assert kda.kda_version() >= 1


P = 0x10000   # a 16-byte aligned fake address; never dereferenced by these calls


def _chunk(L, q=P, k=P, v=P, g=P, beta=P, h0=None, cu=None, out=P, hT=None,
           B=1, T=64, H=2, dk=64, dv=64, dt=0):
    return L.kda_chunk_fwd(q, k, v, g, beta, h0, cu, out, hT, B, T, H, dk, dv, dt, None)


def _decode(L, q=P, k=P, v=P, g=P, beta=P, S=P, out=P, N=1, H=1, dk=64, dv=64, dt=0):
    return L.kda_decode_step(q, k, v, g, beta, S, out, N, H, dk, dv, dt, None)


@pytest.mark.parametrize("bad", [dict(q=None), dict(k=None), dict(v=None), dict(g=None),
                                 dict(beta=None), dict(out=None), dict(q=P + 4),
                                 dict(h0=P + 8), dict(hT=P + 2), dict(cu=P + 4),
                                 dict(B=0), dict(T=-1), dict(H=0), dict(dt=7)])
def test_chunk_fwd_rejects_invalid(L, bad):
    assert _chunk(L, **bad) == kda.KDA_ERR_INVALID_ARG


@pytest.mark.parametrize("dims", [dict(dk=32), dict(dv=96), dict(dk=256, dv=256)])
def test_chunk_fwd_rejects_unsupported_heads(L, dims):
    assert _chunk(L, **dims) == kda.KDA_ERR_UNSUPPORTED


@pytest.mark.parametrize("bad", [dict(q=None), dict(S=None), dict(out=None), dict(S=P + 4),
                                 dict(N=0), dict(H=0), dict(dt=-1)])
def test_decode_rejects_invalid(L, bad):
    assert _decode(L, **bad) == kda.KDA_ERR_INVALID_ARG


def test_decode_rejects_unsupported_heads(L):
    assert _decode(L, dk=48) == kda.KDA_ERR_UNSUPPORTED


def test_binding_rejects_cpu_tensors(L):
    import torch
    x = torch.zeros(1, 4, 1, 64)
    with pytest.raises(ValueError):
        kda.kda_chunk_fwd(x, x, x, x, torch.zeros(1, 4, 1))


def _tokens(L, q=P, k=P, v=P, g=P, beta=P, S=P, out=P, N=1, Lt=4, H=1, dk=64, dv=64, dt=0):
    return L.kda_decode_tokens(q, k, v, g, beta, S, out, N, Lt, H, dk, dv, dt, None)


@pytest.mark.parametrize("bad", [dict(q=None), dict(g=None), dict(S=None), dict(out=P + 4),
                                 dict(N=0), dict(Lt=0), dict(Lt=-3), dict(H=0), dict(dt=3)])
def test_decode_tokens_rejects_invalid(L, bad):
    assert _tokens(L, **bad) == kda.KDA_ERR_INVALID_ARG


def test_decode_tokens_rejects_unsupported_heads(L):
    assert _tokens(L, dv=80) == kda.KDA_ERR_UNSUPPORTED


@pytest.mark.parametrize("G", [0, 3, 96, 256])
def test_grouped_rejects_bad_group(L, G):
    assert L.kda_chunk_fwd_grouped(P, P, P, P, P, None, None, P, None, 1, 4, 1, 128, 128, G, 0,
                                   None) == kda.KDA_ERR_INVALID_ARG
    assert L.kda_decode_tokens_grouped(P, P, P, P, P, P, P, 1, 2, 1, 128, 128, G, 0,
                                       None) == kda.KDA_ERR_INVALID_ARG


def _bwd(L, q=P, k=P, v=P, g=P, beta=P, h0=None, cu=None, dout=P, dhT=None, dq=P, dk_=P,
         dv_=P, dg=P, dbeta=P, dh0=None, B=1, T=64, H=2, dk=64, dv=64, dt=0):
    return L.kda_chunk_bwd(q, k, v, g, beta, h0, cu, dout, dhT, dq, dk_, dv_, dg, dbeta, dh0,
                           B, T, H, dk, dv, dt, None)


@pytest.mark.parametrize("bad", [dict(q=None), dict(dout=None), dict(dq=None), dict(dk_=None),
                                 dict(dv_=None), dict(dg=None), dict(dbeta=None),
                                 dict(dout=P + 4), dict(dhT=P + 8), dict(dh0=P + 2),
                                 dict(B=0), dict(T=-1), dict(H=0), dict(dt=5)])
def test_chunk_bwd_rejects_invalid(L, bad):
    assert _bwd(L, **bad) == kda.KDA_ERR_INVALID_ARG


@pytest.mark.parametrize("dims", [dict(dk=32), dict(dv=96)])
def test_chunk_bwd_rejects_unsupported_heads(L, dims):
    assert _bwd(L, **dims) == kda.KDA_ERR_UNSUPPORTED


def _fused(L, qr=P, kr=P, v=P, cq=P, ck=P, W=4, g=P, beta=P, gate=None, h0=None, cu=None,
           out=P, hT=None, B=1, T=64, H=2, dk=128, dv=128, dt=0):
    return L.kda_chunk_fwd_fused(qr, kr, v, cq, ck, W, g, beta, gate, h0, cu, out, hT,
                                 B, T, H, dk, dv, dt, None)


@pytest.mark.parametrize("bad", [dict(qr=None), dict(v=None), dict(out=None), dict(cq=None),
                                 dict(ck=None), dict(W=0), dict(W=5), dict(gate=P + 4),
                                 dict(cq=P + 4), dict(B=0), dict(H=0), dict(dt=2)])
def test_chunk_fwd_fused_rejects_invalid(L, bad):
    assert _fused(L, **bad) == kda.KDA_ERR_INVALID_ARG


@pytest.mark.parametrize("dims", [dict(dk=32), dict(dt=1)])
def test_chunk_fwd_fused_rejects_unsupported(L, dims):
    assert _fused(L, **dims) == kda.KDA_ERR_UNSUPPORTED


@pytest.mark.parametrize("G", [0, 3, 96, 256])
def test_bwd_grouped_rejects_bad_group(L, G):
    assert L.kda_chunk_bwd_grouped(P, P, P, P, P, None, None, P, None, P, P, P, P, P, None,
                                   1, 4, 1, 128, 128, G, 0, None) == kda.KDA_ERR_INVALID_ARG


@pytest.mark.parametrize("polls", [0, (1 << 20) + 1])
def test_selftest_rejects_poll_counts(L, polls):
    assert L.kda_selftest_bounded_wait(polls, None) == kda.KDA_ERR_INVALID_ARG


def _dchunk(L_, q=P, S=P, out=P, N=1, Lt=4, H=1, dk=128, dv=128, dt=0):
    return L_.kda_decode_chunk(q, P, P, P, P, S, out, N, Lt, H, dk, dv, dt, None)


@pytest.mark.parametrize("bad", [dict(q=None), dict(S=None), dict(out=P + 4), dict(N=0),
                                 dict(Lt=0), dict(H=0), dict(dt=4)])
def test_decode_chunk_rejects_invalid(L, bad):
    assert _dchunk(L, **bad) == kda.KDA_ERR_INVALID_ARG


@pytest.mark.parametrize("dims", [dict(Lt=17), dict(dk=64), dict(dv=64), dict(dt=1)])
def test_decode_chunk_rejects_unsupported(L, dims):
    assert _dchunk(L, **dims) == kda.KDA_ERR_UNSUPPORTED
