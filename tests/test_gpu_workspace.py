"""kda_chunk_fwd_ws / kda_chunk_bwd_ws: the prefill and its backward on workspace the
caller allocates (here with torch), matched against the float64 oracle, with the
library's own memory pool left untouched (kda_pool_usage's high-water mark stays
at zero), and too-small or misaligned workspace rejected with nothing launched."""
import pytest
import torch

import gated_delta_rule_74_b200 as kda
import kda_inputs as ki
import oracle
from _helpers import TOL, rel_err, to_dev

pytestmark = pytest.mark.gpu


def _ws(nbytes):
    # torch's caching allocator hands out 512-byte aligned blocks
    return torch.empty(max(nbytes, 1), dtype=torch.uint8, device="cuda")


def _fwd_case(name):
    if name == "headline_shape":
        return ki.make_prefill("t8k_h12")
    if name == "segmented":
        return ki.make_prefill(ki.PrefillSpec("ws", B=1, T=4000, H=2, dk=128, dv=128, dtype="bf16",
                                              decay="alog", seed=21, h0=True))
    if name == "packed":
        spec = ki.PrefillSpec("ws", B=0, T=0, H=3, dk=128, dv=128, dtype="bf16", decay="alog",
                              seed=22, h0=True, varlen=True)
        return ki.make_prefill(spec, doc_lens=[700, 3, 0, 1300])
    if name == "d64":
        return ki.make_prefill("b16_t512_d64")
    return ki.make_prefill("fp32_t256")


@pytest.mark.parametrize("name", ["headline_shape", "segmented", "packed", "d64", "fp32"])
def test_forward_on_caller_workspace(name):
    x = _fwd_case(name)
    d = to_dev(x)
    packed = x["cu_seqlens"] is not None
    dt = kda.KDA_BF16 if x["dtype"] == "bf16" else kda.KDA_F32
    need = kda.kda_workspace_size(kda.KDA_OP_CHUNK_FWD, x["B"], x["T"], x["H"], x["dk"], x["dv"],
                                  packed=packed, dtype=dt)
    ws = _ws(need) if need else None
    torch.cuda.synchronize()
    kda.kda_pool_usage(reset=True)
    for _ in range(2):
        out, hT = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], h0=d["h0"],
                                    cu_seqlens=d["cu_seqlens"], workspace=ws)
        torch.cuda.synchronize()
    assert kda.kda_pool_usage() == 0
    o_ref, s_ref = oracle.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"],
                                  x["cu_seqlens"])
    assert rel_err(out, o_ref) <= TOL[x["dtype"]]
    assert rel_err(hT, s_ref) <= TOL[x["dtype"]]
    # the same call without a workspace takes its scratch from the pool (bf16 only)
    kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], h0=d["h0"],
                      cu_seqlens=d["cu_seqlens"])
    torch.cuda.synchronize()
    assert (kda.kda_pool_usage() > 0) == (need > 0)


def test_grouped_decay_on_caller_workspace():
    x = ki.make_prefill(ki.PrefillSpec("wsg", B=2, T=300, H=3, dk=128, dv=128, dtype="bf16",
                                       decay="alog", seed=23, h0=True))
    gc = x["g"].view(2, 300, 3, 2, 64)[..., 0].contiguous()
    d = to_dev(x)
    need = kda.kda_workspace_size(kda.KDA_OP_CHUNK_FWD, 2, 300, 3, 128, 128)
    ws = _ws(need)
    kda.kda_pool_usage(reset=True)
    out, hT = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], gc.cuda(), d["beta"], h0=d["h0"],
                                workspace=ws)
    torch.cuda.synchronize()
    assert kda.kda_pool_usage() == 0
    g_full = gc.repeat_interleave(64, dim=-1).contiguous()
    o_ref, s_ref = oracle.prefill(x["q"], x["k"], x["v"], g_full, x["beta"], x["h0"])
    assert rel_err(out, o_ref) <= TOL["bf16"]
    assert rel_err(hT, s_ref) <= TOL["bf16"]


def test_too_small_or_misaligned_workspace_is_rejected():
    x = _fwd_case("segmented")
    d = to_dev(x)
    need = kda.kda_workspace_size(kda.KDA_OP_CHUNK_FWD, 1, 4000, 2, 128, 128)
    out = torch.full_like(d["v"], 3.0)
    for ws in (_ws(need - 16), _ws(need + 256)[16:]):
        with pytest.raises(kda.KdaError) as e:
            kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], h0=d["h0"], out=out,
                              workspace=ws)
        assert e.value.status == kda.KDA_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert bool((out == 3.0).all())


@pytest.mark.parametrize("dtype,packed", [("bf16", False), ("bf16", True), ("f32", True)])
def test_backward_on_caller_workspace(dtype, packed):
    """bf16 runs the chunked form (bf16 bound), fp32 the recurrent sweep (fp32 bound)."""
    spec = ki.PrefillSpec("wsb", B=0 if packed else 2, T=0 if packed else 200, H=2, dk=128,
                          dv=128, dtype=dtype, decay="alog", seed=24, h0=True, varlen=packed)
    x = ki.make_prefill(spec, doc_lens=[150, 2, 90] if packed else None)
    gen = torch.Generator().manual_seed(24)
    dout = torch.randn(x["v"].shape, generator=gen).to(x["v"].dtype)
    dhT = torch.randn(x["h0"].shape, generator=gen) * 0.1
    d = to_dev(x)
    dt = kda.KDA_BF16 if dtype == "bf16" else kda.KDA_F32
    need = kda.kda_workspace_size(kda.KDA_OP_CHUNK_BWD, x["B"], x["T"], 2, 128, 128,
                                  packed=packed, dtype=dt)
    ws = _ws(need)
    torch.cuda.synchronize()
    kda.kda_pool_usage(reset=True)
    r = kda.kda_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], dout.cuda(), h0=d["h0"],
                          dhT=dhT.cuda(), cu_seqlens=d["cu_seqlens"], workspace=ws)
    torch.cuda.synchronize()
    assert kda.kda_pool_usage() == 0
    ref = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], dout, x["h0"], dhT,
                          x["cu_seqlens"])
    tol = TOL["bf16"] if dtype == "bf16" else 1e-4
    for n in ("dq", "dk", "dv", "dg", "dbeta", "dh0"):
        assert rel_err(r[n], ref[n]) <= tol, n
