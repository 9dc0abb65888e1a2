"""The C ABI's calls inside captured CUDA graphs.  The split prefill takes its scratch
with stream-ordered allocation from a private pool and launches its kernels with
programmatic stream serialization (each may start while its predecessor drains); a
captured call must replay to exactly the results of the same call made eagerly, and a
replay after the inputs change in place must follow the new inputs."""
import pytest
import torch

import gated_delta_rule_74_b200 as kda
import kda_inputs as ki
from _helpers import to_dev

pytestmark = pytest.mark.gpu


def _capture(fn):
    """Warm `fn` up on a side stream, then capture it into a graph (torch's recipe)."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


@pytest.mark.parametrize("T,decay", [(4100, "logsigmoid"), (1000, "alog")])
def test_prefill_graph_replay_matches_eager(T, decay):
    """B=1, H=2: T = 4100 runs the segment split with half points (pass A, combine, pass C
    in two chains per middle segment), T = 1000 the split without them (tests/test_plan.py
    pins both plans)."""
    x = ki.make_prefill(ki.PrefillSpec("graph", B=1, T=T, H=2, dk=128, dv=128, dtype="bf16",
                                       decay=decay, seed=T, h0=True))
    d = to_dev(x)
    args = (d["q"], d["k"], d["v"], d["g"], d["beta"])
    out_e, hT_e = kda.kda_chunk_fwd(*args, h0=d["h0"])
    torch.cuda.synchronize()
    out, hT = torch.empty_like(out_e), torch.empty_like(hT_e)
    g = _capture(lambda: kda.kda_chunk_fwd(*args, h0=d["h0"], out=out, hT=hT))
    for _ in range(2):
        out.zero_()
        hT.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, out_e) and torch.equal(hT, hT_e)
    # new inputs in the captured buffers: the replay follows them
    x2 = ki.make_prefill(ki.PrefillSpec("graph", B=1, T=T, H=2, dk=128, dv=128, dtype="bf16",
                                        decay=decay, seed=T + 1, h0=True))
    d2 = to_dev(x2)
    for n in ("q", "k", "v", "g", "beta", "h0"):
        d[n].copy_(d2[n])
    out2_e, hT2_e = kda.kda_chunk_fwd(d2["q"], d2["k"], d2["v"], d2["g"], d2["beta"], h0=d2["h0"])
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, out2_e) and torch.equal(hT, hT2_e)


def test_decode_chunk_graph_replay_matches_eager():
    dd = ki.make_decode(ki.DecodeSpec("graph", N=8, H=4, dk=128, dv=128, steps=16, dtype="bf16",
                                      decay="alog", seed=9))
    x = {n: dd[n].transpose(0, 1).contiguous().cuda() for n in ("q", "k", "v", "g", "beta")}
    S0 = dd["S0"].cuda()
    S_e = S0.clone()
    out_e = kda.kda_decode_chunk(x["q"], x["k"], x["v"], x["g"], x["beta"], S_e)
    torch.cuda.synchronize()
    S = S0.clone()
    out = torch.empty_like(out_e)
    g = _capture(lambda: kda.kda_decode_chunk(x["q"], x["k"], x["v"], x["g"], x["beta"], S,
                                              out=out))
    S.copy_(S0)                 # the warm-up and the capture ran once on S already
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, out_e) and torch.equal(S, S_e)


@pytest.mark.parametrize("packed", [False, True])
def test_backward_graph_replay_matches_eager(packed):
    """The chunked backward (its prep, chain and gradient launches under programmatic
    stream serialization, scratch from the stream-ordered pool) captured into a graph:
    dq, dk, dv and dh0 replay bit for bit, dg and dbeta (shared-memory atomics) to fp32
    rounding, and a replay after the cotangent changes in place follows it."""
    if packed:
        spec = ki.PrefillSpec("varlen", B=0, T=0, H=2, dk=128, dv=128, dtype="bf16",
                              decay="alog", seed=51, h0=True, varlen=True)
        x = ki.make_prefill(spec, doc_lens=[300, 65, 1, 200])
    else:
        x = ki.make_prefill(ki.PrefillSpec("graph", B=2, T=700, H=2, dk=128, dv=128,
                                           dtype="bf16", decay="logsigmoid", seed=52, h0=True))
    d = to_dev(x)
    nseq = d["h0"].shape[0]
    gen = torch.Generator().manual_seed(53)
    dout = torch.randn(d["v"].shape, generator=gen).to(torch.bfloat16).cuda()
    dhT = (0.1 * torch.randn((nseq, 2, 128, 128), generator=gen)).cuda()

    def call(grads=None):
        return kda.kda_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], dout, h0=d["h0"],
                                 dhT=dhT, cu_seqlens=d["cu_seqlens"], grads=grads)

    eager = call()
    torch.cuda.synchronize()
    grads = {n: torch.empty_like(t) for n, t in eager.items() if t is not None}
    g = _capture(lambda: call(grads))

    def check(ref):
        for n in ("dq", "dk", "dv", "dh0"):
            assert torch.equal(grads[n], ref[n]), n
        for n in ("dg", "dbeta"):
            torch.testing.assert_close(grads[n], ref[n], rtol=1e-5, atol=1e-6)

    for _ in range(2):
        for t in grads.values():
            t.zero_()
        g.replay()
        torch.cuda.synchronize()
        check(eager)
    dout.copy_(torch.randn(dout.shape, generator=gen).to(torch.bfloat16).cuda())
    eager2 = call()
    g.replay()
    torch.cuda.synchronize()
    check(eager2)
