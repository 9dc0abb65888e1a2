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
