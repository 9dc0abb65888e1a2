"""kda_chunk_fwd_noalloc: the prefill for callers that cannot allocate device
memory (code that runs under a fixed memory budget or inside captured graphs,
embedders that only hand over pre-sized buffers).  It must give the same
results as kda_chunk_fwd, call after call, using only its fixed in-library
scratch array.  Collected last on purpose: it runs after every other test and
must also pass alone in a fresh process."""
import ctypes

import pytest
import torch

import gated_delta_rule_74_b200 as kda
import kda_inputs as ki
import oracle
from _helpers import TOL, rel_err, to_dev

pytestmark = pytest.mark.gpu


def _noalloc():
    L = kda.lib()
    fn = L.kda_chunk_fwd_noalloc
    vp, ip = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [vp] * 9 + [ip] * 6 + [vp]
    fn.restype = ctypes.c_int
    return fn


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _call_noalloc(d, out, hT, dtype=None):
    nseq = d["B"]
    dt = kda.KDA_BF16 if dtype in (None, "bf16") else kda.KDA_F32
    rc = _noalloc()(_ptr(d["q"]), _ptr(d["k"]), _ptr(d["v"]), _ptr(d["g"]), _ptr(d["beta"]),
                    _ptr(d["h0"]), _ptr(d["cu_seqlens"]), _ptr(out), _ptr(hT),
                    nseq, d["T"], d["H"], d["dk"], d["dv"], dt,
                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc


@pytest.mark.parametrize("shape", ["fixed", "packed"])
def test_noalloc_matches_chunk_fwd_twice(shape):
    if shape == "fixed":
        # B*H = 6 with 64 chunks: the call is split into segments (uses scratch)
        x = ki.make_prefill("t8k_h12", H=6, T=4096)
    else:
        spec = ki.PrefillSpec("varlen", B=0, T=0, H=3, dk=128, dv=128, dtype="bf16",
                              decay="alog", seed=12, h0=True, varlen=True)
        x = ki.make_prefill(spec, doc_lens=[2600, 300, 1500])
    d = to_dev(x)
    ref_out, ref_hT = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], h0=d["h0"],
                                        cu_seqlens=d["cu_seqlens"])
    for _ in range(2):                                   # two calls in a row
        out = torch.full_like(ref_out, float("nan"))
        hT = torch.full_like(ref_hT, float("nan"))
        assert _call_noalloc(d, out, hT) == kda.KDA_OK
        torch.cuda.synchronize()
        assert rel_err(out, ref_out.double().cpu().numpy()) <= TOL["bf16"]
        assert rel_err(hT, ref_hT.double().cpu().numpy()) <= TOL["bf16"]
    # and against the float64 oracle directly, on the same inputs
    o_ref, s_ref = oracle.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"],
                                  x["cu_seqlens"])
    assert rel_err(out, o_ref) <= TOL["bf16"]
    assert rel_err(hT, s_ref) <= TOL["bf16"]


@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 64, 64), ("f32", 64, 64), ("f32", 128, 128),
                                         ("bf16", 128, 64)])
def test_noalloc_other_shapes_match_oracle(dtype, dk, dv):
    """64-wide heads and fp32 inputs run on the CUDA-core path (no scratch at all)."""
    spec = ki.PrefillSpec("na", B=2, T=200, H=3, dk=dk, dv=dv, dtype=dtype, decay="alog",
                          seed=dk + dv, h0=True)
    x = ki.make_prefill(spec)
    d = to_dev(x)
    for _ in range(2):
        out = torch.full_like(d["v"], float("nan"))
        hT = torch.full_like(d["h0"], float("nan"))
        assert _call_noalloc(d, out, hT, dtype) == kda.KDA_OK
        torch.cuda.synchronize()
        o_ref, s_ref = oracle.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"])
        assert rel_err(out, o_ref) <= TOL[dtype]
        assert rel_err(hT, s_ref) <= TOL[dtype]


def test_noalloc_empty_sequence_without_hT():
    """T = 0 with no final state: nothing to write, and the call succeeds."""
    spec = ki.PrefillSpec("na0", B=2, T=0, H=2, dk=128, dv=128, dtype="bf16", decay="alog",
                          seed=3, h0=True)
    d = to_dev(ki.make_prefill(spec))
    out = torch.empty_like(d["v"])
    assert _call_noalloc(d, out, None) == kda.KDA_OK
    torch.cuda.synchronize()


def test_noalloc_rejects_scratch_beyond_its_array():
    """One 16384-token document with H = 32 would need 2 * 17 * 32 * 64 KB of
    segment scratch, more than the fixed array holds: rejected, nothing run."""
    T, H = 16384, 32
    z = lambda *s, dt=torch.bfloat16: torch.zeros(*s, dtype=dt, device="cuda")
    d = dict(q=z(1, T, H, 128), k=z(1, T, H, 128), v=z(1, T, H, 128),
             g=z(1, T, H, 128, dt=torch.float32), beta=z(1, T, H, dt=torch.float32), h0=None,
             cu_seqlens=torch.tensor([0, T], dtype=torch.int32, device="cuda"),
             B=1, T=T, H=H, dk=128, dv=128)
    out = torch.full((1, T, H, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    assert _call_noalloc(d, out, None) == kda.KDA_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())
