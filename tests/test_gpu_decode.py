"""GPU parity of kda_decode_step against the float64 oracle."""
import numpy as np
import pytest
import torch

import kda_inputs as ki
import oracle
from _helpers import TOL, rel_err

pytestmark = pytest.mark.gpu


def _run_steps(d, steps, sample=None):
    import gated_delta_rule_74_b200 as kda
    S = d["S0"].cuda()
    outs = []
    for t in range(steps):
        o = kda.kda_decode_step(d["q"][t].cuda(), d["k"][t].cuda(), d["v"][t].cuda(),
                                d["g"][t].cuda(), d["beta"][t].cuda(), S)
        outs.append(o if sample is None else o.reshape(-1, o.shape[-1])[sample])
    torch.cuda.synchronize()
    return outs, S


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
def test_decode_small(dtype, dk, dv):
    spec = ki.DecodeSpec("t", N=5, H=3, dk=dk, dv=dv, steps=4, dtype=dtype, decay="alog", seed=7)
    d = ki.make_decode(spec)
    outs, S = _run_steps(d, 4)
    S_ref = d["S0"]
    for t in range(4):
        o_ref, S_ref = oracle.decode(d["q"][t], d["k"][t], d["v"][t], d["g"][t], d["beta"][t], S_ref)
        assert rel_err(outs[t], o_ref) <= TOL[dtype], t
    assert rel_err(S, S_ref) <= TOL[dtype]


def test_decode_cfg4_sampled():
    """Full config-4 shape (N=256, H=96, d=128, 16 consecutive tokens, 1.61 GB of
    fp32 state) on the GPU; the oracle checks 96 sampled (n, h) pairs."""
    d = ki.make_decode("cfg4")
    N, H = d["N"], d["H"]
    rng = np.random.default_rng(0)
    pairs = np.sort(rng.choice(N * H, size=96, replace=False))
    outs, S = _run_steps(d, d["steps"], sample=torch.from_numpy(pairs).cuda())
    flat = lambda t: t.reshape(-1, *t.shape[2:])[pairs][:, None]   # [P, 1, ...]
    S_ref = d["S0"].reshape(N * H, 128, 128)[pairs][:, None]
    for t in range(d["steps"]):
        o_ref, S_ref = oracle.decode(flat(d["q"][t]), flat(d["k"][t]), flat(d["v"][t]),
                                     flat(d["g"][t]), d["beta"][t].reshape(-1)[pairs][:, None],
                                     S_ref)
        assert rel_err(outs[t], o_ref[:, 0]) <= TOL["bf16"], t
    S_got = S.reshape(N * H, 128, 128)[torch.from_numpy(pairs).cuda()]
    assert rel_err(S_got, S_ref[:, 0]) <= TOL["bf16"]
