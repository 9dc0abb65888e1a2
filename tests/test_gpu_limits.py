"""Large and extreme sizes against the oracle: thousands of packed documents (many
empty or a single token), one very long sequence (the segmented state pass at its
largest segment count), and a decode step over hundreds of thousands of (sequence,
head) pairs, checked on a sample."""
import numpy as np
import pytest
import torch

import gated_delta_rule_74_b200 as kda
import kda_inputs as ki
import oracle
from _helpers import TOL, gpu_prefill, oracle_prefill, rel_err

pytestmark = pytest.mark.gpu


def test_thousands_of_tiny_documents():
    rng = np.random.default_rng(5)
    lens = [int(x) for x in rng.integers(0, 21, 3000)]        # includes empty documents
    spec = ki.PrefillSpec("varlen", B=0, T=0, H=2, dk=128, dv=128, dtype="bf16",
                          decay="alog", seed=51, h0=True, varlen=True)
    x = ki.make_prefill(spec, doc_lens=lens)
    out, hT = gpu_prefill(x)
    o_ref, s_ref = oracle_prefill(x)
    assert rel_err(out, o_ref) <= TOL["bf16"]
    assert rel_err(hT, s_ref) <= TOL["bf16"]


def test_one_very_long_sequence():
    """T = 131072, one head of 64: 2048 chunks, the state pass split into segments."""
    spec = ki.PrefillSpec("long", B=1, T=131072, H=1, dk=64, dv=64, dtype="bf16",
                          decay="alog", seed=52, h0=True)
    x = ki.make_prefill(spec)
    out, hT = gpu_prefill(x)
    o_ref, s_ref = oracle_prefill(x)
    assert rel_err(out, o_ref) <= TOL["bf16"]
    assert rel_err(hT, s_ref) <= TOL["bf16"]


def test_decode_step_many_pairs_sampled():
    """N x H = 200,000 state pairs in one kda_decode_step; 2,000 sampled pairs checked."""
    N, H, d = 50000, 4, 64
    dd = ki.make_decode(ki.DecodeSpec("big", N=N, H=H, dk=d, dv=d, steps=1, dtype="bf16",
                                      decay="alog", seed=53))
    S = dd["S0"].cuda()
    o = kda.kda_decode_step(dd["q"][0].cuda(), dd["k"][0].cuda(), dd["v"][0].cuda(),
                            dd["g"][0].cuda(), dd["beta"][0].cuda(), S)
    torch.cuda.synchronize()
    idx = torch.tensor(np.random.default_rng(54).choice(N, 500, replace=False))
    pick = lambda t: t[idx]
    o_ref, S_ref = oracle.decode(pick(dd["q"][0]), pick(dd["k"][0]), pick(dd["v"][0]),
                                 pick(dd["g"][0]), pick(dd["beta"][0]), pick(dd["S0"]))
    assert rel_err(o[idx.cuda()], o_ref) <= TOL["bf16"]
    assert rel_err(S[idx.cuda()], S_ref) <= TOL["bf16"]
