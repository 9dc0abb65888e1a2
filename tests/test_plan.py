"""The split prefill's planner (host logic, no GPU): which segment length G and which
half point Gh kda_chunk_fwd takes for a shape, through kda_prefill_plan.  The shapes
pinned here are the ones the GPU tests rely on to reach each path."""
import math

import pytest

import gated_delta_rule_74_b200 as kda


@pytest.mark.parametrize("B,T,H,expect", [
    (1, 8192, 12, (20, 10)),      # headline shape: 7 segments of 20 chunks, halves of 10
    (1, 4100, 2, (10, 5)),        # GPU test_split_half_points
    (1, 8000, 2, (12, 6)),
    (1, 20000, 2, (22, 11)),
    (1, 131072, 1, (58, 29)),     # GPU test_split_long_sequences
    (1, 32768, 96, (0, 0)),       # 96 chains already fill most of 148 SMs: one chain each
    (16, 512, 8, (0, 0)),         # 8 chunks per sequence: not worth splitting
    (1, 1300, 2, (6, 3)),
    (1, 1000, 2, (4, 0)),         # split without half points (GPU graph test)
    (2, 1000, 2, (4, 0)),         # GPU test_split_fixed_length
])
def test_pinned_plans(B, T, H, expect):
    assert kda.kda_prefill_plan(B, T, H, sms=148) == expect


def _check(B, T, H, sms, packed):
    G, half = kda.kda_prefill_plan(B, T, H, packed=packed, sms=sms)
    nch = math.ceil(T / 64)
    NH = B * H
    assert G >= 0 and half >= 0
    if G == 0:
        assert half == 0
        return
    P = math.ceil(nch / G)
    assert P >= 2 and G < nch
    assert NH < sms                              # split only when (sequence, head) pairs are few
    if packed:                                   # packed documents: fixed 16-chunk segments
        assert (G, half) == (16, 0)
        return
    assert P <= 64
    if half:
        assert P >= 3 and half == (G + 1) // 2
        # pass C's longest chain is a half segment or the last segment
        last = nch - (P - 1) * G
        assert 1 <= last <= G
    # at most two waves of pass A chains: beyond that the split costs more than it saves
    assert NH * (2 * P - 3) <= 2 * sms


@pytest.mark.parametrize("sms", [148, 132])
def test_plan_invariants(sms):
    for B in (1, 2, 4):
        for H in (1, 2, 4, 8, 12, 16, 48, 96, 160):
            for T in (0, 64, 511, 512, 513, 4096, 8192, 8193, 32768, 100000):
                _check(B, T, H, sms, packed=False)
                _check(B, T, H, sms, packed=True)


def test_rejects_bad_arguments():
    with pytest.raises(kda.KdaError):
        kda.kda_prefill_plan(0, 64, 1)
    with pytest.raises(kda.KdaError):
        kda.kda_prefill_plan(1, -1, 1)
    with pytest.raises(kda.KdaError):
        kda.kda_prefill_plan(1, 64, 1, sms=0)
