"""kda_workspace_size (host only) against the workspace layout kda.h states:
forward -- 74,240 B of chunk record per (head, chunk slot), ceil(T/64) * B slots
(ceil(T/64) + B packed), plus 2 (4 with half points) x 64 KB per (segment slot,
head) when the prefill splits sequences (kda_prefill_plan); none for fp32 inputs.
backward -- in the chunked form (bf16, dk = dv = 128) 213,504 B per (chunk slot,
head): the 98,816-byte record (the forward's 74,240 B, T as an 8 KB bf16 image, A in
fp32) and the bf16 images of S, dS (32 KB each), Delta, and dDelta as a hi/lo pair
(16 KB each); otherwise (the
recurrent sweep) 4 dk dv B per (chunk slot + sequence, head) plus 64 x 4 dk dv B
per (sequence, head)."""
import math

import pytest

import gated_delta_rule_74_b200 as kda

REC = 74240


def _fwd_expected(B, T, H, packed, sms):
    nch = math.ceil(T / 64)
    slots = nch + B if packed else nch * B
    G, half = kda.kda_prefill_plan(B, T, H, packed, sms)
    seg = 0
    if G > 0 and math.ceil(nch / G) >= 2:
        P = math.ceil(nch / G)
        seg_slots = P + B if packed else B * P
        seg = (4 if half else 2) * seg_slots * H * 128 * 128 * 4
    return slots * H * REC + seg


@pytest.mark.parametrize("B,T,H,packed", [(1, 8192, 12, False), (16, 512, 8, False),
                                          (1, 32768, 96, False), (7, 16384, 12, True),
                                          (1, 4000, 2, False), (3, 0, 4, False), (2, 1, 1, True)])
@pytest.mark.parametrize("sms", [148, 132, 8])
def test_forward_size_matches_the_header(B, T, H, packed, sms):
    for dk, dv in ((128, 128), (64, 64), (64, 128)):
        got = kda.kda_workspace_size(kda.KDA_OP_CHUNK_FWD, B, T, H, dk, dv, packed=packed, sms=sms)
        assert got == _fwd_expected(B, T, H, packed, sms)


@pytest.mark.parametrize("B,T,H,packed", [(1, 8192, 12, False), (5, 300, 3, True), (2, 0, 1, False)])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (64, 64)])
def test_backward_size_matches_the_header(B, T, H, packed, dk, dv):
    nch = math.ceil(T / 64)
    slots = nch + B if packed else nch * B
    recurrent = ((slots + B) * H + B * H * 64) * dk * dv * 4
    chunked = slots * H * (74240 + 64 * 64 * 2 + 64 * 64 * 4 + 2 * 128 * 128 * 2
                           + 3 * 64 * 128 * 2)
    assert chunked == slots * H * 213504
    for dtype in (kda.KDA_BF16, kda.KDA_F32):
        got = kda.kda_workspace_size(kda.KDA_OP_CHUNK_BWD, B, T, H, dk, dv, packed=packed,
                                     dtype=dtype, sms=148)
        use_chunked = dtype == kda.KDA_BF16 and dk == dv == 128
        assert got == (chunked if use_chunked else recurrent)


def test_fp32_forward_needs_none():
    assert kda.kda_workspace_size(kda.KDA_OP_CHUNK_FWD, 4, 8192, 8, 64, 64,
                                  dtype=kda.KDA_F32, sms=148) == 0


@pytest.mark.parametrize("args,status", [
    ((2, 1, 64, 1, 128, 128), kda.KDA_ERR_INVALID_ARG),     # unknown op
    ((0, 0, 64, 1, 128, 128), kda.KDA_ERR_INVALID_ARG),     # B < 1
    ((0, 1, -1, 1, 128, 128), kda.KDA_ERR_INVALID_ARG),     # T < 0
    ((0, 1, 64, 0, 128, 128), kda.KDA_ERR_INVALID_ARG),     # H < 1
    ((0, 1, 64, 1, 96, 128), kda.KDA_ERR_UNSUPPORTED),      # head size
])
def test_invalid_arguments(args, status):
    with pytest.raises(kda.KdaError) as e:
        kda.kda_workspace_size(*args, sms=148)
    assert e.value.status == status
