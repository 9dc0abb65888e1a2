"""Bounded device-side waits: a wait that never completes gives up, raises the flag
kda_device_status reports, and leaves the device usable (no hang, no fault)."""
import pytest
import torch

import gated_delta_rule_74_b200 as kda
import kda_inputs as ki
from _helpers import TOL, gpu_prefill, oracle_prefill, rel_err

pytestmark = pytest.mark.gpu


def test_normal_calls_leave_no_timeout():
    kda.kda_device_status(reset=True)
    x = ki.make_prefill(ki.PrefillSpec("s", B=1, T=300, H=2, dk=128, dv=128, dtype="bf16",
                                       decay="alog", seed=3, h0=True))
    gpu_prefill(x)
    assert kda.kda_device_status(reset=False) == kda.KDA_OK


def test_expired_wait_is_reported_and_cleared():
    kda.kda_device_status(reset=True)
    kda.kda_selftest_bounded_wait(polls=1000)
    assert kda.kda_device_status(reset=False) == kda.KDA_ERR_TIMEOUT
    assert kda.kda_device_status(reset=True) == kda.KDA_ERR_TIMEOUT     # read, then cleared
    assert kda.kda_device_status(reset=False) == kda.KDA_OK
    # the device is still usable: a prefill afterwards matches the oracle
    x = ki.make_prefill(ki.PrefillSpec("s", B=1, T=200, H=2, dk=128, dv=128, dtype="bf16",
                                       decay="alog", seed=4, h0=True))
    out, hT = gpu_prefill(x)
    o_ref, s_ref = oracle_prefill(x)
    assert rel_err(out, o_ref) <= TOL["bf16"] and rel_err(hT, s_ref) <= TOL["bf16"]
    assert kda.kda_device_status(reset=False) == kda.KDA_OK
