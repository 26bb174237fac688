"""Failure detection on the GPU without a fault: the time-bounded wait every
kernel uses runs out on an mbarrier nothing arrives on, reports
SR_DEVERR_TIMEOUT after about its bound, and the context stays usable (a decode
step afterwards still matches the oracle)."""
from __future__ import annotations

import pytest
import torch

from kv_cache_routing_sr_b200 import inputs, native
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_reports():
    for limit_us in (20000, 200000):
        status, waited_ns = native.selftest_bounded_wait(limit_us)
        assert status == native.SR_DEVERR_TIMEOUT
        assert limit_us * 1000 <= waited_ns < limit_us * 1000 + 50_000_000  # the bound, plus at most 50 ms


def test_context_usable_after_a_timeout():
    native.selftest_bounded_wait(50000)
    x = inputs.make("tiny_4k", seed=61, device="cuda", max_ctx=2000)
    mask_g, act_g, out_g, dec = H.gpu_step(x)
    assert dec.workspace.device_error() == 0
    ref = H.oracle_full(x, x.tau)
    H.assert_route_equal(mask_g, act_g, ref.mask, ref.active_list)
    H.check_against_oracle(x, out_g, mask_g, what="after a bounded-wait timeout")
