"""The failure-detection contract on the device: a bounded wait that runs
out records MOE_ERR_TIMEOUT, returns, and leaves the context usable.

The wait is made to run out by an mbarrier that nothing arrives on (1 ms
limit); no copy, MMA or other kernel waits on it, so nothing faults or
hangs.  The header promises the status; this test produces it."""
import numpy as np
import pytest
import torch

from mixture_experts_routing_top_b200 import libmoe as M, synth
from oracle import oracle as O
from tests.helpers import needs_gpu, to_dev, to_np

pytestmark = [pytest.mark.gpu, needs_gpu]

MOE_ERR_TIMEOUT = 7


def test_expired_wait_reports_timeout_and_the_context_stays_usable():
    assert M.device_error() == 0                              # start from a clean word
    r = to_np(M.selftest_bounded_wait(False, 1_000_000))      # nothing arrives; 1 ms limit
    assert r[0] == 0                                          # the wait gave up ...
    assert 1000 <= r[1] < 1_000_000                           # ... after its limit, well inside a second
    assert M.device_error(clear=False) == MOE_ERR_TIMEOUT     # recorded, still set
    assert M.device_error() == MOE_ERR_TIMEOUT                # read and cleared
    assert M.device_error() == 0                              # clean again
    # the control: the barrier completed first, the same wait returns at once
    r = to_np(M.selftest_bounded_wait(True, 1_000_000))
    assert r[0] == 1 and r[1] < 1000
    assert M.device_error() == 0
    # a normal call afterwards runs and is right
    logits = synth.normal_f32(3, 1, (500, 16))
    idx, gate = M.route_topk(to_dev(logits), 4)
    want_idx, want_gate = O.route_topk(logits, 4)
    assert np.array_equal(to_np(idx), want_idx)
    np.testing.assert_allclose(to_np(gate), want_gate, rtol=1e-6)
    assert M.device_error() == 0
