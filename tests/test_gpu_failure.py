"""Failure detection on the GPU without a fault: a device-side wait that runs
out reports DROPKV_ERR_TIMEOUT through the status word and leaves the context
usable.

The self-test kernel waits on an mbarrier that nothing arrives on, with the
same bounded wait (a %globaltimer limit) that the scoring and select kernels
use for every barrier, so an expired wait is seen by the host as a status, not
as a hang.
"""

import time

import pytest
import torch

import kv_cache_eviction_scores_b200 as dk
from kv_cache_eviction_scores_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("limit_ms", [5.0, 50.0])
def test_expired_wait_reports_timeout(limit_ms):
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    st = dk.selftest_wait_timeout(limit_ms)
    dt = (time.perf_counter() - t0) * 1e3
    assert st == dk.ERR_TIMEOUT
    assert dt >= 0.9 * limit_ms  # the wait held for its limit before giving up


def test_context_is_usable_after_an_expired_wait():
    assert dk.selftest_wait_timeout(5.0) == dk.ERR_TIMEOUT
    wl = W.generate(W.config_spec(0), 42)
    s = dk.dropkv_scores(wl.q.cuda(), wl.k.cuda(), wl.v.cuda(), wl.spec.window, wl.spec.pool,
                         wl.lengths)
    torch.cuda.synchronize()
    assert torch.isfinite(s[0, :, : wl.lengths[0] - wl.spec.window]).all()
