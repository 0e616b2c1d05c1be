"""Failure detection on the GPU without a fault: a device-side wait that runs
out reports DROPKV_ERR_TIMEOUT through the status word and leaves the context
usable.  The select kernel's own failure path is exercised the same way: one
CTA of every cluster withholds an arrival, the waits are limited to a few
milliseconds, and the caller must see the timeout status and lists of -1.

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


def _select_scores(B, Hkv, n_max, lengths, seed):
    import numpy as np
    rng = np.random.default_rng(seed)
    s = rng.integers(0, 40, size=(B, Hkv, n_max)).astype(np.float32) / 8.0
    for b, L in enumerate(lengths):
        s[b, :, L:] = np.nan
    return torch.from_numpy(s).cuda()


def test_select_timeout_reaches_the_caller_and_leaves_no_stale_index():
    B, Hkv, n_max, lengths = 2, 3, 5000, [5000, 3001]
    keep = [1000, 3001]  # row 1 keeps everything: no eviction, no wait to run out
    scores = _select_scores(B, Hkv, n_max, lengths, 1)
    t0 = time.perf_counter()
    st, keep_idx, ev_idx = dk.selftest_select_timeout(scores, keep, lengths, limit_ms=10.0)
    dt = (time.perf_counter() - t0) * 1e3
    assert st == dk.ERR_TIMEOUT
    assert dt >= 9.0  # a wait held for its limit before giving up
    assert bool((keep_idx[0] == -1).all()) and bool((ev_idx[0] == -1).all())
    # the row without evictions never waits: its lists are the normal ones
    ok_keep, ok_ev = dk.dropkv_select(scores, keep, lengths, sync=True)
    assert torch.equal(keep_idx[1, :, :3001], ok_keep[1, :, :3001])
    # the context is usable and the status path reports success afterwards
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    k2, e2 = dk.dropkv_select(scores, keep, lengths, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == dk.OK
    assert torch.equal(k2, ok_keep) and torch.equal(e2, ok_ev)
