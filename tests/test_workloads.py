"""The seeded synthetic workloads follow their recipe (CPU only).

The generator holds none of the method's arithmetic; these checks pin what
the parity tests and the benchmark rely on: determinism, the keep budgets, the
outlier channels, the planted heavy keys (peaked but never singular) and the
NaN-poisoned padding.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from kv_cache_eviction_scores_b200 import workloads as W


def test_generation_is_deterministic_per_seed():
    spec = W.small_spec(3)
    a, b, c = W.generate(spec, 42), W.generate(spec, 42), W.generate(spec, 43)
    for x, y in ((a.q, b.q), (a.k, b.k), (a.v, b.v)):
        assert torch.equal(x, y)
    assert not torch.equal(a.k, c.k)


def test_keep_budgets_of_the_configurations():
    assert W.config_spec(0).keep == [22 - 7]
    assert W.config_spec(1).keep == [819]
    assert W.config_spec(2).keep == [1638]
    assert W.config_spec(3).keep == [6553]
    assert W.config_spec(4).keep == [819, 3276, 13107, 6553]
    for i in range(5):
        s = W.config_spec(i)
        assert all(s.window <= kp <= L for kp, L in zip(s.keep, s.lengths))


def test_outlier_channels_are_scaled():
    spec = W.small_spec(3)
    wl = W.generate(spec, 42)
    chans = wl.extras["outlier_channels"]
    k = wl.k.to(torch.float64)
    for h in range(spec.Hkv):
        c = chans[0, h]
        others = torch.ones(spec.d, dtype=torch.bool)
        others[c] = False
        rms_out = k[0, h][:, c].pow(2).mean().sqrt()
        rms_in = k[0, h][:, others].pow(2).mean().sqrt()
        assert 6.0 < float(rms_out / rms_in) < 10.0  # nominal x8


def test_heavy_keys_are_aligned_peaked_and_not_singular():
    spec = W.small_spec(2)
    wl = W.generate(spec, 42)
    G, w, d = spec.G, spec.window, spec.d
    q, k = wl.q.to(torch.float64), wl.k.to(torch.float64)
    pos = wl.extras["heavy_positions"]
    for h in range(spec.Hkv):
        for i in range(spec.heavy_per_head):
            row = i % (G * w)
            qv = q[0, h * G + row // w, row % w]
            kv = k[0, h, int(pos[0, h, i])]
            cos = float(qv @ kv / (qv.norm() * kv.norm()))
            assert abs(cos - spec.heavy_cos) < 0.02
            assert abs(float(kv.norm()) - math.sqrt(d)) < 0.05 * math.sqrt(d)
    # peaked attention on the planted keys, yet every fp32 p stays below 1
    hq = 0
    P = wl.lengths[0] - w  # window query 0 of query head 0
    x = (q[0, hq, 0] @ k[0, 0, : P + 1].T) / math.sqrt(d)
    p = torch.softmax(x, 0)
    heavy = [int(j) for j in pos[0, 0] if int(j) <= P]
    assert float(p[heavy].max()) > 0.05
    oracle.scores(wl.q, wl.k, wl.v, wl.lengths, w, spec.pool)  # raises if singular


def test_padding_is_nan_poisoned_and_history_finite():
    spec = W.small_spec(4)
    wl = W.generate(spec, 42)
    for b, L in enumerate(spec.lengths):
        assert torch.isnan(wl.k[b, :, L:].float()).all() and torch.isnan(wl.v[b, :, L:].float()).all()
        assert torch.isfinite(wl.k[b, :, :L].float()).all() and torch.isfinite(wl.v[b, :, :L].float()).all()


@pytest.mark.parametrize("idx", [1, 2, 3, 4])
def test_scaled_configurations_keep_the_full_shapes(idx):
    small, full = W.small_spec(idx), W.config_spec(idx)
    assert (small.Hq, small.Hkv, small.d, small.window, small.pool, small.dtype) == \
        (full.Hq, full.Hkv, full.d, full.window, full.pool, full.dtype)
    # several 128-token tiles and a ragged tail
    assert max(small.lengths) > 3 * 128 and any(L % 128 for L in small.lengths)
    assert np.all(np.asarray(small.keep) >= small.window)
