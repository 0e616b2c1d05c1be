"""dropkv_scores_select (scoring and eviction in one call) on the GPU.

Its contract is "the results of dropkv_scores followed by dropkv_select":
the scores must be the same bits and the keep / evict lists the same
integers, and both agree with the fp64 oracle where that is cheap.
"""

import numpy as np
import pytest
import torch

import oracle
import kv_cache_eviction_scores_b200 as dk
from kv_cache_eviction_scores_b200 import workloads as W

from parity import assert_evict_sets_match, assert_scores_close, assert_select_exact

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _paths(spec):
    shape = dk.Shape(spec.B, spec.Hq, spec.Hkv, spec.n_max, spec.d, spec.window, spec.pool,
                     0 if spec.dtype == "bf16" else 1)
    out = ["simt"]
    if dk.auto_path(shape) == dk.PATH_TENSOR:
        out.append("tensor")
    return out


def _both(wl, path):
    """(separate calls, one call): each (scores, keep_idx, evict_idx) on the host."""
    q, k, v = wl.q.to(DEV), wl.k.to(DEV), wl.v.to(DEV)
    spec = wl.spec
    s1 = dk.dropkv_scores(q, k, v, spec.window, spec.pool, wl.lengths, path=path)
    k1, e1 = dk.dropkv_select(s1, wl.keep, wl.lengths)
    s2, k2, e2 = dk.dropkv_scores_select(q, k, v, spec.window, spec.pool, wl.keep, wl.lengths,
                                         path=path)
    torch.cuda.synchronize()
    return ((s1.cpu().numpy(), k1.cpu().numpy(), e1.cpu().numpy()),
            (s2.cpu().numpy(), k2.cpu().numpy(), e2.cpu().numpy()))


def _same(a, b, what):
    s1, k1, e1 = a
    s2, k2, e2 = b
    # the same bits (NaN padding included)
    assert np.array_equal(s1.view(np.uint32), s2.view(np.uint32)), f"{what}: scores differ"
    assert np.array_equal(k1, k2), f"{what}: keep lists differ"
    assert np.array_equal(e1, e2), f"{what}: evict lists differ"


SPECS = [W.config_spec(0)] + [W.small_spec(i) for i in (1, 2, 3, 4)] + [
    # ragged tails, pooling off; wide pooling, head dim 256; fp32 odd head dim
    W.Spec("ragged_pool1", B=3, Hq=8, Hkv=2, d=64, lengths=[129, 255, 300], window=4, pool=1,
           keep=[20, 40, 100], dtype="bf16", n_max=301),
    W.Spec("pool31_d256", B=1, Hq=4, Hkv=1, d=256, lengths=[400], window=8, pool=31,
           keep=[50], dtype="bf16"),
    W.Spec("f32_d5_g3", B=2, Hq=6, Hkv=2, d=5, lengths=[70, 33], window=5, pool=5,
           keep=[35, 6], dtype="f32"),
    # more rows than one launch slice; NaN-poisoned padding on the tensor path
    W.Spec("batch66_tc", B=66, Hq=4, Hkv=1, d=128,
           lengths=[130 + (b * 37) % 170 for b in range(66)], window=8, pool=5,
           keep=[20 + (b % 7) for b in range(66)], dtype="bf16", n_max=300),
    W.Spec("nan_pad_tc", B=2, Hq=8, Hkv=2, d=128, lengths=[140, 389], window=16, pool=7,
           keep=[16, 100], dtype="bf16", n_max=400, nan_pad=True),
    # a row longer than 8 CTAs' key caches hold (262144 keys: uncached ranges)
    W.Spec("long_row", B=1, Hq=2, Hkv=1, d=8, lengths=[270000], window=2, pool=3,
           keep=[27000], dtype="f32"),
]


@pytest.mark.parametrize("spec", SPECS, ids=[s.name for s in SPECS])
def test_one_call_equals_two_calls_and_the_oracle(spec):
    wl = W.generate(spec, 5)
    tol = 1e-6 if spec.dtype == "f32" else 1e-3
    ref = oracle.scores(wl.q, wl.k, wl.v, wl.lengths, spec.window, spec.pool)
    for path in _paths(spec):
        sep, one = _both(wl, path)
        _same(sep, one, f"{spec.name} {path}")
        s, k_idx, e_idx = one
        assert_scores_close(s, ref, tol, f"{spec.name} {path}")
        assert_evict_sets_match(e_idx, ref, wl.lengths, wl.keep, tol, f"{spec.name} {path}")
        assert_select_exact(s, wl.lengths, wl.keep, k_idx, e_idx, f"{spec.name} {path}")


@pytest.mark.parametrize("idx", [1, 2, 3, 4])
def test_full_configs_one_call_equals_two_calls(idx):
    # the full-size configurations; the two-call results are checked against
    # the oracle in the full-size whole-array tests
    wl = W.generate(W.config_spec(idx), 42)
    sep, one = _both(wl, "tensor")
    _same(sep, one, f"config {idx}")


def test_launch_counts():
    spec = W.config_spec(3)
    shape = dk.Shape(spec.B, spec.Hq, spec.Hkv, spec.n_max, spec.d, spec.window, spec.pool, 0)
    n_two = dk.scores_launches(shape, spec.lengths) + dk.select_launches(
        spec.B, spec.Hkv, spec.n_max, spec.lengths)
    assert dk.scores_select_launches(shape, spec.lengths) == n_two
    rows = dk.Shape(70, 2, 1, 60, 8, 3, 3, 1)  # two batch slices
    n_two = dk.scores_launches(rows, None) + dk.select_launches(70, 1, 60, None)
    assert dk.scores_select_launches(rows, None) == n_two


def test_async_status_and_singular():
    wl = W.generate(W.config_spec(0), 42)
    q, k, v = wl.q.to(DEV), wl.k.to(DEV), wl.v.to(DEV)
    status = torch.full((1,), -1, dtype=torch.int32, device=DEV)
    dk.dropkv_scores_select(q, k, v, 3, 3, wl.keep, wl.lengths, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == dk.OK
    # one key that takes all the probability: the call reports it
    d, L, w = 16, 40, 2
    qs = torch.zeros(1, 2, w, d)
    qs[..., 0] = 1.0
    ks = torch.zeros(1, 1, L, d)
    ks[0, 0, 0, 0] = 400.0
    vs = torch.randn(1, 1, L, d)
    with pytest.raises(dk.SingularError):
        dk.dropkv_scores_select(qs.to(DEV), ks.to(DEV), vs.to(DEV), w, 1, [10], [L])
