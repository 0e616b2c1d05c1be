"""GPU parity at full depth: every score and the oracle's evict sets.

The write-up ("DropKV：精确单项输出扰动评分组件", section 结果与独立对照)
checks its closed form against a full, independent recomputation.  Here the
whole [B, Hkv, n_max] score array of the CUDA path is compared with the fp64
oracle on:

* the four full-size bf16 configurations (4K near-uniform, 32K with planted
  heavy keys, 128K with outlier channels, and the batched mixed-length case
  with NaN-poisoned padding), on every path the shape allows;
* "deep pipeline" cases in which every tensor-path CTA walks a long run of
  tiles (16 to 64), so the steady state of both passes -- every TMEM buffer
  and shared-memory ring slot reused many times, the deferred O rescale, the
  barriers' parity flips -- is compared element by element, including a
  ragged-length case and one with planted heavy keys (p up to about 0.97);
* the same input scored with several CTA budgets (``tc_ctas``), which changes
  how the tokens are split across CTAs but not the result.

Tolerances and set rules are those of tests/parity.py: relative 1e-3 for bf16
inputs; evict sets equal to the oracle's except for tolerance-level ties; the
GPU selection equal to the oracle's selection of the GPU's own scores.
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
TOL_BF16 = 1e-3
TILE = 128


def _paths(spec):
    shape = dk.Shape(spec.B, spec.Hq, spec.Hkv, spec.n_max, spec.d, spec.window, spec.pool,
                     0 if spec.dtype == "bf16" else 1)
    out = ["simt"]
    if dk.auto_path(shape) == dk.PATH_TENSOR:
        out.append("tensor")
    return out


def _gpu(wl, path, **kw):
    q, k, v = wl.q.to(DEV), wl.k.to(DEV), wl.v.to(DEV)
    s = dk.dropkv_scores(q, k, v, wl.spec.window, wl.spec.pool, wl.lengths, path=path, **kw)
    keep_idx, ev_idx = dk.dropkv_select(s, wl.keep, wl.lengths)
    torch.cuda.synchronize()
    out = s.cpu().numpy(), keep_idx.cpu().numpy(), ev_idx.cpu().numpy()
    del q, k, v, s
    torch.cuda.empty_cache()
    return out


def _compare(wl, ref, got, what):
    s, keep_idx, ev_idx = got
    worst = assert_scores_close(s, ref, TOL_BF16, what)
    assert_evict_sets_match(ev_idx, ref, wl.lengths, wl.keep, TOL_BF16, what)
    assert_select_exact(s, wl.lengths, wl.keep, keep_idx, ev_idx, what)
    return worst


def _split_runs(lengths, units, budget):
    """The library's split rule: one more split to the row whose runs are
    longest while the budget allows; returns every run's tile count."""
    nts = [(L + TILE - 1) // TILE for L in lengths]
    splits = [1] * len(lengths)
    total = units * len(lengths)
    budget = max(budget, total)
    while True:
        best, worst = -1, 0.0
        for b, nt in enumerate(nts):
            per = nt / splits[b]
            if splits[b] < nt and per > worst:
                best, worst = b, per
        if best < 0 or total + units > budget:
            break
        splits[best] += 1
        total += units
    return [(sp + 1) * nt // splits[b] - sp * nt // splits[b]
            for b, nt in enumerate(nts) for sp in range(splits[b])]


def tiles_per_cta(spec, tc_ctas=0, sms=148):
    """Tile runs of the tensor path's CTAs, (min, max) over both passes: pass 1
    runs one CTA per (b, h, chunk of <= 256 query rows, split) within the CTA
    budget; the DropKV second pass runs CTA pairs (half the budget) and each
    CTA of a pair takes half of the pair's run."""
    nq = (spec.Hq // spec.Hkv) * spec.window
    units = spec.Hkv * ((nq + 255) // 256)
    budget = min(tc_ctas if tc_ctas > 0 else sms, 160)
    r1 = _split_runs(spec.lengths, units, budget)
    r2 = [x // 2 for x in _split_runs(spec.lengths, units, budget // 2)]
    return min(r1 + r2), max(r1 + r2)


# ---- the four full-size configurations, whole arrays -------------------------

@pytest.mark.parametrize("idx", [1, 2, 3, 4])
def test_full_config_whole(idx):
    spec = W.config_spec(idx)
    wl = W.generate(spec, 42)
    ref = oracle.scores(wl.q, wl.k, wl.v, wl.lengths, spec.window, spec.pool)
    for b, L in enumerate(wl.lengths):
        assert np.all(np.isnan(ref[b, :, L:])) and np.all(np.isposinf(ref[b, :, L - spec.window:L]))
    for path in _paths(spec):
        worst = _compare(wl, ref, _gpu(wl, path), f"{spec.name} {path}")
        print(f"{spec.name} {path}: worst relative error {worst:.2e}")


# ---- deep pipelines: long tile runs per CTA ----------------------------------

# A CTA budget of 64 gives every (b, h) unit one pass-1 CTA walking all 32
# tiles of its 4096 tokens, and one CTA pair in the second pass (16 tiles each).
DEEP = [
    W.Spec("deep_b8_w64_outlier", B=8, Hq=32, Hkv=8, d=128, lengths=[4096] * 8, window=64,
           pool=7, keep=[W.budget(0.05, 4096)] * 8, outlier_channels=4),
    # ragged lengths with NaN-poisoned padding: runs ending in a partial tile
    # at a different offset
    W.Spec("deep_b8_ragged_nan", B=8, Hq=32, Hkv=8, d=128,
           lengths=[4096, 3001, 4000, 2500, 3333, 4095, 1800, 3900], window=64, pool=7,
           keep=[W.budget(0.05, L) for L in (4096, 3001, 4000, 2500, 3333, 4095, 1800, 3900)],
           n_max=4096, nan_pad=True, outlier_channels=4),
    # planted heavy keys (p up to about 0.97): the careful path and the moving
    # reference max fire in the middle of long runs
    W.Spec("deep_b8_heavy", B=8, Hq=32, Hkv=8, d=128, lengths=[4096] * 8, window=32, pool=7,
           keep=[W.budget(0.05, 4096)] * 8, heavy_per_head=16),
]
DEEP_CTAS = 64


@pytest.mark.parametrize("spec", DEEP, ids=[s.name for s in DEEP])
def test_deep_pipeline_whole(spec):
    tc_ctas = DEEP_CTAS
    lo, hi = tiles_per_cta(spec, tc_ctas)
    assert lo >= 7, (lo, hi)  # every CTA's run is long: the steady state is compared
    wl = W.generate(spec, 7)
    ref = oracle.scores(wl.q, wl.k, wl.v, wl.lengths, spec.window, spec.pool)
    for path in _paths(spec):
        _compare(wl, ref, _gpu(wl, path, tc_ctas=tc_ctas), f"{spec.name} {path}")


@pytest.mark.parametrize("tc_ctas", [16, 48, 0])
def test_cta_budget_gives_the_same_scores(tc_ctas):
    # 128K-token workload shape at n = 16384: with 16 CTAs, pass-1 CTAs walk 64
    # tiles and each second-pass CTA 64 (one pair per KV head); 48 gives
    # uneven runs of 21/22
    spec = W.Spec("cfg3_shape_16k", B=1, Hq=32, Hkv=8, d=128, lengths=[16384], window=64,
                  pool=7, keep=[W.budget(0.05, 16384)], outlier_channels=4)
    lo, hi = tiles_per_cta(spec, tc_ctas)
    wl = W.generate(spec, 11)
    ref = oracle.scores(wl.q, wl.k, wl.v, wl.lengths, spec.window, spec.pool)
    got = _gpu(wl, "tensor", tc_ctas=tc_ctas)
    _compare(wl, ref, got, f"tc_ctas={tc_ctas} (tiles per CTA {lo}..{hi})")
    if tc_ctas == 16:
        assert lo == hi == 64


def test_window_attention_outputs_deep():
    spec = DEEP[0]
    wl = W.generate(spec, 7)
    raw, attn_ref, stats_ref, st, _ = oracle.raw_scores(wl.q, wl.k, wl.v, wl.lengths,
                                                        want_attn=True)
    q, k, v = wl.q.to(DEV), wl.k.to(DEV), wl.v.to(DEV)
    for path in _paths(spec):
        s, attn, stats = dk.dropkv_scores(q, k, v, spec.window, spec.pool, wl.lengths,
                                          path=path, return_attn=True)
        torch.cuda.synchronize()
        a = attn.cpu().numpy().astype(np.float64)
        scale = np.abs(attn_ref).max(axis=-1, keepdims=True)
        assert np.all(np.abs(a - attn_ref) <= 1e-4 * scale + 1e-6), path
        st_g = stats.cpu().numpy().astype(np.float64)
        l_at_ref = st_g[..., 1] * np.exp(st_g[..., 0] - stats_ref[..., 0])
        np.testing.assert_allclose(l_at_ref, stats_ref[..., 1], rtol=1e-4)
