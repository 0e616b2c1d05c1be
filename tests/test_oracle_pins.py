"""Pins for the fp64 oracle: it is checked against things other than itself.

Each test ties one part of the oracle to something the pages or mathematics
fix: brute-force deletion, closed forms of special cases, invariants, textbook
routines.  See the oracle package docstring for which test pins which function.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import bruteforce
from kv_cache_eviction_scores_b200 import workloads as W

from conftest import GOLDEN


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _np(x):
    return np.asarray(x, dtype=np.float64)


# ---- the closed form against actual deletion (core formula; the write-up's
#      independent delete-and-re-softmax check) -----------------------------

@pytest.mark.parametrize("seed", [42, 43, 44])
def test_closed_form_equals_deletion_on_protocol_shapes(seed):
    proto = _load("writeup_protocol.json")
    spec = W.config_spec(0)
    assert (spec.B, spec.Hq, spec.Hkv, spec.d, spec.window) == (
        proto["batch"], proto["query_heads"], proto["kv_heads"], proto["head_dim"],
        proto["window"])
    assert spec.lengths[0] == proto["history_slots"] + proto["window"]
    assert spec.lengths[0] - spec.keep[0] == proto["evict"]
    wl = W.generate(spec, seed)
    raw, _, _, st, _ = oracle.raw_scores(wl.q, wl.k, wl.v, wl.lengths)
    assert st == oracle.OK
    bf = bruteforce.raw_scores(_np(wl.q.double()), _np(wl.k.double()), _np(wl.v.double()),
                               wl.lengths)
    m = np.isfinite(bf)
    err = np.abs(raw[m] - bf[m])
    # Same order as the page's 5.55e-16 largest error (its inputs differ).
    assert err.max() <= 4 * proto["max_abs_err_closed_form_vs_deletion"]
    assert np.all(err <= 1e-12 * np.abs(bf[m]) + 1e-15)


def test_closed_form_equals_deletion_on_random_tiny_shapes():
    rng = torch.Generator().manual_seed(7)
    for i in range(30):
        spec = W.random_spec(rng, max_n=30)
        wl = W.generate(spec, 1000 + i)
        raw, _, _, st, _ = oracle.raw_scores(wl.q, wl.k, wl.v, wl.lengths)
        assert st == oracle.OK
        bf = bruteforce.raw_scores(_np(wl.q.double()), _np(wl.k.double()),
                                   _np(wl.v.double()), wl.lengths)
        assert np.array_equal(np.isnan(raw), np.isnan(bf))
        m = ~np.isnan(bf)
        assert np.all(np.abs(raw[m] - bf[m]) <= 1e-11 * np.abs(bf[m]) + 1e-14), spec


# ---- closed forms of special cases --------------------------------------

def test_uniform_attention_closed_form():
    """q = 0: p_j = 1/N_t over the N_t = P_t + 1 visible keys, a_t = their mean,
    p/(1-p) = 1/(N_t - 1), so s_j = sum_{t: P_t >= j} ||mean_t - v_j||^2 / (N_t-1)^2."""
    g = torch.Generator().manual_seed(3)
    B, Hkv, G, w, d, L = 1, 2, 2, 4, 5, 17
    q = torch.zeros(B, Hkv * G, w, d, dtype=torch.float64)
    k = torch.randn(B, Hkv, L, d, generator=g, dtype=torch.float64)
    v = torch.randn(B, Hkv, L, d, generator=g, dtype=torch.float64)
    raw, _, _, st, _ = oracle.raw_scores(q, k, v, [L])
    assert st == oracle.OK
    vv = v.numpy()
    for hq in range(Hkv * G):
        h = hq // G
        expect = np.zeros(L)
        for t in range(w):
            P = L - w + t
            N = P + 1
            mean = vv[0, h, :N].mean(axis=0)
            for j in range(N):
                expect[j] += np.sum((mean - vv[0, h, j]) ** 2) / (N - 1) ** 2
        np.testing.assert_allclose(raw[0, hq], expect, rtol=1e-12, atol=1e-15)


def test_golden_uniform_three_tokens():
    gd = _load("uniform_three_tokens.json")
    q, k, v = _np(gd["q"]), _np(gd["k"]), _np(gd["v"])
    raw, _, _, st, _ = oracle.raw_scores(q, k, v, gd["lengths"])
    np.testing.assert_allclose(raw[0, 0], gd["raw"], rtol=1e-14, atol=1e-15)
    for case in gd["cases"]:
        s = oracle.scores(q, k, v, gd["lengths"], gd["window"], case["pool"])
        want = np.array([float(x) for x in case["scores"]])
        np.testing.assert_allclose(s[0, 0], want, rtol=1e-14, atol=1e-15)
        keep, ev = oracle.select(s, gd["lengths"], [case["keep"]])
        assert keep[0, 0].tolist() == case["keep_idx"]
        assert ev[0, 0].tolist() == case["evict_idx"]


def test_golden_two_token_closed_form():
    gd = _load("two_token_closed_form.json")
    q, k, v = _np(gd["q"]), _np(gd["k"]), _np(gd["v"])
    raw, _, _, st, _ = oracle.raw_scores(q, k, v, gd["lengths"])
    p0 = 1.0 / (1.0 + math.exp(gd["logit_gap"]))
    p1 = 1.0 - p0
    np.testing.assert_allclose(raw[0, 0], [p0 * p0 * gd["sq_dist"], p1 * p1 * gd["sq_dist"]],
                               rtol=1e-13)


# ---- invariants ----------------------------------------------------------

def test_value_scaling_scales_scores_by_c_squared():
    wl = W.generate(W.config_spec(0), 42)
    raw, *_ = oracle.raw_scores(wl.q, wl.k, wl.v, wl.lengths)
    raw3, *_ = oracle.raw_scores(wl.q, wl.k, wl.v.double() * 3.0, wl.lengths)
    np.testing.assert_allclose(raw3, 9.0 * raw, rtol=1e-13)


def test_history_permutation_permutes_scores():
    """Every window query sees all history positions, so permuting history
    tokens (keys and values together) permutes their raw scores."""
    wl = W.generate(W.config_spec(0), 43)
    L, w = wl.lengths[0], wl.spec.window
    perm = torch.randperm(L - w, generator=torch.Generator().manual_seed(5))
    full = torch.cat([perm, torch.arange(L - w, L)])
    k2, v2 = wl.k.clone(), wl.v.clone()
    k2[:, :, :L] = wl.k[:, :, full]
    v2[:, :, :L] = wl.v[:, :, full]
    raw, *_ = oracle.raw_scores(wl.q, wl.k, wl.v, wl.lengths)
    raw2, *_ = oracle.raw_scores(wl.q, k2, v2, wl.lengths)
    np.testing.assert_allclose(raw2[:, :, :L], raw[:, :, full.numpy()], rtol=1e-12)


def test_gqa_merge_identity_for_one_query_head_per_kv_head():
    spec = W.Spec("g1", B=2, Hq=3, Hkv=3, d=6, lengths=[20, 14], window=3, pool=1,
                  keep=[10, 7], dtype="f32")
    wl = W.generate(spec, 11)
    s, merged, raw, st = oracle.scores(wl.q, wl.k, wl.v, wl.lengths, 3, 1, intermediates=True)
    np.testing.assert_array_equal(np.isnan(merged), np.isnan(raw))
    m = ~np.isnan(raw)
    np.testing.assert_array_equal(merged[m], raw[m])


def test_gqa_merge_of_duplicated_query_heads_equals_one_head():
    spec = W.Spec("dup", B=1, Hq=6, Hkv=2, d=4, lengths=[25], window=4, pool=1, keep=[12],
                  dtype="f32")
    wl = W.generate(spec, 12)
    q = wl.q.clone()
    for h in range(2):
        for g in range(3):
            q[:, h * 3 + g] = wl.q[:, h * 3]
    s, merged, raw, st = oracle.scores(q, wl.k, wl.v, wl.lengths, 4, 1, intermediates=True)
    for h in range(2):
        np.testing.assert_allclose(merged[0, h, :25], raw[0, h * 3, :25], rtol=1e-14)


def test_gqa_merge_is_mean_of_group():
    spec = W.Spec("mean", B=1, Hq=4, Hkv=2, d=4, lengths=[15], window=2, pool=1, keep=[8],
                  dtype="f32")
    wl = W.generate(spec, 13)
    s, merged, raw, st = oracle.scores(wl.q, wl.k, wl.v, wl.lengths, 2, 1, intermediates=True)
    np.testing.assert_allclose(merged[0, 0, :15], raw[0, 0:2, :15].mean(axis=0), rtol=1e-14)
    np.testing.assert_allclose(merged[0, 1, :15], raw[0, 2:4, :15].mean(axis=0), rtol=1e-14)


# ---- MaxPool1D and protection (Algorithm 1) ------------------------------

@pytest.mark.parametrize("pool", [1, 3, 5, 7, 9])
def test_pool_matches_sliding_max(pool):
    rng = np.random.default_rng(pool)
    B, Hkv, n_max, w = 2, 3, 40, 4
    lengths = [40, 23]
    merged = rng.integers(0, 6, size=(B, Hkv, n_max)).astype(np.float64)  # plateaus
    out = oracle.pool_protect(merged, w, pool, lengths)
    r = pool // 2
    for b in range(B):
        L = lengths[b]
        for h in range(Hkv):
            x = merged[b, h, :L]
            # textbook sliding window maximum with -inf padding (numpy)
            padded = np.concatenate([np.full(r, -np.inf), x, np.full(r, -np.inf)])
            win = np.lib.stride_tricks.sliding_window_view(padded, pool).max(axis=1)
            assert np.array_equal(out[b, h, : L - w], win[: L - w])
            assert np.all(out[b, h, : L - w] >= x[: L - w])
            assert np.all(np.isposinf(out[b, h, L - w: L]))
            assert np.all(np.isnan(out[b, h, L:]))
            if pool == 1:
                assert np.array_equal(out[b, h, : L - w], x[: L - w])


def test_window_is_protected_and_never_evicted():
    wl = W.generate(W.config_spec(0), 44)
    s = oracle.scores(wl.q, wl.k, wl.v, wl.lengths, 3, 3)
    L, w = wl.lengths[0], 3
    assert np.all(np.isposinf(s[0, :, L - w: L]))
    keep, ev = oracle.select(s, wl.lengths, [w])  # keep only as many as the window
    for h in range(s.shape[1]):
        assert sorted(keep[0, h].tolist()) == list(range(L - w, L))
        assert not set(ev[0, h].tolist()) & set(range(L - w, L))


# ---- singular input (Algorithm 1 paragraph: rejected, no epsilon) --------

def test_singular_input_is_rejected():
    d, L, w = 8, 12, 2
    q = torch.zeros(1, 1, w, d, dtype=torch.float64)
    q[..., 0] = 1.0
    k = torch.zeros(1, 1, L, d, dtype=torch.float64)
    v = torch.randn(1, 1, L, d, generator=torch.Generator().manual_seed(1), dtype=torch.float64)
    k[0, 0, 3, 0] = 100.0 * math.sqrt(d)  # logit 100 above every other one
    with pytest.raises(oracle.SingularError):
        oracle.scores(q, k, v, [L], w, 3)
    raw, _, _, st, where = oracle.raw_scores(q, k, v, [L], raise_singular=False)
    assert st == oracle.ERR_SINGULAR and where[3] == 3


def test_peaked_but_nonsingular_input_is_accepted():
    d, L, w = 8, 12, 2
    q = torch.zeros(1, 1, w, d, dtype=torch.float64)
    q[..., 0] = 1.0
    k = torch.zeros(1, 1, L, d, dtype=torch.float64)
    v = torch.randn(1, 1, L, d, generator=torch.Generator().manual_seed(1), dtype=torch.float64)
    k[0, 0, 3, 0] = 5.0 * math.sqrt(d)  # p about 0.93, far from 1
    s = oracle.scores(q, k, v, [L], w, 1)
    assert np.all(np.isfinite(s[0, 0, : L - w]))


# The rule at its boundary: "rounds to 1" is the fp32 rounding of the exact
# p_j (the inputs' precision), with no epsilon.  fp32 has 1 - 2^-24 as its
# largest value below 1, so p rounds to 1 exactly when 1 - p <= 2^-25 (the
# midpoint rounds to even, i.e. to 1).  A threshold rule such as
# p > 1 - 1e-5 or p > 1 - 1e-7 fails the accepted cases below, and a rule
# that only catches exact cancellation (1 - p == 0 in fp64) fails the
# rejected ones.
BOUNDARY = [
    (1e-6, False),      # far below the boundary in fp32 terms: scored
    (4e-8, False),      # between 2^-25 and 2^-24: rounds to 1 - 2^-24, scored
    (2.5e-8, True),     # just above 1 - 2^-25: rounds to 1, rejected
    (1e-9, True),       # rounds to 1, rejected
]


@pytest.mark.parametrize("tau,singular", BOUNDARY)
def test_singular_rule_at_the_fp32_boundary(tau, singular):
    from parity import dominant_key_case
    L, w = 40, 1
    q, k, v, t = dominant_key_case(tau, dtype=torch.float32, d=1, L=L, Hq=1, w=w)
    assert (np.float32(1.0 - t) == np.float32(1.0)) == singular  # the construction
    assert abs(t - tau) <= 0.01 * tau
    if singular:
        with pytest.raises(oracle.SingularError):
            oracle.scores(q, k, v, [L], w, 1)
        _, _, _, st, where = oracle.raw_scores(q, k, v, [L], raise_singular=False)
        assert st == oracle.ERR_SINGULAR and where[3] == 0
        return
    raw, _, _, st, _ = oracle.raw_scores(q, k, v, [L])
    assert st == oracle.OK
    # the accepted case is scored exactly: closed form against deletion.  For
    # the dominant token both sides lose about 1e-16 / tau of relative
    # precision in 1 - p (squared in the score); for the others deletion
    # subtracts two O(1) outputs that differ by about p_j, so it carries a
    # relative error of order 1e-16 / p_j (p_j about tau / 39 here)
    bf = bruteforce.raw_scores(q.double().numpy(), k.double().numpy(), v.double().numpy(), [L])
    np.testing.assert_allclose(raw[0, 0, 0], bf[0, 0, 0], rtol=1e-7)
    np.testing.assert_allclose(raw[0, 0, 1:L], bf[0, 0, 1:L], rtol=1e-4)
    # the dominant token's perturbation is about ||mean of the others - v_0||^2
    assert raw[0, 0, 0] > 1e-3


def test_argument_errors():
    wl = W.generate(W.config_spec(0), 42)
    with pytest.raises(ValueError):
        oracle.scores(wl.q, wl.k, wl.v, wl.lengths, 3, 2)      # even pool kernel
    with pytest.raises(ValueError):
        oracle.scores(wl.q, wl.k, wl.v, [3], 3, 3)             # L must exceed w
    with pytest.raises(ValueError):
        oracle.scores(wl.q, wl.k, wl.v, [23], 3, 3)            # L beyond n_max


# ---- selection -----------------------------------------------------------

def _brute_select(s, L, keep):
    order = sorted(range(L), key=lambda j: (s[j], j))
    E = L - keep
    return sorted(order[E:]), sorted(order[:E])


def test_select_matches_full_sort_with_ties():
    rng = np.random.default_rng(0)
    B, Hkv, n_max = 3, 2, 300
    lengths = [300, 123, 7]
    keep = [30, 100, 7]
    s = rng.integers(0, 20, size=(B, Hkv, n_max)).astype(np.float64) / 7.0
    for b, L in enumerate(lengths):
        s[b, :, L - 3: L] = np.inf
        s[b, :, L:] = np.nan
    keep_idx, ev_idx = oracle.select(s, lengths, keep)
    for b, L in enumerate(lengths):
        for h in range(Hkv):
            kk, ee = _brute_select(s[b, h].tolist(), L, keep[b])
            got_k = [x for x in keep_idx[b, h].tolist() if x >= 0]
            got_e = [x for x in ev_idx[b, h].tolist() if x >= 0]
            assert got_k == kk and got_e == ee
            assert all(x == -1 for x in keep_idx[b, h, len(kk):])


def test_constant_values_give_zero_scores_and_all_ties():
    """All v_j equal => a = v_j => every Delta is 0; eviction falls back to the
    position order among the tied zeros.  (v = 0 keeps a = sum p_j v_j exactly
    0 in floating point; any other constant leaves rounding residues ~1e-33.)"""
    spec = W.Spec("constv", B=1, Hq=2, Hkv=1, d=4, lengths=[16], window=3, pool=3, keep=[6],
                  dtype="f32")
    wl = W.generate(spec, 21)
    v = torch.zeros_like(wl.v)
    s = oracle.scores(wl.q, wl.k, v, wl.lengths, 3, 3)
    assert np.all(s[0, 0, :13] == 0.0)
    keep, ev = oracle.select(s, wl.lengths, [6])
    assert ev[0, 0].tolist() == list(range(10))
    assert keep[0, 0].tolist() == [10, 11, 12, 13, 14, 15]


# ---- sampled scoring equals the whole-problem oracle ---------------------

def test_scores_at_equals_full_oracle():
    spec = W.Spec("mid", B=1, Hq=4, Hkv=2, d=16, lengths=[90], window=5, pool=5, keep=[30],
                  dtype="bf16")
    wl = W.generate(spec, 31)
    full = oracle.scores(wl.q, wl.k, wl.v, wl.lengths, 5, 5)
    pos = [0, 1, 2, 40, 83, 84, 85, 86, 89]
    for h in range(2):
        got = oracle.scores_at(wl.q[0, 2 * h: 2 * h + 2], wl.k[0, h, :90], wl.v[0, h, :90],
                               5, 5, pos)
        np.testing.assert_allclose(got, full[0, h, pos], rtol=1e-13)


# ---- attention-only score (the write-up's negative control) -----------------

def test_attention_only_mass_sums_to_the_window():
    # every window query spreads probability 1 over the keys it sees
    rng = np.random.default_rng(7)
    q = rng.standard_normal((2, 4, 5, 16))
    k = rng.standard_normal((2, 2, 40, 16)) * 2.0
    raw = oracle.attn_raw(q, k, [40, 23])
    for b, L in enumerate([40, 23]):
        np.testing.assert_allclose(raw[b, :, :L].sum(axis=1), 5.0, rtol=1e-13)
        assert np.all(np.isnan(raw[b, :, L:]))


def test_attention_only_uniform_keys_closed_form():
    # equal keys: query t sees P_t + 1 keys, each with p = 1 / (P_t + 1)
    L, w, d = 12, 4, 8
    q = np.random.default_rng(1).standard_normal((1, 1, w, d))
    k = np.tile(np.random.default_rng(2).standard_normal(d), (1, 1, L, 1))
    raw = oracle.attn_raw(q, k, [L])[0, 0]
    want = np.zeros(L)
    for t in range(w):
        P = L - w + t
        want[: P + 1] += 1.0 / (P + 1)
    np.testing.assert_allclose(raw, want, rtol=1e-13)


def test_attention_only_three_key_closed_form():
    # d = 4, q = (2,0,0,0), keys (1,0,0,0), 0, (-1,0,0,0): logits / sqrt(4) = 1, 0, -1
    q = np.zeros((1, 1, 1, 4)); q[0, 0, 0, 0] = 2.0
    k = np.zeros((1, 1, 3, 4)); k[0, 0, 0, 0] = 1.0; k[0, 0, 2, 0] = -1.0
    raw = oracle.attn_raw(q, k, [3])[0, 0]
    e = np.array([math.e, 1.0, 1.0 / math.e])
    np.testing.assert_allclose(raw, e / e.sum(), rtol=1e-14)


def test_attention_only_dominant_key_and_pipeline():
    # a key far above the rest takes (almost) all the mass of every query that
    # sees it; after merge / pool / protect the window is +inf and padding NaN
    rng = np.random.default_rng(3)
    L, w, d, G = 20, 3, 8, 2
    u = rng.standard_normal(d)
    u /= np.linalg.norm(u)
    q = u + 0.01 * rng.standard_normal((1, G, w, d))  # every query points along u
    k = rng.standard_normal((1, 1, L, d)) * 0.1
    k[0, 0, 5] = 60.0 * u  # logit about 60 / sqrt(8) = 21 above the others
    raw = oracle.attn_raw(q, k, [L])
    assert np.all(raw[0, :, 5] > w - 1e-3)
    s = oracle.attn_scores(q, k, [L], w, 1)
    np.testing.assert_allclose(s[0, 0, : L - w], raw[0, :, : L - w].mean(axis=0), rtol=1e-14)
    assert np.all(np.isposinf(s[0, 0, L - w: L]))


def test_attention_only_accepts_bf16_tensors_as_their_exact_upcast():
    # bf16 torch inputs are read as their exact fp64 values
    g = torch.Generator().manual_seed(4)
    q = torch.randn(1, 4, 3, 16, generator=g).to(torch.bfloat16)
    k = torch.randn(1, 2, 30, 16, generator=g).to(torch.bfloat16)
    s_t = oracle.attn_scores(q, k, [30], 3, 3)
    s_n = oracle.attn_scores(q.double().numpy(), k.double().numpy(), [30], 3, 3)
    assert np.array_equal(s_t, s_n, equal_nan=True)


def test_negative_control_differs_from_dropkv():
    # the attention-only score is a different ranking from DropKV's: on a seeded
    # workload the two orders are not the same and the evict sets differ
    spec = W.small_spec(1)
    wl = W.generate(spec, 42)
    s_dk = oracle.scores(wl.q, wl.k, wl.v, wl.lengths, spec.window, spec.pool)
    s_at = oracle.attn_scores(wl.q, wl.k, wl.lengths, spec.window, spec.pool)
    L = wl.lengths[0]
    hist = L - spec.window
    for h in range(spec.Hkv):
        a, b = s_dk[0, h, :hist], s_at[0, h, :hist]
        ra, rb = np.argsort(np.argsort(a)), np.argsort(np.argsort(b))
        rho = np.corrcoef(ra, rb)[0, 1]  # Spearman rank correlation
        assert rho < 0.9, (h, rho)
    _, ev_dk = oracle.select(s_dk, wl.lengths, wl.keep)
    _, ev_at = oracle.select(s_at, wl.lengths, wl.keep)
    assert not np.array_equal(ev_dk, ev_at)
