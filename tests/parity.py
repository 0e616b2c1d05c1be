"""Comparison rules shared by the GPU parity tests.

Scores: per element |gpu - oracle| <= tol * |oracle|; elements whose oracle
value is below 1e-30 in magnitude are compared absolutely (<= 1e-30); +inf and
NaN positions must coincide exactly.
Evict sets: identical, except that a position may differ when its oracle score
lies within tol * |T| of T, the oracle's E-th smallest score (a tie at the
tolerance level).  Separately, the GPU selection must equal the oracle's
selection run on the GPU's own scores exactly (integer work on the same input).
"""

import numpy as np

import oracle


def assert_scores_close(gpu, ref, tol, what=""):
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.array_equal(np.isnan(g), np.isnan(r)), f"{what}: NaN pattern differs"
    assert np.array_equal(np.isposinf(g), np.isposinf(r)), f"{what}: +inf pattern differs"
    m = np.isfinite(r)
    assert np.all(np.isfinite(g[m])), f"{what}: non-finite GPU score where the oracle is finite"
    err = np.abs(g[m] - r[m])
    tiny = np.abs(r[m]) < 1e-30
    bad = np.where(tiny, err > 1e-30, err > tol * np.abs(r[m]))
    if bad.any():
        rel = err / np.maximum(np.abs(r[m]), 1e-300)
        i = int(np.argmax(np.where(tiny, 0, rel)))
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} scores outside rel {tol}; "
                             f"worst rel {rel[i]:.3e} (gpu {g[m][i]!r}, oracle {r[m][i]!r})")
    finite = np.abs(r[m]) >= 1e-30
    return float((err[finite] / np.abs(r[m][finite])).max()) if finite.any() else 0.0


def assert_evict_sets_match(gpu_evict, ref_scores, lengths, keep, tol, what=""):
    ref_scores = np.asarray(ref_scores, dtype=np.float64)
    B, Hkv, _ = ref_scores.shape
    _, ref_ev = oracle.select(ref_scores, lengths, keep, max_evict=gpu_evict.shape[2])
    for b in range(B):
        E = int(lengths[b]) - int(keep[b])
        for h in range(Hkv):
            g = set(int(x) for x in gpu_evict[b, h] if x >= 0)
            r = set(int(x) for x in ref_ev[b, h] if x >= 0)
            assert len(g) == E, f"{what}: ({b},{h}) evicted {len(g)} of {E}"
            if g == r:
                continue
            s = ref_scores[b, h, : lengths[b]]
            T = np.sort(s)[E - 1]
            for j in g ^ r:
                assert abs(s[j] - T) <= tol * abs(T) + 1e-30, (
                    f"{what}: ({b},{h}) position {j} differs; oracle score {s[j]!r}, "
                    f"threshold {T!r}")


def assert_select_exact(gpu_scores, lengths, keep, gpu_keep, gpu_evict, what=""):
    ref_keep, ref_ev = oracle.select(np.asarray(gpu_scores, dtype=np.float64), lengths, keep,
                                     max_keep=gpu_keep.shape[2], max_evict=gpu_evict.shape[2])
    assert np.array_equal(ref_keep, gpu_keep), f"{what}: keep lists differ"
    assert np.array_equal(ref_ev, gpu_evict), f"{what}: evict lists differ"


def dominant_key_case(tau, *, dtype, d, L, Hq, Hkv=1, w=1, seed=9):
    """One dominant key at position 0 whose probability misses 1 by about tau
    for every window query: q rows are the unit vector e_0, key 0 is
    x0 sqrt(d) e_0 with x0 = ln((L - 1)(1 - tau) / tau), every other key is 0
    (logit 0), values are N(0, 1).  Returns (q, k, v, tau_exact) where
    tau_exact = 1 - p_0 of the first window query, computed in fp64 from the
    stored tensors (the later window queries see more zero keys, so their
    1 - p_0 is a little larger)."""
    import torch
    P = L - w  # position of the first window query: it sees keys 0..P
    x0 = np.log(P * (1.0 - tau) / tau)
    q = torch.zeros(1, Hq, w, d, dtype=torch.float64)
    q[..., 0] = 1.0
    k = torch.zeros(1, Hkv, L, d, dtype=torch.float64)
    k[:, :, 0, 0] = x0 * np.sqrt(d)
    g = torch.Generator().manual_seed(seed)
    v = torch.randn(1, Hkv, L, d, generator=g, dtype=torch.float64)
    q, k, v = q.to(dtype), k.to(dtype), v.to(dtype)
    logit0 = float(k[0, 0, 0, 0].double()) * float(q[0, 0, 0, 0].double()) / np.sqrt(d)
    s = P * np.exp(-logit0)  # the other P visible keys have logit 0
    return q, k, v, s / (1.0 + s)
