"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Tolerances: relative 1e-6 for fp32 inputs (the 4-head d=8 protocol shape),
relative 1e-3 for bf16 inputs (fp32 arithmetic from bf16-stored Q/K/V), with
the evict-set and exact-selection rules of tests/parity.py.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import kv_cache_eviction_scores_b200 as dk
from kv_cache_eviction_scores_b200 import workloads as W

from parity import (assert_evict_sets_match, assert_scores_close, assert_select_exact,
                    dominant_key_case)

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
TOL_F32 = 1e-6
TOL_BF16 = 1e-3


def _paths(spec):
    shape = dk.Shape(spec.B, spec.Hq, spec.Hkv, spec.n_max, spec.d, spec.window, spec.pool,
                     0 if spec.dtype == "bf16" else 1)
    out = ["simt"]
    if dk.auto_path(shape) == dk.PATH_TENSOR:
        out.append("tensor")
    return out


def _dev(wl):
    return wl.q.to(DEV), wl.k.to(DEV), wl.v.to(DEV)


def _run(wl, path):
    q, k, v = _dev(wl)
    s = dk.dropkv_scores(q, k, v, wl.spec.window, wl.spec.pool, wl.lengths, path=path)
    keep_idx, ev_idx = dk.dropkv_select(s, wl.keep, wl.lengths)
    torch.cuda.synchronize()
    return s.cpu().numpy(), keep_idx.cpu().numpy(), ev_idx.cpu().numpy()


def _check_whole(wl, tol, path, what):
    ref = oracle.scores(wl.q, wl.k, wl.v, wl.lengths, wl.spec.window, wl.spec.pool)
    s, keep_idx, ev_idx = _run(wl, path)
    worst = assert_scores_close(s, ref, tol, what)
    assert_evict_sets_match(ev_idx, ref, wl.lengths, wl.keep, tol, what)
    assert_select_exact(s, wl.lengths, wl.keep, keep_idx, ev_idx, what)
    return worst


# ---- the write-up's protocol shape, fp32 inputs, seeds 42/43/44 -----------

@pytest.mark.parametrize("seed", [42, 43, 44])
@pytest.mark.parametrize("path", ["auto", "simt"])
def test_protocol_shape_fp32(seed, path):
    wl = W.generate(W.config_spec(0), seed)
    _check_whole(wl, TOL_F32, path, f"cfg0 seed {seed} {path}")


# ---- scaled-down versions of the four bf16 configurations -----------------

@pytest.mark.parametrize("idx", [1, 2, 3, 4])
def test_small_configs(idx):
    spec = W.small_spec(idx)
    wl = W.generate(spec, 42)
    for path in _paths(spec):
        _check_whole(wl, TOL_BF16, path, f"{spec.name} {path}")


# The full-size configurations are compared whole, with the oracle's evict
# sets, in tests/test_gpu_full.py.

# ---- edge cases -------------------------------------------------------------

EDGE = [
    # minimum length (w + 1), single window query, one query head per KV head
    W.Spec("min_len", B=2, Hq=2, Hkv=2, d=16, lengths=[2, 5], window=1, pool=3, keep=[1, 3],
           dtype="f32", n_max=6),
    # ragged tails around the 128-token tiles, pooling off
    W.Spec("ragged_pool1", B=3, Hq=8, Hkv=2, d=64, lengths=[129, 255, 300], window=4, pool=1,
           keep=[20, 40, 100], dtype="bf16", n_max=301),
    # wide pooling window, head dim 256
    W.Spec("pool31_d256", B=1, Hq=4, Hkv=1, d=256, lengths=[400], window=8, pool=31,
           keep=[50], dtype="bf16"),
    # fp32, odd head dim, GQA group 3
    W.Spec("f32_d5_g3", B=2, Hq=6, Hkv=2, d=5, lengths=[70, 33], window=5, pool=5,
           keep=[35, 6], dtype="f32"),
    # more batch rows than one launch slice holds
    W.Spec("batch70", B=70, Hq=2, Hkv=1, d=8, lengths=[10 + (b * 7) % 40 for b in range(70)],
           window=3, pool=3, keep=[5 + (b % 4) for b in range(70)], dtype="f32", n_max=60),
    # more batch rows than one launch slice holds, on the tensor path
    W.Spec("batch66_tc", B=66, Hq=4, Hkv=1, d=128,
           lengths=[130 + (b * 37) % 170 for b in range(66)], window=8, pool=5,
           keep=[20 + (b % 7) for b in range(66)], dtype="bf16", n_max=300),
    # NaN-poisoned padding with the tensor-path shape
    W.Spec("nan_pad_tc", B=2, Hq=8, Hkv=2, d=128, lengths=[140, 389], window=16, pool=7,
           keep=[16, 100], dtype="bf16", n_max=400, nan_pad=True),
]


@pytest.mark.parametrize("spec", EDGE, ids=[s.name for s in EDGE])
def test_edge_cases(spec):
    wl = W.generate(spec, 5)
    tol = TOL_F32 if spec.dtype == "f32" else TOL_BF16
    for path in _paths(spec):
        _check_whole(wl, tol, path, f"{spec.name} {path}")


# ---- singular input: rejected, no epsilon ----------------------------------

def _singular_case(dtype):
    d, L, w = 128, 300, 4
    g = torch.Generator().manual_seed(9)
    q = torch.randn(1, 2, w, d, generator=g) * 0.1
    q[..., 0] = 1.0
    k = torch.randn(1, 1, L, d, generator=g) * 0.1
    v = torch.randn(1, 1, L, d, generator=g)
    k[0, 0, 77, 0] = 100.0 * math.sqrt(d)  # logit about 100 above every other one
    return q.to(dtype), k.to(dtype), v.to(dtype), L, w


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_singular_input_is_rejected(dtype):
    q, k, v, L, w = _singular_case(dtype)
    with pytest.raises(oracle.SingularError):
        oracle.scores(q, k, v, [L], w, 3)
    shape = dk.make_shape(q, k, w, 3)
    for path in _paths(W.Spec("s", 1, 2, 1, 128, [L], w, 3, [10],
                              "bf16" if dtype == torch.bfloat16 else "f32")):
        with pytest.raises(dk.SingularError):
            dk.dropkv_scores(q.to(DEV), k.to(DEV), v.to(DEV), w, 3, [L], path=path)
        status = torch.full((1,), -1, dtype=torch.int32, device=DEV)
        dk.dropkv_scores(q.to(DEV), k.to(DEV), v.to(DEV), w, 3, [L], path=path, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == dk.ERR_SINGULAR
    assert dk.auto_path(shape) in (dk.PATH_SIMT, dk.PATH_TENSOR)


# The rule at its boundary (write-up, Algorithm 1 paragraph: rejected, no
# epsilon).  fp32 inputs run in fp64 on the SIMT path, which applies the
# oracle's reading exactly: p_j rounding to 1 in fp32 (1 - p <= 2^-25) is
# singular, 1 - p = 4e-8 (rounds to 1 - 2^-24) is scored, at 1e-6.
@pytest.mark.parametrize("tau,singular", [(1e-6, False), (4e-8, False), (2.5e-8, True),
                                          (1e-9, True)])
def test_singular_boundary_fp32_simt(tau, singular):
    L, w = 40, 1
    q, k, v, t = dominant_key_case(tau, dtype=torch.float32, d=1, L=L, Hq=1, w=w)
    assert (np.float32(1.0 - t) == np.float32(1.0)) == singular
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    if singular:
        with pytest.raises(oracle.SingularError):
            oracle.scores(q, k, v, [L], w, 1)
        with pytest.raises(dk.SingularError):
            dk.dropkv_scores(qd, kd, vd, w, 1, [L], path="simt")
        return
    ref = oracle.scores(q, k, v, [L], w, 1)
    s = dk.dropkv_scores(qd, kd, vd, w, 1, [L], path="simt")
    torch.cuda.synchronize()
    assert_scores_close(s.cpu().numpy(), ref, TOL_F32, f"tau {tau}")


# On the fp32-arithmetic paths (bf16 inputs: SIMT and tensor core) the rule is
# the fp32 complement L - e not > 0.  Where it can differ from the oracle's
# (1 - p within a few fp32 ulps of 2^-25) the fp32 paths cannot score to 1e-3
# anyway, so the margins are: 1 - p ~ 1e-9 must be rejected, and p ~ 0.9
# (1 - p ~ 0.1) must be scored to the bf16 tolerance.
@pytest.mark.parametrize("tau,singular", [(0.1, False), (1e-9, True)])
def test_singular_boundary_bf16(tau, singular):
    L, w, Hq = 200, 1, 16  # G * w = 16: the tensor-core shape
    q, k, v, t = dominant_key_case(tau, dtype=torch.bfloat16, d=128, L=L, Hq=Hq, w=w)
    spec = W.Spec("dominant", 1, Hq, 1, 128, [L], w, 1, [10], "bf16")
    paths = _paths(spec)
    assert "tensor" in paths
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    if singular:
        with pytest.raises(oracle.SingularError):
            oracle.scores(q, k, v, [L], w, 1)
        for path in paths:
            with pytest.raises(dk.SingularError):
                dk.dropkv_scores(qd, kd, vd, w, 1, [L], path=path)
        return
    ref = oracle.scores(q, k, v, [L], w, 1)
    for path in paths:
        s = dk.dropkv_scores(qd, kd, vd, w, 1, [L], path=path)
        torch.cuda.synchronize()
        assert_scores_close(s.cpu().numpy(), ref, TOL_BF16, f"tau {tau} {path}")


def test_nonsingular_async_status_is_ok():
    wl = W.generate(W.config_spec(0), 42)
    q, k, v = _dev(wl)
    status = torch.full((1,), -1, dtype=torch.int32, device=DEV)
    dk.dropkv_scores(q, k, v, 3, 3, wl.lengths, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == dk.OK


# ---- selection on constructed scores (ties, +inf, NaN padding) --------------

# The launch picks the cluster size (1, 2, 4 or 8 CTAs) from the longest row
# and, when 8-CTA clusters would need a second wave, 4-CTA clusters with
# 32768-key ranges: the cases below reach every kind.  "ties" and the other
# short cases: one CTA per segment; "long": 2; "mid": 4; "eight": 8 CTAs with
# ragged rows; "wide": 8 CTAs with 32768-key ranges; "many_rows": 20 segments
# of ~100K keys on 4-CTA clusters with 32768-key ranges; "huge": uncached
# ranges.
@pytest.mark.parametrize("case", ["ties", "keep_all", "evict_all", "long", "mid", "eight",
                                  "wide", "many_rows", "huge", "nan_in_range"])
def test_select_exact_on_constructed_scores(case):
    rng = np.random.default_rng(3)
    if case == "long":
        B, Hkv, n_max, lengths = 2, 3, 20000, [20000, 13001]
    elif case == "mid":
        B, Hkv, n_max, lengths = 2, 2, 60000, [60000, 33001]
    elif case == "eight":
        B, Hkv, n_max, lengths = 2, 2, 120000, [120000, 70001]
    elif case == "wide":
        B, Hkv, n_max, lengths = 1, 2, 200000, [200000]
    elif case == "many_rows":
        B, Hkv, n_max = 20, 1, 100000
        lengths = [100000 - 997 * b for b in range(B)]
    elif case == "huge":
        # per-CTA ranges of 37500 keys: past the shared-memory key cache, three
        # sub-ranges per CTA read from global memory
        B, Hkv, n_max, lengths = 2, 2, 300000, [300000, 140001]
    else:
        B, Hkv, n_max, lengths = 3, 2, 5000, [5000, 4097, 1]
    s = rng.integers(0, 50, size=(B, Hkv, n_max)).astype(np.float32) / 8.0
    for b, L in enumerate(lengths):
        s[b, :, max(0, L - 3): L] = np.inf
        s[b, :, L:] = np.nan
    if case == "nan_in_range":  # NaN scores inside [0, L) order above +inf
        s[0, :, 17:40] = np.nan
        s[1, 1, :100] = np.nan
    if case == "keep_all":
        keep = list(lengths)
    elif case == "evict_all":
        keep = [0] * B
    else:
        keep = [max(0, L // 3) for L in lengths]
    gs = torch.from_numpy(s).to(DEV)
    keep_idx, ev_idx = dk.dropkv_select(gs, keep, lengths)
    torch.cuda.synchronize()
    assert_select_exact(s, lengths, keep, keep_idx.cpu().numpy(), ev_idx.cpu().numpy(), case)


# ---- window attention outputs (optional extra outputs) ----------------------

@pytest.mark.parametrize("spec", [W.config_spec(0), W.small_spec(4)], ids=["cfg0", "cfg4_small"])
def test_window_attention_outputs(spec):
    wl = W.generate(spec, 42)
    raw, attn_ref, stats_ref, st, _ = oracle.raw_scores(wl.q, wl.k, wl.v, wl.lengths,
                                                        want_attn=True)
    q, k, v = _dev(wl)
    for path in _paths(spec):
        s, attn, stats = dk.dropkv_scores(q, k, v, spec.window, spec.pool, wl.lengths,
                                          path=path, return_attn=True)
        torch.cuda.synchronize()
        a = attn.cpu().numpy().astype(np.float64)
        scale = np.abs(attn_ref).max(axis=-1, keepdims=True)
        assert np.all(np.abs(a - attn_ref) <= 1e-4 * scale + 1e-6), path
        # the (max, normaliser) pair is defined up to a common shift: compare
        # the normaliser at the oracle's max (= l * exp(m_gpu - m_oracle)).
        st_g = stats.cpu().numpy().astype(np.float64)
        l_at_ref = st_g[..., 1] * np.exp(st_g[..., 0] - stats_ref[..., 0])
        np.testing.assert_allclose(l_at_ref, stats_ref[..., 1], rtol=1e-4)
