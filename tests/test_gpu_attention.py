"""GPU parity of the attention-only score against the fp64 CPU oracle.

The write-up ("DropKV：精确单项输出扰动评分组件", section 结果与独立对照)
measures DropKV against a control that scores each cached token by the
attention probability it receives, summed over the window queries.  The
library computes it through the same C ABI (dropkv_options.score =
DROPKV_SCORE_ATTENTION) with the same GQA mean-merge, MaxPool1D and +inf on
the window; the oracle is ``oracle.attn_scores``.  Tolerances and the
evict-set / exact-selection rules are those of the perturbation score.
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
TOL_F32 = 1e-6
TOL_BF16 = 1e-3


def _paths(spec):
    shape = dk.Shape(spec.B, spec.Hq, spec.Hkv, spec.n_max, spec.d, spec.window, spec.pool,
                     0 if spec.dtype == "bf16" else 1)
    out = ["simt"]
    if dk.auto_path(shape) == dk.PATH_TENSOR:
        out.append("tensor")
    return out


def _check_whole(wl, tol, path, what):
    ref = oracle.attn_scores(wl.q, wl.k, wl.lengths, wl.spec.window, wl.spec.pool)
    q, k, v = wl.q.to(DEV), wl.k.to(DEV), wl.v.to(DEV)
    s = dk.dropkv_scores(q, k, v, wl.spec.window, wl.spec.pool, wl.lengths, path=path,
                         score="attention")
    keep_idx, ev_idx = dk.dropkv_select(s, wl.keep, wl.lengths)
    torch.cuda.synchronize()
    s, keep_idx, ev_idx = s.cpu().numpy(), keep_idx.cpu().numpy(), ev_idx.cpu().numpy()
    assert_scores_close(s, ref, tol, what)
    assert_evict_sets_match(ev_idx, ref, wl.lengths, wl.keep, tol, what)
    assert_select_exact(s, wl.lengths, wl.keep, keep_idx, ev_idx, what)


@pytest.mark.parametrize("seed", [42, 43, 44])
@pytest.mark.parametrize("path", ["auto", "simt"])
def test_attention_protocol_shape_fp32(seed, path):
    wl = W.generate(W.config_spec(0), seed)
    _check_whole(wl, TOL_F32, path, f"attn cfg0 seed {seed} {path}")


@pytest.mark.parametrize("idx", [1, 2, 3, 4])
def test_attention_small_configs(idx):
    spec = W.small_spec(idx)
    wl = W.generate(spec, 42)
    for path in _paths(spec):
        _check_whole(wl, TOL_BF16, path, f"attn {spec.name} {path}")


EDGE = [
    W.Spec("min_len", B=2, Hq=2, Hkv=2, d=16, lengths=[2, 5], window=1, pool=3, keep=[1, 3],
           dtype="f32", n_max=6),
    W.Spec("ragged_pool1", B=3, Hq=8, Hkv=2, d=64, lengths=[129, 255, 300], window=4, pool=1,
           keep=[20, 40, 100], dtype="bf16", n_max=301),
    W.Spec("f32_d5_g3", B=2, Hq=6, Hkv=2, d=5, lengths=[70, 33], window=5, pool=5,
           keep=[35, 6], dtype="f32"),
    # tensor-path shape with NaN-poisoned padding and tails inside the window
    W.Spec("nan_pad_tc", B=2, Hq=8, Hkv=2, d=128, lengths=[140, 389], window=16, pool=7,
           keep=[16, 100], dtype="bf16", n_max=400, nan_pad=True),
    # several query chunks per KV head on the tensor path (G * w = 256 rows)
    W.Spec("chunks_tc", B=1, Hq=8, Hkv=1, d=128, lengths=[777], window=32, pool=5,
           keep=[100], dtype="bf16"),
]


@pytest.mark.parametrize("spec", EDGE, ids=[s.name for s in EDGE])
def test_attention_edge_cases(spec):
    wl = W.generate(spec, 5)
    tol = TOL_F32 if spec.dtype == "f32" else TOL_BF16
    for path in _paths(spec):
        _check_whole(wl, tol, path, f"attn {spec.name} {path}")


def test_attention_full_128k_head_rows():
    """The 128K-token configuration at full size: the whole score row of two
    KV heads against the oracle run on those heads alone."""
    spec = W.config_spec(3)
    wl = W.generate(spec, 42)
    G = spec.G
    q, k, v = wl.q.to(DEV), wl.k.to(DEV), wl.v.to(DEV)
    for path in _paths(spec):
        s = dk.dropkv_scores(q, k, v, spec.window, spec.pool, wl.lengths, path=path,
                             score="attention")
        torch.cuda.synchronize()
        s = s.cpu().numpy()
        for (b, h) in [(0, 0), (0, spec.Hkv - 1)]:
            L = wl.lengths[b]
            ref = oracle.attn_scores(wl.q[b:b + 1, h * G:(h + 1) * G], wl.k[b:b + 1, h:h + 1],
                                     [L], spec.window, spec.pool)
            assert_scores_close(s[b, h, :L], ref[0, 0, :L], TOL_BF16, f"attn 128k {path} ({b},{h})")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_attention_score_is_never_singular(dtype):
    """A window probability that rounds to 1 makes the removal score singular
    but leaves the attention score well defined (p itself)."""
    import math
    d, L, w = 128, 300, 4
    g = torch.Generator().manual_seed(9)
    q = torch.randn(1, 2, w, d, generator=g) * 0.1
    q[..., 0] = 1.0
    k = torch.randn(1, 1, L, d, generator=g) * 0.1
    v = torch.randn(1, 1, L, d, generator=g)
    k[0, 0, 77, 0] = 100.0 * math.sqrt(d)
    q, k, v = q.to(dtype), k.to(dtype), v.to(dtype)
    ref = oracle.attn_scores(q, k, [L], w, 3)
    spec = W.Spec("s", 1, 2, 1, 128, [L], w, 3, [10], "bf16" if dtype == torch.bfloat16 else "f32")
    for path in _paths(spec):
        status = torch.full((1,), -1, dtype=torch.int32, device=DEV)
        s = dk.dropkv_scores(q.to(DEV), k.to(DEV), v.to(DEV), w, 3, [L], path=path,
                             status=status, score="attention")
        torch.cuda.synchronize()
        assert int(status.item()) == dk.OK
        tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
        assert_scores_close(s.cpu().numpy(), ref, tol, f"attn singular-input {path}")
