"""Seeded synthetic inputs for DropKV prefill-time eviction scoring.

This module only draws numbers; it holds none of the scoring arithmetic, so
both the CUDA path and the CPU oracle can read the same stored tensors.

Shapes follow the write-up's local protocol ("DropKV：精确单项输出扰动评分组件",
section 数据协议与运行: 1 batch, 4 query heads, 2 KV heads, 19 history slots,
3 window queries, d=8, seeds 42/43/44, evict 7) and Llama-3.1-8B-shaped long
contexts (Hq=32, Hkv=8, d=128; the atlas summary's "Key results" and
"Experimental setup" name Llama-3.1-8B, Qwen2.5-7B-1M and Mistral-7B-512K at
4K-128K).  RULER/LongBench items are not used; these synthetic tensors stand in
for them.

Draw order (fixed, so a seed names one input set): q, k, v as fp32 N(0,1)
from ``torch.Generator().manual_seed(seed)``, then the optional extras
(outlier channels, heavy keys), then the cast to the storage dtype with
round-to-nearest-even.  Padding rows (positions >= the sequence length) can be
poisoned with NaN.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional

import torch


@dataclass
class Spec:
    """Shape and value recipe of one synthetic scoring problem."""

    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    lengths: List[int]
    window: int
    pool: int
    keep: List[int]
    dtype: str = "bf16"            # storage dtype of q, k, v: "bf16" or "f32"
    n_max: Optional[int] = None     # padded cache length (default: max length)
    k_scale: float = 1.0            # multiply K before the cast
    outlier_channels: int = 0       # per KV head, this many K channels scaled
    outlier_scale: float = 8.0
    heavy_per_head: int = 0         # planted keys aligned with window queries
    heavy_cos: float = 0.9
    nan_pad: bool = False           # poison K/V rows at positions >= length

    def __post_init__(self):
        if self.n_max is None:
            self.n_max = max(self.lengths)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv


@dataclass
class Workload:
    spec: Spec
    seed: int
    q: torch.Tensor          # [B, Hq, w, d]  window queries (tail-aligned)
    k: torch.Tensor          # [B, Hkv, n_max, d]
    v: torch.Tensor          # [B, Hkv, n_max, d]
    lengths: List[int]
    keep: List[int]
    extras: dict = field(default_factory=dict)

    @property
    def tokens(self) -> int:
        return int(sum(self.lengths))


def budget(frac: float, length: int) -> int:
    """Keep count for a keep-budget fraction: floor(frac * length)."""
    return int(math.floor(frac * length))


def config_spec(idx: int) -> Spec:
    """The five benchmark configurations (full sizes)."""
    if idx == 0:
        # 19 history slots + 3 window queries, evict 7 of 22.
        return Spec("cfg0_tiny_f32", B=1, Hq=4, Hkv=2, d=8, lengths=[22], window=3,
                    pool=3, keep=[22 - 7], dtype="f32")
    if idx == 1:
        n = 4096
        return Spec("cfg1_gqa_4k", B=1, Hq=32, Hkv=8, d=128, lengths=[n], window=32,
                    pool=7, keep=[budget(0.20, n)], k_scale=1.0 / math.sqrt(128))
    if idx == 2:
        n = 32768
        return Spec("cfg2_llama_32k_heavy", B=1, Hq=32, Hkv=8, d=128, lengths=[n],
                    window=32, pool=7, keep=[budget(0.05, n)], heavy_per_head=16)
    if idx == 3:
        n = 131072
        return Spec("cfg3_llama_128k", B=1, Hq=32, Hkv=8, d=128, lengths=[n], window=64,
                    pool=7, keep=[budget(0.05, n)], outlier_channels=4)
    if idx == 4:
        ls = [16384, 32768, 65536, 131072]
        fr = [0.05, 0.10, 0.20, 0.05]
        return Spec("cfg4_batched_mixed", B=4, Hq=28, Hkv=4, d=128, lengths=ls, window=32,
                    pool=7, keep=[budget(f, L) for f, L in zip(fr, ls)], nan_pad=True)
    raise ValueError(f"no config {idx}")


def small_spec(idx: int) -> Spec:
    """Scaled-down versions of configs 1-4 with the same structure.

    Sizes span several 128-token tiles and end in a ragged tail, so the oracle
    finishes in seconds while every tile-boundary case of the kernels is hit.
    """
    if idx == 1:
        n = 1000
        return Spec("cfg1_small", B=1, Hq=32, Hkv=8, d=128, lengths=[n], window=32,
                    pool=7, keep=[budget(0.20, n)], k_scale=1.0 / math.sqrt(128))
    if idx == 2:
        n = 1500
        return Spec("cfg2_small_heavy", B=1, Hq=32, Hkv=8, d=128, lengths=[n], window=32,
                    pool=7, keep=[budget(0.05, n)], heavy_per_head=16)
    if idx == 3:
        n = 1337
        return Spec("cfg3_small_outlier", B=1, Hq=32, Hkv=8, d=128, lengths=[n], window=64,
                    pool=7, keep=[budget(0.05, n)], outlier_channels=4)
    if idx == 4:
        ls = [200, 517, 1024, 1300]
        fr = [0.05, 0.10, 0.20, 0.05]
        return Spec("cfg4_small_mixed", B=4, Hq=28, Hkv=4, d=128, lengths=ls, window=32,
                    pool=7, keep=[max(32, budget(f, L)) for f, L in zip(fr, ls)],
                    n_max=1400, nan_pad=True)
    raise ValueError(f"no small config {idx}")


def generate(spec: Spec, seed: int = 42) -> Workload:
    """Draw one seeded input set for ``spec`` on the CPU."""
    B, Hq, Hkv, d, w, n_max = spec.B, spec.Hq, spec.Hkv, spec.d, spec.window, spec.n_max
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, w, d, generator=g)
    k = torch.randn(B, Hkv, n_max, d, generator=g)
    v = torch.randn(B, Hkv, n_max, d, generator=g)
    if spec.k_scale != 1.0:
        k.mul_(spec.k_scale)
    extras = {}
    if spec.outlier_channels:
        chans = torch.empty(B, Hkv, spec.outlier_channels, dtype=torch.long)
        for b in range(B):
            for h in range(Hkv):
                c = torch.randperm(d, generator=g)[: spec.outlier_channels]
                chans[b, h] = c
                k[b, h][:, c] *= spec.outlier_scale
        extras["outlier_channels"] = chans
    store = torch.bfloat16 if spec.dtype == "bf16" else torch.float32
    q = q.to(store)
    if spec.heavy_per_head:
        # Heavy key i of a KV head is aligned (cosine heavy_cos) with one window
        # query of its group, taken round-robin over the group's (g, t) rows.
        qd = q.to(torch.float64)
        pos_all = torch.empty(B, Hkv, spec.heavy_per_head, dtype=torch.long)
        c = spec.heavy_cos
        for b in range(B):
            hist = spec.lengths[b] - w
            for h in range(Hkv):
                pos = torch.randperm(hist, generator=g)[: spec.heavy_per_head]
                pos_all[b, h] = pos
                for i in range(spec.heavy_per_head):
                    row = i % (G * w)
                    qv = qd[b, h * G + row // w, row % w]
                    qhat = qv / qv.norm()
                    u = torch.randn(d, generator=g).to(torch.float64)
                    u = u - (u @ qhat) * qhat
                    u = u / u.norm()
                    key = math.sqrt(d) * (c * qhat + math.sqrt(1.0 - c * c) * u)
                    k[b, h, int(pos[i])] = key.to(torch.float32)
        extras["heavy_positions"] = pos_all
    k = k.to(store)
    v = v.to(store)
    if spec.nan_pad:
        for b in range(B):
            L = spec.lengths[b]
            k[b, :, L:] = float("nan")
            v[b, :, L:] = float("nan")
    return Workload(spec, seed, q.contiguous(), k.contiguous(), v.contiguous(),
                    list(spec.lengths), list(spec.keep), extras)


def random_spec(rng: "torch.Generator", max_n: int = 40, dtype: str = "f32") -> Spec:
    """A small random shape (used for brute-force checks on tiny inputs)."""
    def ri(lo, hi):
        return int(torch.randint(lo, hi + 1, (1,), generator=rng))
    Hkv = ri(1, 3)
    G = ri(1, 3)
    d = ri(1, 9)
    w = ri(1, 5)
    B = ri(1, 3)
    lengths = [ri(w + 1, max_n) for _ in range(B)]
    n_max = max(lengths) + ri(0, 3)
    pool = 2 * ri(0, 3) + 1
    keep = [ri(w, L) for L in lengths]
    return Spec("random", B=B, Hq=Hkv * G, Hkv=Hkv, d=d, lengths=lengths, window=w,
                pool=pool, keep=keep, dtype=dtype, n_max=n_max)
