"""fp64 CPU oracle for DropKV eviction scoring -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  It shares no code with the CUDA library:
``dropkv_oracle.c`` is plain C compiled with gcc, and ``bruteforce.py`` is an
independent numpy delete-and-re-softmax checker.

Parity status of each function (how it is pinned, see tests/test_oracle_pins.py):
  raw_scores      pinned: brute-force deletion, uniform-attention closed form,
                  two-token closed form (tests/golden), scaling, permutation
  merge           pinned: G=1 identity, duplicated query heads
  pool_protect    pinned: brute-force sliding max, k=1 identity, window = +inf
  select          pinned: brute-force full sort, constant-V all-ties case
  scores_at       pinned: equals the whole-problem oracle on sampled positions
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

from . import build as _build

OK, ERR_ARG, ERR_SINGULAR = 0, 1, 2

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int32)
        i = ctypes.c_int
        L.oracle_raw_scores.argtypes = [i, i, i, i, i, i, dp, dp, dp, ip, dp, dp, dp, ip]
        L.oracle_raw_scores.restype = i
        L.oracle_merge.argtypes = [i, i, i, i, dp, ip, dp]
        L.oracle_merge.restype = None
        L.oracle_pool_protect.argtypes = [i, i, i, i, i, dp, ip, dp]
        L.oracle_pool_protect.restype = None
        L.oracle_scores.argtypes = [i, i, i, i, i, i, i, dp, dp, dp, ip, dp, dp, dp, dp, dp, ip]
        L.oracle_scores.restype = i
        L.oracle_scores_at.argtypes = [i, i, i, i, i, dp, dp, dp, i, ip, dp]
        L.oracle_scores_at.restype = i
        L.oracle_select.argtypes = [i, i, i, dp, ip, ip, i, i, ip, ip]
        L.oracle_select.restype = i
        L.oracle_attn_raw.argtypes = [i, i, i, i, i, i, dp, dp, ip, dp]
        L.oracle_attn_raw.restype = i
        _lib = L
    return _lib


class SingularError(RuntimeError):
    """A window probability rounds to 1: exact single removal is undefined."""


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor: exact upcast of bf16 / fp32
        import torch
        a = a.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _p(a, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def raw_scores(q, k, v, lengths, *, want_attn=False, raise_singular=True):
    """Per query head scores s[b, hq, j] summed over the window; NaN padding.

    Returns (raw, attn_out or None, stats or None, status, singular_at).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, w, d = q.shape
    _, Hkv, n_max, _ = k.shape
    lens = _i32(lengths)
    raw = np.empty((B, Hq, n_max))
    attn = np.empty((B, Hq, w, d)) if want_attn else None
    stats = np.empty((B, Hq, w, 2)) if want_attn else None
    sing = np.full(4, -1, dtype=np.int32)
    st = lib().oracle_raw_scores(
        B, Hq, Hkv, n_max, d, w, _p(q, ctypes.c_double), _p(k, ctypes.c_double),
        _p(v, ctypes.c_double), _p(lens, ctypes.c_int32), _p(raw, ctypes.c_double),
        _p(attn, ctypes.c_double) if attn is not None else None,
        _p(stats, ctypes.c_double) if stats is not None else None, _p(sing, ctypes.c_int32))
    if st == ERR_ARG:
        raise ValueError("oracle: bad shape or lengths")
    if st == ERR_SINGULAR and raise_singular:
        raise SingularError(f"singular at (b, hq, t, j) = {tuple(sing)}")
    return raw, attn, stats, st, tuple(int(x) for x in sing)


def merge(raw, Hkv, lengths):
    raw = _f64(raw)
    B, Hq, n_max = raw.shape
    out = np.empty((B, Hkv, n_max))
    lens = _i32(lengths)
    lib().oracle_merge(B, Hq, Hkv, n_max, _p(raw, ctypes.c_double), _p(lens, ctypes.c_int32),
                       _p(out, ctypes.c_double))
    return out


def pool_protect(merged, window, pool, lengths):
    merged = _f64(merged)
    B, Hkv, n_max = merged.shape
    out = np.empty_like(merged)
    lens = _i32(lengths)
    lib().oracle_pool_protect(B, Hkv, n_max, window, pool, _p(merged, ctypes.c_double),
                              _p(lens, ctypes.c_int32), _p(out, ctypes.c_double))
    return out


def scores(q, k, v, lengths, window, pool, *, raise_singular=True, intermediates=False):
    """Final fp64 scores [B, Hkv, n_max]: merged, pooled, window = +inf, pad NaN."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, w, d = q.shape
    if w != window:
        raise ValueError("q must hold exactly the window rows")
    _, Hkv, n_max, _ = k.shape
    lens = _i32(lengths)
    out = np.empty((B, Hkv, n_max))
    merged = np.empty((B, Hkv, n_max))
    raw = np.empty((B, Hq, n_max))
    sing = np.full(4, -1, dtype=np.int32)
    st = lib().oracle_scores(
        B, Hq, Hkv, n_max, d, w, pool, _p(q, ctypes.c_double), _p(k, ctypes.c_double),
        _p(v, ctypes.c_double), _p(lens, ctypes.c_int32), _p(out, ctypes.c_double),
        _p(merged, ctypes.c_double), _p(raw, ctypes.c_double), None, None,
        _p(sing, ctypes.c_int32))
    if st == ERR_ARG:
        raise ValueError("oracle: bad shape, lengths or pool kernel")
    if st == ERR_SINGULAR and raise_singular:
        raise SingularError(f"singular at (b, hq, t, j) = {tuple(sing)}")
    if intermediates:
        return out, merged, raw, st
    return out


def attn_raw(q, k, lengths):
    """Attention-only raw score per query head: sum over the window queries of
    the attention probability each token receives (NaN padding)."""
    q, k = _f64(q), _f64(k)
    B, Hq, w, d = q.shape
    _, Hkv, n_max, _ = k.shape
    lens = _i32(lengths)
    raw = np.empty((B, Hq, n_max))
    st = lib().oracle_attn_raw(B, Hq, Hkv, n_max, d, w, _p(q, ctypes.c_double),
                               _p(k, ctypes.c_double), _p(lens, ctypes.c_int32),
                               _p(raw, ctypes.c_double))
    if st == ERR_ARG:
        raise ValueError("oracle: bad shape or lengths")
    return raw


def attn_scores(q, k, lengths, window, pool):
    """Final attention-only scores [B, Hkv, n_max]: merged, pooled, window = +inf."""
    q = _f64(q)
    if q.shape[2] != window:
        raise ValueError("q must hold exactly the window rows")
    k = _f64(k)
    return pool_protect(merge(attn_raw(q, k, lengths), k.shape[1], lengths), window, pool, lengths)


def scores_at(Qg, K, V, window, pool, positions: Sequence[int]):
    """Final scores of one KV head at ``positions``.

    Qg: [G, w, d] query group, K, V: [L, d] (exactly the valid rows).
    """
    Qg, K, V = _f64(Qg), _f64(K), _f64(V)
    G, w, d = Qg.shape
    L = K.shape[0]
    pos = _i32(positions)
    out = np.empty(len(pos))
    st = lib().oracle_scores_at(G, L, d, w, pool, _p(Qg, ctypes.c_double),
                                _p(K, ctypes.c_double), _p(V, ctypes.c_double), len(pos),
                                _p(pos, ctypes.c_int32), _p(out, ctypes.c_double))
    if st == ERR_ARG:
        raise ValueError("oracle: bad arguments")
    if st == ERR_SINGULAR:
        raise SingularError("singular input")
    return out


def select(scores_arr, lengths, keep, max_keep: Optional[int] = None,
           max_evict: Optional[int] = None):
    """Keep / evict position lists per (b, h), sorted, padded with -1."""
    s = np.ascontiguousarray(scores_arr, dtype=np.float64)
    B, Hkv, n_max = s.shape
    lens, kp = _i32(lengths), _i32(keep)
    if max_keep is None:
        max_keep = int(kp.max())
    if max_evict is None:
        max_evict = int((lens - kp).max())
    keep_idx = np.empty((B, Hkv, max(max_keep, 0)), dtype=np.int32)
    evict_idx = np.empty((B, Hkv, max(max_evict, 0)), dtype=np.int32)
    st = lib().oracle_select(B, Hkv, n_max, _p(s, ctypes.c_double), _p(lens, ctypes.c_int32),
                             _p(kp, ctypes.c_int32), max_keep, max_evict,
                             _p(keep_idx, ctypes.c_int32), _p(evict_idx, ctypes.c_int32))
    if st != OK:
        raise ValueError("oracle_select: bad arguments")
    return keep_idx, evict_idx


def num_threads() -> int:
    """OpenMP threads the oracle uses (OMP_NUM_THREADS, else the core count)."""
    env = os.environ.get("OMP_NUM_THREADS")
    if env:
        return int(env)
    return os.cpu_count() or 1
