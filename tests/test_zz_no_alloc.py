"""dropkv_select_noalloc: the eviction step for callers that cannot allocate.

Callers such as a serving engine that owns every byte of device memory through
its own pool (or a path that cannot afford cudaMalloc's implicit device
synchronisation) cannot hand dropkv_select a workspace.  dropkv_select_noalloc
takes none and uses a 4 KiB scratch array compiled into the library.  This
test calls it through the C ABI twice in a row and checks that both calls give
exactly the keep / evict lists of dropkv_select and of the oracle's selection
on the same scores (integer outputs: exact), also for a launch of more than 64
batch rows (sliced on the host).

The file is named so that pytest collects it last.
"""

import ctypes

import numpy as np
import pytest
import torch

import kv_cache_eviction_scores_b200 as dk
import oracle

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _bind():
    L = dk.lib()
    i32, vp = ctypes.c_int32, ctypes.c_void_p
    ip = ctypes.POINTER(ctypes.c_int32)
    L.dropkv_select_noalloc.argtypes = [i32, i32, i32, vp, ip, ip, vp, i32, vp, i32, vp]
    L.dropkv_select_noalloc.restype = i32
    return L


def _arr(vals):
    return (ctypes.c_int32 * len(vals))(*[int(x) for x in vals])


def _scores(B, Hkv, n_max, lengths, seed):
    rng = np.random.default_rng(seed)
    s = rng.integers(0, 64, size=(B, Hkv, n_max)).astype(np.float32) / 16.0  # many ties
    for b, L in enumerate(lengths):
        s[b, :, max(0, L - 4): L] = np.inf
        s[b, :, L:] = np.nan
    return torch.from_numpy(s).to(DEV)


def test_noalloc_select_matches_select_on_two_calls_in_a_row():
    L = _bind()
    B, Hkv, n_max = 3, 4, 20000
    lengths = [20000, 9000, 4097]
    keep = [1000, 4500, 4097]
    scores = _scores(B, Hkv, n_max, lengths, 11)
    ref_keep, ref_ev = dk.dropkv_select(scores, keep, lengths)
    torch.cuda.synchronize()
    max_keep, max_evict = ref_keep.shape[2], ref_ev.shape[2]
    o_keep, o_ev = oracle.select(scores.cpu().numpy(), lengths, keep, max_keep, max_evict)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        keep_idx = torch.full((B, Hkv, max_keep), 7, dtype=torch.int32, device=DEV)
        ev_idx = torch.full((B, Hkv, max_evict), 7, dtype=torch.int32, device=DEV)
        st = L.dropkv_select_noalloc(B, Hkv, n_max, ctypes.c_void_p(scores.data_ptr()),
                                     _arr(lengths), _arr(keep), ctypes.c_void_p(keep_idx.data_ptr()),
                                     max_keep, ctypes.c_void_p(ev_idx.data_ptr()), max_evict, stream)
        assert st == dk.OK, f"call {call}: status {st}"
        torch.cuda.synchronize()
        assert torch.equal(keep_idx, ref_keep), f"call {call}: keep lists differ"
        assert torch.equal(ev_idx, ref_ev), f"call {call}: evict lists differ"
        assert np.array_equal(keep_idx.cpu().numpy(), o_keep), f"call {call}: keep vs oracle"
        assert np.array_equal(ev_idx.cpu().numpy(), o_ev), f"call {call}: evict vs oracle"


def test_noalloc_select_many_rows_matches_select():
    L = _bind()
    B, Hkv, n_max = 70, 4, 300  # more than 64 rows: two host-side slices
    rng = np.random.default_rng(5)
    lengths = [int(x) for x in rng.integers(1, n_max + 1, size=B)]
    keep = [int(rng.integers(0, Lb + 1)) for Lb in lengths]
    scores = _scores(B, Hkv, n_max, lengths, 3)
    ref_keep, ref_ev = dk.dropkv_select(scores, keep, lengths)
    torch.cuda.synchronize()
    max_keep, max_evict = ref_keep.shape[2], ref_ev.shape[2]
    keep_idx = torch.full((B, Hkv, max_keep), 7, dtype=torch.int32, device=DEV)
    ev_idx = torch.full((B, Hkv, max_evict), 7, dtype=torch.int32, device=DEV)
    st = L.dropkv_select_noalloc(B, Hkv, n_max, ctypes.c_void_p(scores.data_ptr()), _arr(lengths),
                                 _arr(keep), ctypes.c_void_p(keep_idx.data_ptr()), max_keep,
                                 ctypes.c_void_p(ev_idx.data_ptr()), max_evict, None)
    assert st == dk.OK
    torch.cuda.synchronize()
    assert torch.equal(keep_idx, ref_keep) and torch.equal(ev_idx, ref_ev)
    o_keep, o_ev = oracle.select(scores.cpu().numpy(), lengths, keep, max_keep, max_evict)
    assert np.array_equal(keep_idx.cpu().numpy(), o_keep)
    assert np.array_equal(ev_idx.cpu().numpy(), o_ev)
