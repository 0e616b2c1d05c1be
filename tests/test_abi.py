"""The C ABI loads, exports every declared symbol and rejects bad arguments on
the host, before any device work (no GPU needed).

Only arguments that fail host-side validation are passed here, so no call
below can reach a kernel launch even on a machine with a GPU.
"""

import ctypes
import os
import re

import pytest
import torch

import kv_cache_eviction_scores_b200 as dk

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dropkv.h")


def _declared():
    text = open(HEADER).read()
    return re.findall(r"DROPKV_API\s+[\w\s\*]+?\b(dropkv_\w+)\s*\(", text)


def test_header_declares_the_entry_points():
    names = set(_declared())
    assert {"dropkv_scores", "dropkv_scores_async", "dropkv_scores_ex", "dropkv_select",
            "dropkv_select_ex", "dropkv_scores_workspace_bytes", "dropkv_select_workspace_bytes",
            "dropkv_status_string", "dropkv_abi_version"} <= names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(dk.lib_path())
    for name in _declared():
        assert hasattr(lib, name), f"{name} declared in include/dropkv.h but not exported"


def test_abi_version_matches_header():
    text = open(HEADER).read()
    ver = int(re.search(r"#define DROPKV_ABI_VERSION (\d+)", text).group(1))
    assert dk.lib().dropkv_abi_version() == ver


def test_status_strings():
    L = dk.lib()
    for s in range(6):
        assert L.dropkv_status_string(s)
    assert b"singular" in L.dropkv_status_string(dk.ERR_SINGULAR)


def _shape(**kw):
    base = dict(B=1, Hq=32, Hkv=8, n_max=4096, d=128, window=32, pool_kernel=7, dtype=0)
    base.update(kw)
    return dk.Shape(*[base[n] for n in ("B", "Hq", "Hkv", "n_max", "d", "window",
                                        "pool_kernel", "dtype")])


def test_workspace_sizes():
    good = _shape()
    ws = dk.scores_workspace_bytes(good)
    assert ws > 0
    # at least stats + attention output + one partial-score plane
    assert ws >= 32 * 32 * (128 + 2) * 4 + 8 * 4096 * 4
    assert dk.scores_workspace_bytes(_shape(pool_kernel=4)) == 0
    assert dk.scores_workspace_bytes(_shape(Hq=30)) == 0
    assert dk.scores_workspace_bytes(_shape(d=300)) == 0
    assert dk.scores_workspace_bytes(_shape(window=4096)) == 0
    assert dk.select_workspace_bytes(1, 8, 131072) >= 4  # the device status word
    assert dk.select_workspace_bytes(0, 8, 10) == 0


@pytest.mark.parametrize("bad", [
    dict(B=0), dict(Hq=0), dict(Hkv=3), dict(d=0), dict(d=257), dict(window=0),
    dict(n_max=32), dict(pool_kernel=0), dict(pool_kernel=6), dict(pool_kernel=1025),
    dict(dtype=7),
])
def test_bad_shapes_are_rejected_on_the_host(bad):
    s = _shape(**bad)
    fake = ctypes.c_void_p(0x100000)
    st = dk.lib().dropkv_scores(ctypes.byref(s), fake, fake, fake, None, fake, fake, 1 << 30,
                                None)
    assert st == dk.ERR_ARG


def test_bad_lengths_and_pointers_are_rejected_on_the_host():
    s = _shape()
    fake = ctypes.c_void_p(0x100000)
    L = dk.lib()
    for lens in ([32], [4097], [0]):
        arr = (ctypes.c_int32 * 1)(*lens)
        assert L.dropkv_scores(ctypes.byref(s), fake, fake, fake, arr, fake, fake, 1 << 30,
                               None) == dk.ERR_ARG
    assert L.dropkv_scores(ctypes.byref(s), None, fake, fake, None, fake, fake, 1 << 30,
                           None) == dk.ERR_ARG
    odd = ctypes.c_void_p(0x100004)  # not 16-byte aligned
    assert L.dropkv_scores(ctypes.byref(s), odd, fake, fake, None, fake, fake, 1 << 30,
                           None) == dk.ERR_ARG
    # async variant needs a status pointer
    assert L.dropkv_scores_async(ctypes.byref(s), fake, fake, fake, None, fake, fake, 1 << 30,
                                 None, None) == dk.ERR_ARG


def test_unknown_score_kind_is_rejected_on_the_host():
    s = _shape()
    fake = ctypes.c_void_p(0x100000)
    L = dk.lib()
    for bad in (-1, 2, 99):
        opts = dk.Options(dk.PATH_AUTO, bad, None, None, None, 0, 0)
        assert L.dropkv_scores_ex(ctypes.byref(s), fake, fake, fake, None, fake, fake, 1 << 30,
                                  None, None, ctypes.byref(opts)) == dk.ERR_ARG
    with pytest.raises(ValueError):
        dk.dropkv_scores(torch.zeros(1, 4, 2, 8), torch.zeros(1, 2, 8, 8), torch.zeros(1, 2, 8, 8),
                         2, 1, score="bogus")


def test_small_or_missing_workspace_is_rejected_on_the_host():
    s = _shape()
    fake = ctypes.c_void_p(0x100000)
    need = dk.scores_workspace_bytes(s)
    L = dk.lib()
    assert L.dropkv_scores(ctypes.byref(s), fake, fake, fake, None, fake, fake, need - 1,
                           None) == dk.ERR_WORKSPACE
    assert L.dropkv_scores(ctypes.byref(s), fake, fake, fake, None, fake, None, need,
                           None) == dk.ERR_WORKSPACE


def test_select_rejects_bad_arguments_on_the_host():
    L = dk.lib()
    fake = ctypes.c_void_p(0x100000)
    lens = (ctypes.c_int32 * 2)(100, 50)
    keep_ok = (ctypes.c_int32 * 2)(10, 5)
    keep_bad = (ctypes.c_int32 * 2)(10, 51)
    ws = dk.select_workspace_bytes(2, 4, 100)
    assert L.dropkv_select(2, 4, 100, fake, lens, keep_bad, fake, 64, fake, 90, fake, ws,
                           None) == dk.ERR_ARG
    assert L.dropkv_select(2, 4, 100, fake, lens, keep_ok, fake, 5, fake, 90, fake, ws,
                           None) == dk.ERR_ARG   # max_keep too small
    assert L.dropkv_select(2, 4, 100, fake, lens, keep_ok, fake, 10, fake, 80, fake, ws,
                           None) == dk.ERR_ARG   # max_evict too small
    assert L.dropkv_select(2, 4, 100, fake, lens, keep_ok, fake, 10, fake, 90, fake, ws - 1,
                           None) == dk.ERR_WORKSPACE


def test_path_planning_is_host_only():
    s = _shape()
    p = dk.auto_path(s)
    assert p in (dk.PATH_SIMT, dk.PATH_TENSOR)
    assert dk.auto_path(_shape(dtype=1)) == dk.PATH_SIMT        # fp32 inputs
    assert dk.auto_path(_shape(d=64)) == dk.PATH_SIMT           # other head dims
    assert dk.auto_path(_shape(pool_kernel=2)) == -1
    assert dk.scores_launches(s, None, "simt") == 3
    assert dk.scores_launches(_shape(B=65, n_max=64, window=4), None, "simt") == 6  # 2 slices
    assert dk.select_launches(1, 8, 131072) >= 1


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_no_device_means_unsupported_not_a_cpu_fallback():
    s = _shape(B=1, Hq=2, Hkv=1, n_max=8, d=4, window=2, pool_kernel=3, dtype=1)
    fake = ctypes.c_void_p(0x100000)
    need = dk.scores_workspace_bytes(s)
    st = dk.lib().dropkv_scores(ctypes.byref(s), fake, fake, fake, None, fake, fake, need, None)
    assert st == dk.ERR_UNSUPPORTED


def test_last_cuda_error_starts_clear():
    L = dk.lib()
    assert L.dropkv_last_cuda_error() == 0
    assert L.dropkv_last_cuda_error_string() == b"cudaSuccess"


def test_wait_selftest_rejects_bad_arguments_on_the_host():
    L = dk.lib()
    fake = ctypes.c_void_p(0x100000)
    assert L.dropkv_selftest_wait_timeout(None, 1000, None) == dk.ERR_ARG
    assert L.dropkv_selftest_wait_timeout(ctypes.c_void_p(0x100002), 1000, None) == dk.ERR_ARG
    assert L.dropkv_selftest_wait_timeout(fake, 0, None) == dk.ERR_ARG
    assert L.dropkv_selftest_wait_timeout(fake, 2_000_000_000, None) == dk.ERR_ARG
    if not torch.cuda.is_available():
        assert L.dropkv_selftest_wait_timeout(fake, 1000, None) == dk.ERR_UNSUPPORTED


def test_noalloc_select_rejects_bad_arguments_on_the_host():
    L = dk.lib()
    i32, vp = ctypes.c_int32, ctypes.c_void_p
    ip = ctypes.POINTER(ctypes.c_int32)
    fn = L.dropkv_select_noalloc
    fn.argtypes = [i32, i32, i32, vp, ip, ip, vp, i32, vp, i32, vp]
    fn.restype = i32
    fake = ctypes.c_void_p(0x100000)
    lens = (ctypes.c_int32 * 2)(100, 50)
    keep_ok = (ctypes.c_int32 * 2)(10, 5)
    keep_bad = (ctypes.c_int32 * 2)(10, 51)
    assert fn(0, 4, 100, fake, lens, keep_ok, fake, 10, fake, 90, None) == dk.ERR_ARG
    assert fn(2, 4, 100, None, lens, keep_ok, fake, 10, fake, 90, None) == dk.ERR_ARG
    assert fn(2, 4, 100, fake, lens, keep_bad, fake, 64, fake, 90, None) == dk.ERR_ARG
    assert fn(2, 4, 100, fake, lens, keep_ok, fake, 5, fake, 90, None) == dk.ERR_ARG   # max_keep
    assert fn(2, 4, 100, fake, lens, keep_ok, fake, 10, fake, 80, None) == dk.ERR_ARG  # max_evict
    odd = ctypes.c_void_p(0x100004)  # scores not 16-byte aligned
    assert fn(2, 4, 100, odd, lens, keep_ok, fake, 10, fake, 90, None) == dk.ERR_ARG
    if not torch.cuda.is_available():
        assert fn(2, 4, 100, fake, lens, keep_ok, fake, 10, fake, 90, None) == dk.ERR_UNSUPPORTED


def test_negative_cta_budget_is_rejected_on_the_host():
    s = _shape()
    fake = ctypes.c_void_p(0x100000)
    opts = dk.Options(dk.PATH_AUTO, dk.SCORE_PERTURBATION, None, None, None, 0, -1)
    assert dk.lib().dropkv_scores_ex(ctypes.byref(s), fake, fake, fake, None, fake, fake,
                                     1 << 30, None, None, ctypes.byref(opts)) == dk.ERR_ARG


def test_select_ex_rejects_bad_arguments_on_the_host():
    L = dk.lib()
    fake = ctypes.c_void_p(0x100000)
    lens = (ctypes.c_int32 * 2)(100, 50)
    keep_ok = (ctypes.c_int32 * 2)(10, 5)
    keep_bad = (ctypes.c_int32 * 2)(10, 51)
    ws = dk.select_workspace_bytes(2, 4, 100)
    assert L.dropkv_select_ex(2, 4, 100, fake, lens, keep_bad, fake, 64, fake, 90, fake, ws,
                              None, fake) == dk.ERR_ARG
    assert L.dropkv_select_ex(2, 4, 100, fake, lens, keep_ok, fake, 10, fake, 90, fake, ws,
                              None, ctypes.c_void_p(0x100002)) == dk.ERR_ARG  # status misaligned
    assert L.dropkv_select_ex(2, 4, 100, fake, lens, keep_ok, fake, 10, fake, 90, fake, ws - 1,
                              None, fake) == dk.ERR_WORKSPACE
    if not torch.cuda.is_available():
        for status in (None, fake):
            assert L.dropkv_select_ex(2, 4, 100, fake, lens, keep_ok, fake, 10, fake, 90, fake,
                                      ws, None, status) == dk.ERR_UNSUPPORTED


def test_select_selftest_rejects_bad_arguments_on_the_host():
    L = dk.lib()
    fake = ctypes.c_void_p(0x100000)
    lens = (ctypes.c_int32 * 2)(100, 50)
    keep_ok = (ctypes.c_int32 * 2)(10, 5)
    fn = L.dropkv_selftest_select_timeout
    assert fn(2, 4, 100, fake, lens, keep_ok, fake, 10, fake, 90, None, 1000, None) == dk.ERR_ARG
    assert fn(2, 4, 100, fake, lens, keep_ok, fake, 10, fake, 90, fake, 0, None) == dk.ERR_ARG
    assert fn(2, 4, 100, fake, lens, keep_ok, fake, 10, fake, 90, fake, 2_000_000_000,
              None) == dk.ERR_ARG
    lens65 = (ctypes.c_int32 * 65)(*([100] * 65))
    keep65 = (ctypes.c_int32 * 65)(*([10] * 65))
    assert fn(65, 1, 100, fake, lens65, keep65, fake, 10, fake, 90, fake, 1000,
              None) == dk.ERR_ARG  # one launch slice at most
    if not torch.cuda.is_available():
        assert fn(2, 4, 100, fake, lens, keep_ok, fake, 10, fake, 90, fake, 1000,
                  None) == dk.ERR_UNSUPPORTED
