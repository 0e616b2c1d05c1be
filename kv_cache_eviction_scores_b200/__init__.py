"""DropKV prefill-time KV-cache eviction scoring on NVIDIA B200 (sm_100a).

A thin ctypes binding over ``libdropkv.so`` (C ABI: ``include/dropkv.h``).
It only marshals arguments: PyTorch supplies device memory and the current
stream, and every step of the scoring path runs in the library's CUDA kernels.
There is no CPU fallback; without the built library every call raises.

What is scored (write-up "DropKV：精确单项输出扰动评分组件", section 核心公式
and the Algorithm 1 paragraph): for the last ``window`` prompt queries,
p = softmax(K q / sqrt d), a = sum_j p_j v_j, Delta_j = p_j/(1-p_j) (a - v_j),
s_j = sum_t ||Delta_j||^2; scores are averaged over the query heads of each KV
head, max-pooled, the window is set to +inf, and the lowest scores are evicted.

Usage (CUDA tensors; q holds the last ``window`` query rows of each sequence)::

    import kv_cache_eviction_scores_b200 as dk
    # q [B, Hq, window, d], k / v [B, Hkv, n_max, d], bf16 or fp32
    scores = dk.dropkv_scores(q, k, v, window, pool_kernel, lengths)   # [B, Hkv, n_max]
    keep_idx, evict_idx = dk.dropkv_select(scores, keep_counts, lengths)
    # or both at once:
    scores, keep_idx, evict_idx = dk.evict(q, k, v, window, pool_kernel, keep_counts, lengths)
    # the attention-only control score through the same pipeline:
    control = dk.dropkv_scores(q, k, v, window, pool_kernel, lengths, score="attention")
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import torch

__all__ = [
    "DropKVError", "SingularError", "Shape", "Options", "lib", "lib_path",
    "make_shape", "scores_workspace_bytes", "select_workspace_bytes", "dropkv_scores",
    "dropkv_select", "evict", "auto_path", "scores_launches", "select_launches",
    "selftest_wait_timeout", "selftest_select_timeout",
    "OK", "ERR_ARG", "ERR_SINGULAR", "ERR_CUDA", "ERR_UNSUPPORTED", "ERR_WORKSPACE", "ERR_TIMEOUT",
    "PATH_AUTO", "PATH_SIMT", "PATH_TENSOR", "SCORE_PERTURBATION", "SCORE_ATTENTION",
]

OK, ERR_ARG, ERR_SINGULAR, ERR_CUDA, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_TIMEOUT = range(7)
PATH_AUTO, PATH_SIMT, PATH_TENSOR = 0, 1, 2
_PATHS = {"auto": PATH_AUTO, "simt": PATH_SIMT, "tensor": PATH_TENSOR}
SCORE_PERTURBATION, SCORE_ATTENTION = 0, 1
_SCORES = {"perturbation": SCORE_PERTURBATION, "attention": SCORE_ATTENTION}
BF16, F32 = 0, 1

_HERE = os.path.dirname(os.path.abspath(__file__))


def lib_path() -> str:
    return os.path.join(_HERE, "libdropkv.so")


class DropKVError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        msg = _status_string(status)
        super().__init__(f"{what}: {msg} (status {status})" if what else msg)


class SingularError(DropKVError):
    """Some window probability rounds to 1: exact single removal is undefined."""


class Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "Hq", "Hkv", "n_max", "d", "window", "pool_kernel", "dtype")]


class Options(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int32), ("score", ctypes.c_int32),
                ("attn_out", ctypes.c_void_p), ("stats_out", ctypes.c_void_p),
                ("events", ctypes.c_void_p), ("n_events", ctypes.c_int32),
                ("tc_ctas", ctypes.c_int32)]


_lib = None


def lib():
    """Load libdropkv.so (built in-tree by ``python -m kv_cache_eviction_scores_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    path = lib_path()
    if not os.path.exists(path):
        raise RuntimeError(f"libdropkv.so is not built ({path}); run "
                           "`python -m kv_cache_eviction_scores_b200.build`")
    L = ctypes.CDLL(path)
    vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
    ip = ctypes.POINTER(ctypes.c_int32)
    sp = ctypes.POINTER(Shape)
    L.dropkv_scores_workspace_bytes.argtypes = [sp]
    L.dropkv_scores_workspace_bytes.restype = sz
    L.dropkv_scores.argtypes = [sp, vp, vp, vp, ip, vp, vp, sz, vp]
    L.dropkv_scores.restype = i32
    L.dropkv_scores_async.argtypes = [sp, vp, vp, vp, ip, vp, vp, sz, vp, vp]
    L.dropkv_scores_async.restype = i32
    L.dropkv_scores_ex.argtypes = [sp, vp, vp, vp, ip, vp, vp, sz, vp, vp,
                                   ctypes.POINTER(Options)]
    L.dropkv_scores_ex.restype = i32
    L.dropkv_select_workspace_bytes.argtypes = [i32, i32, i32]
    L.dropkv_select_workspace_bytes.restype = sz
    L.dropkv_select.argtypes = [i32, i32, i32, vp, ip, ip, vp, i32, vp, i32, vp, sz, vp]
    L.dropkv_select.restype = i32
    L.dropkv_select_ex.argtypes = [i32, i32, i32, vp, ip, ip, vp, i32, vp, i32, vp, sz, vp, vp]
    L.dropkv_select_ex.restype = i32
    L.dropkv_auto_path.argtypes = [sp]
    L.dropkv_auto_path.restype = i32
    L.dropkv_scores_launches.argtypes = [sp, ip, i32]
    L.dropkv_scores_launches.restype = i32
    L.dropkv_select_launches.argtypes = [i32, i32, i32, ip]
    L.dropkv_select_launches.restype = i32
    L.dropkv_scores_select.argtypes = [sp, vp, vp, vp, ip, ip, vp, vp, i32, vp, i32, vp, sz, vp,
                                       vp, ctypes.POINTER(Options)]
    L.dropkv_scores_select.restype = i32
    L.dropkv_scores_select_launches.argtypes = [sp, ip, i32]
    L.dropkv_scores_select_launches.restype = i32
    L.dropkv_status_string.argtypes = [i32]
    L.dropkv_status_string.restype = ctypes.c_char_p
    L.dropkv_abi_version.argtypes = []
    L.dropkv_abi_version.restype = i32
    L.dropkv_selftest_wait_timeout.argtypes = [vp, ctypes.c_uint64, vp]
    L.dropkv_selftest_wait_timeout.restype = i32
    L.dropkv_selftest_select_timeout.argtypes = [i32, i32, i32, vp, ip, ip, vp, i32, vp, i32, vp,
                                                 ctypes.c_uint64, vp]
    L.dropkv_selftest_select_timeout.restype = i32
    L.dropkv_last_cuda_error.argtypes = []
    L.dropkv_last_cuda_error.restype = i32
    L.dropkv_last_cuda_error_string.argtypes = []
    L.dropkv_last_cuda_error_string.restype = ctypes.c_char_p
    _lib = L
    return L


def _status_string(status: int) -> str:
    try:
        return lib().dropkv_status_string(status).decode()
    except Exception:
        return f"status {status}"


def _check(status: int, what: str):
    if status == OK:
        return
    if status == ERR_SINGULAR:
        raise SingularError(status, what)
    if status == ERR_CUDA:
        what = f"{what} [{lib().dropkv_last_cuda_error_string().decode()}]"
    raise DropKVError(status, what)


def _i32_array(vals: Optional[Sequence[int]]):
    if vals is None:
        return None
    arr = (ctypes.c_int32 * len(vals))(*[int(x) for x in vals])
    return arr


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def make_shape(q: torch.Tensor, k: torch.Tensor, window: int, pool_kernel: int) -> Shape:
    B, Hq, w, d = q.shape
    Bk, Hkv, n_max, dk = k.shape
    if (B, d) != (Bk, dk) or w != window:
        raise ValueError("q must be [B, Hq, window, d] and k, v [B, Hkv, n_max, d]")
    if q.dtype == torch.bfloat16:
        dt = BF16
    elif q.dtype == torch.float32:
        dt = F32
    else:
        raise TypeError("q, k, v must be bfloat16 or float32")
    return Shape(B, Hq, Hkv, n_max, d, window, pool_kernel, dt)


def scores_workspace_bytes(shape: Shape) -> int:
    return int(lib().dropkv_scores_workspace_bytes(ctypes.byref(shape)))


def select_workspace_bytes(B: int, Hkv: int, n_max: int) -> int:
    return int(lib().dropkv_select_workspace_bytes(B, Hkv, n_max))


def auto_path(shape: Shape) -> int:
    return int(lib().dropkv_auto_path(ctypes.byref(shape)))


def scores_launches(shape: Shape, lengths=None, path: str = "auto") -> int:
    return int(lib().dropkv_scores_launches(ctypes.byref(shape), _i32_array(lengths),
                                            _PATHS[path]))


def select_launches(B: int, Hkv: int, n_max: int, lengths=None) -> int:
    return int(lib().dropkv_select_launches(B, Hkv, n_max, _i32_array(lengths)))


def scores_select_launches(shape: Shape, lengths=None, path: str = "auto") -> int:
    return int(lib().dropkv_scores_select_launches(ctypes.byref(shape), _i32_array(lengths),
                                                   _PATHS[path]))


def _check_inputs(q, k, v):
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA tensor (there is no CPU path)")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k and v must share one dtype")
    if k.shape != v.shape:
        raise ValueError("k and v must have the same shape")
    if not (q.device == k.device == v.device):
        raise ValueError("q, k and v must be on one device")


def dropkv_scores(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, window: int,
                  pool_kernel: int, lengths: Optional[Sequence[int]] = None, *,
                  path: str = "auto", out: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, return_attn: bool = False,
                  status: Optional[torch.Tensor] = None, kernel_events=None,
                  score: str = "perturbation", tc_ctas: int = 0):
    """fp32 scores [B, Hkv, n_max] (pooled, window = +inf, padding = NaN).

    q: [B, Hq, window, d] window queries; k, v: [B, Hkv, n_max, d]; lengths:
    per-row lengths (host ints) or None for n_max.  With ``status`` (a CUDA
    int32 tensor of one element) the call is asynchronous and the singular flag
    lands there; otherwise it synchronises and raises SingularError.
    With ``return_attn`` also returns the window attention outputs
    [B, Hq, window, d] and (max logit, normaliser) stats [B, Hq, window, 2].
    ``kernel_events``: torch.cuda.Event objects (each recorded once already so
    that its handle exists); events 2i / 2i+1 bracket the i-th kernel launch.
    ``score``: "perturbation" (DropKV's exact single-removal score) or
    "attention" (the accumulated window attention probability, the control
    score), same merge / pool / window handling.
    ``tc_ctas``: on the tensor path, the most CTAs a scoring pass launches
    (0 = one per SM); fewer CTAs walk longer runs of tiles each.
    """
    if score not in _SCORES:
        raise ValueError(f"score must be one of {sorted(_SCORES)}")
    _check_inputs(q, k, v)
    shape = make_shape(q, k, window, pool_kernel)
    dev = q.device
    if out is None:
        out = torch.empty(shape.B, shape.Hkv, shape.n_max, dtype=torch.float32, device=dev)
    need = scores_workspace_bytes(shape)
    if need == 0:
        raise DropKVError(ERR_ARG, "dropkv_scores_workspace_bytes")
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    opts = Options(_PATHS[path], _SCORES[score], None, None, None, 0, int(tc_ctas))
    ev_arr = None
    if kernel_events:
        # raw cudaEvent_t handles of (already recorded once) torch.cuda.Event objects
        ev_arr = (ctypes.c_void_p * len(kernel_events))(*[e.cuda_event for e in kernel_events])
        opts.events = ctypes.cast(ev_arr, ctypes.c_void_p)
        opts.n_events = len(kernel_events)
    attn = stats = None
    if return_attn:
        attn = torch.empty(shape.B, shape.Hq, window, shape.d, dtype=torch.float32, device=dev)
        stats = torch.empty(shape.B, shape.Hq, window, 2, dtype=torch.float32, device=dev)
        opts.attn_out = attn.data_ptr()
        opts.stats_out = stats.data_ptr()
    st = lib().dropkv_scores_ex(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v),
                                _i32_array(lengths), _ptr(out), _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _stream(dev),
                                _ptr(status), ctypes.byref(opts))
    _check(st, "dropkv_scores")
    if return_attn:
        return out, attn, stats
    return out


def selftest_wait_timeout(limit_ms: float = 20.0, device=None) -> int:
    """Runs the bounded-wait self-test (a wait on an mbarrier nothing arrives
    on) and returns the status word it leaves: ERR_TIMEOUT when the device-side
    wait gave up as designed."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    _check(lib().dropkv_selftest_wait_timeout(_ptr(status), int(limit_ms * 1e6), _stream(dev)),
           "dropkv_selftest_wait_timeout")
    torch.cuda.synchronize(dev)
    return int(status.item())


def selftest_select_timeout(scores: torch.Tensor, keep_counts: Sequence[int],
                            lengths: Optional[Sequence[int]] = None, limit_ms: float = 20.0):
    """Runs the select kernel with one CTA of every segment withholding an
    arrival and waits limited to ``limit_ms``; returns (status word, keep_idx,
    evict_idx).  Segments with evictions report ERR_TIMEOUT and lists of -1."""
    B, Hkv, n_max = scores.shape
    lens = list(lengths) if lengths is not None else [n_max] * B
    keep = [int(x) for x in keep_counts]
    max_keep = max(keep)
    max_evict = max(L - kc for L, kc in zip(lens, keep))
    dev = scores.device
    keep_idx = torch.full((B, Hkv, max_keep), 7, dtype=torch.int32, device=dev)
    evict_idx = torch.full((B, Hkv, max_evict), 7, dtype=torch.int32, device=dev)
    status = torch.full((1,), -1, dtype=torch.int32, device=dev)
    _check(lib().dropkv_selftest_select_timeout(
        B, Hkv, n_max, _ptr(scores), _i32_array(lengths), _i32_array(keep), _ptr(keep_idx),
        max_keep, _ptr(evict_idx), max_evict, _ptr(status), int(limit_ms * 1e6), _stream(dev)),
        "dropkv_selftest_select_timeout")
    torch.cuda.synchronize(dev)
    return int(status.item()), keep_idx, evict_idx


def dropkv_select(scores: torch.Tensor, keep_counts: Sequence[int],
                  lengths: Optional[Sequence[int]] = None, *, max_keep: Optional[int] = None,
                  max_evict: Optional[int] = None,
                  workspace: Optional[torch.Tensor] = None,
                  status: Optional[torch.Tensor] = None,
                  sync: bool = False) -> Tuple[torch.Tensor, torch.Tensor]:
    """Keep / evict positions per (b, h), ascending, padded with -1 (int32).

    Asynchronous by default.  With ``status`` (a CUDA int32 tensor of one
    element) the device-side status of the kernels (OK, or ERR_TIMEOUT if a
    bounded wait gave up) lands there; with ``sync=True`` the call waits for
    the stream and raises on a device-side error.
    """
    if not scores.is_cuda or scores.dtype != torch.float32 or not scores.is_contiguous():
        raise TypeError("scores must be a contiguous CUDA float32 tensor")
    B, Hkv, n_max = scores.shape
    lens = list(lengths) if lengths is not None else [n_max] * B
    keep = [int(x) for x in keep_counts]
    if len(keep) != B or len(lens) != B:
        raise ValueError("keep_counts and lengths need one entry per batch row")
    if max_keep is None:
        max_keep = max(keep)
    if max_evict is None:
        max_evict = max(L - kc for L, kc in zip(lens, keep))
    dev = scores.device
    keep_idx = torch.empty(B, Hkv, max_keep, dtype=torch.int32, device=dev)
    evict_idx = torch.empty(B, Hkv, max_evict, dtype=torch.int32, device=dev)
    need = select_workspace_bytes(B, Hkv, n_max)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    args = (B, Hkv, n_max, _ptr(scores), _i32_array(lengths), _i32_array(keep), _ptr(keep_idx),
            max_keep, _ptr(evict_idx), max_evict, _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream(dev))
    if status is not None or sync:
        if status is not None and (not status.is_cuda or status.dtype != torch.int32):
            raise TypeError("status must be a CUDA int32 tensor")
        st = lib().dropkv_select_ex(*args, _ptr(status))
    else:
        st = lib().dropkv_select(*args)
    _check(st, "dropkv_select")
    return keep_idx, evict_idx


def dropkv_scores_select(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, window: int,
                         pool_kernel: int, keep_counts: Sequence[int],
                         lengths: Optional[Sequence[int]] = None, *, path: str = "auto",
                         score: str = "perturbation", out: Optional[torch.Tensor] = None,
                         keep_idx: Optional[torch.Tensor] = None,
                         evict_idx: Optional[torch.Tensor] = None,
                         workspace: Optional[torch.Tensor] = None,
                         status: Optional[torch.Tensor] = None, kernel_events=None,
                         tc_ctas: int = 0):
    """Scores and the keep / evict lists in one call (dropkv_scores_select):
    (scores, keep_idx, evict_idx), the same results as dropkv_scores followed
    by dropkv_select.  With ``status`` the call is asynchronous (the device
    status lands there); otherwise it synchronises and raises on a
    device-side error.  ``kernel_events`` as for dropkv_scores."""
    if score not in _SCORES:
        raise ValueError(f"score must be one of {sorted(_SCORES)}")
    _check_inputs(q, k, v)
    shape = make_shape(q, k, window, pool_kernel)
    dev = q.device
    B, Hkv, n_max = shape.B, shape.Hkv, shape.n_max
    lens = list(lengths) if lengths is not None else [n_max] * B
    keep = [int(x) for x in keep_counts]
    if len(keep) != B or len(lens) != B:
        raise ValueError("keep_counts and lengths need one entry per batch row")
    max_keep = max(keep)
    max_evict = max(L - kc for L, kc in zip(lens, keep))
    if out is None:
        out = torch.empty(B, Hkv, n_max, dtype=torch.float32, device=dev)
    if keep_idx is None:
        keep_idx = torch.empty(B, Hkv, max_keep, dtype=torch.int32, device=dev)
    if evict_idx is None:
        evict_idx = torch.empty(B, Hkv, max_evict, dtype=torch.int32, device=dev)
    need = scores_workspace_bytes(shape)
    if need == 0:
        raise DropKVError(ERR_ARG, "dropkv_scores_workspace_bytes")
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    opts = Options(_PATHS[path], _SCORES[score], None, None, None, 0, int(tc_ctas))
    ev_arr = None
    if kernel_events:
        ev_arr = (ctypes.c_void_p * len(kernel_events))(*[e.cuda_event for e in kernel_events])
        opts.events = ctypes.cast(ev_arr, ctypes.c_void_p)
        opts.n_events = len(kernel_events)
    if status is not None and (not status.is_cuda or status.dtype != torch.int32):
        raise TypeError("status must be a CUDA int32 tensor")
    st = lib().dropkv_scores_select(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v),
                                    _i32_array(lengths), _i32_array(keep), _ptr(out),
                                    _ptr(keep_idx), keep_idx.shape[2], _ptr(evict_idx),
                                    evict_idx.shape[2], _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(dev),
                                    _ptr(status), ctypes.byref(opts))
    _check(st, "dropkv_scores_select")
    return out, keep_idx, evict_idx


def evict(q, k, v, window: int, pool_kernel: int, keep_counts: Sequence[int],
          lengths: Optional[Sequence[int]] = None, *, path: str = "auto",
          score: str = "perturbation"):
    """Scores and the keep / evict lists in one call: (scores, keep_idx, evict_idx)."""
    return dropkv_scores_select(q, k, v, window, pool_kernel, keep_counts, lengths, path=path,
                                score=score)
