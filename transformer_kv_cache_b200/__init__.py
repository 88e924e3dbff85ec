"""Python binding of libkvc: the paged KV cache hot path for streaming visual-geometry
transformers on B200 (sm_100a).

Argument marshalling only: every function here has the name of the C entry point it
calls (include/kvc.h) and converts torch tensors to device pointers and statuses to
exceptions. All computation happens in the CUDA library; importing this package fails
loudly when the built library is missing.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvc.so")

KVC_F32, KVC_BF16, KVC_FP8_E4M3 = 0, 1, 2
DTYPES = {"f32": KVC_F32, "bf16": KVC_BF16, "fp8_e4m3": KVC_FP8_E4M3}
STATUS = ["KVC_OK", "KVC_ERR_ARG", "KVC_ERR_OOM", "KVC_ERR_CUDA", "KVC_ERR_STATE", "KVC_ERR_BUDGET",
          "KVC_ERR_TIMEOUT", "KVC_ERR_DEVICE", "KVC_ERR_UNSUPPORTED"]

# every symbol include/kvc.h declares
EXPORTS = ["kvc_create", "kvc_destroy", "kvc_set_stream", "kvc_reset", "kvc_append_frame", "kvc_attend",
           "kvc_attend_all", "kvc_prune_all",
           "kvc_compress", "kvc_compress_all", "kvc_page_table", "kvc_token_meta", "kvc_last_merge", "kvc_export_pages",
           "kvc_step_host", "kvc_synchronize", "kvc_last_error", "kvc_status_string", "kvc_version",
           "kvc_debug_fail_allocs", "kvc_debug_bounded_wait", "kvc_attend_paged_noalloc", "kvc_append_frame_all",
           "kvc_step_host_async", "kvc_set_layer_budgets", "kvc_prune", "kvc_layer_diversity",
           "kvc_head_tokens", "kvc_scale_phase", "kvc_export_fp8_group_scales", "kvc_last_raw_scores",
           "kvc_adapt_layer_budgets"]


class kvc_config(ctypes.Structure):
    _fields_ = [("num_layers", ctypes.c_int32), ("num_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("tokens_per_frame", ctypes.c_int32), ("num_special_tokens", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("window_frames", ctypes.c_int32), ("scale_frames", ctypes.c_int32),
                ("io_dtype", ctypes.c_int32), ("kv_dtype", ctypes.c_int32), ("softmax_scale", ctypes.c_float),
                ("budget_tokens", ctypes.c_int32), ("keep_frac", ctypes.c_float), ("lambda_", ctypes.c_float),
                ("rank_window", ctypes.c_int32), ("residual_dim", ctypes.c_int32),
                ("protect_first_frame", ctypes.c_int32), ("max_frames", ctypes.c_int32),
                ("kv_splits", ctypes.c_int32), ("diversity_budget", ctypes.c_int32),
                ("special_frames", ctypes.c_int32), ("fp8_dim_adaptive", ctypes.c_int32),
                ("model_heads", ctypes.c_int32), ("head_begin", ctypes.c_int32),
                ("reserved", ctypes.c_int32 * 2)]


class kvc_info(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in (
        "tokens", "pages_used", "pages_total", "pool_bytes", "high_water_pages", "frames_appended",
        "frames_committed", "frames_skipped", "frames_evicted", "compress_events", "device_error",
        "kernel_launches")]

    def as_dict(self):
        return {n: int(getattr(self, n)) for n, _ in self._fields_}


class KVCError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        self.status_name = STATUS[status] if 0 <= status < len(STATUS) else str(status)
        super().__init__(f"{self.status_name}: {message}")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libkvc.so is not built ({LIB_PATH}); run `python transformer_kv_cache_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64p, i32p, fp = ctypes.c_void_p, ctypes.c_int32, ctypes.POINTER(ctypes.c_int64), \
        ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_float)
    sig = {
        "kvc_create": ([ctypes.POINTER(kvc_config), vp, ctypes.POINTER(vp)], i32),
        "kvc_destroy": ([vp], i32),
        "kvc_set_stream": ([vp, vp], i32),
        "kvc_reset": ([vp], i32),
        "kvc_append_frame": ([vp, i32, i32, vp, vp, i32], i32),
        "kvc_attend": ([vp, i32, vp, vp], i32),
        "kvc_append_frame_all": ([vp, i32, ctypes.POINTER(vp), ctypes.POINTER(vp), i32], i32),
        "kvc_attend_all": ([vp, ctypes.POINTER(vp), ctypes.POINTER(vp)], i32),
        "kvc_compress": ([vp, i32, vp, i32p], i32),
        "kvc_compress_all": ([vp, ctypes.POINTER(vp), i32p], i32),
        "kvc_page_table": ([vp, i32, i32p, i32, i32p, ctypes.POINTER(kvc_info)], i32),
        "kvc_token_meta": ([vp, i32, i64p, i32p, fp, i32, i32p], i32),
        "kvc_last_merge": ([vp, i32, i64p, i64p, i32, i32p], i32),
        "kvc_last_raw_scores": ([vp, vp, i32, i32p], i32),
        "kvc_export_pages": ([vp, i32, i32, i32, vp, vp, fp, fp], i32),
        "kvc_step_host": ([vp, i32, i32, i32, vp, vp, vp, vp], i32),
        "kvc_step_host_async": ([vp, i32, i32, i32, vp, vp, vp, vp], i32),
        "kvc_set_layer_budgets": ([vp, vp, i32], i32),
        "kvc_adapt_layer_budgets": ([vp, ctypes.c_double, i32, vp], i32),
        "kvc_prune": ([vp, i32], i32),
        "kvc_prune_all": ([vp], i32),
        "kvc_scale_phase": ([vp, i32, i32, vp, vp, vp, vp], i32),
        "kvc_export_fp8_group_scales": ([vp, i32, i32, i32, vp, vp], i32),
        "kvc_layer_diversity": ([vp, i32, vp], i32),
        "kvc_head_tokens": ([vp, i32, i32, vp, i32, vp], i32),
        "kvc_synchronize": ([vp], i32),
        "kvc_last_error": ([vp], ctypes.c_char_p),
        "kvc_status_string": ([i32], ctypes.c_char_p),
        "kvc_version": ([], i32),
        "kvc_debug_fail_allocs": ([i32], i32),
        "kvc_debug_bounded_wait": ([vp, i32], i32),
        "kvc_attend_paged_noalloc": ([vp, vp, vp, vp, ctypes.c_int64, vp, i32, i32, i32, i32, i32, ctypes.c_float,
                                      i32, vp], i32),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    return lib


_lib = _load()


def _ptr(x) -> Optional[int]:
    """Device/host pointer of a torch tensor, numpy array, or an int."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if isinstance(x, np.ndarray):
        return x.ctypes.data
    return x.data_ptr()


def _dptr(x) -> Optional[int]:
    """Device pointer of a CUDA tensor, or an int taken as a device address. A host buffer
    (numpy array or CPU tensor) is refused here, before a kernel could read it."""
    if x is None or isinstance(x, int):
        return x
    if isinstance(x, np.ndarray) or not getattr(x, "is_cuda", False):
        raise TypeError("a CUDA tensor (or a device address) is expected here, not a host buffer")
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(handle, st: int):
    if st != 0:
        msg = _lib.kvc_last_error(handle).decode() if handle else ""
        raise KVCError(st, msg)


def make_config(num_layers, num_heads, head_dim, tokens_per_frame, num_special_tokens, page_size,
                window_frames, scale_frames, io_dtype="bf16", kv_dtype="bf16", softmax_scale=0.125,
                budget_tokens=0, keep_frac=0.6, lam=0.5, rank_window=5, residual_dim=1024,
                protect_first_frame=1, max_frames=0, kv_splits=0, diversity_budget=0,
                special_frames=0, fp8_dim_adaptive=0, model_heads=0, head_begin=0) -> kvc_config:
    c = kvc_config()
    c.num_layers, c.num_heads, c.head_dim = num_layers, num_heads, head_dim
    c.tokens_per_frame, c.num_special_tokens, c.page_size = tokens_per_frame, num_special_tokens, page_size
    c.window_frames, c.scale_frames = window_frames, scale_frames
    c.io_dtype = DTYPES[io_dtype] if isinstance(io_dtype, str) else io_dtype
    c.kv_dtype = DTYPES[kv_dtype] if isinstance(kv_dtype, str) else kv_dtype
    c.softmax_scale = softmax_scale
    c.budget_tokens, c.keep_frac, c.lambda_ = budget_tokens, keep_frac, lam
    c.rank_window, c.residual_dim, c.protect_first_frame = rank_window, residual_dim, protect_first_frame
    c.max_frames, c.kv_splits = max_frames, kv_splits
    c.diversity_budget = diversity_budget
    c.special_frames = special_frames
    c.fp8_dim_adaptive = fp8_dim_adaptive
    c.model_heads, c.head_begin = model_heads, head_begin
    return c


def config_from_workload(wl, **over) -> kvc_config:
    d = dict(num_layers=wl.num_layers, num_heads=wl.num_heads, head_dim=wl.head_dim,
             tokens_per_frame=wl.tokens_per_frame, num_special_tokens=wl.num_special_tokens,
             page_size=wl.page_size, window_frames=wl.window_frames, scale_frames=wl.scale_frames,
             io_dtype=wl.io_dtype, kv_dtype=wl.kv_dtype, softmax_scale=wl.softmax_scale,
             budget_tokens=wl.budget_tokens, keep_frac=wl.keep_frac, lam=wl.lam, rank_window=wl.rank_window,
             residual_dim=wl.residual_dim, protect_first_frame=wl.protect_first_frame,
             diversity_budget=getattr(wl, "diversity_budget", 0),
             special_frames=getattr(wl, "special_frames", 0),
             fp8_dim_adaptive=getattr(wl, "fp8_dim_adaptive", 0))
    d.update(over)
    return make_config(**d)


# ---------------------------------------------------------------- entry points (same names as the C ABI)

def kvc_version() -> int:
    return int(_lib.kvc_version())


def kvc_create(cfg: kvc_config, stream=None) -> int:
    h = ctypes.c_void_p()
    st = _lib.kvc_create(ctypes.byref(cfg), _stream(stream), ctypes.byref(h))
    if st != 0:
        raise KVCError(st, "kvc_create failed")
    return h.value


def kvc_destroy(handle) -> None:
    _check(handle, _lib.kvc_destroy(handle))


def kvc_set_stream(handle, stream) -> None:
    _check(handle, _lib.kvc_set_stream(handle, _stream(stream)))


def kvc_reset(handle) -> None:
    _check(handle, _lib.kvc_reset(handle))


def kvc_append_frame(handle, layer: int, frame_idx: int, k, v, is_keyframe: bool = True) -> None:
    _check(handle, _lib.kvc_append_frame(handle, layer, frame_idx, _dptr(k), _dptr(v), int(bool(is_keyframe))))


def kvc_append_frame_all(handle, frame_idx: int, ks, vs, is_keyframe: bool = True) -> None:
    """ks, vs: per-layer device tensors (or pointers), one per layer."""
    n = len(ks)
    ka = (ctypes.c_void_p * n)(*[_dptr(k) for k in ks])
    va = (ctypes.c_void_p * n)(*[_dptr(v) for v in vs])
    _check(handle, _lib.kvc_append_frame_all(handle, frame_idx, ka, va, int(bool(is_keyframe))))


def kvc_attend(handle, layer: int, q, o) -> None:
    _check(handle, _lib.kvc_attend(handle, layer, _dptr(q), _dptr(o)))


def kvc_attend_all(handle, qs, os) -> None:
    """qs, os: per-layer device tensors (or pointers), one per layer of the cache."""
    n = len(qs)
    qa = (ctypes.c_void_p * n)(*[_dptr(q) for q in qs])
    oa = (ctypes.c_void_p * n)(*[_dptr(o) for o in os])
    _check(handle, _lib.kvc_attend_all(handle, qa, oa))


def kvc_compress(handle, layer: int, residual) -> bool:
    fired = ctypes.c_int32(0)
    _check(handle, _lib.kvc_compress(handle, layer, _dptr(residual), ctypes.byref(fired)))
    return bool(fired.value)


def kvc_compress_all(handle, residuals) -> list:
    """residuals: per-layer device fp32 tensors (or pointers), one per layer of the cache.
    Returns, per layer, whether a compression ran."""
    n = len(residuals)
    ra = (ctypes.c_void_p * n)(*[_dptr(r) for r in residuals])
    fired = (ctypes.c_int32 * n)()
    _check(handle, _lib.kvc_compress_all(handle, ra, fired))
    return [bool(f) for f in fired]


def kvc_page_table(handle, layer: int):
    """(rows int32 [n, 4] = owner, page_in_owner, phys_page, valid; info dict)"""
    n = ctypes.c_int32(0)
    info = kvc_info()
    _check(handle, _lib.kvc_page_table(handle, layer, None, 0, ctypes.byref(n), ctypes.byref(info)))
    rows = np.zeros((max(n.value, 1), 4), np.int32)
    _check(handle, _lib.kvc_page_table(handle, layer, rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                       n.value, ctypes.byref(n), ctypes.byref(info)))
    return rows[: n.value], info.as_dict()


def kvc_token_meta(handle, layer: int, capacity: int = 1 << 22):
    ids = np.zeros(capacity, np.int64)
    cnt = np.zeros(capacity, np.int32)
    sh = np.zeros(capacity, np.float32)
    n = ctypes.c_int32(0)
    _check(handle, _lib.kvc_token_meta(handle, layer, ids.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                       cnt.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                       sh.ctypes.data_as(ctypes.POINTER(ctypes.c_float)), capacity,
                                       ctypes.byref(n)))
    k = n.value
    return ids[:k], cnt[:k], sh[:k]


def kvc_last_merge(handle, layer: int, capacity: int = 1 << 20):
    src = np.zeros(capacity, np.int64)
    dst = np.zeros(capacity, np.int64)
    n = ctypes.c_int32(0)
    _check(handle, _lib.kvc_last_merge(handle, layer, src.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                       dst.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), capacity,
                                       ctypes.byref(n)))
    return src[: n.value], dst[: n.value]


def kvc_last_raw_scores(handle, capacity: int = 1 << 16):
    """Raw scores s (fp32, one per token slot) of the last kvc_compress call."""
    s = np.zeros(capacity, np.float32)
    n = ctypes.c_int32(0)
    _check(handle, _lib.kvc_last_raw_scores(handle, s.ctypes.data_as(ctypes.c_void_p), capacity, ctypes.byref(n)))
    return s[: n.value]


def kvc_export_pages(handle, layer: int, first_row: int, n_rows: int, page_bytes: int, num_heads: int,
                     fp8: bool = False):
    """Raw page bytes of rows [first_row, first_row + n_rows): (k uint8 [n, page_bytes], v, k_scale, v_scale)."""
    k = np.zeros((n_rows, page_bytes), np.uint8)
    v = np.zeros((n_rows, page_bytes), np.uint8)
    ks = np.zeros((n_rows, num_heads), np.float32) if fp8 else None
    vs = np.zeros((n_rows, num_heads), np.float32) if fp8 else None
    fptr = lambda a: a.ctypes.data_as(ctypes.POINTER(ctypes.c_float)) if a is not None else None
    _check(handle, _lib.kvc_export_pages(handle, layer, first_row, n_rows, k.ctypes.data, v.ctypes.data,
                                         fptr(ks), fptr(vs)))
    return k, v, ks, vs


def kvc_step_host(handle, layer: int, frame_idx: int, is_keyframe: bool, q_host, k_host, v_host, o_host) -> None:
    _check(handle, _lib.kvc_step_host(handle, layer, frame_idx, int(bool(is_keyframe)), _ptr(q_host),
                                      _ptr(k_host), _ptr(v_host), _ptr(o_host)))


def kvc_step_host_async(handle, layer: int, frame_idx: int, is_keyframe: bool, q_host, k_host, v_host,
                        o_host) -> None:
    """Enqueue one host-buffer step and return; the buffers must stay alive (and o_host
    unread) until kvc_synchronize."""
    _check(handle, _lib.kvc_step_host_async(handle, layer, frame_idx, int(bool(is_keyframe)), _ptr(q_host),
                                            _ptr(k_host), _ptr(v_host), _ptr(o_host)))


def kvc_set_layer_budgets(handle, budgets) -> None:
    arr = (ctypes.c_int32 * len(budgets))(*[int(b) for b in budgets])
    _check(handle, _lib.kvc_set_layer_budgets(handle, arr, len(budgets)))


def kvc_scale_phase(handle, layer: int, n_frames: int, q, k, v, o) -> None:
    """The joint scale-frame phase: frames 0..n_frames-1 ([n_frames*T, H, D] tensors)
    appended, committed, and attended bidirectionally."""
    _check(handle, _lib.kvc_scale_phase(handle, layer, n_frames, _dptr(q), _dptr(k), _dptr(v), _dptr(o)))


def kvc_export_fp8_group_scales(handle, layer: int, first_row: int, n_rows: int, H: int, D: int, P: int):
    """Dimension-adaptive FP8 scales of page-table rows: K [n, H, D], V [n, H, P] (float32)."""
    kc = np.zeros((n_rows, H, D), np.float32)
    vt = np.zeros((n_rows, H, P), np.float32)
    _check(handle, _lib.kvc_export_fp8_group_scales(handle, layer, first_row, n_rows,
                                                    kc.ctypes.data, vt.ctypes.data))
    return kc, vt


def kvc_prune(handle, layer: int) -> None:
    """Prune every head of `layer` to its Top-K candidates (the step before kvc_attend)."""
    _check(handle, _lib.kvc_prune(handle, layer))


def kvc_prune_all(handle) -> None:
    _check(handle, _lib.kvc_prune_all(handle))


def kvc_adapt_layer_budgets(handle, num_layers: int, tau: float, k_avg: int) -> np.ndarray:
    """Budgets floor(L * k_avg * softmax(mean diversity / tau)), clamped to [1, diversity_budget],
    computed by the library from every layer's last pruning and applied from the next one
    (num_layers: the cache's layer count, the length of the returned array)."""
    out = np.zeros(num_layers, np.int32)
    _check(handle, _lib.kvc_adapt_layer_budgets(handle, float(tau), int(k_avg), out.ctypes.data))
    return out


def kvc_layer_diversity(handle, layer: int) -> float:
    out = ctypes.c_double()
    _check(handle, _lib.kvc_layer_diversity(handle, layer, ctypes.byref(out)))
    return float(out.value)


def kvc_head_tokens(handle, layer: int, head: int, capacity: int = 1 << 20):
    ids = np.zeros(capacity, np.int64)
    n = ctypes.c_int32()
    _check(handle, _lib.kvc_head_tokens(handle, layer, head, ids.ctypes.data, capacity, ctypes.byref(n)))
    return ids[: n.value].copy()


def kvc_synchronize(handle) -> None:
    _check(handle, _lib.kvc_synchronize(handle))


def kvc_last_error(handle) -> str:
    return _lib.kvc_last_error(handle).decode()


def kvc_status_string(status: int) -> str:
    return _lib.kvc_status_string(status).decode()


def kvc_debug_fail_allocs(n: int) -> None:
    _lib.kvc_debug_fail_allocs(n)


def kvc_debug_bounded_wait(handle, timeout_us: int) -> None:
    _check(handle, _lib.kvc_debug_bounded_wait(handle, timeout_us))


def kvc_attend_paged_noalloc(q, o, k_pool, v_pool, pool_pages: int, page_table, n_pages: int, tokens: int,
                             num_heads: int, head_dim: int, page_size: int, softmax_scale: float,
                             kv_splits: int = 1, stream=None) -> None:
    """Attention over caller-owned pools with no device allocation (see include/kvc.h)."""
    st = _lib.kvc_attend_paged_noalloc(_dptr(q), _dptr(o), _dptr(k_pool), _dptr(v_pool), pool_pages, _dptr(page_table),
                                       n_pages, tokens, num_heads, head_dim, page_size, softmax_scale, kv_splits,
                                       _stream(stream))
    if st != 0:
        raise KVCError(st, "kvc_attend_paged_noalloc failed")


@dataclass
class KVCache:
    """Owning wrapper: creates the cache and destroys it when closed."""
    cfg: kvc_config
    handle: int = 0

    def __post_init__(self):
        self.handle = kvc_create(self.cfg)

    def close(self):
        if self.handle:
            kvc_destroy(self.handle)
            self.handle = 0

    def __enter__(self):
        return self

    def __exit__(self, *a):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
