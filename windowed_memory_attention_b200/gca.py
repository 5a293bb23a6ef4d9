"""ctypes binding of libgca.so — argument marshalling only.

Every function has the name and meaning of its C entry point in
``include/gca.h``; every step of the path runs in the library's kernels.
Tensors are passed as raw pointers (``tensor.data_ptr()``) with the current
torch CUDA stream; host tensors (pinned or not) are accepted too, the library
stages them.  Loading fails loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgca.so")

GCA_ALL_LAYERS = -1
GCA_HOST_ONLY = -1        # cache-create device: the page table alone (no GPU needed)
GCA_DTYPE_BF16, GCA_DTYPE_F32 = 0, 1
GCA_PAGE_IMAGE, GCA_PAGE_SUMMARY = 0, 1
GCA_MEMORY_SUMMARY, GCA_MEMORY_CAMERA, GCA_MEMORY_NONE = 0, 1, 2
GCA_ROPE_NONE, GCA_ROPE_3D = 0, 1
STATUS = {0: "GCA_OK", 1: "GCA_ERR_INVALID_ARG", 2: "GCA_ERR_CAPACITY", 3: "GCA_ERR_STATE",
          4: "GCA_ERR_UNSUPPORTED", 5: "GCA_ERR_CUDA", 6: "GCA_ERR_DEVICE_CHECK"}
EXPORTS = ("gca_cache_create", "gca_cache_destroy", "gca_append_frame", "gca_evict_to_summary",
           "gca_attend", "gca_reset", "gca_get_layout", "gca_token_slot", "gca_get_info",
           "gca_device_status", "gca_status_string", "gca_attend_pages_noalloc",
           "gca_selftest_bounded_wait", "gca_attend_transient", "gca_frame_attention",
           "gca_frame_attention_batch",
           "gca_visible_prefix")


class gca_config_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "num_layers", "num_heads", "head_dim", "image_tokens", "summary_tokens", "num_anchor",
        "window", "max_frames", "page_size", "dtype", "anchor_block", "max_query_frames",
        "frame_slack")] + [("softmax_scale", ctypes.c_float), ("trajectory_memory", ctypes.c_int32),
                           ("rope", ctypes.c_int32), ("rope_grid_w", ctypes.c_int32),
                           ("rope_base", ctypes.c_float)]


class gca_page_entry_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("page_id", "kind", "frame", "first", "n_valid")]


class gca_info_t(ctypes.Structure):
    _fields_ = [("num_pages", ctypes.c_int32), ("image_pages_per_frame", ctypes.c_int32),
                ("frames", ctypes.c_int32), ("full_frames", ctypes.c_int32),
                ("resident_tokens", ctypes.c_int64), ("k_pool", ctypes.c_void_p),
                ("v_pool", ctypes.c_void_p), ("pool_bytes", ctypes.c_size_t),
                ("scratch_bytes", ctypes.c_size_t), ("kernel_launches", ctypes.c_int64)]


class GCAError(RuntimeError):
    def __init__(self, call: str, status: int):
        super().__init__(f"{call} -> {STATUS.get(status, status)}")
        self.status = status
        self.name = STATUS.get(status, str(status))


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C-ABI library; raises if it is missing (no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libgca.so is not built ({LIB_PATH}); run "
                               "python -m windowed_memory_attention_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        sig = {
            "gca_cache_create": [ctypes.POINTER(gca_config_t), ctypes.c_int, ctypes.POINTER(vp)],
            "gca_cache_destroy": [vp],
            "gca_append_frame": [vp, i32, vp, vp, ctypes.POINTER(i64), vp],
            "gca_evict_to_summary": [vp, ctypes.POINTER(i32)],
            "gca_attend": [vp, i32, vp, i32, vp, vp, vp],
            "gca_attend_transient": [vp, i32, vp, vp, vp, vp, vp, vp],
            "gca_frame_attention": [vp, i32, vp, vp, vp, vp, vp, vp],
            "gca_frame_attention_batch": [vp, i32, i32, vp, vp, vp, vp, vp, vp],
            "gca_visible_prefix": [vp, ctypes.POINTER(gca_page_entry_t), i32, ctypes.POINTER(i32)],
            "gca_reset": [vp],
            "gca_get_layout": [vp, i32, ctypes.POINTER(gca_page_entry_t), i32, ctypes.POINTER(i32)],
            "gca_token_slot": [vp, i32, i32, ctypes.POINTER(i32), ctypes.POINTER(i32)],
            "gca_get_info": [vp, ctypes.POINTER(gca_info_t)],
            "gca_device_status": [vp, ctypes.POINTER(i32), i32],
            "gca_selftest_bounded_wait": [vp, i32, ctypes.POINTER(i32)],
            "gca_attend_pages_noalloc": [vp, vp, i32, i32, i32, i32, i32, vp, i32, vp, i32, i32,
                                         i32, i32, i32, i32, i32, ctypes.c_float, vp, vp, vp, vp],
        }
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.gca_status_string.argtypes = [ctypes.c_int]
        L.gca_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(call: str, rc: int):
    if rc != 0:
        raise GCAError(call, rc)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libgca must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream() if torch.cuda.is_available() else None
    if stream is None:
        return ctypes.c_void_p(0)
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def gca_status_string(status: int) -> str:
    return lib().gca_status_string(status).decode()


def gca_cache_create(*, num_layers: int, num_heads: int, image_tokens: int, num_anchor: int,
                     window: int, max_frames: int, summary_tokens: int = 6, head_dim: int = 64,
                     page_size: int = 128, dtype: str = "bf16", anchor_block: bool = False,
                     max_query_frames: int = 1, frame_slack: int = 0,
                     softmax_scale: float = 0.0, trajectory_memory: int = GCA_MEMORY_SUMMARY,
                     rope: int = GCA_ROPE_NONE, rope_grid_w: int = 0, rope_base: float = 0.0,
                     device: int = 0) -> ctypes.c_void_p:
    cfg = gca_config_t(num_layers, num_heads, head_dim, image_tokens, summary_tokens, num_anchor,
                       window, max_frames, page_size,
                       GCA_DTYPE_BF16 if dtype == "bf16" else GCA_DTYPE_F32,
                       int(bool(anchor_block)), max_query_frames, frame_slack, softmax_scale,
                       trajectory_memory, rope, rope_grid_w, rope_base)
    h = ctypes.c_void_p()
    _check("gca_cache_create", lib().gca_cache_create(ctypes.byref(cfg), device, ctypes.byref(h)))
    return h


def gca_cache_destroy(cache) -> None:
    _check("gca_cache_destroy", lib().gca_cache_destroy(cache))


def gca_append_frame(cache, layer: int, k: torch.Tensor, v: torch.Tensor, stream=None) -> int:
    idx = ctypes.c_int64(-1)
    _check("gca_append_frame", lib().gca_append_frame(cache, layer, _ptr(k), _ptr(v),
                                                      ctypes.byref(idx), _stream(stream)))
    return idx.value


def gca_evict_to_summary(cache) -> int:
    n = ctypes.c_int32(0)
    _check("gca_evict_to_summary", lib().gca_evict_to_summary(cache, ctypes.byref(n)))
    return n.value


def gca_attend(cache, layer: int, q: torch.Tensor, out: torch.Tensor,
               lse: Optional[torch.Tensor] = None, num_query_frames: int = 1, stream=None) -> None:
    _check("gca_attend", lib().gca_attend(cache, layer, _ptr(q), num_query_frames, _ptr(out),
                                          _ptr(lse), _stream(stream)))


def gca_attend_transient(cache, layer: int, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                         out: torch.Tensor, lse: Optional[torch.Tensor] = None, stream=None) -> None:
    _check("gca_attend_transient", lib().gca_attend_transient(cache, layer, _ptr(q), _ptr(k), _ptr(v),
                                                              _ptr(out), _ptr(lse), _stream(stream)))


def gca_frame_attention(cache, layer: int, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                        out: torch.Tensor, lse: Optional[torch.Tensor] = None, stream=None) -> None:
    _check("gca_frame_attention", lib().gca_frame_attention(cache, layer, _ptr(q), _ptr(k), _ptr(v),
                                                            _ptr(out), _ptr(lse), _stream(stream)))


def gca_frame_attention_batch(cache, layer: int, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                              out: torch.Tensor, lse: Optional[torch.Tensor] = None, stream=None) -> None:
    """q, k, v, out: [F][S+M][H][D]; lse: [F][S+M][H]."""
    _check("gca_frame_attention_batch",
           lib().gca_frame_attention_batch(cache, layer, q.shape[0], _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                           _ptr(lse), _stream(stream)))


def gca_reset(cache) -> None:
    _check("gca_reset", lib().gca_reset(cache))


def gca_get_layout(cache, num_query_frames: int = 1) -> List[Tuple[int, int, int, int, int]]:
    n = ctypes.c_int32(0)
    _check("gca_get_layout", lib().gca_get_layout(cache, num_query_frames, None, 0, ctypes.byref(n)))
    buf = (gca_page_entry_t * max(1, n.value))()
    _check("gca_get_layout", lib().gca_get_layout(cache, num_query_frames, buf, n.value,
                                                  ctypes.byref(n)))
    return [(e.page_id, e.kind, e.frame, e.first, e.n_valid) for e in buf[:n.value]]


def gca_token_slot(cache, frame: int, tau: int) -> Tuple[int, int]:
    pid, slot = ctypes.c_int32(), ctypes.c_int32()
    _check("gca_token_slot", lib().gca_token_slot(cache, frame, tau, ctypes.byref(pid),
                                                  ctypes.byref(slot)))
    return pid.value, slot.value


def gca_visible_prefix(cache, entry, query_frame: int) -> int:
    """Visible-prefix length of a walk-list entry (page_id, kind, frame, first, n_valid)."""
    e = gca_page_entry_t(*entry)
    n = ctypes.c_int32(0)
    _check("gca_visible_prefix", lib().gca_visible_prefix(cache, ctypes.byref(e), query_frame,
                                                          ctypes.byref(n)))
    return n.value


def gca_get_info(cache) -> gca_info_t:
    info = gca_info_t()
    _check("gca_get_info", lib().gca_get_info(cache, ctypes.byref(info)))
    return info


def gca_device_status(cache, clear: bool = False) -> int:
    s = ctypes.c_int32(0)
    _check("gca_device_status", lib().gca_device_status(cache, ctypes.byref(s), int(clear)))
    return s.value


def gca_attend_pages_noalloc(k_pool, v_pool, *, num_layers: int, num_pages: int, num_heads: int,
                             page_size: int, layer: int, walk, nwalk: int, q: torch.Tensor,
                             num_query_frames: int, tokens_per_frame: int, first_query_frame: int,
                             num_anchor: int, window: int, summary_tokens: int,
                             anchor_block: bool, softmax_scale: float, out: torch.Tensor,
                             lse: Optional[torch.Tensor] = None, status=None, stream=None) -> None:
    """Attention over caller-owned pools with no device allocation (see gca.h).
    ``walk`` is a ctypes array of gca_page_entry_t or a device pointer."""
    _check("gca_attend_pages_noalloc", lib().gca_attend_pages_noalloc(
        ctypes.c_void_p(k_pool), ctypes.c_void_p(v_pool), num_layers, num_pages, num_heads,
        page_size, layer, walk if not isinstance(walk, int) else ctypes.c_void_p(walk), nwalk,
        _ptr(q), num_query_frames, tokens_per_frame, first_query_frame, num_anchor, window,
        summary_tokens, int(bool(anchor_block)), softmax_scale, _ptr(out), _ptr(lse),
        _ptr(status), _stream(stream)))


def gca_selftest_bounded_wait(cache, timeout_ms: int = 100) -> int:
    s = ctypes.c_int32(0)
    _check("gca_selftest_bounded_wait", lib().gca_selftest_bounded_wait(cache, timeout_ms, ctypes.byref(s)))
    return s.value


class Cache:
    """Owning wrapper: one GCA cache for a workload (see inputs.Workload)."""

    def __init__(self, *, device: int = 0, **cfg):
        self.cfg = dict(cfg)
        self.handle = gca_cache_create(device=device, **cfg)

    @classmethod
    def for_workload(cls, w, *, max_frames: Optional[int] = None, device: int = 0, **extra):
        return cls(num_layers=w.L, num_heads=w.H, image_tokens=w.M, summary_tokens=w.S,
                   head_dim=w.D, num_anchor=w.n, window=w.k,
                   max_frames=max_frames if max_frames is not None else
                   (w.window_frames or w.T), page_size=w.page_size, dtype=w.dtype,
                   softmax_scale=w.softmax_scale, device=device, **extra)

    def append(self, k, v, layer: int = GCA_ALL_LAYERS, stream=None) -> int:
        return gca_append_frame(self.handle, layer, k, v, stream)

    def evict(self) -> int:
        return gca_evict_to_summary(self.handle)

    def attend(self, layer, q, out, lse=None, num_query_frames: int = 1, stream=None):
        gca_attend(self.handle, layer, q, out, lse, num_query_frames, stream)

    def attend_transient(self, layer, q, k, v, out, lse=None, stream=None):
        gca_attend_transient(self.handle, layer, q, k, v, out, lse, stream)

    def frame_attention(self, layer, q, k, v, out, lse=None, stream=None):
        gca_frame_attention(self.handle, layer, q, k, v, out, lse, stream)

    def frame_attention_batch(self, layer, q, k, v, out, lse=None, stream=None):
        gca_frame_attention_batch(self.handle, layer, q, k, v, out, lse, stream)

    def reset(self):
        gca_reset(self.handle)

    def layout(self, num_query_frames: int = 1):
        return gca_get_layout(self.handle, num_query_frames)

    def info(self) -> gca_info_t:
        return gca_get_info(self.handle)

    def visible_prefix(self, entry, query_frame: int) -> int:
        return gca_visible_prefix(self.handle, entry, query_frame)

    def token_slot(self, frame: int, tau: int):
        return gca_token_slot(self.handle, frame, tau)

    def status(self, clear: bool = False) -> int:
        return gca_device_status(self.handle, clear)

    def close(self):
        if self.handle is not None:
            gca_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
