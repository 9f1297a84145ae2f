"""ctypes binding of libuf.so: argument marshalling only.

Every step of the hot path runs in the CUDA library; this module converts
torch tensors to pointers, picks the caller's current CUDA stream and turns a
non-zero status into an exception.  There is no CPU fallback: importing it
without a built libuf.so raises.
"""
from __future__ import annotations

import ctypes
import os

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libuf.so")

UF_OK, UF_EINVAL, UF_ECUDA, UF_ETIMEOUT, UF_EBOUNDS, UF_EUNSUPPORTED = range(6)
UF_APPEND_REPLACE_NEWEST = 1
UF_APPEND_ANCHOR = 2
UF_MASK_LOCAL_ONLY = 1


class UfKvCache(ctypes.Structure):
    """Mirror of ``uf_kv_cache`` in include/uf.h."""

    _fields_ = [
        ("k", ctypes.c_void_p),
        ("v", ctypes.c_void_p),
        ("kpool", ctypes.c_void_p),
        ("meta", ctypes.c_void_p),
        ("B", ctypes.c_int32), ("G", ctypes.c_int32), ("D", ctypes.c_int32),
        ("W", ctypes.c_int32), ("Lc", ctypes.c_int32), ("blk", ctypes.c_int32),
        ("host_start", ctypes.c_int32), ("host_n_valid", ctypes.c_int32), ("host_anchor", ctypes.c_int32),
        ("err", ctypes.c_void_p),
    ]


class UfError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {strerror(status)}"
        if status == UF_ECUDA:
            msg += f" ({lib.uf_last_cuda_error().decode()})"
        super().__init__(msg)


def _load() -> ctypes.CDLL:
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is not built: run `python -m block_sparse_causal_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    i32, vp, sz = ctypes.c_int32, ctypes.c_void_p, ctypes.c_size_t
    pc = ctypes.POINTER(UfKvCache)
    sig = {
        "uf_version": ([], i32),
        "uf_source_hash": ([], ctypes.c_char_p),
        "uf_strerror": ([i32], ctypes.c_char_p),
        "uf_kv_cache_bytes": ([i32, i32, i32, i32, i32, i32, ctypes.POINTER(sz), ctypes.POINTER(sz),
                               ctypes.POINTER(sz)], i32),
        "uf_kv_cache_init": ([pc, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32], i32),
        "uf_kv_cache_set_error_word": ([pc, vp], i32),
        "uf_kv_reset": ([pc, vp], i32),
        "uf_kv_append": ([pc, vp, vp, i32, i32, vp], i32),
        "uf_kv_append_rope": ([pc, vp, vp, i32, i32, ctypes.c_int64, ctypes.c_float, vp], i32),
        "uf_rope": ([vp, vp, i32, i32, i32, ctypes.c_int64, ctypes.c_float, vp], i32),
        "uf_tile_tokens": ([vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, i32, vp], i32),
        "uf_kv_append_tiled": ([pc, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, vp], i32),
        "uf_block_mask": ([vp, i32, pc, i32, vp, vp, vp, vp], i32),
        "uf_block_mask_local": ([vp, i32, pc, i32, i32, i32, vp, vp, vp, vp], i32),
        "uf_block_sparse_attn": ([vp, i32, pc, vp, vp, i32, ctypes.c_float, vp, vp, vp], i32),
        "uf_kv_append_fp8k": ([pc, vp, ctypes.c_float, vp, vp, i32, i32, vp], i32),
        "uf_block_sparse_attn_balanced": ([vp, i32, pc, vp, vp, i32, ctypes.c_float, vp, vp, vp, sz, vp], i32),
        "uf_attn_workspace_bytes": ([ctypes.POINTER(sz)], i32),
        "uf_block_sparse_attn_balanced_noalloc": ([vp, i32, pc, vp, vp, i32, ctypes.c_float, vp, vp, vp], i32),
        "uf_block_sparse_attn_fp8k": ([vp, i32, pc, vp, ctypes.c_float, ctypes.c_float, vp, vp, i32, ctypes.c_float,
                                       vp, vp, vp], i32),
        "uf_check_error": ([vp, vp], i32),
        "uf_get_error": ([ctypes.POINTER(i32), i32], i32),
        "uf_last_cuda_error": ([], ctypes.c_char_p),
        "uf_set_wait_limit": ([ctypes.c_int64], i32),
        "uf_set_clock_counters": ([vp], i32),
        "uf_debug_wait_timeout": ([ctypes.c_int64, vp], i32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


lib = _load()


def _check_source_hash() -> None:
    """Refuse a library built from sources other than the ones beside it."""
    from .build import source_hash
    built = lib.uf_source_hash().decode()
    tree = source_hash()
    if built != tree:
        raise ImportError(f"{_LIB_PATH} was built from other sources (library {built}, tree {tree}): "
                          f"run `python block_sparse_causal_b200/build.py`")


_check_source_hash()


def strerror(status: int) -> str:
    return lib.uf_strerror(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != UF_OK:
        raise UfError(status, where)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def uf_kv_cache_bytes(B, G, D, W, Lc, blk):
    """(kv_bytes, kpool_bytes, meta_bytes) of a window with these dimensions."""
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib.uf_kv_cache_bytes(B, G, D, W, Lc, blk, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)),
           "uf_kv_cache_bytes")
    return a.value, b.value, c.value


def uf_kv_cache_init(k, v, kpool, meta, B, G, D, W, Lc, blk) -> UfKvCache:
    c = UfKvCache()
    _check(lib.uf_kv_cache_init(ctypes.byref(c), _ptr(k), _ptr(v), _ptr(kpool), _ptr(meta), B, G, D, W, Lc, blk),
           "uf_kv_cache_init")
    return c


def uf_kv_cache_set_error_word(cache: UfKvCache, err) -> None:
    _check(lib.uf_kv_cache_set_error_word(ctypes.byref(cache), _ptr(err)), "uf_kv_cache_set_error_word")


def uf_kv_reset(cache: UfKvCache, stream=None) -> None:
    _check(lib.uf_kv_reset(ctypes.byref(cache), _stream(stream)), "uf_kv_reset")


def uf_kv_append(cache: UfKvCache, k_new, v_new, keep_chunks: int, flags: int = 0, stream=None) -> None:
    _check(lib.uf_kv_append(ctypes.byref(cache), _ptr(k_new), _ptr(v_new), keep_chunks, flags, _stream(stream)),
           "uf_kv_append")


def uf_kv_append_rope(cache: UfKvCache, k_new, v_new, keep_chunks: int, flags: int, pos0: int,
                      base: float = 10000.0, stream=None) -> None:
    _check(lib.uf_kv_append_rope(ctypes.byref(cache), _ptr(k_new), _ptr(v_new), keep_chunks, flags, pos0, base,
                                 _stream(stream)), "uf_kv_append_rope")


def uf_rope(x, y, B: int, L: int, heads: int, pos0: int, base: float = 10000.0, stream=None) -> None:
    _check(lib.uf_rope(_ptr(x), _ptr(y), B, L, heads, pos0, base, _stream(stream)), "uf_rope")


def uf_tile_tokens(x, y, B: int, grid, heads: int, tile=(2, 8, 8), inverse: bool = False, stream=None) -> None:
    T, Hg, Wg = grid
    _check(lib.uf_tile_tokens(_ptr(x), _ptr(y), B, T, Hg, Wg, heads, *tile, 1 if inverse else 0, _stream(stream)),
           "uf_tile_tokens")


def uf_kv_append_tiled(cache: UfKvCache, k_new, v_new, keep_chunks: int, flags: int, grid, tile=(2, 8, 8),
                       stream=None) -> None:
    _check(lib.uf_kv_append_tiled(ctypes.byref(cache), _ptr(k_new), _ptr(v_new), keep_chunks, flags, *grid, *tile,
                                  _stream(stream)), "uf_kv_append_tiled")


def uf_block_mask(q, H: int, cache: UfKvCache, k: int, idx, cnt, scores=None, stream=None) -> None:
    _check(lib.uf_block_mask(_ptr(q), H, ctypes.byref(cache), k, _ptr(idx), _ptr(cnt), _ptr(scores),
                             _stream(stream)), "uf_block_mask")


def uf_block_mask_local(q, H: int, cache: UfKvCache, k: int, local: int, flags: int, idx, cnt, scores=None,
                        stream=None) -> None:
    _check(lib.uf_block_mask_local(_ptr(q), H, ctypes.byref(cache), k, local, flags, _ptr(idx), _ptr(cnt),
                                   _ptr(scores), _stream(stream)), "uf_block_mask_local")


def uf_block_sparse_attn(q, H: int, cache: UfKvCache, idx, cnt, k: int, scale: float, o, lse=None,
                         stream=None) -> None:
    _check(lib.uf_block_sparse_attn(_ptr(q), H, ctypes.byref(cache), _ptr(idx), _ptr(cnt), k, scale, _ptr(o),
                                    _ptr(lse), _stream(stream)), "uf_block_sparse_attn")


def uf_attn_workspace_bytes() -> int:
    """Workspace bytes of uf_block_sparse_attn_balanced on the current device."""
    n = ctypes.c_size_t()
    _check(lib.uf_attn_workspace_bytes(ctypes.byref(n)), "uf_attn_workspace_bytes")
    return n.value


def uf_block_sparse_attn_balanced(q, H: int, cache: UfKvCache, idx, cnt, k: int, scale: float, o, lse, workspace,
                                  stream=None) -> None:
    """workspace: a device tensor of at least uf_attn_workspace_bytes() bytes."""
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.uf_block_sparse_attn_balanced(_ptr(q), H, ctypes.byref(cache), _ptr(idx), _ptr(cnt), k, scale,
                                             _ptr(o), _ptr(lse), _ptr(workspace), nbytes, _stream(stream)),
           "uf_block_sparse_attn_balanced")


def uf_block_sparse_attn_balanced_noalloc(q, H: int, cache: UfKvCache, idx, cnt, k: int, scale: float, o, lse=None,
                                          stream=None) -> None:
    """uf_block_sparse_attn_balanced with the library's own fixed scratch array
    (no workspace argument, nothing allocated)."""
    _check(lib.uf_block_sparse_attn_balanced_noalloc(_ptr(q), H, ctypes.byref(cache), _ptr(idx), _ptr(cnt), k,
                                                     scale, _ptr(o), _ptr(lse), _stream(stream)),
           "uf_block_sparse_attn_balanced_noalloc")


def uf_kv_append_fp8k(cache: UfKvCache, k8, k_scale: float, k_new, v_new, keep_chunks: int, flags: int = 0,
                      stream=None) -> None:
    _check(lib.uf_kv_append_fp8k(ctypes.byref(cache), _ptr(k8), k_scale, _ptr(k_new), _ptr(v_new), keep_chunks,
                                 flags, _stream(stream)), "uf_kv_append_fp8k")


def uf_block_sparse_attn_fp8k(q, H: int, cache: UfKvCache, k8, q_scale: float, k_scale: float, idx, cnt, k: int,
                              scale: float, o, lse=None, stream=None) -> None:
    _check(lib.uf_block_sparse_attn_fp8k(_ptr(q), H, ctypes.byref(cache), _ptr(k8), q_scale, k_scale, _ptr(idx),
                                         _ptr(cnt), k, scale, _ptr(o), _ptr(lse), _stream(stream)),
           "uf_block_sparse_attn_fp8k")


def uf_check_error(dev_err_word, stream=None) -> None:
    """Enqueue the move of the library's device error word into ``dev_err_word``
    (a device int32 tensor) on ``stream``; no synchronisation."""
    _check(lib.uf_check_error(_ptr(dev_err_word), _stream(stream)), "uf_check_error")


def uf_get_error(clear: bool = True) -> int:
    st = ctypes.c_int32()
    _check(lib.uf_get_error(ctypes.byref(st), 1 if clear else 0), "uf_get_error")
    return st.value


def uf_set_wait_limit(cycles: int) -> None:
    _check(lib.uf_set_wait_limit(cycles), "uf_set_wait_limit")


def uf_set_clock_counters(counters) -> None:
    """counters: a device int64 tensor of 2 zeroed elements (or None to stop):
    attention launches add their SM cycles and nanoseconds to it."""
    if counters is not None and (counters.numel() < 2 or counters.element_size() != 8 or not counters.is_cuda):
        raise ValueError("counters must be a device tensor of at least 2 eight-byte elements")
    _check(lib.uf_set_clock_counters(_ptr(counters)), "uf_set_clock_counters")


def uf_debug_wait_timeout(cycles: int, stream=None) -> None:
    _check(lib.uf_debug_wait_timeout(cycles, _stream(stream)), "uf_debug_wait_timeout")


def uf_version() -> int:
    return lib.uf_version()


def uf_source_hash() -> str:
    return lib.uf_source_hash().decode()
