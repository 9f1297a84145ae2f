"""Owner of one rolling KV window's device buffers (torch allocations)."""
from __future__ import annotations

import math

import torch

from . import _uf


class KVWindow:
    """Allocates k, v, kpool and meta for a window of W chunks on ``device``
    (sizes from ``uf_kv_cache_bytes``) and holds the ``uf_kv_cache``
    descriptor that the library calls take.  With ``k_scale`` it also owns the
    e4m3 copy of K (``k8``) that the FP8-score calls read and write.  With
    ``error_word`` it owns a device int32 ``err`` in which the kernels of calls
    on this window record their errors (``uf_kv_cache_set_error_word``)."""

    def __init__(self, B: int, G: int, W: int, Lc: int, blk: int = 128, D: int = 128, device="cuda",
                 k_scale: float | None = None, error_word: bool = False):
        kv_bytes, kpool_bytes, meta_bytes = _uf.uf_kv_cache_bytes(B, G, D, W, Lc, blk)
        self.B, self.G, self.D, self.W, self.Lc, self.blk = B, G, D, W, Lc, blk
        self.nb = math.ceil(Lc / blk)
        self.lslot = self.nb * blk
        # k: token rows [B, G, W*Lslot, D]; v: transposed [B, G, D, W*Lslot]
        self.k = torch.zeros(kv_bytes // 2, dtype=torch.bfloat16, device=device).view(B, G, W * self.lslot, D)
        self.v = torch.zeros(kv_bytes // 2, dtype=torch.bfloat16, device=device).view(B, G, D, W * self.lslot)
        self.kpool = torch.zeros(kpool_bytes // 4, dtype=torch.float32, device=device).view(B, G, W * self.nb, D)
        self.meta = torch.zeros(meta_bytes // 4, dtype=torch.int32, device=device)
        self.desc = _uf.uf_kv_cache_init(self.k, self.v, self.kpool, self.meta, B, G, D, W, Lc, blk)
        self.k_scale = k_scale
        self.k8 = None if k_scale is None else torch.zeros(B, G, W * self.lslot, D, dtype=torch.uint8, device=device)
        self.err = None
        if error_word:
            self.err = torch.zeros(1, dtype=torch.int32, device=device)
            _uf.uf_kv_cache_set_error_word(self.desc, self.err)

    @property
    def n_valid(self) -> int:
        """Host mirror of the number of chunks in the window."""
        return self.desc.host_n_valid

    def reset(self, stream=None) -> None:
        _uf.uf_kv_reset(self.desc, stream)

    def append(self, k_new, v_new, keep_chunks: int | None = None, replace_newest: bool = False, stream=None,
               rope_pos0: int | None = None, rope_base: float = 10000.0, anchor: bool = False,
               tile_grid=None, tile=(2, 8, 8)):
        """Append the chunk's K and V (uf_kv_append); with ``rope_pos0``, K is
        rotated at stream positions rope_pos0 + token (uf_kv_append_rope); with
        ``tile_grid`` = (T, Hg, Wg), K and V are stored in tiled token order
        (uf_kv_append_tiled); with ``anchor`` (empty window) the chunk becomes
        the pinned anchor.  A window made with ``k_scale`` also writes the e4m3
        copy of K (uf_kv_append_fp8k)."""
        keep = self.W if keep_chunks is None else keep_chunks
        flags = (_uf.UF_APPEND_REPLACE_NEWEST if replace_newest else 0) | (_uf.UF_APPEND_ANCHOR if anchor else 0)
        if self.k8 is not None:
            if rope_pos0 is not None or tile_grid is not None:
                raise ValueError("the FP8 append neither rotates nor tiles")
            _uf.uf_kv_append_fp8k(self.desc, self.k8, self.k_scale, k_new, v_new, keep, flags, stream)
        elif tile_grid is not None:
            if rope_pos0 is not None:
                raise ValueError("the tiled append does not rotate")
            _uf.uf_kv_append_tiled(self.desc, k_new, v_new, keep, flags, tile_grid, tile, stream)
        elif rope_pos0 is None:
            _uf.uf_kv_append(self.desc, k_new, v_new, keep, flags, stream)
        else:
            _uf.uf_kv_append_rope(self.desc, k_new, v_new, keep, flags, rope_pos0, rope_base, stream)
