"""fp64 CPU oracle for chunk-causal block-sparse attention over a rolling KV window.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this module.  The product path (the
CUDA library and its Python binding) never calls it and shares no code with it.

Every function computes the plain definition of its step, in float64, with no
blocking, fusion or reordering beyond what that definition states.  Inputs are
float64 numpy arrays (exact upcasts of the bf16 values the GPU receives).

Sources (page title, then section / equation):

* Ultra Flash (papernotes.org notes), Method, key design 3: the 3-D token grid
  is cut into non-overlapping blocks; per attention layer the query and key
  tokens of each block are mean-pooled, blocks are scored by the dot product of
  the pooled query and key, and each head keeps its top-k scoring blocks, under
  a strict temporal causal mask.
* Ultra Flash (papernotes.org notes), Method, key design 4: dynamic cache
  management -- reuse of the last denoising step's KV cache instead of a rerun,
  and adaptive cropping of the SR model's KV window length.
* FlashDecoder (xllm-io blog), Sec. 3, Eq. 4: the cached keys/values have shape
  B x G x (W_frm * L_frm) x D_h, with G grouped-query KV heads.
* FlashDecoder (xllm-io blog), Algorithm 1 (streaming inference): after each
  frame the cache becomes the tail (W_frm - 1) frames of the old cache followed
  by the new frame's K/V; causality comes from the processing order, not from a
  token mask (Sec. 3.3).

Readings taken where the pages are silent or ambiguous (each is listed in the
design notes of the repository):

* Blocks are contiguous runs of ``blk`` tokens in the caller's token order,
  counted within each chunk; the last block of a chunk is partial when ``blk``
  does not divide the chunk length.  Blocks never straddle chunks.
* The query chunk is the newest chunk of the window (it was appended just
  before attention).  Inside the window there is no token-level mask: each query
  token may attend to every token of every kept block, including blocks of its
  own chunk (causal at chunk granularity).
* Pooled block score = mean(q_block) . mean(k_block) / sqrt(D); no softmax is
  applied to pooled scores (it would not change the ranking).
* Selection per (batch, query head, q-block i): the diagonal block
  d_i = (n_valid - 1) * nb + i (same block of the newest chunk) is always kept;
  the other blocks are ranked by (score descending, logical index ascending) and
  the first k - 1 are kept.  k is clamped to the number of blocks in the window.
* Under GQA, query head h reads KV head h // (H / G); masks are per query head.
* LSE is the natural log of sum(exp(scale * q . k)) over kept tokens.
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "RollingWindow",
    "block_ranges",
    "window_blocks",
    "pool_blocks",
    "block_scores",
    "select_blocks",
    "block_mask",
    "block_sparse_attention",
    "rope",
    "window_rope",
    "round_bf16",
    "tile_order",
    "to_tile_order",
    "from_tile_order",
    "E4M3_MAX",
    "quantize_e4m3",
    "fp8_scores_attention",
]


# --------------------------------------------------------------------------
# Rolling KV window
# --------------------------------------------------------------------------
class RollingWindow:
    """The last ``keep_chunks`` chunks of K and V, oldest first.

    FlashDecoder, Eq. 4 / Algorithm 1: a fixed window whose memory does not grow
    with the stream (the oldest frame leaves when a new one arrives).  Ultra
    Flash key design 4 adds two cache operations, read here as:

    * ``replace_newest``: the newest chunk's K/V are overwritten by a new
      computation of the same chunk (no eviction);
    * ``keep_chunks``: the window is cropped to at most ``keep_chunks`` chunks
      (oldest dropped first), ``1 <= keep_chunks <= W``.

    HiStream (aipapers summary), innovation 2, anchor-guided sliding window:
    one anchor key frame plus a small cache of neighbouring frames keeps the
    attention context at a fixed size.  ``anchor=True`` on an empty window
    pins the chunk as the window's first chunk: it is never evicted or
    cropped, ``keep_chunks`` counts it (2..W afterwards), and eviction drops
    the oldest of the other chunks.
    """

    def __init__(self, W: int):
        if W < 1:
            raise ValueError("window capacity must be >= 1")
        self.W = W
        self.k: List[np.ndarray] = []
        self.v: List[np.ndarray] = []
        self.anchored = False

    def append(self, k_new: np.ndarray, v_new: np.ndarray,
               keep_chunks: Optional[int] = None, replace_newest: bool = False, anchor: bool = False) -> None:
        keep = self.W if keep_chunks is None else keep_chunks
        if not 1 <= keep <= self.W:
            raise ValueError("keep_chunks must be in [1, W]")
        if anchor:
            if self.k or replace_newest or self.W < 2:
                raise ValueError("an anchor starts an empty window of W >= 2")
            self.anchored = True
            self.k.append(np.array(k_new, dtype=np.float64))
            self.v.append(np.array(v_new, dtype=np.float64))
            return
        if self.anchored and keep < 2:
            raise ValueError("keep_chunks counts the anchor and must leave room for one more chunk")
        if replace_newest:
            if not self.k:
                raise ValueError("replace_newest on an empty window")
            self.k[-1] = np.array(k_new, dtype=np.float64)
            self.v[-1] = np.array(v_new, dtype=np.float64)
        else:
            self.k.append(np.array(k_new, dtype=np.float64))
            self.v.append(np.array(v_new, dtype=np.float64))
        first = 1 if self.anchored else 0          # the anchor is never dropped
        while len(self.k) > keep:
            self.k.pop(first)
            self.v.pop(first)

    @property
    def n_valid(self) -> int:
        return len(self.k)


# --------------------------------------------------------------------------
# Blocks
# --------------------------------------------------------------------------
def block_ranges(Lc: int, blk: int) -> List[Tuple[int, int]]:
    """[start, stop) token ranges of the blocks of one chunk (Ultra Flash key
    design 3: non-overlapping blocks; last one partial)."""
    if Lc < 1 or blk < 1:
        raise ValueError("Lc and blk must be positive")
    return [(s, min(s + blk, Lc)) for s in range(0, Lc, blk)]


def window_blocks(n_chunks: int, Lc: int, blk: int) -> List[Tuple[int, int, int]]:
    """Logical kv blocks of a window of ``n_chunks`` chunks, oldest first:
    block j -> (chunk index c, start, stop) with j = c * nb + r."""
    return [(c, s, e) for c in range(n_chunks) for (s, e) in block_ranges(Lc, blk)]


# --------------------------------------------------------------------------
# Block mask: pooling, scores, top-k
# --------------------------------------------------------------------------
def pool_blocks(x: np.ndarray, blk: int) -> np.ndarray:
    """Mean of each block's own tokens.

    x: [B, L, heads, D] -> [B, heads, nblocks, D] (Ultra Flash key design 3:
    in-block mean pooling of queries and keys).
    """
    B, L, Hx, D = x.shape
    ranges = block_ranges(L, blk)
    out = np.empty((B, Hx, len(ranges), D), dtype=np.float64)
    for n, (s, e) in enumerate(ranges):
        out[:, :, n, :] = x[:, s:e, :, :].mean(axis=1)
    return out


def block_scores(qpool: np.ndarray, kpool: np.ndarray, scale: float) -> np.ndarray:
    """Pooled block scores (Ultra Flash key design 3: dot product of pooled
    query and key blocks), scaled by ``scale``.

    qpool [B, H, NQ, D], kpool [B, G, NKV, D] -> [B, H, NQ, NKV]; query head h
    reads KV head h // (H // G) (grouped-query attention, FlashDecoder Eq. 4).
    """
    B, H, NQ, D = qpool.shape
    G = kpool.shape[1]
    if H % G:
        raise ValueError("H must be a multiple of G")
    rep = H // G
    out = np.empty((B, H, NQ, kpool.shape[2]), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            out[b, h] = (qpool[b, h] @ kpool[b, h // rep].T) * scale
    return out


def select_blocks(scores: np.ndarray, k: int, diag: Sequence[int], local: int = 0, local_only: bool = False):
    """Per-row top-k block selection with forced blocks.

    Ultra Flash (papernotes notes), Method, key design 3: each head keeps its
    top-k blocks by pooled score; the layer's mask also combines a local
    sliding-window mask (and the ablation table's "fixed local window instead
    of adaptive top-k" keeps that window alone).  Forced blocks: the band of
    logical blocks within ``local`` of the diagonal, clipped to the window
    (local = 0: the diagonal alone).  The rest of the row's k blocks are the
    others ranked by (score descending, logical index ascending); with
    ``local_only`` the row is the band alone.

    scores [B, H, NQ, NKV]; diag[i] = logical index of q-block i's own block.
    Returns (idx [B, H, NQ, k_eff] int32, ascending, padded with -1 past cnt;
    cnt [B, H, NQ] int32; boundary [B, H, NQ, 2] float64).  ``boundary`` holds
    the score of the last kept scored block and of the first dropped one (NaN
    when there is none); rows where the two are closer than the near-tie
    tolerance may legitimately differ between two correct implementations.
    """
    B, H, NQ, NKV = scores.shape
    k_eff = min(k, NKV)
    if k_eff < 1:
        raise ValueError("k must be >= 1")
    if local < 0 or 2 * local + 1 > k:
        raise ValueError("the band (2 local + 1 blocks) must fit in k")
    idx = np.full((B, H, NQ, k_eff), -1, dtype=np.int32)
    cnt = np.zeros((B, H, NQ), dtype=np.int32)
    boundary = np.full((B, H, NQ, 2), np.nan)
    all_j = np.arange(NKV)
    for b in range(B):
        for h in range(H):
            for i in range(NQ):
                d = diag[i]
                band = all_j[np.abs(all_j - d) <= local]
                take = 0 if local_only else k_eff - len(band)
                cand = all_j[np.abs(all_j - d) > local]
                s = scores[b, h, i, cand]
                # rank: score descending, then logical index ascending
                order = cand[np.lexsort((cand, -s))]
                chosen = order[:take]
                row = np.sort(np.concatenate([band, chosen]))
                idx[b, h, i, : len(row)] = row
                cnt[b, h, i] = len(row)
                if take >= 1:
                    boundary[b, h, i, 0] = scores[b, h, i, order[take - 1]]
                if not local_only and take < len(order):
                    boundary[b, h, i, 1] = scores[b, h, i, order[take]]
    return idx, cnt, boundary


def block_mask(q: np.ndarray, window: RollingWindow, blk: int, k: int,
               scale: Optional[float] = None, local: int = 0, local_only: bool = False):
    """The whole mask step for the newest chunk's queries (``local`` and
    ``local_only`` as in select_blocks).

    q [B, Lc, H, D]; the window holds n_valid chunks of K [B, Lc, G, D].
    Returns dict(idx, cnt, scores, boundary, qpool, kpool).
    """
    B, Lc, H, D = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    n_valid = window.n_valid
    if n_valid < 1:
        raise ValueError("empty window")
    nb = len(block_ranges(Lc, blk))
    qpool = pool_blocks(q, blk)                                     # [B,H,NQ,D]
    kpool = np.concatenate([pool_blocks(kc, blk) for kc in window.k], axis=2)  # [B,G,NKV,D]
    scores = block_scores(qpool, kpool, scale)
    diag = [(n_valid - 1) * nb + i for i in range(nb)]
    idx, cnt, boundary = select_blocks(scores, k, diag, local, local_only)
    return dict(idx=idx, cnt=cnt, scores=scores, boundary=boundary, qpool=qpool, kpool=kpool)


# --------------------------------------------------------------------------
# Block-sparse attention
# --------------------------------------------------------------------------
def block_sparse_attention(q: np.ndarray, window: RollingWindow, blk: int,
                           idx: Optional[np.ndarray] = None, cnt: Optional[np.ndarray] = None,
                           scale: Optional[float] = None,
                           items: Optional[Sequence[Tuple[int, int, int]]] = None):
    """Softmax attention of the newest chunk's queries over the kept blocks.

    For each (batch b, query head h, q-block i), the queries of block i attend
    to every token of the kept kv blocks idx[b, h, i, :cnt] (all window blocks
    when ``idx`` is None: density 1.0 = dense chunk-causal attention):

        s = scale * q . k,  O = sum(exp(s - m) v) / sum(exp(s - m)),
        LSE = m + ln(sum(exp(s - m)))

    (Ultra Flash key design 3: attention restricted to the kept blocks;
    FlashDecoder Sec. 3.3: no token mask inside the window.)

    q [B, Lc, H, D]; returns (O [B, Lc, H, D], LSE [B, H, Lc]).  When ``items``
    lists (b, h, i) work items, only those rows are computed (others NaN).
    """
    B, Lc, H, D = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    kwin = np.concatenate(window.k, axis=1)     # [B, n*Lc, G, D] logical token order
    vwin = np.concatenate(window.v, axis=1)
    G = kwin.shape[2]
    rep = H // G
    qranges = block_ranges(Lc, blk)
    kvblocks = window_blocks(window.n_valid, Lc, blk)
    nkv = len(kvblocks)
    O = np.full((B, Lc, H, D), np.nan)
    LSE = np.full((B, H, Lc), np.nan)
    if items is None:
        items = [(b, h, i) for b in range(B) for h in range(H) for i in range(len(qranges))]
    for (b, h, i) in items:
        if idx is None:
            kept = range(nkv)
        else:
            n = idx.shape[-1] if cnt is None else int(cnt[b, h, i])
            kept = [int(j) for j in idx[b, h, i, :n]]
        cols = np.concatenate([np.arange(c * Lc + s, c * Lc + e) for (c, s, e) in
                               (kvblocks[j] for j in kept)])
        s0, e0 = qranges[i]
        qi = q[b, s0:e0, h, :]
        kk = kwin[b, cols, h // rep, :]
        vv = vwin[b, cols, h // rep, :]
        s = (qi @ kk.T) * scale
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        l = p.sum(axis=1)
        O[b, s0:e0, h, :] = (p @ vv) / l[:, None]
        LSE[b, h, s0:e0] = m[:, 0] + np.log(l)
    return O, LSE


# --------------------------------------------------------------------------
# Rotary position embedding with window-relative positions
# --------------------------------------------------------------------------
def rope(x: np.ndarray, pos: np.ndarray, base: float = 10000.0) -> np.ndarray:
    """Rotary position embedding of the last axis (RoFormer, Su et al. 2021:
    channel pairs (x_2i, x_2i+1) rotated by the angle pos * theta_i with
    theta_i = base^(-2i / D)).  The pages name RoPE but not its form
    (FlashDecoder, "long video decoding": positions relative to the current
    window; Algorithm 1 offsets the positions by the frame index times the
    tokens per frame); this is the published form.

    x [..., L, heads, D]; pos [L] integer positions of the L tokens.
    """
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    if D % 2:
        raise ValueError("D must be even")
    theta = base ** (-2.0 * np.arange(D // 2) / D)                      # [D/2]
    ang = np.asarray(pos, dtype=np.float64)[:, None] * theta[None, :]   # [L, D/2]
    c = np.cos(ang)[:, None, :]                                         # [L, 1, D/2]
    s = np.sin(ang)[:, None, :]
    x0, x1 = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


def round_bf16(x: np.ndarray) -> np.ndarray:
    """float64 -> nearest bfloat16 value (ties to even), returned as float64:
    the rounding a bf16 store applies.  bf16 keeps 8 significant bits, so the
    grid spacing at x is 2^(floor(log2|x|) - 7); np.round rounds halves to
    even.  (Inputs here are far from the bf16 range limits.)"""
    x = np.asarray(x, dtype=np.float64)
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    ulp = np.exp2(e - 7)
    return np.where(ax > 0, np.round(x / ulp) * ulp, 0.0)


def window_rope(q: np.ndarray, window: RollingWindow, base: float = 10000.0, shift: int = 0,
                to_bf16: bool = False):
    """The window and the newest chunk's queries with RoPE at window-relative
    positions (FlashDecoder, "long video decoding": RoPE positions are assigned
    relative to the current window, not by absolute frame index): token r of
    the window's chunk c (c = 0 the oldest) sits at c * Lc + r, so the query
    chunk (the newest) sits at (n_valid - 1) * Lc + r.  Returns (q_rot, a new
    RollingWindow holding the rotated K and the unchanged V), ready for
    block_mask and block_sparse_attention.

    ``shift`` adds a common offset to every position (rotary scores depend
    only on position differences, so exact results do not change); with
    ``to_bf16`` the rotated values are rounded to bf16 as a bf16 cache stores
    them.  Together they give the rotated values a stream-position cache holds.
    """
    Lc = q.shape[1]
    n = window.n_valid
    out = RollingWindow(window.W)
    fin = round_bf16 if to_bf16 else (lambda a: a)
    for c in range(n):
        out.append(fin(rope(window.k[c], shift + c * Lc + np.arange(Lc), base)), window.v[c])
    q_rot = fin(rope(q, shift + (n - 1) * Lc + np.arange(Lc), base))
    return q_rot, out


# --------------------------------------------------------------------------
# 3-D block token order
# --------------------------------------------------------------------------
def tile_order(T: int, Hg: int, Wg: int, tile: Tuple[int, int, int] = (2, 8, 8)) -> np.ndarray:
    """Token order of a chunk cut into 3-D tiles (Ultra Flash notes, Method, key
    design 3: the spatio-temporal token grid is divided into non-overlapping
    (2, 8, 8) blocks).

    The chunk's tokens are a (T, Hg, Wg) grid in row-major order (token
    t * Hg * Wg + y * Wg + x).  Tiles of ``tile`` = (bt, by, bx) are taken in
    row-major tile order, the tokens inside a tile in row-major order; tiles at
    the grid's far edges are clipped.  Returns ``order`` with
    order[p] = the row-major index of the token at position p of the tiled
    order (a permutation of range(T * Hg * Wg)).
    """
    bt, by, bx = tile
    t, y, x = np.meshgrid(np.arange(T), np.arange(Hg), np.arange(Wg), indexing="ij")
    t, y, x = t.ravel(), y.ravel(), x.ravel()
    # sort keys, most significant last for lexsort
    keys = (x % bx, y % by, t % bt, x // bx, y // by, t // bt)
    return np.lexsort(keys)


def to_tile_order(x: np.ndarray, order: np.ndarray) -> np.ndarray:
    """x [B, L, heads, D] in row-major token order -> tiled order."""
    return x[:, order]


def from_tile_order(x: np.ndarray, order: np.ndarray) -> np.ndarray:
    """Inverse of to_tile_order."""
    out = np.empty_like(x)
    out[:, order] = x
    return out


# --------------------------------------------------------------------------
# FP8 (e4m3) scores
# --------------------------------------------------------------------------
E4M3_MAX = 448.0


def quantize_e4m3(x: np.ndarray, scale: float) -> np.ndarray:
    """Static-scale FP8 quantisation (FlashDecoder, inference optimisations:
    statically calibrated FP8): the e4m3 value nearest to the quotient
    x / scale (ties to even; e4m3 keeps 4 significant bits, exponent bias 7,
    subnormal spacing 2^-9, saturating at +-448), returned in e4m3 units as
    float64.

    The pages fix no precision for the quotient, so this takes its plain
    definition: x / scale in float64 (relative error 2^-53, far below any
    e4m3 spacing), then the rounding."""
    v = np.asarray(x, dtype=np.float64) / float(scale)
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    ulp = np.exp2(np.maximum(e, -6.0) - 3.0)             # normal spacing 2^(e-3); below 2^-6 the subnormal 2^-9
    q = np.round(v / ulp) * ulp
    return np.clip(q, -E4M3_MAX, E4M3_MAX)


def fp8_scores_attention(q: np.ndarray, window: RollingWindow, blk: int, q_scale: float, k_scale: float,
                         idx: Optional[np.ndarray] = None, cnt: Optional[np.ndarray] = None,
                         scale: Optional[float] = None,
                         items: Optional[Sequence[Tuple[int, int, int]]] = None):
    """block_sparse_attention with the scores taken from FP8 queries and keys:
    q8 = quantize_e4m3(q, q_scale), k8 = quantize_e4m3(k, k_scale), and
    s = scale * q_scale * k_scale * (q8 . k8); V and the softmax are as in
    block_sparse_attention."""
    w8 = RollingWindow(window.W)
    w8.anchored = window.anchored
    for kc, vc in zip(window.k, window.v):
        w8.k.append(quantize_e4m3(kc, k_scale))
        w8.v.append(vc)
    D = q.shape[-1]
    s0 = 1.0 / math.sqrt(D) if scale is None else scale
    return block_sparse_attention(quantize_e4m3(q, q_scale), w8, blk, idx, cnt, s0 * q_scale * k_scale, items)
