"""Helpers shared by the parity tests: run the CUDA path through the binding,
run the oracle per head on the same seeded inputs, compare with the
acceptance tolerances.

Acceptance (fixed for this path):
  * masks bit-exact, except rows whose oracle boundary scores (last kept and
    first dropped non-diagonal block) differ by less than 1e-4 relative;
  * O within max-abs 2e-2 and mean-abs 2e-3 of the oracle;
  * LSE within 1e-3 absolute.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np
import torch

import oracle
from workloads import Config, chunk_inputs, to_f64

O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_ABS = 1e-3
NEAR_TIE_REL = 1e-4
# The kernels form the e4m3 quotient x / scale in fp32 as x * fp32(1 / scale):
# two roundings, within 2^-23 relative of the exact quotient (plus 2^-48).
E4M3_QUOTIENT_REL = 2.0 ** -22


# ------------------------------------------------------------------ GPU side --
class GpuStream:
    """Rolling window on the GPU fed chunk by chunk through the C ABI."""

    def __init__(self, cfg: Config, device="cuda", k_scale: Optional[float] = None):
        import block_sparse_causal_b200 as uf
        self.uf = uf
        self.cfg = cfg
        self.win = uf.KVWindow(cfg.B, cfg.G, cfg.W, cfg.Lc, cfg.blk, cfg.D, device=device, k_scale=k_scale)
        self.win.reset()
        self.device = device

    def append(self, inp, keep=None, replace=False, anchor=False):
        k = inp["k"].to(self.device)
        v = inp["v"].to(self.device)
        self.win.append(k, v, keep_chunks=keep, replace_newest=replace, anchor=anchor)

    def mask(self, q_cpu, k: int, want_scores=True, local: int = 0, local_only: bool = False):
        cfg = self.cfg
        q = q_cpu.to(self.device)
        nb = cfg.nb
        idx = torch.full((cfg.B, cfg.H, nb, k), -7, dtype=torch.int32, device=self.device)
        cnt = torch.full((cfg.B, cfg.H, nb), -7, dtype=torch.int32, device=self.device)
        scores = (torch.full((cfg.B, cfg.H, nb, cfg.W * nb), float("nan"), device=self.device)
                  if want_scores else None)
        if local == 0 and not local_only:
            self.uf.uf_block_mask(q, cfg.H, self.win.desc, k, idx, cnt, scores)
        else:
            flags = self.uf.UF_MASK_LOCAL_ONLY if local_only else 0
            self.uf.uf_block_mask_local(q, cfg.H, self.win.desc, k, local, flags, idx, cnt, scores)
        return idx, cnt, scores

    def attention(self, q_cpu, idx=None, cnt=None, k=0, scale=None):
        cfg = self.cfg
        q = q_cpu.to(self.device)
        o = torch.full((cfg.B, cfg.Lc, cfg.H, cfg.D), float("nan"), dtype=torch.bfloat16, device=self.device)
        lse = torch.full((cfg.B, cfg.H, cfg.Lc), float("nan"), dtype=torch.float32, device=self.device)
        scale = 1.0 / math.sqrt(cfg.D) if scale is None else scale
        self.uf.uf_block_sparse_attn(q, cfg.H, self.win.desc, idx, cnt, k, scale, o, lse)
        return o, lse

    def attention_fp8(self, q_cpu, q_scale: float, idx=None, cnt=None, k=0, scale=None):
        """FP8-score attention over the window's e4m3 K (window made with k_scale)."""
        cfg = self.cfg
        q = q_cpu.to(self.device)
        o = torch.full((cfg.B, cfg.Lc, cfg.H, cfg.D), float("nan"), dtype=torch.bfloat16, device=self.device)
        lse = torch.full((cfg.B, cfg.H, cfg.Lc), float("nan"), dtype=torch.float32, device=self.device)
        scale = 1.0 / math.sqrt(cfg.D) if scale is None else scale
        self.uf.uf_block_sparse_attn_fp8k(q, cfg.H, self.win.desc, self.win.k8, q_scale, self.win.k_scale, idx,
                                          cnt, k, scale, o, lse)
        return o, lse


# --------------------------------------------------------------- oracle side --
class OracleStream:
    """The same stream replayed on the oracle, one window per head group
    (slicing by head keeps full-size cases in memory; heads are independent)."""

    def __init__(self, cfg: Config):
        self.cfg = cfg
        self.windows = [oracle.RollingWindow(cfg.W) for _ in range(cfg.G)]

    def append(self, inp, keep=None, replace=False, anchor=False):
        for g, w in enumerate(self.windows):
            w.append(to_f64(inp["k"][:, :, g:g + 1]), to_f64(inp["v"][:, :, g:g + 1]),
                     keep_chunks=keep, replace_newest=replace, anchor=anchor)

    @property
    def n_valid(self):
        return self.windows[0].n_valid

    def head_window(self, h):
        return self.windows[h // (self.cfg.H // self.cfg.G)]

    def mask(self, q_cpu, k: int, heads: Optional[Sequence[int]] = None, local: int = 0, local_only: bool = False):
        cfg = self.cfg
        heads = range(cfg.H) if heads is None else heads
        out = {}
        for h in heads:
            r = oracle.block_mask(to_f64(q_cpu[:, :, h:h + 1]), self.head_window(h), cfg.blk, k,
                                  local=local, local_only=local_only)
            out[h] = r
        return out

    def attention(self, q_cpu, items: Sequence[Tuple[int, int, int]], idx=None, cnt=None, scale=None):
        """items: (b, h, i).  idx/cnt: numpy [B, H, nb, k] / [B, H, nb] or None."""
        cfg = self.cfg
        res = {}
        by_head: Dict[int, List[Tuple[int, int, int]]] = {}
        for it in items:
            by_head.setdefault(it[1], []).append(it)
        for h, its in by_head.items():
            qh = to_f64(q_cpu[:, :, h:h + 1])
            sub_idx = None if idx is None else idx[:, h:h + 1]
            sub_cnt = None if cnt is None else cnt[:, h:h + 1]
            O, L = oracle.block_sparse_attention(qh, self.head_window(h), cfg.blk, sub_idx, sub_cnt, scale,
                                                 items=[(b, 0, i) for (b, _, i) in its])
            for (b, _, i) in its:
                s0, e0 = i * cfg.blk, min(cfg.Lc, (i + 1) * cfg.blk)
                res[(b, h, i)] = (O[b, s0:e0, 0, :], L[b, 0, s0:e0])
        return res

    def attention_fp8(self, q_cpu, items: Sequence[Tuple[int, int, int]], q_scale: float, k_scale: float,
                      idx=None, cnt=None, scale=None):
        """oracle.fp8_scores_attention per head, as ``attention``."""
        cfg = self.cfg
        res = {}
        by_head: Dict[int, List[Tuple[int, int, int]]] = {}
        for it in items:
            by_head.setdefault(it[1], []).append(it)
        for h, its in by_head.items():
            qh = to_f64(q_cpu[:, :, h:h + 1])
            sub_idx = None if idx is None else idx[:, h:h + 1]
            sub_cnt = None if cnt is None else cnt[:, h:h + 1]
            O, L = oracle.fp8_scores_attention(qh, self.head_window(h), cfg.blk, q_scale, k_scale, sub_idx,
                                               sub_cnt, scale, items=[(b, 0, i) for (b, _, i) in its])
            for (b, _, i) in its:
                s0, e0 = i * cfg.blk, min(cfg.Lc, (i + 1) * cfg.blk)
                res[(b, h, i)] = (O[b, s0:e0, 0, :], L[b, 0, s0:e0])
        return res


# --------------------------------------------------------------- comparison --
def compare_masks(cfg: Config, gpu_idx, gpu_cnt, orc: Dict[int, dict], k: int):
    """Bit-exact per row except near-ties.  Returns (rows, exact_rows, tie_rows, bad_rows)."""
    gi = gpu_idx.cpu().numpy()
    gc = gpu_cnt.cpu().numpy()
    rows = exact = ties = 0
    bad = []
    for h, r in orc.items():
        oi, oc, bnd = r["idx"], r["cnt"], r["boundary"]
        k_eff = oi.shape[-1]
        for b in range(cfg.B):
            for i in range(cfg.nb):
                rows += 1
                g_row = gi[b, h, i]
                if gc[b, h, i] != oc[b, 0, i]:
                    bad.append((b, h, i, "cnt", int(gc[b, h, i]), int(oc[b, 0, i])))
                    continue
                if np.array_equal(g_row[:k_eff], oi[b, 0, i]) and np.all(g_row[k_eff:] == -1):
                    exact += 1
                    continue
                a, c = bnd[b, 0, i]
                rel = abs(a - c) / max(abs(a), abs(c), 1e-300) if np.isfinite(a) and np.isfinite(c) else np.inf
                nkv = r["scores"].shape[-1]
                diag = (nkv // cfg.nb - 1) * cfg.nb + i
                sel = g_row[:k_eff]
                valid = (np.all(np.diff(sel) > 0) and sel.min() >= 0 and sel.max() < nkv and diag in sel)
                if rel < NEAR_TIE_REL and valid:
                    ties += 1
                else:
                    bad.append((b, h, i, "idx", g_row[:k_eff].tolist(), oi[b, 0, i].tolist(), rel))
    return rows, exact, ties, bad


def e4m3_codes_agree(gpu_codes: np.ndarray, x: np.ndarray, scale: float):
    """Compare e4m3 values written by the kernels with the oracle's codes of
    the exact quotient x / scale.  A value may differ only where an e4m3
    rounding boundary lies within E4M3_QUOTIENT_REL (relative) of the exact
    quotient, and it must then be one of the two values on either side of
    that boundary: the kernels' fp32 quotient, within that distance of the
    exact one, may fall on the other side.  Returns (mismatches accepted by
    that rule, boolean mask of elements that break it)."""
    want = oracle.quantize_e4m3(x, scale)
    a = oracle.quantize_e4m3(x * (1.0 - E4M3_QUOTIENT_REL), scale)
    b = oracle.quantize_e4m3(x * (1.0 + E4M3_QUOTIENT_REL), scale)
    lo, hi = np.minimum(a, b), np.maximum(a, b)
    same = gpu_codes == want
    near = (~same) & (lo != hi) & (gpu_codes >= lo) & (gpu_codes <= hi)
    return int(near.sum()), ~(same | near)


def compare_attention(cfg: Config, o_gpu, lse_gpu, orc_res):
    """Max-abs / mean-abs of O and max-abs of LSE over the oracle's items."""
    og = o_gpu.float().cpu().numpy()
    lg = lse_gpu.cpu().numpy()
    max_o = 0.0
    sum_o = 0.0
    n_o = 0
    max_l = 0.0
    for (b, h, i), (O, L) in orc_res.items():
        s0, e0 = i * cfg.blk, min(cfg.Lc, (i + 1) * cfg.blk)
        d = np.abs(og[b, s0:e0, h, :].astype(np.float64) - O)
        max_o = max(max_o, float(d.max()))
        sum_o += float(d.sum())
        n_o += d.size
        max_l = max(max_l, float(np.abs(lg[b, h, s0:e0].astype(np.float64) - L).max()))
    return max_o, sum_o / max(n_o, 1), max_l


def assert_attention_ok(cfg, o_gpu, lse_gpu, orc_res, what=""):
    max_o, mean_o, max_l = compare_attention(cfg, o_gpu, lse_gpu, orc_res)
    assert max_o <= O_MAX_ABS, f"{what}: O max-abs {max_o:.3e}"
    assert mean_o <= O_MEAN_ABS, f"{what}: O mean-abs {mean_o:.3e}"
    assert max_l <= LSE_ABS, f"{what}: LSE max-abs {max_l:.3e}"
    return max_o, mean_o, max_l


def oracle_idx_array(cfg: Config, orc_masks: Dict[int, dict]):
    """[B, H, nb, k_eff] idx and [B, H, nb] cnt from per-head oracle masks."""
    k_eff = next(iter(orc_masks.values()))["idx"].shape[-1]
    idx = np.full((cfg.B, cfg.H, cfg.nb, k_eff), -1, dtype=np.int32)
    cnt = np.zeros((cfg.B, cfg.H, cfg.nb), dtype=np.int32)
    for h, r in orc_masks.items():
        idx[:, h] = r["idx"][:, 0]
        cnt[:, h] = r["cnt"][:, 0]
    return idx, cnt


def sample_items(cfg: Config, n: int, seed: int = 0):
    """Work items (b, h, i) spread over heads and q-blocks; always includes the
    first and the ragged last q-block."""
    r = np.random.default_rng(seed)
    items = {(0, 0, 0), (cfg.B - 1, cfg.H - 1, cfg.nb - 1), (0, cfg.H // 2, cfg.nb - 1)}
    while len(items) < min(n, cfg.B * cfg.H * cfg.nb):
        items.add((int(r.integers(cfg.B)), int(r.integers(cfg.H)), int(r.integers(cfg.nb))))
    return sorted(items)


def fill_window(cfg: Config, seed: int, n_chunks: int, gpu: GpuStream, orc: OracleStream, keep=None):
    """Append chunks 0..n_chunks-1 of the seeded stream to both sides; returns
    the inputs of the last chunk."""
    last = None
    for t in range(n_chunks):
        last = chunk_inputs(cfg, seed, t)
        gpu.append(last, keep=keep)
        orc.append(last, keep=keep)
    return last
