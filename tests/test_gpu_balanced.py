"""Parity of the balanced attention schedule (uf_block_sparse_attn_balanced):
the kept blocks of all work items are divided evenly over the SMs, items cut
between thread blocks are computed in parts and merged in-kernel by the part
that finishes last.  Checked against the fp64 oracle on every element at
reduced sizes (items cut into 2 to 18 parts, dense and sparse, rows shorter
than the nominal length, empty rows and bad indices) and at the full GQA
decoder and 480P sizes; with many items per SM the call must give the plain
schedule's output bit for bit."""
import math

import numpy as np
import pytest
import torch

from uf_testlib import (GpuStream, OracleStream, assert_attention_ok, fill_window, oracle_idx_array, sample_items)
from workloads import CONFIGS, chunk_inputs, scaled

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

CASES = {
    # 8 items of 4 kept blocks on all SMs: every block of an item in another part
    "tiny": CONFIGS["tiny"],
    # dense, grouped-query heads (3 per KV head), batch 2, window of 3: 72 items of 18 blocks
    "gqa_b2": scaled(CONFIGS["gqa_decoder"], B=2, H=6, G=2, Lc=700, W=3),
    # sparse top-k with block offsets: 32 items of 4 blocks, ragged last block
    "sr_small": scaled(CONFIGS["1k_sr"], H=4, G=4, Lc=1000),
    # 64-token blocks, dense, 3-chunk window: 60 items of 30 blocks
    "blk64_dense": scaled(CONFIGS["tiny"], H=4, G=2, Lc=600, W=3, density=1.0, offsets=False),
}


@pytest.fixture(scope="module", autouse=True)
def _lib(built_lib):
    uf = built_lib
    uf.uf_get_error(clear=True)
    yield uf
    assert uf.uf_get_error(clear=True) == 0, "a kernel recorded a device-side error"


@pytest.fixture(scope="module")
def ws(_lib):
    return torch.empty(_lib.uf_attn_workspace_bytes(), dtype=torch.uint8, device="cuda")


def balanced(uf, gpu, cfg, q_cpu, ws, idx=None, cnt=None, k=0):
    q = q_cpu.cuda()
    o = torch.full((cfg.B, cfg.Lc, cfg.H, cfg.D), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((cfg.B, cfg.H, cfg.Lc), float("nan"), dtype=torch.float32, device="cuda")
    uf.uf_block_sparse_attn_balanced(q, cfg.H, gpu.win.desc, idx, cnt, k, 1.0 / math.sqrt(cfg.D), o, lse, ws)
    return o, lse


def _all_items(cfg):
    return [(b, h, i) for b in range(cfg.B) for h in range(cfg.H) for i in range(cfg.nb)]


@pytest.mark.parametrize("name", sorted(CASES))
def test_balanced_parity_every_element(_lib, ws, name):
    cfg = CASES[name]
    gpu, orc = GpuStream(cfg), OracleStream(cfg)
    last = fill_window(cfg, 51, cfg.W, gpu, orc)
    items = _all_items(cfg)
    if cfg.dense:
        o, lse = balanced(_lib, gpu, cfg, last["q"], ws)
        ref = orc.attention(last["q"], items)
    else:
        oidx, ocnt = oracle_idx_array(cfg, orc.mask(last["q"], cfg.k_for()))
        idx, cnt = torch.from_numpy(oidx).cuda(), torch.from_numpy(ocnt).cuda()
        o, lse = balanced(_lib, gpu, cfg, last["q"], ws, idx, cnt, oidx.shape[-1])
        ref = orc.attention(last["q"], items, oidx, ocnt)
    torch.cuda.synchronize()
    assert_attention_ok(cfg, o, lse, ref, name)
    # and close to the plain schedule (same blocks, fp32 merge of the parts)
    if cfg.dense:
        o2, lse2 = gpu.attention(last["q"])
    else:
        o2, lse2 = gpu.attention(last["q"], idx, cnt, oidx.shape[-1])
    torch.cuda.synchronize()
    assert float((o.float() - o2.float()).abs().max()) <= 2 ** -7
    assert float((lse - lse2).abs().max()) <= 1e-4


def test_balanced_rows_shorter_than_the_stride(_lib, ws):
    # idx rows with fewer kept blocks than the row stride k (cnt < k), lists in
    # any order: parts past an item's true length are empty and skipped
    cfg = CASES["sr_small"]
    gpu, orc = GpuStream(cfg), OracleStream(cfg)
    last = fill_window(cfg, 52, cfg.W, gpu, orc)
    oidx, ocnt = oracle_idx_array(cfg, orc.mask(last["q"], cfg.k_for()))
    k_wide = 12
    r = np.random.default_rng(5)
    idx = np.full(oidx.shape[:-1] + (k_wide,), -1, dtype=np.int32)
    cnt = np.zeros(ocnt.shape, dtype=np.int32)
    nkv = cfg.nkv()
    for b in range(cfg.B):
        for h in range(cfg.H):
            for i in range(cfg.nb):
                n = int(r.integers(1, k_wide + 1))
                sel = r.permutation(nkv)[:n]
                idx[b, h, i, :n] = sel
                cnt[b, h, i] = n
    o, lse = balanced(_lib, gpu, cfg, last["q"], ws, torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda(),
                      k_wide)
    torch.cuda.synchronize()
    assert_attention_ok(cfg, o, lse, orc.attention(last["q"], _all_items(cfg), idx, cnt), "short rows")


def test_balanced_empty_row_and_bad_index(_lib, ws):
    uf = _lib
    cfg = CASES["sr_small"]
    gpu, orc = GpuStream(cfg), OracleStream(cfg)
    last = fill_window(cfg, 53, cfg.W, gpu, orc)
    oidx, ocnt = oracle_idx_array(cfg, orc.mask(last["q"], cfg.k_for()))
    cnt = ocnt.copy()
    cnt[0, 2, 3] = 0                                   # empty row: O = 0, LSE = -inf
    bad = oidx.copy()
    bad[0, 1, 4, 1] = 99_999                           # replaced by the diagonal block
    fixed = oidx.copy()
    fixed[0, 1, 4, 1] = (cfg.W - 1) * cfg.nb + 4
    o, lse = balanced(uf, gpu, cfg, last["q"], ws, torch.from_numpy(bad).cuda(), torch.from_numpy(cnt).cuda(),
                      bad.shape[-1])
    torch.cuda.synchronize()
    assert uf.uf_get_error(clear=True) == uf.UF_EBOUNDS
    assert torch.all(o[0, 3 * cfg.blk:4 * cfg.blk, 2].float() == 0)
    assert torch.all(torch.isneginf(lse[0, 2, 3 * cfg.blk:4 * cfg.blk]))
    items = [it for it in _all_items(cfg) if it != (0, 2, 3)]
    assert_attention_ok(cfg, o, lse, orc.attention(last["q"], items, fixed, cnt), "others")


def test_balanced_many_items_is_the_plain_schedule(_lib, ws):
    # at least 8 items per SM: the plain schedule, bit for bit, workspace untouched
    cfg = scaled(CONFIGS["1k_sr"], H=12, G=12, Lc=18720)
    gpu, orc = GpuStream(cfg), OracleStream(cfg)
    last = fill_window(cfg, 54, cfg.W, gpu, orc)
    idx, cnt, _ = gpu.mask(last["q"], cfg.k_for(), want_scores=False)
    ws.fill_(0x5A)
    o1, l1 = gpu.attention(last["q"], idx, cnt, idx.shape[-1])
    o2, l2 = balanced(_lib, gpu, cfg, last["q"], ws, idx, cnt, idx.shape[-1])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert bool((ws == 0x5A).all())


def test_balanced_full_size_gqa_stream(_lib, ws):
    cfg = CONFIGS["gqa_decoder"]
    gpu, orc = GpuStream(cfg), OracleStream(cfg)
    for t in range(cfg.stream_len):
        inp = chunk_inputs(cfg, 0, t)
        gpu.append(inp, keep=cfg.W)
        orc.append(inp, keep=cfg.W)
        o, lse = balanced(_lib, gpu, cfg, inp["q"], ws)
        if t in (0, 1, cfg.stream_len - 1):
            torch.cuda.synchronize()
            items = _all_items(cfg) if t == cfg.stream_len - 1 else sample_items(cfg, 12, seed=t)
            assert_attention_ok(cfg, o, lse, orc.attention(inp["q"], items), f"frame {t}: {len(items)} items")


def test_balanced_full_size_480p_dense(_lib, ws):
    cfg = CONFIGS["480p_dense"]
    gpu, orc = GpuStream(cfg), OracleStream(cfg)
    last = fill_window(cfg, 0, cfg.W, gpu, orc)
    o, lse = balanced(_lib, gpu, cfg, last["q"], ws)
    torch.cuda.synchronize()
    items = sample_items(cfg, 24, seed=4)
    assert_attention_ok(cfg, o, lse, orc.attention(last["q"], items), "480p balanced")


def test_balanced_call_replays_in_a_captured_graph(_lib, ws):
    # the call's counter memset and kernel capture into a CUDA graph; each
    # replay (after a new chunk's queries are copied in) equals the eager call
    # bit for bit
    cfg = CASES["gqa_b2"]
    gpu, orc = GpuStream(cfg), OracleStream(cfg)
    fill_window(cfg, 55, cfg.W, gpu, orc)
    qs = [chunk_inputs(cfg, 56, t)["q"].cuda() for t in range(3)]
    q_static = torch.empty_like(qs[0])
    o = torch.empty(cfg.B, cfg.Lc, cfg.H, cfg.D, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(cfg.B, cfg.H, cfg.Lc, dtype=torch.float32, device="cuda")
    scale = 1.0 / math.sqrt(cfg.D)
    eager = []
    for q in qs:
        _lib.uf_block_sparse_attn_balanced(q, cfg.H, gpu.win.desc, None, None, 0, scale, o, lse, ws)
        eager.append((o.clone(), lse.clone()))
    q_static.copy_(qs[0])
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        _lib.uf_block_sparse_attn_balanced(q_static, cfg.H, gpu.win.desc, None, None, 0, scale, o, lse, ws)
    for t, q in enumerate(qs):
        q_static.copy_(q)
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, eager[t][0]) and torch.equal(lse, eager[t][1]), t
    del graph
