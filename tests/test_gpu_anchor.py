"""GPU parity of the anchored rolling window (HiStream, innovation 2: one
anchor key frame plus a small cache of neighbouring frames): the window state
and contents after streams of appends, crops and replaces around a pinned
anchor, and the mask and attention over anchored windows, against the fp64
oracle's RollingWindow(anchor=True)."""
import numpy as np
import pytest
import torch

import oracle
from uf_testlib import (GpuStream, OracleStream, assert_attention_ok, compare_masks, oracle_idx_array,
                        sample_items)
from workloads import CONFIGS, chunk_inputs, scaled

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

CASES = {
    # window of 4: the anchor plus 3 recent chunks, sparse top-k
    "sr_w4": scaled(CONFIGS["1k_sr"], H=4, G=4, Lc=1000, W=4),
    # grouped-query heads, window of 3, dense
    "gqa_w3": scaled(CONFIGS["gqa_decoder"], B=2, H=6, G=2, Lc=700, W=3),
    # 64-token blocks, window of 2: the anchor plus the newest chunk
    "blk64_w2": scaled(CONFIGS["tiny"], H=2, G=1, Lc=300, k_fixed=3),
}


@pytest.fixture(scope="module", autouse=True)
def _lib(built_lib):
    uf = built_lib
    uf.uf_get_error(clear=True)
    yield uf
    assert uf.uf_get_error(clear=True) == 0, "a kernel recorded a device-side error"


def _slot(win, c):
    """Physical slot of logical chunk c (anchored: chunk 0 in slot W - 1, the
    others on a ring over slots 0 .. W - 2)."""
    start, anchor = int(win.meta[0].item()), int(win.meta[3].item())
    if anchor:
        return win.W - 1 if c == 0 else (start + c - 1) % (win.W - 1)
    return (start + c) % win.W


def _stream(cfg, ops, seed=3):
    gpu, orc = GpuStream(cfg), OracleStream(cfg)
    last = None
    for t, (keep, replace, anchor) in enumerate(ops):
        last = chunk_inputs(cfg, seed, t)
        gpu.append(last, keep=keep, replace=replace, anchor=anchor)
        orc.append(last, keep=keep, replace=replace, anchor=anchor)
    torch.cuda.synchronize()
    return gpu, orc, last


@pytest.mark.parametrize("name", ["sr_w4", "gqa_w3", "blk64_w2"])
def test_anchor_window_state_and_contents(name):
    cfg = CASES[name]
    gpu, orc = GpuStream(cfg), OracleStream(cfg)
    W = cfg.W
    ops = ([(None, False, True)] + [(None, False, False)] * (W + 2) + [(None, True, False)]
           + [(2, False, False), (2, True, False), (None, False, False), (None, False, False)])
    for t, (keep, replace, anchor) in enumerate(ops):
        inp = chunk_inputs(cfg, 9, t)
        gpu.append(inp, keep=keep, replace=replace, anchor=anchor)
        orc.append(inp, keep=keep, replace=replace, anchor=anchor)
        torch.cuda.synchronize()
        meta = gpu.win.meta.cpu().tolist()
        assert meta[1] == orc.n_valid and meta[3] == 1 and meta[2] == 0, (t, meta)
        assert meta[0] == gpu.win.desc.host_start and gpu.win.desc.host_anchor == 1
        for g in range(cfg.G):
            w = orc.windows[g]
            for c in range(orc.n_valid):
                slot = _slot(gpu.win, c)
                rows = slice(slot * gpu.win.lslot, slot * gpu.win.lslot + cfg.Lc)
                for b in range(cfg.B):
                    kk = gpu.win.k[b, g, rows].double().cpu().numpy()
                    vv = gpu.win.v[b, g, :, rows].t().double().cpu().numpy()
                    assert np.array_equal(kk, w.k[c][b, :, 0, :]), (t, g, c)
                    assert np.array_equal(vv, w.v[c][b, :, 0, :]), (t, g, c)
                    kp = gpu.win.kpool[b, g, slot * cfg.nb:(slot + 1) * cfg.nb].double().cpu().numpy()
                    assert np.allclose(kp, oracle.pool_blocks(w.k[c][b:b + 1], cfg.blk)[0, 0], rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("name", ["sr_w4", "blk64_w2"])
def test_anchor_mask_and_attention_parity(name):
    cfg = CASES[name]
    ops = [(None, False, True)] + [(None, False, False)] * (cfg.W + 3)
    gpu, orc, last = _stream(cfg, ops)
    k = max(1, min(cfg.k_for(), cfg.nkv()))
    idx, cnt, _ = gpu.mask(last["q"], k, want_scores=False)
    om = orc.mask(last["q"], k)
    torch.cuda.synchronize()
    rows, exact, ties, bad = compare_masks(cfg, idx, cnt, om, k)
    assert not bad, bad[:5]
    assert exact >= rows - 2
    oidx, ocnt = oracle_idx_array(cfg, om)
    o, lse = gpu.attention(last["q"], torch.from_numpy(oidx).cuda(), torch.from_numpy(ocnt).cuda(), oidx.shape[-1])
    items = [(b, h, i) for b in range(cfg.B) for h in range(cfg.H) for i in range(cfg.nb)]
    torch.cuda.synchronize()
    assert_attention_ok(cfg, o, lse, orc.attention(last["q"], items, oidx, ocnt), name)


def test_anchor_dense_attention_after_crop_and_replace():
    cfg = CASES["gqa_w3"]
    ops = [(None, False, True), (None, False, False), (None, False, False), (None, False, False),
           (2, False, False), (2, True, False)]
    gpu, orc, last = _stream(cfg, ops, seed=5)
    assert orc.n_valid == 2
    o, lse = gpu.attention(last["q"])
    items = [(b, h, i) for b in range(cfg.B) for h in range(cfg.H) for i in range(cfg.nb)]
    torch.cuda.synchronize()
    assert_attention_ok(cfg, o, lse, orc.attention(last["q"], items), "gqa anchored dense")


def test_anchor_full_size_1k():
    # the 1K workload with its window of 2: the anchor chunk plus the newest
    cfg = CONFIGS["1k_sr"]
    ops = [(None, False, True)] + [(None, False, False)] * 3
    gpu, orc, last = _stream(cfg, ops, seed=0)
    k = cfg.k_for()
    idx, cnt, _ = gpu.mask(last["q"], k, want_scores=False)
    om = orc.mask(last["q"], k)
    torch.cuda.synchronize()
    rows, exact, ties, bad = compare_masks(cfg, idx, cnt, om, k)
    assert not bad, bad[:3]
    assert exact >= rows - 3
    oidx, ocnt = oracle_idx_array(cfg, om)
    o, lse = gpu.attention(last["q"], torch.from_numpy(oidx).cuda(), torch.from_numpy(ocnt).cuda(), oidx.shape[-1])
    items = sample_items(cfg, 12, seed=4)
    torch.cuda.synchronize()
    assert_attention_ok(cfg, o, lse, orc.attention(last["q"], items, oidx, ocnt), "1k anchored")
