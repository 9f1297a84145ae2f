"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.  Reduced sizes are compared element by element; the full
workload sizes are compared on every mask row and on sampled attention work
items (all rows of each sampled (batch, head, q-block) tile)."""
import math

import numpy as np
import pytest
import torch

import oracle

from uf_testlib import (NEAR_TIE_REL, GpuStream, OracleStream, assert_attention_ok, compare_masks,
                              fill_window, oracle_idx_array, sample_items)
from workloads import CONFIGS, chunk_inputs, scaled, to_f64

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

SMALL = {
    # several q/kv tiles, ragged last block (104 tokens), top-k density 25%
    "small_sr": scaled(CONFIGS["1k_sr"], H=4, G=4, Lc=1000),
    # 2K-like density 15%, last block of 80 tokens, 3 heads
    "small_2k": scaled(CONFIGS["2k_sr"], H=3, G=3, Lc=2000),
    # grouped-query heads (6 q heads over 2 KV heads), batch 2, window of 3, dense
    "small_gqa": scaled(CONFIGS["gqa_decoder"], B=2, H=6, G=2, Lc=700, W=3),
    # 64-token blocks, last block of 44 tokens, fixed k = 3
    "small_blk64": scaled(CONFIGS["tiny"], H=2, G=1, Lc=300, k_fixed=3),
    "tiny": CONFIGS["tiny"],
    # one partial block per chunk (Lc < block)
    "lc100": scaled(CONFIGS["1k_sr"], H=2, G=2, Lc=100, density=1.0, offsets=False),
}


@pytest.fixture(scope="module", autouse=True)
def _lib(built_lib):
    uf = built_lib
    uf.uf_get_error(clear=True)
    yield uf
    assert uf.uf_get_error(clear=True) == 0, "a kernel recorded a device-side error"


def _slot_chunk(win, c, g, b=0):
    start = int(win.meta[0].item())
    slot = (start + c) % win.W
    rows = slice(slot * win.lslot, slot * win.lslot + win.Lc)
    pad = slice(slot * win.lslot + win.Lc, (slot + 1) * win.lslot)
    # v is stored transposed: [B, G, D, W*Lslot]
    return slot, win.k[b, g, rows], win.v[b, g, :, rows].t(), win.k[b, g, pad], win.v[b, g, :, pad].t()


# ----------------------------------------------------------------- append ----
@pytest.mark.parametrize("name", ["small_sr", "small_gqa", "small_blk64", "lc100"])
def test_append_window_state_and_contents(name):
    cfg = SMALL[name]
    gpu, orc = GpuStream(cfg), OracleStream(cfg)
    # plain appends past the capacity, a replace of the newest chunk, crops, regrowth
    ops = [(None, False)] * (cfg.W + 2) + [(None, True)] + [(max(1, cfg.W - 1), False), (1, False),
                                                             (1, True), (None, False), (None, False)]
    for t, (keep, replace) in enumerate(ops):
        inp = chunk_inputs(cfg, 7, t)
        gpu.append(inp, keep=keep, replace=replace)
        orc.append(inp, keep=keep, replace=replace)
        torch.cuda.synchronize()
        meta = gpu.win.meta.cpu().tolist()
        assert meta[1] == orc.n_valid == gpu.win.n_valid, (t, meta)
        assert meta[0] == gpu.win.desc.host_start and meta[2] == 0
        for g in range(cfg.G):
            w = orc.windows[g]
            for c in range(orc.n_valid):
                for b in range(cfg.B):
                    slot, kk, vv, kpad, vpad = _slot_chunk(gpu.win, c, g, b)
                    assert np.array_equal(kk.double().cpu().numpy(), w.k[c][b, :, 0, :]), (t, g, c)
                    assert np.array_equal(vv.double().cpu().numpy(), w.v[c][b, :, 0, :]), (t, g, c)
                    assert kpad.abs().sum().item() == 0 and vpad.abs().sum().item() == 0
                    # pooled K of the slot = fp64 block means (fp32 on the GPU)
                    kp = gpu.win.kpool[b, g, slot * cfg.nb:(slot + 1) * cfg.nb].double().cpu().numpy()
                    ref = oracle.pool_blocks(w.k[c][b:b + 1], cfg.blk)[0, 0]
                    assert np.allclose(kp, ref, rtol=1e-5, atol=1e-6), (t, g, c)


# ------------------------------------------------------------------- mask -----
def _mask_case(cfg, seed=0, n_chunks=None, want_scores=True):
    gpu, orc = GpuStream(cfg), OracleStream(cfg)
    last = fill_window(cfg, seed, cfg.W if n_chunks is None else n_chunks, gpu, orc)
    k = cfg.k_for(orc.n_valid) if not cfg.dense else cfg.nkv(orc.n_valid)
    k_arg = max(1, min(cfg.k_for(), cfg.nkv()))     # the row stride the caller allocates
    idx, cnt, scores = gpu.mask(last["q"], k_arg, want_scores=want_scores)
    om = orc.mask(last["q"], k_arg)
    torch.cuda.synchronize()
    return gpu, orc, last, idx, cnt, scores, om, k


@pytest.mark.parametrize("name", ["small_sr", "small_2k", "small_blk64", "tiny", "small_gqa"])
def test_mask_parity_small(name):
    cfg = SMALL[name]
    gpu, orc, last, idx, cnt, scores, om, k = _mask_case(cfg)
    rows, exact, ties, bad = compare_masks(cfg, idx, cnt, om, k)
    assert not bad, bad[:5]
    assert exact + ties == rows and exact >= rows - 2
    sc = scores.cpu().numpy()
    nkv = cfg.nkv(orc.n_valid)
    for h, r in om.items():
        assert np.allclose(sc[:, h, :, :nkv], r["scores"][:, 0], rtol=1e-5, atol=1e-6)


def test_mask_before_window_fills():
    cfg = SMALL["small_sr"]                      # W = 2, one chunk appended
    gpu, orc, last, idx, cnt, scores, om, k = _mask_case(cfg, seed=3, n_chunks=1)
    assert orc.n_valid == 1
    rows, exact, ties, bad = compare_masks(cfg, idx, cnt, om, k)
    assert not bad, bad[:5]
    assert torch.all(cnt == min(cfg.k_for(), cfg.nkv(1)))


def test_mask_k_one_and_k_all():
    cfg = SMALL["small_2k"]
    gpu, orc = GpuStream(cfg), OracleStream(cfg)
    last = fill_window(cfg, 5, cfg.W, gpu, orc)
    for k in (1, cfg.nkv()):
        idx, cnt, _ = gpu.mask(last["q"], k, want_scores=False)
        torch.cuda.synchronize()
        gi = idx.cpu().numpy()
        if k == 1:
            diag = (cfg.W - 1) * cfg.nb + np.arange(cfg.nb)
            assert np.array_equal(gi[..., 0], np.broadcast_to(diag, gi.shape[:-1]))
        else:
            assert np.array_equal(gi, np.broadcast_to(np.arange(k), gi.shape))


# -------------------------------------------------------------- attention -----
@pytest.mark.parametrize("name", ["small_sr", "small_2k", "small_blk64", "tiny"])
def test_attention_parity_with_oracle_mask(name):
    cfg = SMALL[name]
    gpu, orc, last, idx, cnt, scores, om, k = _mask_case(cfg, seed=1, want_scores=False)
    oidx, ocnt = oracle_idx_array(cfg, om)
    o, lse = gpu.attention(last["q"], torch.from_numpy(oidx).cuda(), torch.from_numpy(ocnt).cuda(), oidx.shape[-1])
    items = [(b, h, i) for b in range(cfg.B) for h in range(cfg.H) for i in range(cfg.nb)]
    ref = orc.attention(last["q"], items, oidx, ocnt)
    torch.cuda.synchronize()
    assert_attention_ok(cfg, o, lse, ref, name)


@pytest.mark.parametrize("name", ["small_gqa", "lc100", "small_sr", "small_blk64"])
def test_attention_dense_parity(name):
    cfg = SMALL[name]
    gpu, orc = GpuStream(cfg), OracleStream(cfg)
    last = fill_window(cfg, 2, cfg.W, gpu, orc)
    o, lse = gpu.attention(last["q"])
    items = [(b, h, i) for b in range(cfg.B) for h in range(cfg.H) for i in range(cfg.nb)]
    ref = orc.attention(last["q"], items)
    torch.cuda.synchronize()
    assert_attention_ok(cfg, o, lse, ref, name)


def test_attention_first_chunk_and_replace_newest():
    cfg = SMALL["small_gqa"]
    gpu, orc = GpuStream(cfg), OracleStream(cfg)
    items = [(b, h, i) for b in range(cfg.B) for h in range(cfg.H) for i in range(cfg.nb)]
    first = chunk_inputs(cfg, 11, 0)
    gpu.append(first)
    orc.append(first)
    o, lse = gpu.attention(first["q"])                     # window of one chunk
    assert_attention_ok(cfg, o, lse, orc.attention(first["q"], items), "first chunk")
    second = chunk_inputs(cfg, 11, 1)
    gpu.append(second)
    orc.append(second)
    redo = chunk_inputs(cfg, 11, 2)                       # recomputed K/V of the newest chunk
    gpu.append(redo, replace=True)
    orc.append(redo, replace=True)
    o, lse = gpu.attention(redo["q"])
    assert_attention_ok(cfg, o, lse, orc.attention(redo["q"], items), "replace newest")


def test_attention_end_to_end_on_agreeing_rows():
    cfg = SMALL["small_sr"]
    gpu, orc, last, idx, cnt, scores, om, k = _mask_case(cfg, seed=4, want_scores=False)
    o, lse = gpu.attention(last["q"], idx, cnt, idx.shape[-1])
    oidx, ocnt = oracle_idx_array(cfg, om)
    gi = idx.cpu().numpy()
    items = [(b, h, i) for b in range(cfg.B) for h in range(cfg.H) for i in range(cfg.nb)
             if np.array_equal(gi[b, h, i, :ocnt[b, h, i]], oidx[b, h, i, :ocnt[b, h, i]])]
    assert len(items) >= cfg.B * cfg.H * cfg.nb - 2
    ref = orc.attention(last["q"], items, oidx, ocnt)
    assert_attention_ok(cfg, o, lse, ref, "gpu mask -> gpu attention")


def test_attention_unordered_index_list():
    # the attention accepts kept blocks in any order
    cfg = SMALL["small_2k"]
    gpu, orc, last, idx, cnt, scores, om, k = _mask_case(cfg, seed=6, want_scores=False)
    oidx, ocnt = oracle_idx_array(cfg, om)
    rev = np.ascontiguousarray(oidx[..., ::-1])
    o, lse = gpu.attention(last["q"], torch.from_numpy(rev).cuda(), torch.from_numpy(ocnt).cuda(), rev.shape[-1])
    items = sample_items(cfg, 12, seed=2)
    assert_attention_ok(cfg, o, lse, orc.attention(last["q"], items, oidx, ocnt), "reversed idx")


# ------------------------------------------------------- device-side errors ---
def test_out_of_range_index_is_replaced_and_reported(_lib):
    uf = _lib
    cfg = SMALL["small_sr"]
    gpu, orc, last, idx, cnt, scores, om, k = _mask_case(cfg, seed=8, want_scores=False)
    oidx, ocnt = oracle_idx_array(cfg, om)
    bad = oidx.copy()
    bad[0, 1, 2, 0] = 10_000                       # out of range -> replaced by the diagonal block
    fixed = oidx.copy()
    fixed[0, 1, 2, 0] = (cfg.W - 1) * cfg.nb + 2
    o, lse = gpu.attention(last["q"], torch.from_numpy(bad).cuda(), torch.from_numpy(ocnt).cuda(), bad.shape[-1])
    assert uf.uf_get_error(clear=True) == uf.UF_EBOUNDS
    ref = orc.attention(last["q"], [(0, 1, 2), (0, 0, 0)], fixed, ocnt)
    assert_attention_ok(cfg, o, lse, ref, "substituted index")


def test_empty_row_gives_zero_output_and_reports(_lib):
    uf = _lib
    cfg = SMALL["small_sr"]
    gpu, orc, last, idx, cnt, scores, om, k = _mask_case(cfg, seed=9, want_scores=False)
    c2 = cnt.clone()
    c2[0, 3, 1] = 0
    o, lse = gpu.attention(last["q"], idx, c2, idx.shape[-1])
    assert uf.uf_get_error(clear=True) == uf.UF_EBOUNDS
    assert torch.all(o[0, cfg.blk:2 * cfg.blk, 3].float() == 0)
    assert torch.all(torch.isneginf(lse[0, 3, cfg.blk:2 * cfg.blk]))
    oidx, ocnt = oracle_idx_array(cfg, om)
    assert_attention_ok(cfg, o, lse, orc.attention(last["q"], [(0, 3, 0), (0, 2, 1)], oidx, ocnt), "others")


def test_bounded_wait_times_out_without_hanging(_lib):
    uf = _lib
    assert uf.uf_get_error(clear=True) == 0
    uf.uf_debug_wait_timeout(200_000)
    assert uf.uf_get_error(clear=True) == uf.UF_ETIMEOUT
    assert uf.uf_get_error(clear=True) == 0


# ------------------------------------------------------------- full sizes -----
@pytest.mark.parametrize("name", ["1k_sr", "2k_sr"])
def test_full_size_sparse(name):
    cfg = CONFIGS[name]
    gpu, orc, last, idx, cnt, scores, om, k = _mask_case(cfg, seed=0, want_scores=False)
    rows, exact, ties, bad = compare_masks(cfg, idx, cnt, om, k)
    assert not bad, bad[:3]
    assert exact >= rows - 3
    # attention fed with the oracle's mask, sampled work items (incl. the ragged last q-block)
    oidx, ocnt = oracle_idx_array(cfg, om)
    o, lse = gpu.attention(last["q"], torch.from_numpy(oidx).cuda(), torch.from_numpy(ocnt).cuda(), oidx.shape[-1])
    items = sample_items(cfg, 16, seed=1)
    assert_attention_ok(cfg, o, lse, orc.attention(last["q"], items, oidx, ocnt), name)
    # and the end-to-end GPU mask -> GPU attention on the same items
    o2, lse2 = gpu.attention(last["q"], idx, cnt, idx.shape[-1])
    gi = idx.cpu().numpy()
    agree = [it for it in items if np.array_equal(gi[it][:ocnt[it]], oidx[it][:ocnt[it]])]
    assert_attention_ok(cfg, o2, lse2, orc.attention(last["q"], agree, oidx, ocnt), name + " e2e")


def test_single_chunk_window():
    # W = 1: every append replaces the only chunk; the window is the newest chunk
    cfg = scaled(CONFIGS["1k_sr"], H=4, G=2, Lc=1000, W=1)
    gpu, orc, last, idx, cnt, scores, om, k = _mask_case(cfg, seed=13, n_chunks=3, want_scores=True)
    rows, exact, ties, bad = compare_masks(cfg, idx, cnt, om, k)
    assert not bad, bad[:3]
    assert exact >= rows - 1
    assert gpu.win.meta[1].item() == 1
    oidx, ocnt = oracle_idx_array(cfg, om)
    o, lse = gpu.attention(last["q"], torch.from_numpy(oidx).cuda(), torch.from_numpy(ocnt).cuda(), oidx.shape[-1])
    items = [(b, h, i) for b in range(cfg.B) for h in range(cfg.H) for i in range(cfg.nb)]
    assert_attention_ok(cfg, o, lse, orc.attention(last["q"], items, oidx, ocnt), "W = 1")
    od, lsed = gpu.attention(last["q"])
    assert_attention_ok(cfg, od, lsed, orc.attention(last["q"], items), "W = 1 dense")


def test_large_scores_exercise_the_rescale_path():
    # queries scaled by 30: scores in the hundreds, rows sharply peaked, so the
    # reference max rises by more than 2^8 many times within an item and O is
    # rescaled in tensor memory; blocks in reversed order make it rise late
    cfg = scaled(CONFIGS["1k_sr"], H=4, G=4, Lc=1000)
    gpu, orc = GpuStream(cfg), OracleStream(cfg)
    last = fill_window(cfg, 17, cfg.W, gpu, orc)
    q = (last["q"].float() * 30).to(torch.bfloat16)
    k = cfg.k_for()
    oidx, ocnt = oracle_idx_array(cfg, orc.mask(q, k))
    rev = np.ascontiguousarray(oidx[..., ::-1])
    items = [(b, h, i) for b in range(cfg.B) for h in range(cfg.H) for i in range(cfg.nb)]
    ref = orc.attention(q, items, oidx, ocnt)
    for idx_arr in (oidx, rev):
        o, lse = gpu.attention(q, torch.from_numpy(idx_arr).cuda(), torch.from_numpy(ocnt).cuda(), idx_arr.shape[-1])
        assert_attention_ok(cfg, o, lse, ref, "large scores")
    o, lse = gpu.attention(q)
    assert_attention_ok(cfg, o, lse, orc.attention(q, items), "large scores dense")


def test_largest_window_the_mask_supports():
    # W * nb = 1024 window blocks (32 selection keys per lane): 8 chunks of 128
    # blocks, 64-token blocks with a ragged last one (8191 = 127 * 64 + 63)
    cfg = scaled(CONFIGS["1k_sr"], H=2, G=1, Lc=8191, W=8, blk=64, density=0.1)
    assert cfg.W * cfg.nb == 1024
    gpu, orc, last, idx, cnt, scores, om, k = _mask_case(cfg, seed=12, want_scores=False)
    rows, exact, ties, bad = compare_masks(cfg, idx, cnt, om, k)
    assert not bad, bad[:3]
    assert exact >= rows - 2
    oidx, ocnt = oracle_idx_array(cfg, om)
    o, lse = gpu.attention(last["q"], torch.from_numpy(oidx).cuda(), torch.from_numpy(ocnt).cuda(), oidx.shape[-1])
    items = sample_items(cfg, 8, seed=3)
    assert_attention_ok(cfg, o, lse, orc.attention(last["q"], items, oidx, ocnt), "1024-block window")


def test_full_size_480p_dense():
    cfg = CONFIGS["480p_dense"]
    gpu, orc = GpuStream(cfg), OracleStream(cfg)
    last = fill_window(cfg, 0, cfg.W, gpu, orc)
    o, lse = gpu.attention(last["q"])
    items = sample_items(cfg, 12, seed=3)
    assert_attention_ok(cfg, o, lse, orc.attention(last["q"], items), "480p dense")


def test_full_size_gqa_rolling_stream():
    cfg = CONFIGS["gqa_decoder"]
    gpu, orc = GpuStream(cfg), OracleStream(cfg)
    for t in range(cfg.stream_len):
        inp = chunk_inputs(cfg, 0, t)
        gpu.append(inp, keep=cfg.W)
        orc.append(inp, keep=cfg.W)
        o, lse = gpu.attention(inp["q"])
        if t in (0, 1, 7, cfg.stream_len - 1):
            items = sample_items(cfg, 6, seed=t)
            assert_attention_ok(cfg, o, lse, orc.attention(inp["q"], items), f"frame {t}")
    # memory independent of stream length: the window holds W frames
    assert gpu.win.n_valid == cfg.W and int(gpu.win.meta[1].item()) == cfg.W


def test_full_size_tiny_everything():
    cfg = CONFIGS["tiny"]
    gpu, orc, last, idx, cnt, scores, om, k = _mask_case(cfg, seed=0)
    rows, exact, ties, bad = compare_masks(cfg, idx, cnt, om, k)
    assert not bad and exact == rows
    o, lse = gpu.attention(last["q"], idx, cnt, idx.shape[-1])
    items = [(0, h, i) for h in range(cfg.H) for i in range(cfg.nb)]
    oidx, ocnt = oracle_idx_array(cfg, om)
    assert_attention_ok(cfg, o, lse, orc.attention(last["q"], items, oidx, ocnt), "tiny")
