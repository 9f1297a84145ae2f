"""GPU parity of the local-band block mask (uf_block_mask_local) against the
fp64 oracle: the band [diag - local, diag + local] is always kept, the rest of
each row is the top-scored other blocks (Ultra Flash notes, Method, key design
3: local sliding-window mask combined with per-head top-k), or the row is the
band alone (the ablation's fixed local window).  Masks bit-exact except
near-ties; attention fed with the oracle's local mask within the O / LSE
tolerances."""
import numpy as np
import pytest
import torch

from uf_testlib import (GpuStream, OracleStream, assert_attention_ok, compare_masks, fill_window,
                        oracle_idx_array, sample_items)
from workloads import CONFIGS, scaled

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

CASES = {
    # 8 blocks per chunk of 125 tokens (last block 104), window of 2, 4 heads
    "small_sr": scaled(CONFIGS["1k_sr"], H=4, G=4, Lc=1000),
    # 64-token blocks, grouped-query heads, window of 3
    "small_gqa64": scaled(CONFIGS["gqa_decoder"], H=4, G=2, Lc=700, W=3, blk=64, density=0.3),
    "tiny": CONFIGS["tiny"],
}


@pytest.fixture(scope="module", autouse=True)
def _lib(built_lib):
    uf = built_lib
    uf.uf_get_error(clear=True)
    yield uf
    assert uf.uf_get_error(clear=True) == 0, "a kernel recorded a device-side error"


def _case(cfg, k, local, local_only, seed=0, n_chunks=None):
    gpu, orc = GpuStream(cfg), OracleStream(cfg)
    last = fill_window(cfg, seed, cfg.W if n_chunks is None else n_chunks, gpu, orc)
    idx, cnt, _ = gpu.mask(last["q"], k, want_scores=False, local=local, local_only=local_only)
    om = orc.mask(last["q"], k, local=local, local_only=local_only)
    torch.cuda.synchronize()
    return gpu, orc, last, idx, cnt, om


@pytest.mark.parametrize("name,local,kplus", [("small_sr", 1, 2), ("small_sr", 3, 0), ("small_gqa64", 2, 5),
                                              ("tiny", 1, 1)])
def test_local_band_mask_parity(name, local, kplus):
    cfg = CASES[name]
    k = 2 * local + 1 + kplus
    gpu, orc, last, idx, cnt, om = _case(cfg, k, local, False)
    rows, exact, ties, bad = compare_masks(cfg, idx, cnt, om, k)
    assert not bad, bad[:5]
    assert exact + ties == rows and exact >= rows - 2
    # every row holds its clipped band
    gi, gc = idx.cpu().numpy(), cnt.cpu().numpy()
    nkv = cfg.nkv(orc.n_valid)
    for i in range(cfg.nb):
        d = (orc.n_valid - 1) * cfg.nb + i
        band = set(range(max(0, d - local), min(nkv - 1, d + local) + 1))
        for b in range(cfg.B):
            for h in range(cfg.H):
                assert band <= set(gi[b, h, i, :gc[b, h, i]].tolist())


@pytest.mark.parametrize("name,local", [("small_sr", 2), ("small_gqa64", 1), ("tiny", 0)])
def test_local_only_mask_is_the_band(name, local):
    cfg = CASES[name]
    k = 2 * local + 3
    gpu, orc, last, idx, cnt, om = _case(cfg, k, local, True, seed=2)
    rows, exact, ties, bad = compare_masks(cfg, idx, cnt, om, k)
    assert not bad and exact == rows


def test_local_band_before_window_fills():
    cfg = CASES["small_sr"]
    gpu, orc, last, idx, cnt, om = _case(cfg, 6, 2, False, seed=4, n_chunks=1)
    rows, exact, ties, bad = compare_masks(cfg, idx, cnt, om, 6)
    assert not bad, bad[:5]


@pytest.mark.parametrize("name,local", [("small_sr", 2), ("small_gqa64", 1)])
def test_attention_with_local_band_mask(name, local):
    cfg = CASES[name]
    k = cfg.k_for() if cfg.k_for() >= 2 * local + 1 else 2 * local + 1
    gpu, orc, last, idx, cnt, om = _case(cfg, k, local, False, seed=5)
    oidx, ocnt = oracle_idx_array(cfg, om)
    o, lse = gpu.attention(last["q"], torch.from_numpy(oidx).cuda(), torch.from_numpy(ocnt).cuda(), oidx.shape[-1])
    items = [(b, h, i) for b in range(cfg.B) for h in range(cfg.H) for i in range(cfg.nb)]
    torch.cuda.synchronize()
    assert_attention_ok(cfg, o, lse, orc.attention(last["q"], items, oidx, ocnt), name)


def test_full_size_1k_local_band():
    # the 1K workload (k = 74) with a band of 9 blocks around the diagonal
    cfg = CONFIGS["1k_sr"]
    k, local = cfg.k_for(), 4
    gpu, orc = GpuStream(cfg), OracleStream(cfg)
    last = fill_window(cfg, 0, cfg.W, gpu, orc)
    idx, cnt, _ = gpu.mask(last["q"], k, want_scores=False, local=local)
    heads = [0, 5, 11]
    om = orc.mask(last["q"], k, heads=heads, local=local)
    torch.cuda.synchronize()
    rows, exact, ties, bad = compare_masks(cfg, idx, cnt, om, k)
    assert not bad, bad[:3]
    assert exact >= rows - 3
    # attention with the GPU's local mask on sampled items of those heads whose rows agree with the oracle
    o, lse = gpu.attention(last["q"], idx, cnt, k)
    oi = {h: om[h]["idx"] for h in heads}
    gi = idx.cpu().numpy()
    items = [it for it in sample_items(cfg, 40, seed=3) if it[1] in heads
             and np.array_equal(gi[it], oi[it[1]][it[0], 0, it[2]])]
    assert len(items) >= 3
    oidx, ocnt = oracle_idx_array(cfg, {h: om[h] for h in heads})
    assert_attention_ok(cfg, o, lse, orc.attention(last["q"], items, oidx, ocnt), "1k local")


def test_full_size_1k_fixed_local_window_every_item_of_a_head():
    # the fixed-local-window workload at the full 1K size (band of 9 blocks, the
    # row stride k = 74): the mask is exactly the band on every row of two heads,
    # and the attention matches the oracle on every item of one of them
    cfg = CONFIGS["1k_sr"]
    k, local = cfg.k_for(), 4
    gpu, orc = GpuStream(cfg), OracleStream(cfg)
    last = fill_window(cfg, 7, cfg.W, gpu, orc)
    idx, cnt, _ = gpu.mask(last["q"], k, want_scores=False, local=local, local_only=True)
    o, lse = gpu.attention(last["q"], idx, cnt, k)
    heads = [0, 11]
    om = orc.mask(last["q"], k, heads=heads, local=local, local_only=True)
    torch.cuda.synchronize()
    rows, exact, ties, bad = compare_masks(cfg, idx, cnt, om, k)
    assert not bad and exact == rows == cfg.B * cfg.nb * len(heads)
    oidx, ocnt = oracle_idx_array(cfg, om)
    items = [(b, 11, i) for b in range(cfg.B) for i in range(cfg.nb)]
    assert_attention_ok(cfg, o, lse, orc.attention(last["q"], items, oidx, ocnt),
                        f"1k fixed local window, {len(items)} items of head 11")
