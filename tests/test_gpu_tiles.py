"""GPU parity of the (2, 8, 8) tile token order (Ultra Flash notes, Method,
key design 3): uf_tile_tokens and uf_kv_append_tiled move tokens exactly
(bit-exact against the oracle's tile_order), and the whole step run in tiled
order -- tiled queries, tiled window, mask, attention, O back to row-major --
matches the oracle run on the same permutation."""
import numpy as np
import pytest
import torch

import oracle
from uf_testlib import (GpuStream, OracleStream, assert_attention_ok, compare_masks, oracle_idx_array,
                        sample_items)
from workloads import CONFIGS, chunk_inputs, scaled, to_f64

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module", autouse=True)
def _lib(built_lib):
    uf = built_lib
    uf.uf_get_error(clear=True)
    yield uf
    assert uf.uf_get_error(clear=True) == 0, "a kernel recorded a device-side error"


@pytest.mark.parametrize("B,grid,heads,tile", [(1, (3, 60, 104), 2, (2, 8, 8)), (2, (3, 10, 13), 3, (2, 8, 8)),
                                               (1, (1, 45, 80), 12, (2, 8, 8)), (1, (5, 9, 7), 1, (2, 4, 4))])
def test_tile_tokens_bit_exact(_lib, B, grid, heads, tile):
    L = int(np.prod(grid))
    x = torch.randn(B, L, heads, 128).to(torch.bfloat16)
    xd = x.cuda()
    y = torch.empty_like(xd)
    z = torch.empty_like(xd)
    _lib.uf_tile_tokens(xd, y, B, grid, heads, tile)
    _lib.uf_tile_tokens(y, z, B, grid, heads, tile, inverse=True)
    order = oracle.tile_order(*grid, tile)
    want = oracle.to_tile_order(x.float().numpy(), order)
    assert np.array_equal(y.float().cpu().numpy(), want)
    assert torch.equal(z, xd)


def _tiled_stream(cfg, seed, n_chunks, tile=(2, 8, 8)):
    """GPU: chunks appended in tiled order, queries tiled.  Oracle: the same
    chunks permuted with tile_order, appended as they are."""
    import block_sparse_causal_b200 as uf
    order = oracle.tile_order(*cfg.grid, tile)
    gpu, orc = GpuStream(cfg), OracleStream(cfg)
    for t in range(n_chunks):
        last = chunk_inputs(cfg, seed, t)
        gpu.win.append(last["k"].cuda(), last["v"].cuda(), tile_grid=cfg.grid, tile=tile)
        orc.append({n: torch.from_numpy(oracle.to_tile_order(last[n].float().numpy(), order)).to(torch.bfloat16)
                    for n in ("k", "v")})
    q = last["q"].cuda()
    q_t = torch.empty_like(q)
    uf.uf_tile_tokens(q, q_t, cfg.B, cfg.grid, cfg.H, tile)
    q_t_cpu = torch.from_numpy(oracle.to_tile_order(last["q"].float().numpy(), order)).to(torch.bfloat16)
    return gpu, orc, last, q_t, q_t_cpu, order


def test_append_tiled_stores_the_tiled_chunk(_lib):
    cfg = scaled(CONFIGS["1k_sr"], H=2, G=2, Lc=3 * 12 * 20, grid=(3, 12, 20))
    gpu, orc, last, q_t, q_t_cpu, order = _tiled_stream(cfg, 3, 3)
    torch.cuda.synchronize()
    start = int(gpu.win.meta[0].item())
    for c in range(orc.n_valid):
        slot = (start + c) % cfg.W
        rows = slice(slot * gpu.win.lslot, slot * gpu.win.lslot + cfg.Lc)
        for g in range(cfg.G):
            w = orc.windows[g]
            assert np.array_equal(gpu.win.k[0, g, rows].double().cpu().numpy(), w.k[c][0, :, 0, :])
            assert np.array_equal(gpu.win.v[0, g, :, rows].t().double().cpu().numpy(), w.v[c][0, :, 0, :])
            kp = gpu.win.kpool[0, g, slot * cfg.nb:(slot + 1) * cfg.nb].double().cpu().numpy()
            assert np.allclose(kp, oracle.pool_blocks(w.k[c], cfg.blk)[0, 0], rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("name", ["small_sr", "gqa"])
def test_tiled_step_parity(name):
    import block_sparse_causal_b200 as uf
    cfg = {"small_sr": scaled(CONFIGS["1k_sr"], H=4, G=4, Lc=3 * 16 * 24, grid=(3, 16, 24)),
           "gqa": scaled(CONFIGS["gqa_decoder"], H=6, G=2, Lc=45 * 24, grid=(1, 45, 24), density=0.5)}[name]
    gpu, orc, last, q_t, q_t_cpu, order = _tiled_stream(cfg, 5, cfg.W + 1)
    k = cfg.k_for()
    idx, cnt, _ = gpu.mask(q_t.cpu(), k, want_scores=False)
    om = orc.mask(q_t_cpu, k)
    torch.cuda.synchronize()
    rows, exact, ties, bad = compare_masks(cfg, idx, cnt, om, k)
    assert not bad, bad[:5]
    assert exact >= rows - 2
    oidx, ocnt = oracle_idx_array(cfg, om)
    o_t, lse = gpu.attention(q_t.cpu(), torch.from_numpy(oidx).cuda(), torch.from_numpy(ocnt).cuda(), oidx.shape[-1])
    items = [(b, h, i) for b in range(cfg.B) for h in range(cfg.H) for i in range(cfg.nb)]
    ref = orc.attention(q_t_cpu, items, oidx, ocnt)
    torch.cuda.synchronize()
    assert_attention_ok(cfg, o_t, lse, ref, name + " tiled")
    # O back to row-major order equals the oracle's output put back the same way
    o = torch.empty_like(o_t)
    uf.uf_tile_tokens(o_t, o, cfg.B, cfg.grid, cfg.H, inverse=True)
    O_t = np.full((cfg.B, cfg.Lc, cfg.H, cfg.D), np.nan)
    for (b, h, i), (O, _) in ref.items():
        O_t[b, i * cfg.blk:i * cfg.blk + O.shape[0], h] = O
    O_row = oracle.from_tile_order(O_t, order)
    assert np.abs(o.float().cpu().numpy() - O_row).max() <= 2e-2


def test_tiled_full_size_1k():
    cfg = CONFIGS["1k_sr"]
    gpu, orc, last, q_t, q_t_cpu, order = _tiled_stream(cfg, 0, 2)
    k = cfg.k_for()
    idx, cnt, _ = gpu.mask(q_t.cpu(), k, want_scores=False)
    om = orc.mask(q_t_cpu, k)
    torch.cuda.synchronize()
    rows, exact, ties, bad = compare_masks(cfg, idx, cnt, om, k)
    assert not bad, bad[:3]
    assert exact >= rows - 3
    oidx, ocnt = oracle_idx_array(cfg, om)
    o_t, lse = gpu.attention(q_t.cpu(), torch.from_numpy(oidx).cuda(), torch.from_numpy(ocnt).cuda(), oidx.shape[-1])
    items = sample_items(cfg, 12, seed=6)
    torch.cuda.synchronize()
    assert_attention_ok(cfg, o_t, lse, orc.attention(q_t_cpu, items, oidx, ocnt), "1k tiled")
