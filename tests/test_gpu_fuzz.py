"""Seeded random configurations against the fp64 oracle: batch, heads and
grouped-query ratio, chunk length (ragged last blocks), window capacity, block
size, density, stream length (window not yet full, wrapped ring, crops,
replace-newest), anchored windows and the local band.  For each: the GPU mask
on every row (bit-exact up to the near-tie rule), and the attention with the
oracle's mask through the plain and the balanced schedule on every item."""
import math

import numpy as np
import pytest
import torch

from uf_testlib import GpuStream, OracleStream, assert_attention_ok, compare_masks, oracle_idx_array
from workloads import CONFIGS, chunk_inputs, scaled

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _random_case(seed):
    r = np.random.default_rng(1000 + seed)
    G = int(r.choice([1, 2, 3]))
    H = G * int(r.choice([1, 2, 4]))
    blk = int(r.choice([64, 128]))
    Lc = int(r.integers(40, 1300))
    W = int(r.integers(1, 5))
    B = int(r.choice([1, 1, 2]))
    dense = bool(r.random() < 0.25)
    cfg = scaled(CONFIGS["1k_sr"], B=B, H=H, G=G, Lc=Lc, W=W, blk=blk, density=1.0 if dense else float(r.uniform(0.1, 0.6)),
                 offsets=bool(r.random() < 0.7))
    n_chunks = int(r.integers(1, W + 3))
    anchor = W >= 2 and r.random() < 0.25
    ops = []
    for t in range(n_chunks):
        keep = None if r.random() < 0.7 else int(r.integers(2 if anchor else 1, W + 1))
        replace = t > 0 and r.random() < 0.15
        ops.append((keep, replace, anchor and t == 0))
    local = int(r.integers(0, 3)) if not dense and r.random() < 0.3 else 0
    return cfg, ops, local


@pytest.fixture(scope="module", autouse=True)
def _lib(built_lib):
    uf = built_lib
    uf.uf_get_error(clear=True)
    yield uf
    assert uf.uf_get_error(clear=True) == 0, "a kernel recorded a device-side error"


@pytest.mark.parametrize("seed", range(40))
def test_random_configuration(_lib, seed):
    uf = _lib
    cfg, ops, local = _random_case(seed)
    gpu, orc = GpuStream(cfg), OracleStream(cfg)
    last = None
    for t, (keep, replace, anchor) in enumerate(ops):
        last = chunk_inputs(cfg, 77 + seed, t)
        gpu.append(last, keep=keep, replace=replace, anchor=anchor)
        orc.append(last, keep=keep, replace=replace, anchor=anchor)
    nkv = cfg.nb * orc.n_valid
    items = [(b, h, i) for b in range(cfg.B) for h in range(cfg.H) for i in range(cfg.nb)]
    scale = 1.0 / math.sqrt(cfg.D)
    ws = torch.empty(uf.uf_attn_workspace_bytes(), dtype=torch.uint8, device="cuda")
    if cfg.dense:
        idx_t = cnt_t = None
        k = 0
        ref = orc.attention(last["q"], items)
    else:
        k = max(min(cfg.k_for(), cfg.W * cfg.nb), 2 * local + 1)
        if 2 * local + 1 > cfg.W * cfg.nb:
            local = 0
            k = max(1, min(cfg.k_for(), cfg.W * cfg.nb))
        idx, cnt, _ = gpu.mask(last["q"], k, want_scores=False, local=local)
        om = orc.mask(last["q"], k, local=local)
        torch.cuda.synchronize()
        rows, exact, ties, bad = compare_masks(cfg, idx, cnt, om, k)
        assert not bad, (seed, bad[:3])
        oidx, ocnt = oracle_idx_array(cfg, om)
        idx_t, cnt_t = torch.from_numpy(oidx).cuda(), torch.from_numpy(ocnt).cuda()
        k = oidx.shape[-1]
        ref = orc.attention(last["q"], items, oidx, ocnt)
    q = last["q"].cuda()
    for balanced in (False, True):
        o = torch.full((cfg.B, cfg.Lc, cfg.H, cfg.D), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((cfg.B, cfg.H, cfg.Lc), float("nan"), dtype=torch.float32, device="cuda")
        if balanced:
            uf.uf_block_sparse_attn_balanced(q, cfg.H, gpu.win.desc, idx_t, cnt_t, k, scale, o, lse, ws)
        else:
            uf.uf_block_sparse_attn(q, cfg.H, gpu.win.desc, idx_t, cnt_t, k, scale, o, lse)
        torch.cuda.synchronize()
        assert_attention_ok(cfg, o, lse, ref, f"seed {seed} balanced={balanced} nkv={nkv}")
