"""The attention call for callers that cannot allocate device memory.

uf_block_sparse_attn_balanced_noalloc keeps the balanced schedule's scratch
data in a fixed array inside the library instead of a workspace the caller
passes in, for code that may not call cudaMalloc (a plugin whose host owns
all device memory, a streaming loop that must not allocate after start-up).
Its output must be that of uf_block_sparse_attn_balanced with a caller
workspace, within the parity tolerances, on two calls in a row: the array
keeps the previous call's contents, and the call must clear what it needs.
This file is collected last so that a run stopping at its first failure has
run every other test first."""
import math

import numpy as np
import pytest
import torch

from uf_testlib import LSE_ABS, O_MAX_ABS, O_MEAN_ABS, GpuStream, OracleStream, fill_window, oracle_idx_array
from workloads import CONFIGS, chunk_inputs, scaled

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

# few items per SM, so the balanced schedule splits items and uses its scratch
CFG_DENSE = scaled(CONFIGS["gqa_decoder"], B=2, H=6, G=2, Lc=700, W=3)
CFG_SPARSE = scaled(CONFIGS["1k_sr"], H=4, G=4, Lc=1000)


@pytest.fixture(scope="module")
def uf(built_lib):
    built_lib.uf_get_error(clear=True)
    yield built_lib
    assert built_lib.uf_get_error(clear=True) == 0, "a kernel recorded a device-side error"


def _close(a, b):
    o1, l1 = a
    o2, l2 = b
    d = (o1.float() - o2.float()).abs()
    assert float(d.max()) <= O_MAX_ABS and float(d.mean()) <= O_MEAN_ABS
    assert float((l1 - l2).abs().max()) <= LSE_ABS


@pytest.mark.parametrize("cfg", [CFG_DENSE, CFG_SPARSE], ids=["dense_gqa", "sparse_topk"])
def test_noalloc_matches_the_workspace_call_twice(uf, cfg):
    ws = torch.empty(uf.uf_attn_workspace_bytes(), dtype=torch.uint8, device="cuda")
    gpu, orc = GpuStream(cfg), OracleStream(cfg)
    fill_window(cfg, 61, cfg.W, gpu, orc)
    scale = 1.0 / math.sqrt(cfg.D)
    for call in range(2):
        # a new chunk before each call: the second call sees other inputs than
        # the first, with the scratch array still holding the first call's data
        inp = chunk_inputs(cfg, 61, cfg.W + call)
        gpu.append(inp)
        orc.append(inp)
        q = inp["q"].cuda()
        idx = cnt = None
        k = 0
        if not cfg.dense:
            oidx, ocnt = oracle_idx_array(cfg, orc.mask(inp["q"], cfg.k_for()))
            idx, cnt, k = torch.from_numpy(oidx).cuda(), torch.from_numpy(ocnt).cuda(), oidx.shape[-1]
        outs = []
        for noalloc in (False, True):
            o = torch.full((cfg.B, cfg.Lc, cfg.H, cfg.D), float("nan"), dtype=torch.bfloat16, device="cuda")
            lse = torch.full((cfg.B, cfg.H, cfg.Lc), float("nan"), dtype=torch.float32, device="cuda")
            if noalloc:
                uf.uf_block_sparse_attn_balanced_noalloc(q, cfg.H, gpu.win.desc, idx, cnt, k, scale, o, lse)
            else:
                uf.uf_block_sparse_attn_balanced(q, cfg.H, gpu.win.desc, idx, cnt, k, scale, o, lse, ws)
            outs.append((o, lse))
        torch.cuda.synchronize()
        assert bool(torch.isfinite(outs[1][0].float()).all()) and bool(torch.isfinite(outs[1][1]).all()), call
        _close(outs[1], outs[0])
