"""Full-size attention parity over the persistent pipeline's item depth.

The attention kernel runs one thread block per SM, each looping over work
items c, c + grid, c + 2 grid, ... with barrier phases, S-buffer parities
and the Q staging tile carried from item to item.  A fault that shows only at
some depth of that loop, or at some head, is caught by comparing, at the 1K
and 2K workloads: every item of the first, the middle and the last query
head (depths 0, about half and the deepest of every thread block), every
head's last (ragged) q-block, and the last item each thread block takes.  The
same set is compared for the FP8-score and the RoPE variants at 1K.  Every
row's O and LSE must also be finite.  The item count is part of each test id."""
import numpy as np
import pytest
import torch

from test_gpu_fp8 import static_scales
from test_gpu_rope import _oracle_rope, _rope_stream
from uf_testlib import (GpuStream, OracleStream, assert_attention_ok, compare_masks, fill_window,
                        oracle_idx_array)
from workloads import CONFIGS, chunk_inputs

pytestmark = [pytest.mark.gpu, pytest.mark.slow,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

B200_SMS = 148


def coverage_items(cfg, sms=B200_SMS):
    """(b, h, i) work items: all of heads 0, H // 2 and H - 1, the last q-block
    of every head, and the last item of each of the min(items, sms) thread
    blocks."""
    nb, H = cfg.nb, cfg.H
    n_items = cfg.B * H * nb
    grid = min(n_items, sms)

    def unpack(item):
        return (item // nb // H, item // nb % H, item % nb)

    s = set()
    for b in range(cfg.B):
        for h in sorted({0, H // 2, H - 1}):
            s.update((b, h, i) for i in range(nb))
        s.update((b, h, nb - 1) for h in range(H))
    for c in range(grid):
        s.add(unpack(c + (n_items - 1 - c) // grid * grid))
    return sorted(s)


def _ids(name):
    return f"{name}-items={len(coverage_items(CONFIGS[name]))}"


@pytest.fixture(scope="module", autouse=True)
def _lib(built_lib):
    uf = built_lib
    uf.uf_get_error(clear=True)
    yield uf
    assert uf.uf_get_error(clear=True) == 0, "a kernel recorded a device-side error"


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def _finite(o, lse):
    assert bool(torch.isfinite(o.float()).all()), "non-finite O"
    assert bool(torch.isfinite(lse).all()), "non-finite LSE"


@pytest.mark.parametrize("name", ["1k_sr", "2k_sr"], ids=_ids)
def test_full_size_item_depth(name):
    cfg = CONFIGS[name]
    gpu, orc = GpuStream(cfg), OracleStream(cfg)
    last = fill_window(cfg, 2, cfg.W, gpu, orc)
    k = cfg.k_for()
    om = orc.mask(last["q"], k)
    oidx, ocnt = oracle_idx_array(cfg, om)
    o, lse = gpu.attention(last["q"], torch.from_numpy(oidx).cuda(), torch.from_numpy(ocnt).cuda(), oidx.shape[-1])
    torch.cuda.synchronize()
    _finite(o, lse)
    items = coverage_items(cfg, _sms())
    assert_attention_ok(cfg, o, lse, orc.attention(last["q"], items, oidx, ocnt), f"{name}: {len(items)} items")
    # the GPU's own mask, on every row, for the same inputs
    idx, cnt, _ = gpu.mask(last["q"], k, want_scores=False)
    rows, exact, ties, bad = compare_masks(cfg, idx, cnt, om, k)
    assert not bad, bad[:3]


def test_full_size_item_depth_fp8_1k():
    cfg = CONFIGS["1k_sr"]
    qs, ks = static_scales(cfg, 3)
    gpu, orc = GpuStream(cfg, k_scale=ks), OracleStream(cfg)
    last = None
    for t in range(cfg.W):
        last = chunk_inputs(cfg, 3, t)
        gpu.append(last)
        orc.append(last)
    oidx, ocnt = oracle_idx_array(cfg, orc.mask(last["q"], cfg.k_for()))
    o, lse = gpu.attention_fp8(last["q"], qs, torch.from_numpy(oidx).cuda(), torch.from_numpy(ocnt).cuda(),
                               oidx.shape[-1])
    torch.cuda.synchronize()
    _finite(o, lse)
    items = coverage_items(cfg, _sms())
    assert_attention_ok(cfg, o, lse, orc.attention_fp8(last["q"], items, qs, ks, oidx, ocnt),
                        f"1k fp8: {len(items)} items")


def test_full_size_item_depth_rope_1k():
    cfg = CONFIGS["1k_sr"]
    k = cfg.k_for()
    gpu, orc, last, q_rot, shift = _rope_stream(cfg, 4, 3)
    items = coverage_items(cfg, _sms())
    heads = sorted({h for (_, h, _) in items})
    om = _oracle_rope(cfg, orc, last["q"], k, shift, to_bf16=True, heads=heads)
    oidx = np.full((cfg.B, cfg.H, cfg.nb, k), -1, dtype=np.int32)
    ocnt = np.zeros((cfg.B, cfg.H, cfg.nb), dtype=np.int32)
    for h, r in om.items():
        oidx[:, h] = r["idx"][:, 0]
        ocnt[:, h] = r["cnt"][:, 0]
    o, lse = gpu.attention(q_rot.cpu(), torch.from_numpy(oidx).cuda(), torch.from_numpy(ocnt).cuda(), k)
    torch.cuda.synchronize()
    _finite(o, lse)
    ref = _oracle_rope(cfg, orc, last["q"], k, shift, True, heads=heads, items=items, idx=oidx, cnt=ocnt)
    assert_attention_ok(cfg, o, lse, ref, f"1k rope: {len(items)} items")
