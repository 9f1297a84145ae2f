"""GPU parity of the rotary-position path: uf_rope and uf_kv_append_rope
against the fp64 oracle (RoFormer rotation, FlashDecoder's window-relative
positions).  The GPU rotates each chunk once, at its stream position; rotary
scores depend only on position differences, so the oracle's window-relative
definition is met exactly up to rounding (pinned on the CPU).  Mask decisions
are compared on the same bf16-rounded rotated values the cache holds (oracle
shift = the oldest chunk's stream position), attention also against the
plain window-relative definition in fp64."""
import math

import numpy as np
import pytest
import torch

import oracle
from uf_testlib import (O_MAX_ABS, O_MEAN_ABS, GpuStream, OracleStream, assert_attention_ok, compare_attention,
                        compare_masks, fill_window, oracle_idx_array, sample_items)
from workloads import CONFIGS, chunk_inputs, scaled, to_f64

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

# Against the unrounded definition, the bf16 storage of the rotated Q and K
# (relative rounding up to 2^-9 per element) moves a score scale * q . k by up
# to 2^-8 * scale * sum|q_d k_d| -- about 3e-3 typical and 3e-2 worst for
# N(0, 1) channels at D = 128 -- and LSE by a weighted mean of those moves.
LSE_ABS_UNROUNDED = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _lib(built_lib):
    uf = built_lib
    uf.uf_get_error(clear=True)
    yield uf
    assert uf.uf_get_error(clear=True) == 0, "a kernel recorded a device-side error"


def _bf16_step(v):
    """Spacing of the bf16 grid at |v| (8 significant bits)."""
    a = np.maximum(np.abs(v), 2.0 ** -120)
    return np.exp2(np.floor(np.log2(a)) - 7)


def _rope_bound(x, ref, max_pos):
    """Allowed |GPU - exact| per element: one bf16 step of the result (the
    final rounding) plus the rotation error, which scales with the norm of the
    channel pair (a rotated component near zero is a cancellation): fp32
    arithmetic, and the angle pos * theta, whose fp64 product is off by up to
    an ulp of pos (the header's bound: 1.2e-4 rad below 2^40)."""
    pair = np.sqrt(x[..., 0::2] ** 2 + x[..., 1::2] ** 2)
    pair = np.repeat(pair, 2, axis=-1)
    angle_err = 2.0 * max_pos * 2.0 ** -52
    return _bf16_step(ref) + (2.0 ** -18 + angle_err) * pair


@pytest.mark.parametrize("B,L,heads,pos0", [(1, 37, 3, 0), (2, 64, 2, 123456789), (1, 5, 12, 2 ** 40 - 5)])
def test_rope_kernel_within_one_bf16_step(_lib, B, L, heads, pos0):
    g = torch.Generator().manual_seed(B * 1000 + L)
    x = (torch.randn(B, L, heads, 128, generator=g) * 2).to(torch.bfloat16)
    xd = x.cuda()
    y = torch.empty_like(xd)
    _lib.uf_rope(xd, y, B, L, heads, pos0)
    ref = oracle.rope(to_f64(x), pos0 + np.arange(L))
    got = y.float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= _rope_bound(to_f64(x), ref, pos0 + L))
    _lib.uf_rope(xd, xd, B, L, heads, pos0)          # in place gives the same values
    assert torch.equal(xd, y)


def test_rope_position_zero_is_identity(_lib):
    x = torch.randn(1, 1, 4, 128).to(torch.bfloat16).cuda()
    y = torch.empty_like(x)
    _lib.uf_rope(x, y, 1, 1, 4, 0)
    assert torch.equal(x, y)


def test_append_rope_stores_rotated_keys(_lib):
    import block_sparse_causal_b200 as uf
    cfg = scaled(CONFIGS["1k_sr"], H=2, G=2, Lc=300)      # 3 blocks per chunk, last one 44 tokens
    win = uf.KVWindow(cfg.B, cfg.G, cfg.W, cfg.Lc, cfg.blk, cfg.D)
    win.reset()
    for t in range(3):                                   # the window slides once
        c = chunk_inputs(cfg, 7, t)
        win.append(c["k"].cuda(), c["v"].cuda(), rope_pos0=t * cfg.Lc)
    torch.cuda.synchronize()
    start = int(win.meta[0].item())
    slot = (start + 1) % cfg.W                           # the newest chunk (t = 2)
    rows = slice(slot * win.lslot, slot * win.lslot + cfg.Lc)
    ref = oracle.rope(to_f64(c["k"]), 2 * cfg.Lc + np.arange(cfg.Lc))[0]    # [Lc, G, D]
    for g in range(cfg.G):
        got = win.k[0, g, rows].float().cpu().numpy().astype(np.float64)
        assert np.all(np.abs(got - ref[:, g]) <= _rope_bound(to_f64(c["k"])[0][:, g], ref[:, g], 3 * cfg.Lc))
        vt = win.v[0, g, :, rows].t().cpu()
        assert torch.equal(vt, c["v"][0, :, g])          # V is stored as is
        # pooled K: block means of the rotated keys
        pooled = win.kpool[0, g, slot * cfg.nb:(slot + 1) * cfg.nb].cpu().numpy()
        for r0, (s0, e0) in enumerate(oracle.block_ranges(cfg.Lc, cfg.blk)):
            assert np.allclose(pooled[r0], ref[s0:e0, g].mean(axis=0), atol=2.0 ** -7, rtol=0)


def _rope_stream(cfg, seed, n_chunks, keep=None):
    """GPU: every chunk appended with RoPE at its stream position, the last
    chunk's queries rotated at the same position.  Oracle: the raw stream."""
    import block_sparse_causal_b200 as uf
    gpu, orc = GpuStream(cfg), OracleStream(cfg)
    firsts = []
    for t in range(n_chunks):
        last = chunk_inputs(cfg, seed, t)
        gpu.win.append(last["k"].cuda(), last["v"].cuda(), keep_chunks=keep, rope_pos0=t * cfg.Lc)
        orc.append(last, keep=keep)
        firsts.append(t * cfg.Lc)
    q = last["q"].cuda()
    q_rot = torch.empty_like(q)
    uf.uf_rope(q, q_rot, cfg.B, cfg.Lc, cfg.H, (n_chunks - 1) * cfg.Lc)
    shift = firsts[n_chunks - orc.n_valid]               # stream position of the window's oldest chunk
    return gpu, orc, last, q_rot, shift


def _oracle_rope(cfg, orc, q_cpu, k, shift, to_bf16, heads=None, items=None, idx=None, cnt=None):
    masks, att = {}, {}
    heads = range(cfg.H) if heads is None else heads
    for h in heads:
        qr, wr = oracle.window_rope(to_f64(q_cpu[:, :, h:h + 1]), orc.head_window(h), shift=shift, to_bf16=to_bf16)
        if idx is None:
            masks[h] = oracle.block_mask(qr, wr, cfg.blk, k)
        else:
            its = [(b, 0, i) for (b, hh, i) in items if hh == h]
            if its:
                O, L = oracle.block_sparse_attention(qr, wr, cfg.blk, idx[:, h:h + 1], cnt[:, h:h + 1], items=its)
                for (b, _, i) in its:
                    s0, e0 = i * cfg.blk, min(cfg.Lc, (i + 1) * cfg.blk)
                    att[(b, h, i)] = (O[b, s0:e0, 0, :], L[b, 0, s0:e0])
    return masks if idx is None else att


@pytest.mark.parametrize("name,n_chunks", [("small_sr", 4), ("tiny", 3), ("small_gqa", 3)])
def test_rope_stream_mask_and_attention(name, n_chunks):
    cases = {"small_sr": scaled(CONFIGS["1k_sr"], H=4, G=4, Lc=1000),
             "tiny": CONFIGS["tiny"],
             "small_gqa": scaled(CONFIGS["gqa_decoder"], B=2, H=6, G=2, Lc=700, W=3, density=0.4)}
    cfg = cases[name]
    k = cfg.k_for()
    gpu, orc, last, q_rot, shift = _rope_stream(cfg, 11, n_chunks)
    idx, cnt, _ = gpu.mask(q_rot.cpu(), k, want_scores=False)
    om = _oracle_rope(cfg, orc, last["q"], k, shift, to_bf16=True)
    torch.cuda.synchronize()
    rows, exact, ties, bad = compare_masks(cfg, idx, cnt, om, k)
    assert not bad, bad[:5]
    assert exact >= rows - 2
    # attention with the oracle's mask: against the stored-precision values and
    # against the plain window-relative definition (fp64, no rounding)
    oidx, ocnt = oracle_idx_array(cfg, om)
    o, lse = gpu.attention(q_rot.cpu(), torch.from_numpy(oidx).cuda(), torch.from_numpy(ocnt).cuda(), oidx.shape[-1])
    items = [(b, h, i) for b in range(cfg.B) for h in range(cfg.H) for i in range(cfg.nb)]
    torch.cuda.synchronize()
    ref = _oracle_rope(cfg, orc, last["q"], k, shift, True, items=items, idx=oidx, cnt=ocnt)
    assert_attention_ok(cfg, o, lse, ref, f"{name} rope")
    ref = _oracle_rope(cfg, orc, last["q"], k, 0, False, items=items, idx=oidx, cnt=ocnt)
    max_o, mean_o, max_l = compare_attention(cfg, o, lse, ref)
    assert max_o <= O_MAX_ABS and mean_o <= O_MEAN_ABS and max_l <= LSE_ABS_UNROUNDED, (max_o, mean_o, max_l)


def test_rope_full_size_1k():
    cfg = CONFIGS["1k_sr"]
    k = cfg.k_for()
    gpu, orc, last, q_rot, shift = _rope_stream(cfg, 0, 3)
    idx, cnt, _ = gpu.mask(q_rot.cpu(), k, want_scores=False)
    heads = [0, 7]                                       # attention samples; the mask is checked on every head
    om = _oracle_rope(cfg, orc, last["q"], k, shift, to_bf16=True)
    torch.cuda.synchronize()
    rows, exact, ties, bad = compare_masks(cfg, idx, cnt, om, k)
    assert not bad, bad[:3]
    assert exact >= rows - 3
    oidx, ocnt = oracle_idx_array(cfg, om)
    o, lse = gpu.attention(q_rot.cpu(), torch.from_numpy(oidx).cuda(), torch.from_numpy(ocnt).cuda(), oidx.shape[-1])
    items = [it for it in sample_items(cfg, 30, seed=2) if it[1] in heads]
    torch.cuda.synchronize()
    ref = _oracle_rope(cfg, orc, last["q"], k, shift, True, heads=heads, items=items, idx=oidx, cnt=ocnt)
    assert_attention_ok(cfg, o, lse, ref, "1k rope")
    ref = _oracle_rope(cfg, orc, last["q"], k, 0, False, heads=heads, items=items, idx=oidx, cnt=ocnt)
    max_o, mean_o, max_l = compare_attention(cfg, o, lse, ref)
    assert max_o <= O_MAX_ABS and mean_o <= O_MEAN_ABS and max_l <= LSE_ABS_UNROUNDED, (max_o, mean_o, max_l)
