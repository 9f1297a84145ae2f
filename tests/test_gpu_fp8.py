"""GPU parity of the FP8-score variant (FlashDecoder, inference optimisations:
statically calibrated FP8): the e4m3 copy of K that the append writes, bit
for bit, and the attention whose scores are e4m3 q . e4m3 k on the tensor
cores, against the fp64 oracle's fp8_scores_attention on the same codes.

The oracle rounds the exact quotient x / scale; the kernels form it in fp32
as x * fp32(1 / scale), within 2^-23 relative of the exact one.  With an
arbitrary scale the codes are compared with a near-boundary rule
(uf_testlib.e4m3_codes_agree): equal, except where an e4m3 rounding boundary
lies within that distance of the exact quotient.  One such flip moves a score
by one e4m3 step of one element, up to 1/8 of a large code, which can move an
LSE by 1e-2; so the attention is compared at the bf16 path's tolerances
unchanged on (a) power-of-two scales, where the quotient is exact in fp32 and
both sides hold the same codes, and (b) arbitrary scales, on every row that no
near-boundary element of q or of its kept keys touches."""
import math

import numpy as np
import pytest
import torch

import oracle
from uf_testlib import (E4M3_QUOTIENT_REL, LSE_ABS, O_MAX_ABS, O_MEAN_ABS, GpuStream, OracleStream,
                        assert_attention_ok, e4m3_codes_agree, fill_window, oracle_idx_array, sample_items)
from workloads import CONFIGS, chunk_inputs, scaled

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

CASES = {
    # 64-token blocks, top-4 of 8, ragged last block (300 = 4 * 64 + 44)
    "blk64": scaled(CONFIGS["tiny"], H=2, G=1, Lc=300, k_fixed=3),
    # grouped-query heads (4 per KV head), window of 3, dense
    "gqa_w3": scaled(CONFIGS["gqa_decoder"], B=2, H=8, G=2, Lc=700, W=3),
    # block-offset inputs, window of 3, top-k density 25%
    "sr_w3": scaled(CONFIGS["1k_sr"], H=4, G=4, Lc=1000, W=3),
}


@pytest.fixture(scope="module", autouse=True)
def _lib(built_lib):
    uf = built_lib
    uf.uf_get_error(clear=True)
    yield uf
    assert uf.uf_get_error(clear=True) == 0, "a kernel recorded a device-side error"


def static_scales(cfg, seed, pow2=True):
    """Per-tensor scales calibrated once on chunk 0 of the stream: amax / 448,
    rounded up to a power of two unless pow2 is False.  With a power-of-two
    scale the quotient x / scale is exact in fp32, so the codes do not depend
    on how it is formed."""
    inp = chunk_inputs(cfg, seed, 0)
    qs = float(inp["q"].float().abs().max()) / oracle.E4M3_MAX
    ks = float(inp["k"].float().abs().max()) / oracle.E4M3_MAX
    if pow2:
        qs, ks = 2.0 ** math.ceil(math.log2(qs)), 2.0 ** math.ceil(math.log2(ks))
    else:   # the values the library receives (fp32)
        qs, ks = float(np.float32(qs)), float(np.float32(ks))
    return qs, ks


def _stream(cfg, n, seed, anchor=False, pow2=True):
    qs, ks = static_scales(cfg, seed, pow2)
    gpu, orc = GpuStream(cfg, k_scale=ks), OracleStream(cfg)
    last = None
    for t in range(n):
        last = chunk_inputs(cfg, seed, t)
        gpu.append(last, anchor=anchor and t == 0)
        orc.append(last, anchor=anchor and t == 0)
    torch.cuda.synchronize()
    return gpu, orc, last, qs, ks


def _slot(win, c):
    start, anchor = int(win.meta[0].item()), int(win.meta[3].item())
    if anchor:
        return win.W - 1 if c == 0 else (start + c - 1) % (win.W - 1)
    return (start + c) % win.W


@pytest.mark.parametrize("name,anchor", [("blk64", False), ("gqa_w3", False), ("sr_w3", True)])
def test_fp8_k_codes_bit_exact(name, anchor):
    # arbitrary (not power-of-two) scales: codes equal up to the near-boundary rule
    cfg = CASES[name]
    gpu, orc, _, _, ks = _stream(cfg, cfg.W + 2, seed=21, anchor=anchor, pow2=False)
    n_near = 0
    k8 = gpu.win.k8.view(torch.float8_e4m3fn).to(torch.float64).cpu().numpy()
    raw = gpu.win.k8.cpu().numpy()
    for g in range(cfg.G):
        w = orc.windows[g]
        for c in range(orc.n_valid):
            slot = _slot(gpu.win, c)
            r0 = slot * gpu.win.lslot
            near, bad = e4m3_codes_agree(k8[:, g, r0:r0 + cfg.Lc], w.k[c][:, :, 0, :], ks)
            assert not bad.any(), (g, c, int(bad.sum()))
            n_near += near
            assert not raw[:, g, r0 + cfg.Lc:r0 + gpu.win.lslot].any(), "padding rows must be zero"
    print(f"{name}: {n_near} e4m3 codes differ from the oracle's, each next to a rounding boundary")


def test_fp8_k_code_at_an_exact_midpoint():
    # K = 175/512 with k_scale = 7/64: the exact quotient 3.125 is the midpoint
    # between the e4m3 values 3.0 and 3.25 (the oracle takes 3.0, ties to even);
    # the kernel's fp32 product lies just above it.  The near-boundary rule
    # accepts either value there and nothing else
    cfg = CASES["blk64"]
    ks = 7.0 / 64.0
    gpu = GpuStream(cfg, k_scale=ks)
    inp = chunk_inputs(cfg, 25, 0)
    inp["k"][:, : cfg.Lc // 2] = 175.0 / 512.0
    gpu.append(inp)
    torch.cuda.synchronize()
    k8 = gpu.win.k8.view(torch.float8_e4m3fn).to(torch.float64).cpu().numpy()
    r0 = _slot(gpu.win, 0) * gpu.win.lslot
    got = k8[:, :, r0:r0 + cfg.Lc // 2]
    assert set(np.unique(got).tolist()) <= {3.0, 3.25}
    x = inp["k"][:, : cfg.Lc].double().numpy().transpose(0, 2, 1, 3)
    near, bad = e4m3_codes_agree(k8[:, :, r0:r0 + cfg.Lc], x, ks)
    assert not bad.any()


@pytest.mark.parametrize("name", ["blk64", "gqa_w3", "sr_w3"])
def test_fp8_attention_parity(name):
    cfg = CASES[name]
    gpu, orc, last, qs, ks = _stream(cfg, cfg.W + 1, seed=22)
    items = [(b, h, i) for b in range(cfg.B) for h in range(cfg.H) for i in range(cfg.nb)]
    if cfg.dense:
        o, lse = gpu.attention_fp8(last["q"], qs)
        torch.cuda.synchronize()
        assert_attention_ok(cfg, o, lse, orc.attention_fp8(last["q"], items, qs, ks), name)
        return
    k = cfg.k_for()
    oidx, ocnt = oracle_idx_array(cfg, orc.mask(last["q"], k))
    o, lse = gpu.attention_fp8(last["q"], qs, torch.from_numpy(oidx).cuda(), torch.from_numpy(ocnt).cuda(),
                               oidx.shape[-1])
    torch.cuda.synchronize()
    assert_attention_ok(cfg, o, lse, orc.attention_fp8(last["q"], items, qs, ks, oidx, ocnt), name)


def _near_boundary(x, scale):
    """Elements of x whose exact quotient x / scale lies within the kernels'
    fp32 quotient error of an e4m3 rounding boundary."""
    rel = E4M3_QUOTIENT_REL
    return oracle.quantize_e4m3(x * (1 - rel), scale) != oracle.quantize_e4m3(x * (1 + rel), scale)


@pytest.mark.parametrize("name", ["blk64", "sr_w3"])
def test_fp8_attention_arbitrary_scales_untouched_rows(name):
    # scales that are not powers of two: every row whose q and whose kept keys
    # hold no near-boundary element must meet the bf16 tolerances.  The scales
    # are amax / 448 times 1.0123457, not a simple fraction of the bf16 data's
    # amax (amax / 448 itself puts many bf16 values exactly on e4m3 midpoints,
    # e.g. 0.75 amax on 336; those cases are the code test's), so the rows
    # touched are few
    cfg = CASES[name]
    qs, ks = (float(np.float32(x * 1.0123457)) for x in static_scales(cfg, 26, pow2=False))
    gpu, orc = GpuStream(cfg, k_scale=ks), OracleStream(cfg)
    last = fill_window(cfg, 26, cfg.W + 1, gpu, orc)
    k = cfg.k_for()
    oidx, ocnt = oracle_idx_array(cfg, orc.mask(last["q"], k))
    o, lse = gpu.attention_fp8(last["q"], qs, torch.from_numpy(oidx).cuda(), torch.from_numpy(ocnt).cuda(),
                               oidx.shape[-1])
    items = [(b, h, i) for b in range(cfg.B) for h in range(cfg.H) for i in range(cfg.nb)]
    ref = orc.attention_fp8(last["q"], items, qs, ks, oidx, ocnt)
    torch.cuda.synchronize()
    og, lg = o.float().cpu().numpy(), lse.cpu().numpy()
    qnear = _near_boundary(last["q"].double().numpy(), qs).any(axis=-1)            # [B, Lc, H]
    kv_near = []                                                                    # per head group: [B, NKV*blk]
    for g in range(cfg.G):
        w = orc.windows[g]
        toks = np.concatenate([_near_boundary(kc[:, :, 0, :], ks).any(axis=-1) for kc in w.k], axis=1)
        kv_near.append(toks)
    max_o = max_l = sum_o = 0.0
    n_o = touched = rows = 0
    for (b, h, i), (O, L) in ref.items():
        g = h // (cfg.H // cfg.G)
        s0, e0 = i * cfg.blk, min(cfg.Lc, (i + 1) * cfg.blk)
        kept_touched = False
        for j in oidx[b, h, i, :ocnt[b, h, i]]:
            c, r = divmod(int(j), cfg.nb)
            t0 = c * cfg.Lc + r * cfg.blk
            kept_touched |= bool(kv_near[g][b, t0:min(t0 + cfg.blk, (c + 1) * cfg.Lc)].any())
        for rr in range(e0 - s0):
            rows += 1
            if kept_touched or qnear[b, s0 + rr, h]:
                touched += 1
                continue
            d = np.abs(og[b, s0 + rr, h] - O[rr])
            max_o, sum_o, n_o = max(max_o, float(d.max())), sum_o + float(d.sum()), n_o + d.size
            max_l = max(max_l, abs(float(lg[b, h, s0 + rr]) - float(L[rr])))
    assert touched <= rows // 4, (touched, rows)
    assert max_o <= O_MAX_ABS and sum_o / n_o <= O_MEAN_ABS and max_l <= LSE_ABS, (max_o, sum_o / n_o, max_l)


def test_fp8_anchored_window_and_saturation():
    # anchored window; the scales are calibrated on a quarter of chunk 0's
    # amax, so the largest q and k saturate at +-448 on both sides
    cfg = CASES["sr_w3"]
    qs, ks = static_scales(cfg, 23)
    qs, ks = qs / 4, ks / 4
    gpu, orc = GpuStream(cfg, k_scale=ks), OracleStream(cfg)
    last = None
    for t in range(cfg.W + 2):
        last = chunk_inputs(cfg, 23, t)
        gpu.append(last, anchor=t == 0)
        orc.append(last, anchor=t == 0)
    k8 = gpu.win.k8.view(torch.float8_e4m3fn).to(torch.float64).cpu().numpy()
    assert (np.abs(k8) == oracle.E4M3_MAX).any()
    o, lse = gpu.attention_fp8(last["q"], qs)
    items = [(b, h, i) for b in range(cfg.B) for h in range(cfg.H) for i in range(cfg.nb)]
    torch.cuda.synchronize()
    assert_attention_ok(cfg, o, lse, orc.attention_fp8(last["q"], items, qs, ks), "anchored saturated")


def test_fp8_is_close_to_bf16_scores():
    # the two variants differ only by the e4m3 rounding of q and k (scales
    # calibrated on every chunk here, so nothing saturates).  With
    # |dq| <= 2^-4 (|q| + 2^-6 q_scale) and the same for k, each score moves by
    # at most D = (2^-3 + 2^-8) scale max_j sum_i (|q_i| + 2^-6 q_scale)(|k_ji| + 2^-6 k_scale),
    # so |LSE8 - LSE16| <= D and each probability by a factor within e^(+-2D)
    cfg = CASES["gqa_w3"]
    chunks = [chunk_inputs(cfg, 24, t) for t in range(cfg.W)]
    qs = float(chunks[-1]["q"].float().abs().max()) / oracle.E4M3_MAX
    ks = max(float(c["k"].float().abs().max()) for c in chunks) / oracle.E4M3_MAX
    gpu = GpuStream(cfg, k_scale=ks)
    for c in chunks:
        gpu.append(c)
    q = chunks[-1]["q"]
    o8, l8 = gpu.attention_fp8(q, qs)
    o16, l16 = gpu.attention(q)
    torch.cuda.synchronize()
    scale = cfg.D ** -0.5
    delta = 0.0
    for b in range(cfg.B):
        for h in range(cfg.H):
            g = h // (cfg.H // cfg.G)
            a = q[b, :, h, :].double().abs() + qs / 64
            kk = torch.cat([c["k"][b, :, g, :] for c in chunks]).double().abs() + ks / 64
            delta = max(delta, (2.0 ** -3 + 2.0 ** -8) * scale * float((a @ kk.t()).max()))
    assert float((l8 - l16).abs().max()) <= delta
    vmax = max(float(c["v"].float().abs().max()) for c in chunks)
    # both outputs also carry bf16 probabilities (2^-9 relative each) and bf16 O
    bound = (np.expm1(2 * delta) + 2.0 ** -7) * vmax
    assert float((o8.float() - o16.float()).abs().max()) <= bound


def test_fp8_full_size_1k():
    cfg = CONFIGS["1k_sr"]
    gpu, orc, last, qs, ks = _stream(cfg, cfg.W + 1, seed=0)
    k = cfg.k_for()
    oidx, ocnt = oracle_idx_array(cfg, orc.mask(last["q"], k))
    o, lse = gpu.attention_fp8(last["q"], qs, torch.from_numpy(oidx).cuda(), torch.from_numpy(ocnt).cuda(),
                               oidx.shape[-1])
    items = sample_items(cfg, 12, seed=5)
    torch.cuda.synchronize()
    assert_attention_ok(cfg, o, lse, orc.attention_fp8(last["q"], items, qs, ks, oidx, ocnt), "1k fp8")


def test_fp8_full_size_2k():
    cfg = CONFIGS["2k_sr"]
    gpu, orc, last, qs, ks = _stream(cfg, cfg.W + 1, seed=1)
    k = cfg.k_for()
    oidx, ocnt = oracle_idx_array(cfg, orc.mask(last["q"], k))
    o, lse = gpu.attention_fp8(last["q"], qs, torch.from_numpy(oidx).cuda(), torch.from_numpy(ocnt).cuda(),
                               oidx.shape[-1])
    items = sample_items(cfg, 10, seed=6)
    torch.cuda.synchronize()
    assert_attention_ok(cfg, o, lse, orc.attention_fp8(last["q"], items, qs, ks, oidx, ocnt), "2k fp8")
