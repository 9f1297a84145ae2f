"""ChunkPipeline (copy in / compute / copy out on three streams) gives the
same outputs, bit for bit, as running each chunk's copies and calls one after
the other on one stream: the overlap changes when work runs, not what it
computes or the order in which the window sees its appends."""
import math

import pytest
import torch

from workloads import CONFIGS, chunk_inputs, scaled

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module", autouse=True)
def _lib(built_lib):
    uf = built_lib
    uf.uf_get_error(clear=True)
    yield uf
    assert uf.uf_get_error(clear=True) == 0, "a kernel recorded a device-side error"


@pytest.mark.parametrize("depth", [2, 3])
def test_pipeline_matches_serial(_lib, depth):
    uf = _lib
    cfg = scaled(CONFIGS["1k_sr"], H=4, G=2, Lc=1000, W=2)
    n_chunks = 6
    chunks = [{n: x.pin_memory() for n, x in chunk_inputs(cfg, 31, t).items()} for t in range(n_chunks)]
    k = cfg.k_for()
    scale = 1.0 / math.sqrt(cfg.D)
    o_shape, lse_shape = (cfg.B, cfg.Lc, cfg.H, cfg.D), (cfg.B, cfg.H, cfg.Lc)

    def make(device="cuda"):
        win = uf.KVWindow(cfg.B, cfg.G, cfg.W, cfg.Lc, cfg.blk, cfg.D)
        win.reset()
        idx = torch.empty(cfg.B, cfg.H, cfg.nb, k, dtype=torch.int32, device=device)
        cnt = torch.empty(cfg.B, cfg.H, cfg.nb, dtype=torch.int32, device=device)

        def step(din, dout, stream=None):
            win.append(din["k"], din["v"], stream=stream)
            uf.uf_block_mask(din["q"], cfg.H, win.desc, k, idx, cnt, stream=stream)
            uf.uf_block_sparse_attn(din["q"], cfg.H, win.desc, idx, cnt, k, scale, dout["o"], dout["lse"],
                                    stream=stream)
        return step

    # serial: copy in, compute, copy out, one chunk at a time on one stream
    step = make()
    serial = []
    for c in chunks:
        din = {n: x.cuda() for n, x in c.items()}
        dout = {"o": torch.empty(o_shape, dtype=torch.bfloat16, device="cuda"),
                "lse": torch.empty(lse_shape, dtype=torch.float32, device="cuda")}
        step(din, dout)
        serial.append({n: x.cpu() for n, x in dout.items()})
    torch.cuda.synchronize()

    step = make()
    pipe = uf.ChunkPipeline({n: (tuple(x.shape), x.dtype) for n, x in chunks[0].items()},
                            {"o": (o_shape, torch.bfloat16), "lse": (lse_shape, torch.float32)},
                            step, depth=depth)
    outs = [{"o": torch.full(o_shape, float("nan"), dtype=torch.bfloat16).pin_memory(),
             "lse": torch.full(lse_shape, float("nan"), dtype=torch.float32).pin_memory()} for _ in chunks]
    for c, ho in zip(chunks, outs):
        pipe.submit(c, ho)
    pipe.synchronize()
    for t, (a, b) in enumerate(zip(serial, outs)):
        assert torch.equal(a["o"], b["o"]), t
        assert torch.equal(a["lse"], b["lse"]), t


def test_pipeline_rejects_depth_one():
    from block_sparse_causal_b200 import ChunkPipeline
    with pytest.raises(ValueError):
        ChunkPipeline({}, {}, lambda *a: None, depth=1)
