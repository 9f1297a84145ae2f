"""A per-chunk step (append, mask, attention) captured once in a CUDA graph
and replayed chunk after chunk gives the same outputs, bit for bit, as the
same calls made eagerly: the window state the kernels read lives on the
device, so a replay sees the window the previous replay left behind."""
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


@pytest.mark.parametrize("anchor", [False, True])
def test_graph_replay_matches_eager(_lib, anchor):
    uf = _lib
    cfg = scaled(CONFIGS["1k_sr"], H=4, G=2, Lc=1000, W=3)
    n_chunks = 7
    chunks = [{n: x.cuda() for n, x in chunk_inputs(cfg, 41, t).items()} for t in range(n_chunks)]
    k = cfg.k_for()
    scale = 1.0 / math.sqrt(cfg.D)

    def make():
        win = uf.KVWindow(cfg.B, cfg.G, cfg.W, cfg.Lc, cfg.blk, cfg.D)
        win.reset()
        bufs = {"idx": torch.empty(cfg.B, cfg.H, cfg.nb, k, dtype=torch.int32, device="cuda"),
                "cnt": torch.empty(cfg.B, cfg.H, cfg.nb, dtype=torch.int32, device="cuda"),
                "o": torch.empty(cfg.B, cfg.Lc, cfg.H, cfg.D, dtype=torch.bfloat16, device="cuda"),
                "lse": torch.empty(cfg.B, cfg.H, cfg.Lc, dtype=torch.float32, device="cuda")}

        def step(q, kn, vn, first=False):
            win.append(kn, vn, anchor=anchor and first)
            uf.uf_block_mask(q, cfg.H, win.desc, k, bufs["idx"], bufs["cnt"])
            uf.uf_block_sparse_attn(q, cfg.H, win.desc, bufs["idx"], bufs["cnt"], k, scale, bufs["o"], bufs["lse"])
        return win, bufs, step

    # eager
    _, bufs, step = make()
    eager = []
    for t, c in enumerate(chunks):
        step(c["q"], c["k"], c["v"], first=t == 0)
        eager.append({n: bufs[n].clone() for n in ("o", "lse", "idx", "cnt")})
    torch.cuda.synchronize()

    # chunk 0 eagerly, then one captured step replayed for chunks 1 ..
    win, bufs, step = make()
    step(chunks[0]["q"], chunks[0]["k"], chunks[0]["v"], first=True)
    static = {n: torch.empty_like(x) for n, x in chunks[0].items()}
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(static["q"], static["k"], static["v"])
    for t in range(1, n_chunks):
        for n, x in chunks[t].items():
            static[n].copy_(x)
        graph.replay()
        torch.cuda.synchronize()
        for n in ("o", "lse", "idx", "cnt"):
            assert torch.equal(bufs[n], eager[t][n]), (t, n)
    meta = win.meta.cpu().tolist()
    assert meta[1] == cfg.W and meta[2] == 0 and meta[3] == int(anchor), meta
    del graph
