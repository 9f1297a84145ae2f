"""Failure detection on the GPU without a fault: errors the kernels find (an
out-of-range block index, a pipeline wait that reached its bound) are read in
stream order, also from inside a captured CUDA graph, and a window can carry
its own error word so that concurrent windows do not share one flag.  The
waits are made to run out by a short bound; nothing here hangs or faults."""
import math

import numpy as np
import pytest
import torch

from uf_testlib import GpuStream, OracleStream, assert_attention_ok, fill_window, oracle_idx_array
from workloads import CONFIGS, chunk_inputs, scaled

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

CFG = scaled(CONFIGS["1k_sr"], H=4, G=2, Lc=1000)


@pytest.fixture(scope="module", autouse=True)
def _lib(built_lib):
    uf = built_lib
    uf.uf_get_error(clear=True)
    yield uf
    uf.uf_set_wait_limit(1 << 31)
    assert uf.uf_get_error(clear=True) == 0, "a kernel recorded a device-side error"


def _case(seed):
    gpu, orc = GpuStream(CFG), OracleStream(CFG)
    last = fill_window(CFG, seed, CFG.W, gpu, orc)
    k = CFG.k_for()
    oidx, ocnt = oracle_idx_array(CFG, orc.mask(last["q"], k))
    return gpu, orc, last, oidx, ocnt


def _attend(uf, win, q, idx, cnt, stream=None):
    o = torch.empty(CFG.B, CFG.Lc, CFG.H, CFG.D, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(CFG.B, CFG.H, CFG.Lc, dtype=torch.float32, device="cuda")
    uf.uf_block_sparse_attn(q, CFG.H, win.desc, idx, cnt, idx.shape[-1], 1.0 / math.sqrt(CFG.D), o, lse,
                            stream=stream)
    return o, lse


def test_check_error_reads_the_word_in_stream_order(_lib):
    uf = _lib
    gpu, orc, last, oidx, ocnt = _case(31)
    q = last["q"].cuda()
    word = torch.zeros(1, dtype=torch.int32, device="cuda")
    good = torch.from_numpy(oidx).cuda()
    cnt = torch.from_numpy(ocnt).cuda()
    _attend(uf, gpu.win, q, good, cnt)
    uf.uf_check_error(word)
    torch.cuda.synchronize()
    assert int(word.item()) == 0
    bad = oidx.copy()
    bad[0, 1, 2, 0] = 10_000                        # out of range: UF_EBOUNDS
    _attend(uf, gpu.win, q, torch.from_numpy(bad).cuda(), cnt)
    uf.uf_check_error(word)                         # moves the error into `word`, clears the library's
    _attend(uf, gpu.win, q, good, cnt)
    uf.uf_check_error(word)                         # nothing new; `word` keeps the first error
    torch.cuda.synchronize()
    assert int(word.item()) == uf.UF_EBOUNDS
    assert uf.uf_get_error(clear=True) == 0


def test_check_error_inside_a_captured_graph(_lib):
    uf = _lib
    gpu, orc, last, oidx, ocnt = _case(32)
    q = last["q"].cuda()
    idx = torch.from_numpy(oidx).cuda()
    cnt = torch.from_numpy(ocnt).cuda()
    word = torch.zeros(1, dtype=torch.int32, device="cuda")
    _attend(uf, gpu.win, q, idx, cnt)               # first call outside the capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        o, lse = _attend(uf, gpu.win, q, idx, cnt)
        uf.uf_check_error(word)
    graph.replay()
    torch.cuda.synchronize()
    assert int(word.item()) == 0
    ref = orc.attention(last["q"], [(0, 1, 2), (0, 3, CFG.nb - 1)], oidx, ocnt)
    assert_attention_ok(CFG, o, lse, ref, "replayed")
    idx[0, 1, 2, 0] = -5                            # the next replay meets an out-of-range index
    graph.replay()
    torch.cuda.synchronize()
    assert int(word.item()) == uf.UF_EBOUNDS
    assert uf.uf_get_error(clear=True) == 0
    del graph


def test_each_window_records_in_its_own_word(_lib):
    uf = _lib
    a = uf.KVWindow(CFG.B, CFG.G, CFG.W, CFG.Lc, CFG.blk, CFG.D, error_word=True)
    b = uf.KVWindow(CFG.B, CFG.G, CFG.W, CFG.Lc, CFG.blk, CFG.D, error_word=True)
    orc = OracleStream(CFG)
    for win in (a, b):
        win.reset()
    last = None
    for t in range(CFG.W):
        last = chunk_inputs(CFG, 33, t)
        for win in (a, b):
            win.append(last["k"].cuda(), last["v"].cuda())
        orc.append(last)
    oidx, ocnt = oracle_idx_array(CFG, orc.mask(last["q"], CFG.k_for()))
    q = last["q"].cuda()
    bad = oidx.copy()
    bad[0, 0, 1, 3] = 1 << 20
    side = torch.cuda.Stream()
    _attend(uf, a, q, torch.from_numpy(bad).cuda(), torch.from_numpy(ocnt).cuda())
    with torch.cuda.stream(side):
        _attend(uf, b, q, torch.from_numpy(oidx).cuda(), torch.from_numpy(ocnt).cuda(), stream=side)
    torch.cuda.synchronize()
    assert int(a.err.item()) == uf.UF_EBOUNDS
    assert int(b.err.item()) == 0
    assert uf.uf_get_error(clear=True) == 0         # the library's word saw nothing


def test_short_wait_bound_unwinds_and_the_next_call_is_exact(_lib):
    # a bound of a few thousand cycles makes the attention's pipeline waits give
    # up; every block lets its copies and MMAs in flight finish (their own,
    # longer bound), releases tensor memory and exits with UF_ETIMEOUT recorded.
    # The next call at the default bound computes the right result
    uf = _lib
    gpu, orc, last, oidx, ocnt = _case(34)
    q = last["q"].cuda()
    idx, cnt = torch.from_numpy(oidx).cuda(), torch.from_numpy(ocnt).cuda()
    statuses = []
    for limit in (1000, 20_000):
        uf.uf_set_wait_limit(limit)
        try:
            _attend(uf, gpu.win, q, idx, cnt)
        finally:
            uf.uf_set_wait_limit(1 << 31)
        torch.cuda.synchronize()
        statuses.append(uf.uf_get_error(clear=True))
    assert set(statuses) <= {uf.UF_OK, uf.UF_ETIMEOUT}, statuses
    o, lse = _attend(uf, gpu.win, q, idx, cnt)
    torch.cuda.synchronize()
    assert uf.uf_get_error(clear=True) == 0
    items = [(b, h, i) for b in range(CFG.B) for h in range(CFG.H) for i in range(CFG.nb)]
    assert_attention_ok(CFG, o, lse, orc.attention(last["q"], items, oidx, ocnt), "after the timeout")
