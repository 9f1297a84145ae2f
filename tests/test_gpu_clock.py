"""The attention kernel's clock record (uf_set_clock_counters): while a counter
pair is set, every thread block adds its SM cycles and global-timer
nanoseconds; their ratio is the clock the kernel ran at.  The record changes
nothing in the output, and nothing is added once the pair is unset."""
import pytest
import torch

from uf_testlib import GpuStream
from workloads import CONFIGS, chunk_inputs, scaled

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module", autouse=True)
def _lib(built_lib):
    uf = built_lib
    uf.uf_get_error(clear=True)
    yield uf
    uf.uf_set_clock_counters(None)
    assert uf.uf_get_error(clear=True) == 0, "a kernel recorded a device-side error"


def test_clock_counters_give_the_kernels_clock(_lib):
    uf = _lib
    cfg = scaled(CONFIGS["gqa_decoder"], H=6, G=2, Lc=2000, W=3)      # dense: 96 items of 48 blocks
    gpu = GpuStream(cfg)
    for t in range(cfg.W):
        gpu.append(chunk_inputs(cfg, 5, t))
    q = chunk_inputs(cfg, 5, cfg.W)["q"]
    o_off, lse_off = gpu.attention(q)
    torch.cuda.synchronize()

    clk = torch.zeros(2, dtype=torch.int64, device="cuda")
    uf.uf_set_clock_counters(clk)
    try:
        o_on, lse_on = gpu.attention(q)
        torch.cuda.synchronize()
    finally:
        uf.uf_set_clock_counters(None)
    cycles, ns = (int(v) for v in clk.tolist())
    props = torch.cuda.get_device_properties(0)
    # one record per thread block: each lasted at least a microsecond
    assert cycles > 0 and ns >= min(props.multi_processor_count, 96) * 1000
    mhz = cycles / ns * 1e3
    assert 300.0 < mhz < 2200.0, mhz
    assert torch.equal(o_on, o_off) and torch.equal(lse_on, lse_off)

    # unset: a further launch adds nothing
    gpu.attention(q)
    torch.cuda.synchronize()
    assert clk.tolist() == [cycles, ns]
