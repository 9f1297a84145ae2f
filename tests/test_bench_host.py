"""Host-side checks of bench.py: FLOP / byte accounting, the traffic staleness
rule, the reference arm's JSON line, and the multi-rank timing helpers over
gloo with two ranks (the N > 1 path runs independent replicas; the only
collectives are the barrier and the max over ranks)."""
import json
import math
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from workloads import CONFIGS, scaled  # noqa: E402


def test_kept_flops_dense_and_sparse():
    cfg = scaled(CONFIGS["1k_sr"], H=2, G=2, Lc=300)          # nb = 3, last block 44 tokens
    dense = bench.kept_flops(cfg, None, None, "cpu")
    assert dense == 4 * 128 * 2 * 300 * 600                    # every (query, window token) pair
    idx = torch.tensor([[[[0, 5], [1, 2], [3, 4]], [[2, -1], [0, 1], [5, 5]]]], dtype=torch.int32)
    cnt = torch.tensor([[[2, 2, 2], [1, 2, 1]]], dtype=torch.int32)
    vq = [128, 128, 44]
    vkv = vq * 2
    want = 0
    for h in range(2):
        for i in range(3):
            for t in range(int(cnt[0, h, i])):
                want += vq[i] * vkv[int(idx[0, h, i, t])]
    assert bench.kept_flops(cfg, idx, cnt, "cpu") == 4 * 128 * want


def test_byte_accounting_1k():
    cfg = CONFIGS["1k_sr"]
    chunk = 18720 * 12 * 128 * 2
    slot = 147 * 128 * 12 * 128 * 2
    assert bench.append_bytes(cfg) == 2 * chunk + 2 * slot + 12 * 147 * 128 * 4
    assert bench.mask_bytes(cfg, 74) == chunk + 12 * 294 * 128 * 4 + 12 * 147 * 75 * 4


def test_traffic_is_dropped_when_the_kernel_changes(tmp_path, monkeypatch):
    prof = tmp_path / "attn_1k_sr_traffic.txt"
    prof.write_text(f"source_hash: {bench.kernel_source_hash()}\ntraffic_bytes_per_launch: 123\n")
    monkeypatch.setattr(bench, "PROFILES_DIR", str(tmp_path))
    assert bench.attn_traffic_per_launch("1k_sr") == 123.0
    assert bench.attn_traffic_per_launch("2k_sr") is None
    prof.write_text("source_hash: 0000\ntraffic_bytes_per_launch: 123\n")
    assert bench.attn_traffic_per_launch("1k_sr") is None


def test_clock_rows_summary():
    row = "0, 00000000:1B:00.0, {sm}, 1965, {w}, 0x4, Not Active, Not Active, Not Active, {cap}, 1000.00\n"
    lines = [row.format(sm=1500, w=700.5, cap="Active"), row.format(sm=1550, w=760.2, cap="Not Active"),
             row.format(sm=1600, w=650.0, cap="Not Active"),
             "1, 00000000:2A:00.0, 900, 1965, 100.0, 0x0, Not Active, Active, Not Active, Not Active, 1000.00\n",
             "garbage\n"]
    c = bench.summarise_clock_rows(lines, pci="1b:00.0")
    assert c["sm_mhz"] == 1550 and c["sm_max_mhz"] == 1965 and c["samples"] == 3
    assert c["power_w_max"] == 760.2 and c["power_limit_w"] == 1000.0
    assert c["reasons"] == ["sw_power_cap"]                 # the other GPU's thermal slowdown is not ours
    assert bench.summarise_clock_rows(["garbage\n"]) is None
    na = bench.summarise_clock_rows([row.format(sm=1965, w=300, cap="Not Active").replace("1000.00", "[N/A]")])
    assert na["power_limit_w"] is None and na["reasons"] == []


def test_clock_normalisation_prefers_the_kernels_own_clock():
    assert bench.clock_normalised(1000.0, None) is None
    assert bench.clock_normalised(1000.0, {"sm_max_mhz": 1965.0}) is None
    assert bench.clock_normalised(1000.0, {"sm_max_mhz": 1965.0, "sm_mhz": 1965.0}) == 1000.0
    c = {"sm_max_mhz": 1965.0, "sm_mhz": 1965.0, "attn_sm_mhz": 1572.0}
    assert math.isclose(bench.clock_normalised(1000.0, c), 1000.0 * 1965.0 / 1572.0)


def test_reference_arm_json_line():
    env = dict(os.environ, OMP_NUM_THREADS="2", OPENBLAS_NUM_THREADS="2")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                          "--steps", "3", "--warmup", "3"], capture_output=True, text=True, timeout=600, env=env)
    assert res.returncode == 0, res.stderr
    line = json.loads(res.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["config"]["workload"] == "tiny"


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    bench.barrier(world)
    # each replica reports its own elapsed time; the job time is the slowest rank
    out[rank] = bench.all_max(10.0 + 5.0 * rank, world, "cpu")
    # the job's work is the sum of every replica's kept FLOPs
    out[(rank, "sum")] = bench.all_sum(1.0 + rank, world, "cpu")
    bench.barrier(world)
    dist.destroy_process_group()


def test_max_over_ranks_with_gloo():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == 15.0
    assert out[(0, "sum")] == out[(1, "sum")] == 3.0


def test_world_of_one_needs_no_process_group():
    assert bench.all_max(3.5, 1, "cpu") == 3.5
    assert bench.all_sum(3.5, 1, "cpu") == 3.5
    bench.barrier(1)
