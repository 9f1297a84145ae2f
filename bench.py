#!/usr/bin/env python3
"""Benchmark of the chunk-causal block-sparse attention hot path on B200.

One step = one chunk of one attention layer: uf_kv_append (the new chunk's K/V
into the rolling window) -> uf_block_mask (pool, score, top-k) ->
uf_block_sparse_attn, on seeded synthetic inputs of the chosen workload, with
the window already full (steady state).  Inputs are resident in HBM before
the timed region; every step's working set (Q, new K/V, the window, O) is
larger than the 126 MB L2, so no flush is needed between steps.

The headline workload is the 2K SR-DiT chunk (the largest); the 1K chunk, the
dense 480P chunk and the GQA decoder step are timed after it with fewer steps
and reported under "other_workloads" of the same line (--others '' skips them).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config 2k_sr] [--others LIST] [--impl ours|reference]

Under torchrun (N > 1) every rank runs an independent replica on its own GPU
(weak scaling; the path needs no data exchange).  Rank 0 prints one JSON line.
``--impl reference`` times the fp64 CPU oracle on bounded samples of the same
workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from workloads import CONFIGS, chunk_inputs  # noqa: E402

METRIC = "block-sparse chunk attn ms/chunk & kept-block TFLOP/s (% bf16 peak), 1 B200"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DEFAULT_OTHERS = "1k_sr,480p_dense,gqa_decoder"
PROFILES_DIR = os.path.join(ROOT, "profiles")
ATTN_SOURCES = ["block_sparse_causal_b200/csrc/attention.cuh", "block_sparse_causal_b200/csrc/uf_device.cuh"]


# ----------------------------------------------------------------- helpers --
def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in ATTN_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def attn_traffic_per_launch(config_name: str):
    """DRAM bytes per attention launch from the committed ncu summary of this
    workload (profiles/attn_<workload>_traffic.txt), or None when there is none
    or the kernel changed since."""
    path = os.path.join(PROFILES_DIR, f"attn_{config_name}_traffic.txt")
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    m_hash = re.search(r"^source_hash:\s*(\S+)", txt, flags=re.M)
    m_bytes = re.search(r"^traffic_bytes_per_launch:\s*([0-9.eE+]+)", txt, flags=re.M)
    if not m_hash or not m_bytes or m_hash.group(1) != kernel_source_hash():
        return None
    return float(m_bytes.group(1))


def valid_counts(cfg, device):
    """Valid tokens of each q-block [nb] and of each logical kv block of a full window [W*nb]."""
    vq = torch.full((cfg.nb,), cfg.blk, dtype=torch.float64, device=device)
    vq[-1] = cfg.last_block_tokens
    vkv = vq.repeat(cfg.W)
    return vq, vkv


def kept_flops(cfg, idx, cnt, device):
    """Algorithmic attention FLOPs of one call: 4 * D per (query token, kept kv
    token) pair (QK^T and PV), summed over kept (q-block, kv-block) pairs."""
    vq, vkv = valid_counts(cfg, device)
    if idx is None:
        return 4.0 * cfg.D * cfg.B * cfg.H * float(vq.sum()) * float(vkv.sum())
    k = idx.shape[-1]
    pos = torch.arange(k, device=device)
    live = pos.view(1, 1, 1, k) < cnt.unsqueeze(-1)
    kv_tok = torch.where(live, vkv[idx.clamp(min=0).long()], torch.zeros((), dtype=torch.float64, device=device))
    per_item = kv_tok.sum(-1) * vq.view(1, 1, -1)
    return 4.0 * cfg.D * float(per_item.sum())


def append_bytes(cfg, fp8=False):
    # read K,V of the chunk; write them into the slot (incl. padding rows); write pooled K;
    # FP8 variant: also the e4m3 copy of K's slot rows
    chunk = cfg.B * cfg.Lc * cfg.G * cfg.D * 2
    slot = cfg.B * cfg.lslot * cfg.G * cfg.D * 2
    return 2 * chunk + 2 * slot + cfg.B * cfg.G * cfg.nb * cfg.D * 4 + (slot // 2 if fp8 else 0)


def fp8_scales(chunk):
    """Static per-tensor scales calibrated once on one chunk: amax / 448 (e4m3),
    rounded up to a power of two (the quotient x / scale is then exact)."""
    return tuple(2.0 ** math.ceil(math.log2(float(chunk[n].float().abs().max()) / 448.0)) for n in ("q", "k"))


def rope_q_bytes(cfg):
    # uf_rope of the chunk's queries: read and write Q once (timed with the append)
    return 2 * cfg.B * cfg.Lc * cfg.H * cfg.D * 2


def mask_call_name(args):
    return "uf_block_mask_local + " if (args.mask_local or args.mask_local_only) else "uf_block_mask + "


def mask_bytes(cfg, k):
    # read Q once; pooled K of the window once per KV head; write idx and cnt
    return (cfg.B * cfg.Lc * cfg.H * cfg.D * 2 + cfg.B * cfg.G * cfg.nkv() * cfg.D * 4
            + cfg.B * cfg.H * cfg.nb * (k + 1) * 4)


class ClockSampler:
    """nvidia-smi samples of SM clock, power and throttle reasons while running."""

    FIELDS = ("index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,enforced.power.limit")

    def __init__(self, device=None):
        self.pci = ""
        if device is not None:
            props = torch.cuda.get_device_properties(device)
            bus, dev, dom = (getattr(props, n, None) for n in ("pci_bus_id", "pci_device_id", "pci_domain_id"))
            if isinstance(bus, int) and isinstance(dev, int):
                self.pci = f"{bus:02x}:{dev:02x}.0"       # matches the tail of nvidia-smi's pci.bus_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.15)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        with open(self.path) as f:
            lines = f.readlines()
        os.unlink(self.path)
        return summarise_clock_rows(lines, self.pci)


def summarise_clock_rows(lines, pci=""):
    """Summary of nvidia-smi rows in ClockSampler.FIELDS order (rows of other
    GPUs, when pci is given, and malformed rows are skipped); None if none."""
    rows = []
    for line in lines:
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 11:
            continue
        if pci and not parts[1].lower().endswith(pci):
            continue
        rows.append(parts)
    if not rows:
        return None

    def num(x):
        try:
            return float(x)
        except ValueError:
            return None
    sm = [num(r[2]) for r in rows if num(r[2]) is not None]
    reasons = set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for r in rows:
        for n, v in zip(names, r[6:10]):
            if v.lower().startswith("active"):
                reasons.add(n)
    return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": num(rows[0][3]),
            "power_w_max": max((num(r[4]) or 0.0) for r in rows), "power_limit_w": num(rows[0][10]),
            "samples": len(rows), "reasons": sorted(reasons)}


def clock_normalised(tflops, clocks):
    """tflops scaled to the maximum SM clock from the clock the kernel ran at
    (its in-kernel effective clock, else the sampled median); None if unknown."""
    if not clocks or not clocks.get("sm_max_mhz"):
        return None
    mhz = clocks.get("attn_sm_mhz") or clocks.get("sm_mhz")
    return tflops * clocks["sm_max_mhz"] / mhz if mhz else None


# --------------------------------------------------------------- GPU arm ----
def mask_k(args, cfg):
    """Kept blocks per q-block: the workload's k, widened to hold a forced local band."""
    k = cfg.k_for() if not cfg.dense else cfg.nkv()
    return max(k, 2 * args.mask_local + 1) if not cfg.dense else k


def run_ours(args, cfg, rank, world, device, do_e2e=True):
    import block_sparse_causal_b200 as uf
    stream = torch.cuda.current_stream()
    k = mask_k(args, cfg)
    local_flags = uf.UF_MASK_LOCAL_ONLY if args.mask_local_only else 0
    scale = 1.0 / math.sqrt(cfg.D)

    # seeded chunks, generated on the host, resident in HBM before timing
    n_distinct = 3
    host_chunks = [chunk_inputs(cfg, args.seed + 1000 * rank, t) for t in range(cfg.W + n_distinct)]
    dev_chunks = [{n: x.to(device) for n, x in c.items()} for c in host_chunks]
    q_scale, k_scale = fp8_scales(host_chunks[0]) if args.fp8 else (None, None)
    win = uf.KVWindow(cfg.B, cfg.G, cfg.W, cfg.Lc, cfg.blk, cfg.D, device=device, k_scale=k_scale)
    win.reset()
    tile_grid = cfg.grid if args.tiled else None
    for t in range(cfg.W):                       # fill the window (--anchor: the first chunk is pinned)
        win.append(dev_chunks[t]["k"], dev_chunks[t]["v"], keep_chunks=cfg.W, anchor=bool(args.anchor and t == 0),
                   tile_grid=tile_grid)
    o = torch.empty(cfg.B, cfg.Lc, cfg.H, cfg.D, dtype=torch.bfloat16, device=device)
    lse = torch.empty(cfg.B, cfg.H, cfg.Lc, dtype=torch.float32, device=device)
    n_idx = args.steps + args.warmup
    idx = [torch.empty(cfg.B, cfg.H, cfg.nb, k, dtype=torch.int32, device=device) for _ in range(n_idx)]
    cnt = [torch.empty(cfg.B, cfg.H, cfg.nb, dtype=torch.int32, device=device) for _ in range(n_idx)]

    q_rot = torch.empty_like(dev_chunks[0]["q"]) if (args.rope or args.tiled) else None
    o_tiled = torch.empty_like(o) if args.tiled else None

    balanced = args.schedule == "balanced" and not args.fp8
    ws = torch.empty(uf.uf_attn_workspace_bytes(), dtype=torch.uint8, device=device) if balanced else None

    def attention(q, idx_s, cnt_s, k_s, out, lse_out):
        if args.fp8:
            uf.uf_block_sparse_attn_fp8k(q, cfg.H, win.desc, win.k8, q_scale, k_scale, idx_s, cnt_s, k_s, scale,
                                         out, lse_out)
        elif balanced:
            uf.uf_block_sparse_attn_balanced(q, cfg.H, win.desc, idx_s, cnt_s, k_s, scale, out, lse_out, ws)
        else:
            uf.uf_block_sparse_attn(q, cfg.H, win.desc, idx_s, cnt_s, k_s, scale, out, lse_out)

    def step(s, chunk, ev=None, o_out=None, lse_out=None):
        # every call goes to the current stream; outputs to o / lse unless given
        o_out = o if o_out is None else o_out
        lse_out = lse if lse_out is None else lse_out
        # RoPE variant: the chunk sits at stream position (W + s) * Lc
        pos0 = (cfg.W + s) * cfg.Lc
        if ev is not None:
            ev[0].record(stream)
        if args.rope:
            win.append(chunk["k"], chunk["v"], keep_chunks=cfg.W, rope_pos0=pos0)
            uf.uf_rope(chunk["q"], q_rot, cfg.B, cfg.Lc, cfg.H, pos0)
            q = q_rot
        elif args.tiled:
            # tiled token order: K and V gathered by the append, the queries permuted
            win.append(chunk["k"], chunk["v"], keep_chunks=cfg.W, tile_grid=cfg.grid)
            uf.uf_tile_tokens(chunk["q"], q_rot, cfg.B, cfg.grid, cfg.H)
            q = q_rot
        else:
            win.append(chunk["k"], chunk["v"], keep_chunks=cfg.W)
            q = chunk["q"]
        if ev is not None:
            ev[1].record(stream)
        if cfg.dense:
            if ev is not None:
                ev[2].record(stream)
            attention(q, None, None, 0, o_tiled if args.tiled else o_out, lse_out)
        else:
            if args.mask_local or args.mask_local_only:
                uf.uf_block_mask_local(q, cfg.H, win.desc, k, args.mask_local, local_flags, idx[s], cnt[s])
            else:
                uf.uf_block_mask(q, cfg.H, win.desc, k, idx[s], cnt[s])
            if ev is not None:
                ev[2].record(stream)
            attention(q, idx[s], cnt[s], k, o_tiled if args.tiled else o_out, lse_out)
        if ev is not None:
            ev[3].record(stream)
        if args.tiled:                             # O back to row-major order (in the step, not in "attn")
            uf.uf_tile_tokens(o_tiled, o_out, cfg.B, cfg.grid, cfg.H, inverse=True)

    launches_per_step = (2 if cfg.dense else 3) + (1 if args.rope else 0) + (2 if args.tiled else 0)
    for s in range(args.warmup):
        step(s, dev_chunks[cfg.W + s % n_distinct])
    torch.cuda.synchronize()
    if uf.uf_get_error() != 0:
        raise RuntimeError("device-side error during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    # the attention kernel's own clock: its thread blocks add their SM cycles
    # and global-timer nanoseconds here (atomic adds when each block ends)
    clk = torch.zeros(2, dtype=torch.int64, device=device)
    sampler = ClockSampler(device)
    sampler.start()
    barrier(world)
    torch.cuda.synchronize()
    uf.uf_set_clock_counters(clk)
    t_start.record(stream)
    for s in range(args.steps):
        step(args.warmup + s, dev_chunks[cfg.W + (args.warmup + s) % n_distinct], evs[s])
    t_end.record(stream)
    torch.cuda.synchronize()
    uf.uf_set_clock_counters(None)
    barrier(world)
    clocks = sampler.stop()
    cycles, ns = (int(v) for v in clk.tolist())
    attn_mhz = cycles / ns * 1e3 if ns > 0 else None
    if clocks is None:
        clocks = {}
    clocks["attn_sm_mhz"] = attn_mhz
    elapsed_ms = t_start.elapsed_time(t_end)
    per = {"append": 0.0, "mask": 0.0, "attn": 0.0}
    for ev in evs:
        per["append"] += ev[0].elapsed_time(ev[1])
        per["mask"] += ev[1].elapsed_time(ev[2])
        per["attn"] += ev[2].elapsed_time(ev[3])
    per = {n: v / args.steps for n, v in per.items()}
    if uf.uf_get_error() != 0:
        raise RuntimeError("device-side error during the timed steps")

    flops = [kept_flops(cfg, None if cfg.dense else idx[args.warmup + s],
                        None if cfg.dense else cnt[args.warmup + s], device) for s in range(args.steps)]
    flops_per_step = sum(flops) / len(flops)
    max_ms = all_max(elapsed_ms, world, device)

    e2e = None
    if do_e2e:
        e2e = run_e2e(args, cfg, world, device, host_chunks, dev_chunks, step, o, lse, n_idx, n_distinct)
    ms_per_step = max_ms / args.steps
    # every rank ran its own seeded stream: the job's work is the sum of their kept FLOPs
    job_flops_per_step = all_sum(flops_per_step, world, device)
    value = job_flops_per_step / (ms_per_step * 1e-3) / 1e12
    peaks, peaks_src = load_peaks()
    attn_tflops = flops_per_step / (per["attn"] * 1e-3) / 1e12
    traffic = None if args.fp8 else attn_traffic_per_launch(args.config)
    # FP8 variant: half the FLOPs (QK) at the e4m3 rate, twice bf16's (nominal
    # ratio applied to the measured bf16 peak), half (PV) at the bf16 rate
    peak = peaks["bf16_tflops"] * (4.0 / 3.0 if args.fp8 else 1.0)
    hbm = peaks["hbm_gbs"]
    kernels = {
        "append": {"ms": per["append"],
                   "GB/s": (append_bytes(cfg, args.fp8) + (rope_q_bytes(cfg) if (args.rope or args.tiled) else 0))
                   / (per["append"] * 1e-3) / 1e9},
        "attn": {"ms": per["attn"], "TFLOP/s": attn_tflops},
    }
    kernels["append"]["frac_of_measured_hbm"] = kernels["append"]["GB/s"] / hbm
    if not cfg.dense:
        kernels["mask"] = {"ms": per["mask"], "GB/s": mask_bytes(cfg, k) / (per["mask"] * 1e-3) / 1e9}
        kernels["mask"]["frac_of_measured_hbm"] = kernels["mask"]["GB/s"] / hbm
    result = {
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3 QK, bf16 PV" if args.fp8 else "bf16",
        "data": "synthetic",
        "config": {
            "workload": args.config, "description": cfg.description, "B": cfg.B, "H": cfg.H, "G": cfg.G,
            "D": cfg.D, "Lc": cfg.Lc, "W": cfg.W, "blk": cfg.blk, "k": k,
            "density": cfg.density, "kept_flops_per_step": flops_per_step,
            "mask_local": args.mask_local, "mask_local_only": bool(args.mask_local_only), "rope": bool(args.rope),
            "anchor": bool(args.anchor), "tiled": list(cfg.grid) if args.tiled else None,
            "fp8": {"q_scale": q_scale, "k_scale": k_scale, "calibration": "amax / 448 of the first chunk, rounded up to a power of two"}
            if args.fp8 else None,
            "step": ("uf_kv_append_rope + uf_rope + " if args.rope else
                     "uf_kv_append_tiled + uf_tile_tokens + " if args.tiled else
                     "uf_kv_append_fp8k + " if args.fp8 else "uf_kv_append + ")
                    + ("" if cfg.dense else mask_call_name(args))
                    + ("uf_block_sparse_attn_fp8k" if args.fp8 else
                       "uf_block_sparse_attn_balanced" if balanced else "uf_block_sparse_attn")
                    + (" + uf_tile_tokens (O)" if args.tiled else ""),
            "l2": "no flush: every step's working set (%.0f MB) exceeds the 126 MB L2" % (
                (cfg.B * cfg.Lc * (cfg.H * 2 + cfg.G * 2) * cfg.D * 2
                 + 2 * cfg.B * cfg.G * cfg.nkv() * cfg.blk * cfg.D * 2) / 1e6),
            "parallelism": "replicas" if world > 1 else "single",
            "schedule": "balanced" if balanced else "plain",
        },
        "ms_per_chunk": ms_per_step,
        "kernels": kernels,
        "roofline": {
            "bound": "tensor",
            "achieved": attn_tflops,
            "peak": peak,
            "unit": "TFLOP/s",
            "frac": attn_tflops / peak,
            "frac_of_sustained": attn_tflops / (peaks["bf16_tflops_sustained"] * (4.0 / 3.0 if args.fp8 else 1.0)),
            "traffic": traffic,
            "kernel": "uf::attn_kernel<%d, %s>" % (cfg.blk, "true" if args.fp8 else "false"),
            "peak_source": f"{peaks_src} bf16 dense burst (cuBLAS 8192^3)"
                           + (" x 4/3: QK at the nominal e4m3/bf16 ratio of 2" if args.fp8 else ""),
            # the rate at the maximum SM clock: achieved x (max SM MHz / the SM clock
            # the attention kernel ran at, from its own cycle and timer counts);
            # separates kernel quality from the power cap's clock
            "clock_normalised_tflops": clock_normalised(attn_tflops, clocks),
        },
        "e2e": None if e2e is None else {
            "value": job_flops_per_step / (e2e[0] * 1e-3) / 1e12, "unit": "TFLOP/s",
            "ms_per_step": e2e[0], "h2d_bytes_per_step": e2e[1], "d2h_bytes_per_step": e2e[2],
            "overlap": "ChunkPipeline: copy in / compute / copy out on three streams, two slots"},
        "clocks": clocks,
        "gpu_launches": launches_per_step * args.steps,
    }
    return result


def run_e2e(args, cfg, world, device, host_chunks, dev_chunks, step, o, lse, n_idx, n_distinct):
    """End-to-end rate through the C ABI from pinned host buffers."""
    import block_sparse_causal_b200 as uf
    # e2e: the same steps through the C ABI from pinned host buffers, with each
    # chunk's inputs copied in and its O / LSE copied out inside the timed
    # region; ChunkPipeline overlaps chunk n's copy in and chunk n - 2's copy
    # out with chunk n - 1's compute (three streams, two staging slots)
    from block_sparse_causal_b200.pipeline import ChunkPipeline
    pinned = [{n: x.pin_memory() for n, x in c.items()} for c in host_chunks[cfg.W:]]
    host_out = [{"o": torch.empty(o.shape, dtype=o.dtype).pin_memory(),
                 "lse": torch.empty(lse.shape, dtype=lse.dtype).pin_memory()} for _ in range(2)]
    e2e_steps = max(3, min(args.steps, 50))
    e2e_count = [0]

    def pipe_step(din, dout, st):
        step(e2e_count[0] % n_idx, din, o_out=dout["o"], lse_out=dout["lse"])
        e2e_count[0] += 1

    pipe = ChunkPipeline({n: (tuple(x.shape), x.dtype) for n, x in dev_chunks[0].items()},
                         {"o": (tuple(o.shape), o.dtype), "lse": (tuple(lse.shape), lse.dtype)},
                         pipe_step, depth=2, device=device)
    pipe.submit(pinned[0], host_out[0])
    pipe.synchronize()
    sampler2 = ClockSampler(device)
    sampler2.start()
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(pipe.h2d)
    for s in range(e2e_steps):
        pipe.submit(pinned[(s + 1) % n_distinct], host_out[(s + 1) % 2])
    e1.record(pipe.d2h)          # after the last copy out, which follows every earlier step
    pipe.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    sampler2.stop()
    if uf.uf_get_error() != 0:
        raise RuntimeError("device-side error during the end-to-end steps")
    e2e_ms = all_max(e0.elapsed_time(e1), world, device) / e2e_steps
    h2d = sum(x.numel() * x.element_size() for x in pinned[0].values())
    d2h = o.numel() * o.element_size() + lse.numel() * lse.element_size()

    return e2e_ms, h2d, d2h


def run_others(args, rank, world, device):
    """The other workloads with the same options, fewer steps and no e2e leg:
    per workload its step time, kept-block rate and per-kernel figures."""
    names = [n for n in args.others.split(",") if n and n != args.config]
    out = {}
    for name in names:
        sub = argparse.Namespace(**vars(args))
        sub.config = name
        sub.steps = max(3, min(args.steps, 50))
        sub.warmup = max(3, min(args.warmup, 5))
        torch.cuda.empty_cache()
        r = run_ours(sub, CONFIGS[name], rank, world, device, do_e2e=False)
        out[name] = {"ms_per_step": r["ms_per_step"], "value": r["value"], "unit": r["unit"], "steps": sub.steps,
                     "kernels": r["kernels"],
                     "attn_frac": r["roofline"]["frac"],
                     "attn_clock_normalised_tflops": r["roofline"]["clock_normalised_tflops"],
                     "attn_traffic": r["roofline"]["traffic"],
                     "k": r["config"]["k"], "kept_flops_per_step": r["config"]["kept_flops_per_step"],
                     "clocks": r["clocks"], "gpu_launches": r["gpu_launches"]}
    return out


# --------------------------------------------------------- CPU oracle arm ---
class OracleSample:
    """The fp64 oracle (as it stands) on a bounded sample of the workload: the
    mask of one query head over the full window, then attention for up to
    ``n_items`` work items of that head.  Inputs are prepared once."""

    def __init__(self, cfg, seed, local=0, local_only=False, anchor=False, fp8=False):
        import oracle
        from workloads import to_f64
        self.oracle = oracle
        self.cfg = cfg
        self.local, self.local_only = local, local_only
        chunks = [chunk_inputs(cfg, seed, t) for t in range(cfg.W)]
        self.scales = fp8_scales(chunks[0]) if fp8 else None
        self.win = oracle.RollingWindow(cfg.W)
        for t, c in enumerate(chunks):
            self.win.append(to_f64(c["k"][:, :, 0:1]), to_f64(c["v"][:, :, 0:1]), anchor=anchor and t == 0)
        self.q = to_f64(chunks[-1]["q"][:, :, 0:1])
        self.k = cfg.k_for() if not cfg.dense else cfg.nkv()
        if not cfg.dense:
            self.k = max(self.k, 2 * local + 1)
        self.vq = [cfg.blk] * (cfg.nb - 1) + [cfg.last_block_tokens]
        self.vkv = self.vq * cfg.W

    def run(self, n_items, budget_s, first_item=0):
        """Returns (kept FLOPs computed, seconds, description)."""
        cfg = self.cfg
        t0 = time.perf_counter()
        m = self.oracle.block_mask(self.q, self.win, cfg.blk, self.k, local=self.local, local_only=self.local_only)
        flops = 0.0
        done = 0
        while done < n_items and time.perf_counter() - t0 < budget_s:
            i = (first_item + done) % cfg.nb
            if self.scales:
                self.oracle.fp8_scores_attention(self.q, self.win, cfg.blk, *self.scales, m["idx"], m["cnt"],
                                                 items=[(0, 0, i)])
            else:
                self.oracle.block_sparse_attention(self.q, self.win, cfg.blk, m["idx"], m["cnt"],
                                                   items=[(0, 0, i)])
            flops += 4.0 * cfg.D * self.vq[i] * sum(self.vkv[j] for j in m["idx"][0, 0, i, :m["cnt"][0, 0, i]])
            done += 1
        dt = time.perf_counter() - t0
        return flops, dt, (f"mask of 1 head ({cfg.nb} q-blocks over {cfg.nkv()} kv blocks) "
                           f"+ attention of {done} work items")


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads") for d in threadpool_info() if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def cpu_baseline(cfg, seed, local=0, local_only=False, anchor=False, fp8=False):
    flops, dt, desc = OracleSample(cfg, seed, local, local_only, anchor, fp8).run(n_items=10_000, budget_s=12.0)
    out = {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
           "sample": desc + f", {dt:.1f} s of fp64 numpy", "seconds": dt}
    # the oracle on one core for the tiny workload (its whole mask and attention, repeated)
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(1):
            f1, t1, d1 = OracleSample(CONFIGS["tiny"], seed).run(n_items=10_000, budget_s=3.0)
        out["tiny_1core"] = {"value": f1 / t1 / 1e12, "unit": "TFLOP/s", "cores": 1,
                             "sample": "tiny workload: " + d1 + f", {t1:.1f} s"}
    except ImportError:
        out["tiny_1core"] = None
    return out


def run_reference(args, cfg):
    # each step: the oracle on a bounded sample (one head's mask + 1 work item)
    sample = OracleSample(cfg, args.seed, args.mask_local, args.mask_local_only, args.anchor, args.fp8)
    for s in range(args.warmup):
        sample.run(n_items=1, budget_s=5.0, first_item=s)
    tot_f, tot_t = 0.0, 0.0
    desc = ""
    for s in range(args.steps):
        f, t, desc = sample.run(n_items=1, budget_s=5.0, first_item=s)
        tot_f += f
        tot_t += t
    value = tot_f / tot_t / 1e12
    k = mask_k(args, cfg)
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.config, "description": cfg.description, "B": cfg.B, "H": cfg.H, "G": cfg.G,
                   "D": cfg.D, "Lc": cfg.Lc, "W": cfg.W, "blk": cfg.blk, "k": k, "density": cfg.density,
                   "mask_local": args.mask_local, "mask_local_only": bool(args.mask_local_only),
                   "anchor": bool(args.anchor), "fp8": bool(args.fp8)},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": "per step: " + desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------ distributed ---
def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def all_sum(x, world, device):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def all_max(x, world, device):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="2k_sr", choices=sorted(CONFIGS))
    ap.add_argument("--others", default=DEFAULT_OTHERS,
                    help="comma-separated workloads timed after the headline one (fewer steps, no e2e leg)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing leg")
    ap.add_argument("--mask-local", type=int, default=0,
                    help="radius of the forced local band of blocks around the diagonal (uf_block_mask_local)")
    ap.add_argument("--anchor", action="store_true",
                    help="anchored window: the first chunk stays pinned, the others roll (W >= 2)")
    ap.add_argument("--tiled", action="store_true",
                    help="(2,8,8) tile token order: K/V gathered by the append, Q and O permuted")
    ap.add_argument("--rope", action="store_true",
                    help="rotary position embedding: K rotated in the append, Q by uf_rope, at stream positions")
    ap.add_argument("--fp8", action="store_true",
                    help="FP8 scores: e4m3 K written by the append, e4m3 q . k on the tensor cores (static scales)")
    ap.add_argument("--schedule", default="balanced", choices=["balanced", "plain"],
                    help="attention call: uf_block_sparse_attn_balanced (kept blocks spread evenly over the SMs when "
                         "there are fewer than 8 items per SM; the plain schedule otherwise) or uf_block_sparse_attn")
    ap.add_argument("--mask-local-only", action="store_true",
                    help="keep the local band only (the fixed-local-window mask)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if sum(map(bool, (args.rope, args.tiled, args.fp8))) > 1:
        ap.error("--rope, --tiled and --fp8 are separate variants")
    cfg = CONFIGS[args.config]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, cfg)), flush=True)
        return 0

    if world > 1:
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                             device_id=torch.device("cuda", local_rank))
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    try:
        result = run_ours(args, cfg, rank, world, device)
        result["other_workloads"] = run_others(args, rank, world, device)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                result["cpu_baseline"] = cpu_baseline(cfg, args.seed, args.mask_local, args.mask_local_only,
                                                      args.anchor, args.fp8)
            else:
                result["cpu_baseline"] = None
            print(json.dumps(result), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
