"""Seeded synthetic workloads for the chunk-causal block-sparse attention path.

This module holds only shapes and random inputs.  It contains none of the
method's arithmetic (no pooling, scoring, selection or attention), so both the
CUDA path (through the binding) and the fp64 oracle can draw their inputs from
it without sharing any computation.

Shapes follow the pages' streaming video DiT workloads:

* Ultra Flash (papernotes notes, "Pipeline" diagram of the UltraFlash README):
  LR latents 16x60x104 and HR latents 16x120x208; 2x2 patchify gives token grids
  of 30x52 (480P) and 60x104 (1K); the 3x upsampler gives 180x312 latents,
  i.e. a 90x156 token grid (2K).  A chunk is 3 latent frames.
* FlashDecoder (xllm-io blog, model components table and Table 5): 12 query
  heads over 3 KV groups, head_dim 128, a rolling window of W_frm = 2 frames.

Value distribution: Q, K, V ~ N(0, 1) rounded to bf16 (round-to-nearest-even).
For the sparse SR configs, Q and K additionally get one offset vector per
(head, 128-token block, channel), drawn from N(0, 0.5^2) and added to every
token of that block, so that block scores are not uniform.  V gets no offset.
Every chunk of a stream draws its own values and offsets from its own seed.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional, Tuple

import torch


@dataclasses.dataclass(frozen=True)
class Config:
    """One workload: a streaming chunk of Lc query tokens over a window of W chunks."""

    name: str
    B: int            # batch (streaming: 1)
    H: int            # query heads
    G: int            # KV heads (groups); H % G == 0
    D: int            # head dim
    Lc: int           # tokens per chunk (= query tokens per call)
    W: int            # window capacity in chunks
    blk: int          # tokens per block
    density: Optional[float]   # fraction of kv blocks kept; 1.0 = dense
    k_fixed: Optional[int] = None  # explicit k (tiny config)
    offsets: bool = False      # per-block Q/K mean offsets
    offset_std: float = 0.5
    stream_len: int = 0        # frames in a rolling stream (GQA decoder config)
    description: str = ""
    grid: Optional[Tuple[int, int, int]] = None   # the chunk's (frames, rows, cols) token grid, Lc = product

    @property
    def nb(self) -> int:
        """Blocks per chunk (last one partial when blk does not divide Lc)."""
        return -(-self.Lc // self.blk)

    @property
    def last_block_tokens(self) -> int:
        return self.Lc - (self.nb - 1) * self.blk

    @property
    def lslot(self) -> int:
        """Tokens per ring slot: the chunk padded up to a block multiple."""
        return self.nb * self.blk

    def nkv(self, n_valid: Optional[int] = None) -> int:
        return (self.W if n_valid is None else n_valid) * self.nb

    def k_for(self, n_valid: Optional[int] = None) -> int:
        """Kept kv blocks per q-block, counting the forced diagonal block."""
        nkv = self.nkv(n_valid)
        if self.k_fixed is not None:
            return min(self.k_fixed, nkv)
        if self.density is None or self.density >= 1.0:
            return nkv
        return min(nkv, max(1, math.ceil(self.density * nkv)))

    @property
    def dense(self) -> bool:
        return self.k_fixed is None and (self.density is None or self.density >= 1.0)


CONFIGS: Dict[str, Config] = {
    c.name: c
    for c in [
        Config("tiny", B=1, H=2, G=2, D=128, Lc=256, W=2, blk=64, density=None, k_fixed=4, grid=(1, 16, 16),
               description="1 latent frame of 16x16 tokens, window of 2 frames, block 64, top-4 of 8"),
        Config("480p_dense", B=1, H=12, G=12, D=128, Lc=4680, W=3, blk=128, density=1.0, grid=(3, 30, 52),
               description="3 frames x 30x52 tokens, window of 3 chunks, dense"),
        Config("1k_sr", B=1, H=12, G=12, D=128, Lc=18720, W=2, blk=128, density=0.25, offsets=True,
               grid=(3, 60, 104),
               description="3 frames x 60x104 tokens, window of 2 chunks, top-k density 25%"),
        Config("2k_sr", B=1, H=12, G=12, D=128, Lc=42120, W=2, blk=128, density=0.15, offsets=True,
               grid=(3, 90, 156),
               description="3 frames x 90x156 tokens, window of 2 chunks, top-k density 15%"),
        Config("gqa_decoder", B=1, H=12, G=3, D=128, Lc=3600, W=2, blk=128, density=1.0, stream_len=16,
               grid=(1, 45, 80),
               description="1 frame of 45x80 tokens, 12 q heads / 3 KV groups, rolling window of 2 frames"),
    ]
}


def scaled(cfg: Config, **changes) -> Config:
    """A copy of ``cfg`` with some fields changed (reduced-size parity cases)."""
    return dataclasses.replace(cfg, **changes)


def _gen(seed: int, t: int, stream: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    # splitmix-style mixing so (seed, t, stream) triples never collide
    x = (seed * 0x9E3779B1 + t * 0x85EBCA77 + stream * 0xC2B2AE3D) & 0x7FFFFFFFFFFFFFFF
    g.manual_seed(x)
    return g


def _block_offsets(cfg: Config, heads: int, g: torch.Generator) -> torch.Tensor:
    """[B, Lc, heads, D] fp32 tensor holding one N(0, std^2) vector per
    (head, block, channel), repeated over the block's tokens."""
    off = torch.randn(cfg.B, cfg.nb, heads, cfg.D, generator=g, dtype=torch.float32) * cfg.offset_std
    rep = off.repeat_interleave(cfg.blk, dim=1)[:, : cfg.Lc]
    return rep


def chunk_inputs(cfg: Config, seed: int, t: int) -> Dict[str, torch.Tensor]:
    """Inputs of chunk ``t`` of a seeded stream, as CPU bf16 tensors.

    Returns q [B, Lc, H, D], k [B, Lc, G, D], v [B, Lc, G, D] (token-major, heads
    interleaved, the layout a fused QKV projection writes).
    """
    out = {}
    for name, heads, stream in (("q", cfg.H, 1), ("k", cfg.G, 2), ("v", cfg.G, 3)):
        g = _gen(seed, t, stream)
        x = torch.randn(cfg.B, cfg.Lc, heads, cfg.D, generator=g, dtype=torch.float32)
        if cfg.offsets and name in ("q", "k"):
            x += _block_offsets(cfg, heads, g)
        out[name] = x.to(torch.bfloat16)
    return out


def to_f64(x: torch.Tensor):
    """Exact upcast of a bf16 tensor to a float64 numpy array."""
    return x.detach().to("cpu").to(torch.float64).numpy()
