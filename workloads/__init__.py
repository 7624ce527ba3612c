"""Seeded synthetic workloads for the DiT block hot path.

This module is shared by the tests, the benchmark and the CPU oracle's callers.
It holds the workload shapes and the random draws only -- none of the block's
arithmetic (no norm, projection, attention, RoPE, quantisation, merge or
sampler step) lives here, so that the CUDA path and the oracle stay
independent of each other.

Workload geometry (MiniMax H3 pages: "dense single-stream omni transformer"
over one joint video + audio token sequence, 512x512 / 22-frame and 768x1344
render geometries): a latent video grid of F frames x H rows x W columns
followed by A audio tokens.  Token order is video row-major
``(f*H + r)*W + c`` and then the audio tokens.

Random draws: every tensor has its own generator seed derived from the
workload seed, the layer index and the tensor's slot, so a single block can be
regenerated on its own (the oracle checks blocks one at a time).  Weights are
drawn in fp32 from N(0, sigma_l) and rounded to bf16; RMSNorm gains are ones;
the input tokens are N(0, 1) in fp32.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

BF16, INT8 = 0, 1  # block weight dtypes, same codes as the C ABI


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    frames: int
    rows: int
    cols: int
    n_audio: int
    d: int
    n_heads: int
    head_dim: int
    ffn: int
    n_blocks: int
    dtype: int
    seed: int
    depth_scaled_init: bool  # sigma_l = 0.02/sqrt(l+1) instead of 0.02
    eps: float = 1e-6
    rope_theta: float = 10000.0
    # denoising loop (only the loop workload sets these)
    steps: int = 0
    reuse: int = 1
    merge_first: int = -1
    merge_last: int = -1

    @property
    def n_video(self) -> int:
        return self.frames * self.rows * self.cols

    @property
    def seq(self) -> int:
        return self.n_video + self.n_audio

    @property
    def seq_merged(self) -> int:
        return self.n_video // 2 + self.n_audio

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def init_sigma(self, layer: int) -> float:
        return 0.02 / math.sqrt(layer + 1) if self.depth_scaled_init else 0.02

    def block_flops(self, merged: bool = False) -> float:
        """Dense algorithmic FLOPs of one block: 24*d^2*S linear + 4*S^2*d attention."""
        s = self.seq_merged if merged else self.seq
        lin = 2.0 * s * self.d * (3 * self.d + self.d + 2 * self.ffn)
        return lin + 4.0 * s * s * self.d


WORKLOADS = {
    # Tiny single block (fp32 oracle vs bf16 GPU): 4x8x8 video + 32 audio tokens.
    "block_d256_s288": Workload("block_d256_s288", 4, 8, 8, 32, 256, 4, 64, 1024, 1, BF16, 0, False),
    # Single bf16 block on the 512x512 / 22-frame geometry: 6x32x32 video + 256 audio.
    "block_d3072_s6400": Workload("block_d3072_s6400", 6, 32, 32, 256, 3072, 24, 128, 12288, 1, BF16, 1, False),
    # 8-block bf16 stack, 33B-class width: 6x32x32 video + 384 audio.
    "stack8_d5120_s6528": Workload("stack8_d5120_s6528", 6, 32, 32, 384, 5120, 40, 128, 20480, 8, BF16, 2, True),
    # INT8 W8A8 block on the 768x1344 geometry: 5x48x84 video + 480 audio.
    "block_int8_d5120_s20640": Workload("block_int8_d5120_s20640", 5, 48, 84, 480, 5120, 40, 128, 20480, 1, INT8, 3, False),
    # 20-step flow-matching loop, reuse 2, 45 blocks, token reduction in blocks 15..29.
    "loop45_d5120_s6528": Workload("loop45_d5120_s6528", 6, 32, 32, 384, 5120, 40, 128, 20480, 45, BF16, 4, True,
                                   steps=20, reuse=2, merge_first=15, merge_last=29),
    # The pages' aggressive preview: 320x320 internal canvas (6x20x20 latent video + 384 audio),
    # 40 active blocks, reuse 3, 20 steps, no token reduction.
    "preview40_d5120_s2784": Workload("preview40_d5120_s2784", 6, 20, 20, 384, 5120, 40, 128, 20480, 40, BF16, 5,
                                      True, steps=20, reuse=3),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _slot_seed(wl: Workload, layer: int, slot: int) -> int:
    return (wl.seed * 1_000_003 + layer * 17 + slot) & 0x7FFF_FFFF


def block_weights(wl: Workload, layer: int, device="cpu") -> dict:
    """bf16 weights of block ``layer``: W_qkv [3d,d], W_o [d,d], W_fc1 [f,d], W_fc2 [d,f]
    (row-major [out, in]) and fp32 RMSNorm gains of ones."""
    sig = wl.init_sigma(layer)
    d, f = wl.d, wl.ffn
    shapes = {"w_qkv": (3 * d, d), "w_o": (d, d), "w_fc1": (f, d), "w_fc2": (d, f)}
    out = {}
    for slot, (name, shp) in enumerate(shapes.items()):
        w = torch.empty(shp, dtype=torch.float32, device=device)
        w.normal_(0.0, sig, generator=_gen(_slot_seed(wl, layer, slot), device))
        out[name] = w.to(torch.bfloat16)
    out["g_attn"] = torch.ones(d, dtype=torch.float32, device=device)
    out["g_mlp"] = torch.ones(d, dtype=torch.float32, device=device)
    return out


def initial_tokens(wl: Workload, device="cpu", seq: Optional[int] = None) -> torch.Tensor:
    """Input tokens / initial latent x0 [S, d] fp32 ~ N(0, 1)."""
    s = wl.seq if seq is None else seq
    x = torch.empty((s, wl.d), dtype=torch.float32, device=device)
    x.normal_(0.0, 1.0, generator=_gen(_slot_seed(wl, 1 << 20, 0), device))
    return x


def uniform_tensor(shape, seed: int, device="cpu", lo=-1.0, hi=1.0, dtype=torch.float32) -> torch.Tensor:
    t = torch.empty(shape, dtype=torch.float32, device=device)
    t.uniform_(lo, hi, generator=_gen(seed, device))
    return t.to(dtype)


def normal_tensor(shape, seed: int, device="cpu", std=1.0, dtype=torch.float32) -> torch.Tensor:
    t = torch.empty(shape, dtype=torch.float32, device=device)
    t.normal_(0.0, std, generator=_gen(seed, device))
    return t.to(dtype)


def int8_tensor(shape, seed: int, device="cpu") -> torch.Tensor:
    """Uniform int8 codes in [-127, 127] (the symmetric code range)."""
    g = _gen(seed, device)
    return torch.randint(-127, 128, shape, generator=g, device=device, dtype=torch.int32).to(torch.int8)
