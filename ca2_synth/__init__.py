"""Seeded synthetic inputs for the Ca2-VDM cached-attention path.

This module is shared by the CPU oracle (``oracle/``) and the CUDA path's tests and
benchmark.  It holds only random-number draws, bf16 rounding of those draws and the
workload shapes; none of the attention, ring-buffer or positional-index arithmetic
lives here.

Workloads (the shapes come from the Ca2-VDM paper's setting: Open-Sora v1.0 backbone,
256x256 video -> 32x32 latent -> 16x16 tokens per frame after 2x2 patching, C=1152 split
into 16 heads of 72, chunk length l=8, prefix length P in {1, 1+l, ..., 1+nl}, P'=3,
50 denoising steps; "Ca2-VDM" papernotes page, sections "整体框架", "关键设计 3-4",
"训练策略" and the memory table):

  tiny      B=1, H=2,  D=16, HW=16,   l=4, Pmax=9,  P'=1, 1 layer,  3 AR steps
  os_p25    B=1, H=16, D=72, HW=256,  l=8, Pmax=25, P'=3, 1 layer,  4 AR steps
  os_p41    B=1, H=16, D=72, HW=256,  l=8, Pmax=41, P'=3, 1 layer, 10 AR steps
  os_28blk  B=4, H=16, D=72, HW=256,  l=8, Pmax=41, P'=3, 28 layers, 5 AR steps
  hires     B=2, H=16, D=72, HW=1024, l=8, Pmax=41, P'=3, 1 layer,  3 AR steps (queue pre-filled)

Value recipes:
  "normal"   i.i.d. N(0,1) * scale (scale 1/sqrt(16) for the tiny case)
  "lnhead"   per (token, head) the D-vector of N(0,1) draws is centred and scaled to
             unit variance, then multiplied by a per-head gain g_h ~ U[0.5, 2.0]
             drawn once per generator; rounded to bf16 once.
  "peaky"    i.i.d. N(0,1) * 2 (sharper softmax; exercises the running max)
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Tuple

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "bf16_bits", "bf16_to_f32", "Generator",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads: int
    head_dim: int
    hw: int
    chunk_len: int
    p_max: int
    p_spatial: int
    n_layers: int
    ar_steps: int
    denoise_steps: int
    recipe: str
    scale: float = 1.0
    prefill: bool = False   # queue pre-filled to Pmax before the first AR step

    @property
    def channels(self) -> int:
        return self.heads * self.head_dim

    @property
    def tpe_len(self) -> int:
        return self.p_max + self.chunk_len

    def frame_elems(self) -> int:
        """Elements of one frame-plane: B * HW * H * D."""
        return self.batch * self.hw * self.heads * self.head_dim


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 1, 2, 16, 16, 4, 9, 1, 1, 3, 2, "normal", 0.25),
    "os_p25": Workload("os_p25", 1, 16, 72, 256, 8, 25, 3, 1, 4, 50, "lnhead"),
    "os_p41": Workload("os_p41", 1, 16, 72, 256, 8, 41, 3, 1, 10, 50, "lnhead"),
    "os_28blk": Workload("os_28blk", 4, 16, 72, 256, 8, 41, 3, 28, 5, 50, "normal"),
    "hires": Workload("hires", 2, 16, 72, 1024, 8, 41, 3, 1, 3, 50, "lnhead", prefill=True),
}


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even); return raw bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    nan = (u & 0x7FFFFFFF) > 0x7F800000
    rounding = ((u >> 16) & 1) + 0x7FFF
    out = ((u + rounding) >> 16).astype(np.uint16)
    out[nan] = 0x7FC0
    return out


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen raw bfloat16 bits to float32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


class Generator:
    """Counter-free, order-defined generator: numpy PCG64 seeded once, draws in call order.

    Every tensor is returned as raw bf16 bits (np.uint16) in the caller layout
    [B][n][HW][H][D] (frame-major: video, frame, token, then heads and head dim contiguous).
    """

    def __init__(self, wl: Workload, seed: int = 0):
        self.wl = wl
        self.rng = np.random.default_rng(seed)
        # per-head gains for the "lnhead" recipe, drawn once
        self.gain = self.rng.uniform(0.5, 2.0, size=wl.heads).astype(np.float32)

    def _draw(self, shape: Tuple[int, ...]) -> np.ndarray:
        wl = self.wl
        x = self.rng.standard_normal(size=shape, dtype=np.float32)
        if wl.recipe == "normal":
            x *= np.float32(wl.scale)
        elif wl.recipe == "peaky":
            x *= np.float32(2.0)
        elif wl.recipe == "lnhead":
            mu = x.mean(axis=-1, keepdims=True)
            var = x.var(axis=-1, keepdims=True)
            x = (x - mu) / np.sqrt(var + np.float32(1e-6))
            x = x * self.gain.reshape((1,) * (x.ndim - 2) + (-1, 1))
        else:
            raise ValueError(wl.recipe)
        return bf16_bits(x.astype(np.float32))

    def frames(self, n: int) -> np.ndarray:
        """One tensor of n frames: [B][n][HW][H][D] bf16 bits."""
        wl = self.wl
        return self._draw((wl.batch, n, wl.hw, wl.heads, wl.head_dim))

    def qkv(self, n: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
        """Q, K, V for n frames, drawn in that order."""
        return self.frames(n), self.frames(n), self.frames(n)

    def tpe_offset(self, seed: int = 1) -> int:
        """Random cyclic TPE offset in [0, N_tpe), from its own seeded stream."""
        return int(np.random.default_rng(seed).integers(0, self.wl.tpe_len))

    def table(self, rows: int, cols: int) -> np.ndarray:
        """A bf16 table (e.g. a positional-embedding table) of N(0,1) * 0.02 draws."""
        x = self.rng.standard_normal(size=(rows, cols), dtype=np.float32) * np.float32(0.02)
        return bf16_bits(x)
