"""Named BRA workloads and their seeded synthetic inputs.

This module holds no step of the method: it only names the workload shapes and draws
inputs with numpy, so that the CUDA path and the CPU oracle can be fed the same values.

Shapes follow the BiFormer stage table ("从零构建BiFormer", §3: 56x56 / topk 1 / 2 heads,
28x28 / 4 / 4, 14x14 / 16 / 8, 7x7 / S^2 / 16, head_dim 32 everywhere) and the
high-resolution segmentation setting with a 16x16 region grid ("手把手带你读懂BiFormer源码",
§3.2: S=16 for high-resolution segmentation). No dataset is available, so the values are
synthetic:

* ``iid``            q, k, v ~ N(0, 1) i.i.d.
* ``region_offset``  q, k, v ~ N(0, 1) plus, per tensor, a per-(image, region, channel)
                     offset ~ N(0, 0.5^2) added to every token of the region, so that the
                     region means differ and routing is not decided by noise alone.
* ``grf``            as ``region_offset`` but the offset of each (image, channel) is a
                     Gaussian random field on the region grid: white N(0, 1) noise,
                     circularly smoothed with a Gaussian kernel of sigma = 2 regions,
                     rescaled to empirical std 0.5.

Draw order: q, k, v noise, then the q, k, v offsets. Values are drawn in float64, rounded
to float32 and, for bf16 workloads, rounded to bf16 (round to nearest even). The rounded
values are what both sides see.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    W: int
    C: int
    heads: int
    n_win: int
    topk: int
    dtype: str  # "f32" or "bf16"
    values: str  # "iid", "region_offset" or "grf"
    seed: int

    @property
    def R(self) -> int:
        return self.n_win * self.n_win

    @property
    def rs(self) -> int:
        return (self.H // self.n_win) * (self.W // self.n_win)

    @property
    def N(self) -> int:
        return self.H * self.W

    @property
    def hd(self) -> int:
        return self.C // self.heads

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def tokens(self) -> int:
        """Query tokens per batch: B * H * W."""
        return self.B * self.N

    def unique_bytes(self) -> int:
        """q + k + v read once, out written once."""
        return 4 * self.B * self.N * self.C * self.elem_bytes

    def attention_flops(self) -> int:
        """QK^T plus PV over the routed keys only: 4 * B * N * topk * rs * C."""
        return 4 * self.B * self.N * self.topk * self.rs * self.C

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    def describe(self) -> dict:
        return {"workload": self.name, "B": self.B, "H": self.H, "W": self.W, "C": self.C,
                "heads": self.heads, "head_dim": self.hd, "n_win": self.n_win, "regions": self.R,
                "tokens_per_region": self.rs, "topk": self.topk, "dtype": self.dtype,
                "values": self.values, "seed": self.seed}


WORKLOADS = {
    # tiny oracle check, fp32
    "tiny_f32": Workload("tiny_f32", 1, 28, 28, 64, 2, 7, 4, "f32", "iid", 20261),
    # BiFormer stage-1 shape (the benchmark's headline workload)
    "stage1": Workload("stage1", 64, 56, 56, 64, 2, 7, 1, "bf16", "region_offset", 20262),
    # stage-2 and stage-3 shapes
    "stage2": Workload("stage2", 64, 28, 28, 128, 4, 7, 4, "bf16", "region_offset", 20263),
    "stage3": Workload("stage3", 64, 14, 14, 256, 8, 7, 16, "bf16", "region_offset", 20264),
    # stage-4: one token per region and topk = R, i.e. global attention over 49 tokens
    "stage4": Workload("stage4", 64, 7, 7, 512, 16, 7, 49, "bf16", "iid", 20265),
    # high-resolution segmentation: 16x16 regions of 64 tokens
    "highres": Workload("highres", 8, 128, 128, 64, 2, 16, 4, "bf16", "grf", 20266),
}

HEADLINE = "stage1"


def bf16_bits(x32: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even. Inputs are finite."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _smooth_field(white: np.ndarray, sigma: float) -> np.ndarray:
    """Circular Gaussian smoothing of the last two axes (n x n grids) by FFT."""
    n = white.shape[-1]
    d = np.minimum(np.arange(n), n - np.arange(n)).astype(np.float64)
    kern1 = np.exp(-0.5 * (d / sigma) ** 2)
    kern = np.outer(kern1, kern1)
    kern /= kern.sum()
    return np.real(np.fft.ifft2(np.fft.fft2(white) * np.fft.fft2(kern)))


def _region_grid_to_tokens(off: np.ndarray, H: int, W: int, n_win: int) -> np.ndarray:
    """[B, n, n, C] per-region values -> [B, H, W, C] (each token takes its window's value). When
    H or W is not a multiple of n_win the windows are those of the map padded to the next
    multiple (ceil(H / n_win) tokens high), cropped back to H x W."""
    hr, wr = -(-H // n_win), -(-W // n_win)
    return np.repeat(np.repeat(off, hr, axis=1), wr, axis=2)[:, :H, :W]


def make_inputs(w: Workload, seed: int | None = None) -> dict:
    """Seeded q, k, v for workload ``w``.

    Returns a dict with ``q, k, v`` as float32 numpy arrays ``[B, H, W, C]`` holding exactly
    the values the device sees (bf16-representable for bf16 workloads) and, for bf16,
    ``q_bits, k_bits, v_bits`` (uint16) ready to upload.
    """
    rng = np.random.Generator(np.random.PCG64(w.seed if seed is None else seed))
    shape = (w.B, w.H, w.W, w.C)
    noise = [rng.standard_normal(shape) for _ in range(3)]
    if w.values == "region_offset":
        for t in range(3):
            off = rng.standard_normal((w.B, w.n_win, w.n_win, w.C)) * 0.5
            noise[t] = noise[t] + _region_grid_to_tokens(off, w.H, w.W, w.n_win)
    elif w.values == "grf":
        for t in range(3):
            white = rng.standard_normal((w.B, w.C, w.n_win, w.n_win))
            field = _smooth_field(white, 2.0)
            field = field / field.std(axis=(-2, -1), keepdims=True) * 0.5
            off = np.transpose(field, (0, 2, 3, 1))  # [B, n, n, C]
            noise[t] = noise[t] + _region_grid_to_tokens(off, w.H, w.W, w.n_win)
    elif w.values != "iid":
        raise ValueError(f"unknown value recipe {w.values!r}")
    out = {}
    for name, x in zip(("q", "k", "v"), noise):
        x32 = x.astype(np.float32)
        if w.dtype == "bf16":
            bits = bf16_bits(x32)
            out[name + "_bits"] = bits
            out[name] = bf16_to_f32(bits)
        else:
            out[name] = x32
    return out


def sample_tokens(w: Workload, count: int, seed: int = 7) -> np.ndarray:
    """Flat token ids b*H*W + y*W + x to check one by one: the first and last token of the
    batch, then a seeded uniform sample (sorted, distinct)."""
    total = w.B * w.N
    rng = np.random.Generator(np.random.PCG64(seed))
    pick = rng.choice(total, size=min(count, total), replace=False)
    pick = np.unique(np.concatenate([pick, [0, total - 1]]))
    return pick.astype(np.int64)
