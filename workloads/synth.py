"""Workload descriptions and seeded bf16 input generators (no method arithmetic)."""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence, Tuple

import numpy as np

# Token segment kinds (same numbering as the C ABI's sa_seg_kind).
SEG_TEXT = 0   # live prompt conditioning: pinned
SEG_PAD = 1    # padding: dropped
SEG_IMAGE = 2  # image / video tokens: sparsifiable
SEG_OTHER = 3  # audio / unknown: pinned

T_Q, T_K, T_V, T_P, T_MASK = 0, 1, 2, 3, 4


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    N: int
    segments: Tuple[Tuple[int, int, int], ...]   # (kind, start, len); empty = all image
    grid: Tuple[int, ...]                        # () plain N(0,1); (Gy, Gx) 2D; (T, G, G) 3D
    densities: Tuple[float, ...]
    layers: int = 1
    head_mask: Optional[Tuple[int, ...]] = None  # fixed mask; None = all heads (or per-layer runs)
    mask_runs: int = 0                           # >0: drop mask_drop of mask_runs runs per layer
    mask_drop: int = 0
    min_active: int = 4
    block: int = 64

    @property
    def nB(self) -> int:
        return self.N // self.block

    @property
    def n_text(self) -> int:
        return sum(l for k, s, l in self.segments if k in (SEG_TEXT, SEG_PAD, SEG_OTHER))


WORKLOADS = {
    # 40 live text tokens + 88 padding, then a 16 x 24 image grid; heads {0, 2} kept.
    "tiny": Workload("tiny", B=1, H=4, d=64, N=512,
                     segments=((SEG_TEXT, 0, 40), (SEG_PAD, 40, 88), (SEG_IMAGE, 128, 384)),
                     grid=(), densities=(0.5,), head_mask=(1, 0, 1, 0), min_active=2),
    # SDXL-shape UNet self-attention: CFG pair, 64 x 64 latent grid, no text.
    "sdxl": Workload("sdxl", B=2, H=10, d=64, N=4096, segments=(), grid=(64, 64),
                     densities=(0.3, 0.5, 1.0)),
    # Joint text+image transformer at 2048 x 2048: 20 live text + 492 padding, 128 x 128 grid.
    "joint": Workload("joint", B=1, H=24, d=128, N=16896,
                      segments=((SEG_TEXT, 0, 20), (SEG_PAD, 20, 492), (SEG_IMAGE, 512, 16384)),
                      grid=(128, 128), densities=(0.3,)),
    # Head-masked stack: 64 layers x 32 heads, half the heads dropped as runs of 4.
    "stack": Workload("stack", B=1, H=32, d=128, N=4096, segments=(), grid=(64, 64),
                      densities=(1.0, 0.5), layers=64, mask_runs=8, mask_drop=4),
    # Long video-like sequence: 64 live text + 448 padding, 8 frames of 64 x 64.
    "video": Workload("video", B=1, H=24, d=128, N=33280,
                      segments=((SEG_TEXT, 0, 64), (SEG_PAD, 64, 448), (SEG_IMAGE, 512, 32768)),
                      grid=(8, 64, 64), densities=(0.2,)),
}


def make_workload(name: str, **overrides) -> Workload:
    return dataclasses.replace(WORKLOADS[name], **overrides)


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _phi(w: Workload) -> np.ndarray:
    """Rank-8 sinusoidal position features per token, zero on text/padding tokens."""
    phi = np.zeros((w.N, 8), dtype=np.float64)
    img = [(s, l) for k, s, l in w.segments if k == SEG_IMAGE] or [(0, w.N)]
    start, length = img[0]
    m = np.arange(length, dtype=np.int64)
    if len(w.grid) == 2:
        gy, gx = w.grid
        y = (m // gx).astype(np.float64)
        x = (m % gx).astype(np.float64)
        cols = [np.sin(np.pi * y / gy), np.cos(np.pi * y / gy),
                np.sin(2 * np.pi * y / gy), np.cos(2 * np.pi * y / gy),
                np.sin(np.pi * x / gx), np.cos(np.pi * x / gx),
                np.sin(2 * np.pi * x / gx), np.cos(2 * np.pi * x / gx)]
    elif len(w.grid) == 3:
        T, g, _ = w.grid
        t = (m // (g * g)).astype(np.float64)
        y = ((m // g) % g).astype(np.float64)
        x = (m % g).astype(np.float64)
        cols = [np.sin(np.pi * t / T), np.cos(np.pi * t / T),
                np.sin(2 * np.pi * t / T), np.cos(2 * np.pi * t / T),
                np.sin(np.pi * y / g), np.cos(np.pi * y / g),
                np.sin(np.pi * x / g), np.cos(np.pi * x / g)]
    else:
        return phi
    phi[start:start + length] = np.stack(cols, axis=1)
    return phi


def make_qkv(w: Workload, seed: int = 0, layer: int = 0, heads: Optional[Sequence[int]] = None):
    """Q, K, V as uint16 bf16 bits, shape [B, H, N, d] (or [B, len(heads), N, d])."""
    H = w.H
    hs = list(range(H)) if heads is None else list(heads)
    shape = (w.B, H, w.N, w.d)
    out = []
    phi = _phi(w) if w.grid else None
    if phi is not None:
        P = np.random.default_rng([seed, layer, T_P]).standard_normal((H, 8, w.d)) / np.sqrt(8.0)
    for tid in (T_Q, T_K, T_V):
        rng = np.random.default_rng([seed, layer, tid])
        x = rng.standard_normal(shape, dtype=np.float32)
        if heads is not None:
            x = x[:, hs]
        if phi is not None and tid != T_V:
            x = 0.5 * x
            for j, h in enumerate(hs):
                x[:, j] += (phi @ P[h]).astype(np.float32)[None]
        out.append(bf16_bits_from_f32(x))
    return tuple(out)


def head_mask_for_layer(w: Workload, layer: int = 0, seed: int = 0) -> np.ndarray:
    """Per-(layer, head) mask as uint8[H]: 1 = head computed, 0 = skipped."""
    if w.head_mask is not None:
        return np.array(w.head_mask, dtype=np.uint8)
    m = np.ones(w.H, dtype=np.uint8)
    if w.mask_runs:
        run = w.H // w.mask_runs
        rng = np.random.default_rng([seed, layer, T_MASK])
        for r in rng.choice(w.mask_runs, w.mask_drop, replace=False):
            m[r * run:(r + 1) * run] = 0
    return m


def segments_list(w: Workload) -> List[Tuple[int, int, int]]:
    return list(w.segments)
