"""Seeded synthetic inputs for the W8A8 linear layer: activations X [M, K],
weights W [N, K] (out_features x in_features) and a bias [N], stored as bf16
bit patterns.  Random numbers only; none of the layer's arithmetic.

Shapes of the pages' models: Wan2.1-14B has model width 5120 and FFN width
13824 (Wan2.1-1.3B: 1536 and 8960); a 480P 81-frame latent is 21 x 30 x 52 =
32760 tokens.  Distributions: activations N(0, 1) with 1% of the input
channels scaled by 8 (the outlier channels that motivate per-block scales);
weights N(0, 1/K); bias N(0, 0.01).
"""

from __future__ import annotations

import dataclasses

import numpy as np

from .workloads import f32_to_bf16_bits


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (the same bits as
    f32_to_bf16_bits for finite inputs; torch's threaded cast, for large matrices)."""
    import torch

    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)

OUTLIER_CHANNELS = 0.01
OUTLIER_SCALE = 8.0


@dataclasses.dataclass(frozen=True)
class LinearWorkload:
    name: str
    M: int
    N: int
    K: int
    seed: int
    bias: bool = True

    def describe(self) -> str:
        return (f"{self.name}: Y[M,N] = X[M,K] . W[N,K]^T + b, M={self.M} N={self.N} K={self.K} "
                f"bias={self.bias} seed={self.seed}")


LINEAR_CONFIGS = {
    # Wan2.1-14B FFN up-projection on a 480P 81-frame latent
    "w8a8_14b_ffn": LinearWorkload("w8a8_14b_ffn", 32760, 13824, 5120, 101),
    # Wan2.1-14B attention output projection (square, 5120 x 5120)
    "w8a8_14b_proj": LinearWorkload("w8a8_14b_proj", 32760, 5120, 5120, 102),
    # Wan2.1-1.3B FFN up-projection
    "w8a8_1b3_ffn": LinearWorkload("w8a8_1b3_ffn", 32760, 8960, 1536, 103),
    # a quarter of the 14B projection's rows: the case the profiler captures
    "w8a8_prof": LinearWorkload("w8a8_prof", 8192, 5120, 5120, 105),
    # small ragged case (no dimension a multiple of 128)
    "w8a8_small": LinearWorkload("w8a8_small", 1000, 528, 656, 104),
}


def _rng(seed: int, tag: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([seed, tag]))


def make_linear(M: int, N: int, K: int, seed: int, bias: bool = True, rows=None) -> dict:
    """{"x": bf16 bits [M, K] (or the given rows), "w": [N, K], "bias": [N] or None}."""
    g = _rng(seed, 0)
    chan = np.ones(K, dtype=np.float32)
    chan[g.random(K) < OUTLIER_CHANNELS] = OUTLIER_SCALE
    # X by blocks of 128 rows, each from its own stream, so that any subset of
    # rows is reproducible without drawing the whole matrix
    need = range((M + 127) // 128) if rows is None else sorted({int(r) // 128 for r in rows})
    blocks = {}
    for rb in need:
        n = min(128, M - rb * 128)
        blocks[rb] = _rng(seed, 1000 + rb).standard_normal((n, K), dtype=np.float32)
    if rows is None:
        x = np.concatenate([blocks[rb] for rb in need]) if M > 0 else np.zeros((0, K), np.float32)
    else:
        x = np.stack([blocks[int(r) // 128][int(r) % 128] for r in rows]) if len(rows) else np.zeros((0, K), np.float32)
    x *= chan[None, :]
    w = _rng(seed, 2).standard_normal((N, K), dtype=np.float32) * np.float32(1.0 / np.sqrt(K))
    b = (_rng(seed, 3).standard_normal(N, dtype=np.float32) * np.float32(0.1)) if bias else None
    return {"x": _bf16_bits(x), "w": _bf16_bits(w), "bias": None if b is None else f32_to_bf16_bits(b)}


def make_linear_workload(w: LinearWorkload, rows=None) -> dict:
    return make_linear(w.M, w.N, w.K, w.seed, w.bias, rows)
