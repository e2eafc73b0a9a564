"""Seeded synthetic workloads shaped like the video-DiT attention the pages describe.

The pages benchmark Wan2.1/2.2 video diffusion models at 480P and 720P with
SageSLA top-k 0.1 ("TurboDiffusion技术指南", section on T2V generation and the
performance overview table).  Their latents and weights are not available here,
so seeded synthetic tensors with the same shapes stand in for them:

* ``iid``: Q, K, V i.i.d. N(0, 1).
* ``field``: per (b, h, channel) a smooth spatio-temporal Gaussian random field
  on the (T, Hh, W) latent grid (separable circular convolution of white
  noise with Gaussian taps, sigma 4 tokens, truncated at +-12, taps scaled to
  unit sum of squares and wrapped modulo the axis length), plus i.i.d. noise
  0.5 * N(0, 1).  Tokens are the grid flattened row-major (t, h, w); rows past
  the grid (padding up to N) are all zero.
* ``outliers`` (sweep only): on a Bernoulli(0.01) subset of Q and K entries the
  noise term is 0.5 * Student-t(3) instead of 0.5 * N(0, 1).
* K gets a per-(b, h, channel) offset N(0, 4) (std 2) on every real token,
  which makes some channels outliers - the case that K smoothing targets.
* W_proj is d x d, N(0, 1/d).

Random streams: every (tensor, b, h) slice has its own numpy
``Generator(PCG64(SeedSequence(seed, spawn_key=(t, b, h))))`` with t = 0, 1, 2
for Q, K, V, so any head can be regenerated alone; W_proj uses spawn_key (3,).
Within a slice the draws are: the white field (field mode), the noise, the
outlier mask and Student-t values (outlier mode), then, for K only, the
channel offsets.  All values are generated in float32 and stored as bf16 bit
patterns (round to nearest even), uint16 arrays of shape [B, H, N, d];
W_proj is uint16 [d, d].
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np

SIGMA = 4.0
TRUNC = 12
NOISE_STD = 0.5
K_OFFSET_STD = 2.0
OUTLIER_RATE = 0.01
OUTLIER_DOF = 3.0

SWEEP_FRACS = (0.05, 0.10, 0.20, 0.40)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    block: int
    topk_frac: float
    dist: str              # "iid" or "field"
    seed: int
    grid: tuple | None = None   # (T, Hh, W) for "field"
    outliers: bool = False
    head_fracs: tuple | None = None   # one topk_frac per head (three-class mask), else topk_frac for all
    skip_frac: float | None = None    # fraction of blocks left out of the linear branch (three-class mask)
    gran: int | None = None           # tokens per quantisation scale (None: one scale per block)

    @property
    def classes(self) -> bool:
        return self.head_fracs is not None or self.skip_frac is not None

    @property
    def fracs(self):
        """topk_frac as the operator takes it: per head for the three-class mask."""
        return list(self.head_fracs) if self.head_fracs is not None else self.topk_frac

    @property
    def nblk(self) -> int:
        return nblk_of(self.N, self.block)

    def describe(self) -> str:
        g = "x".join(map(str, self.grid)) if self.grid else "-"
        tf = ",".join(f"{f:g}" for f in self.head_fracs) if self.head_fracs else f"{self.topk_frac}"
        cls = f" skip_frac={self.skip_frac}" if self.skip_frac is not None else ""
        cls += f" gran={self.gran}" if self.gran is not None else ""
        return (f"{self.name}: B={self.B} H={self.H} N={self.N} d={self.d} block={self.block} "
                f"topk_frac={tf}{cls} dist={self.dist} grid={g} outliers={self.outliers} "
                f"seed={self.seed}")


def nblk_of(N: int, block: int) -> int:
    return (N + block - 1) // block


CONFIGS = {
    "tiny": Workload("tiny", 1, 2, 1024, 64, 64, 0.25, "iid", 0),
    "480p": Workload("480p", 1, 12, 32768, 128, 128, 0.10, "field", 1, (21, 30, 52)),
    "720p": Workload("720p", 1, 40, 75600, 128, 128, 0.10, "field", 2, (21, 45, 80)),
    "dense": Workload("dense", 1, 12, 32768, 128, 128, 1.0, "iid", 3),
}
for _i, _f in enumerate(SWEEP_FRACS):
    CONFIGS[f"sweep{_f:.2f}"] = Workload(f"sweep{_f:.2f}", 2, 12, 32768, 128, 128, _f, "field",
                                          4 + _i, (21, 30, 52), outliers=True)
# the 480P shape with per-head fractions (5-20%, mean 12.5%) and the lower
# half of every ranking left out of the linear branch (three-class mask)
# the 480P workload with one quantisation scale per 32 tokens (finer granularity)
CONFIGS["480p_gran32"] = Workload("480p_gran32", 1, 12, 32768, 128, 128, 0.10, "field", 1, (21, 30, 52), gran=32)
CONFIGS["480p_classes"] = Workload("480p_classes", 1, 12, 32768, 128, 128, 0.125, "field", 8, (21, 30, 52),
                                   head_fracs=(0.05, 0.10, 0.15, 0.20) * 3, skip_frac=0.5)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit pattern, round to nearest even (inputs are finite)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def _axis_spectrum(L: int, real_last: bool) -> np.ndarray:
    x = np.arange(-TRUNC, TRUNC + 1, dtype=np.float64)
    w = np.exp(-x * x / (2.0 * SIGMA * SIGMA))
    w /= math.sqrt(float(np.sum(w * w)))
    ker = np.zeros(L, dtype=np.float64)
    np.add.at(ker, np.mod(x.astype(np.int64), L), w)
    spec = np.fft.rfft(ker) if real_last else np.fft.fft(ker)
    return spec.real.astype(np.float32)  # symmetric taps: the spectrum is real


def _field(rng: np.random.Generator, d: int, grid: tuple) -> np.ndarray:
    """[T*Hh*W, d] float32 smooth field, one independent field per channel."""
    import scipy.fft as sfft

    T, Hh, W = grid
    white = rng.standard_normal((d, T, Hh, W), dtype=np.float32)
    F = sfft.rfftn(white, axes=(1, 2, 3), workers=-1)
    F *= _axis_spectrum(T, False)[None, :, None, None]
    F *= _axis_spectrum(Hh, False)[None, None, :, None]
    F *= _axis_spectrum(W, True)[None, None, None, :]
    f = sfft.irfftn(F, s=(T, Hh, W), axes=(1, 2, 3), workers=-1).astype(np.float32)
    return np.ascontiguousarray(f.reshape(d, T * Hh * W).T)


def _rng(seed: int, key: tuple) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=key)))


def _tensor(seed, tid, B, heads, N, d, dist, grid, outliers, k_offset) -> np.ndarray:
    out = np.empty((B, len(heads), N, d), dtype=np.uint16)
    ntok = N if dist == "iid" else int(np.prod(grid))
    if ntok > N:
        raise ValueError("grid larger than N")
    for b in range(B):
        for hi, h in enumerate(heads):
            rng = _rng(seed, (tid, b, h))
            x = np.zeros((N, d), dtype=np.float32)
            if dist == "iid":
                x[:] = rng.standard_normal((N, d), dtype=np.float32)
            elif dist == "field":
                x[:ntok] = _field(rng, d, grid)
                noise = rng.standard_normal((ntok, d), dtype=np.float32)
                if outliers:
                    mask = rng.random((ntok, d)) < OUTLIER_RATE
                    t = rng.standard_t(OUTLIER_DOF, size=int(mask.sum())).astype(np.float32)
                    noise[mask] = t
                x[:ntok] += np.float32(NOISE_STD) * noise
            else:
                raise ValueError(dist)
            if k_offset:
                off = (K_OFFSET_STD * rng.standard_normal(d)).astype(np.float32)
                x[:ntok] += off[None, :]
            out[b, hi] = f32_to_bf16_bits(x)
    return out


def make_inputs(B: int, H: int, N: int, d: int, seed: int, dist: str = "iid",
                grid: tuple | None = None, outliers: bool = False,
                heads: list | None = None) -> dict:
    """Seeded Q, K, V (bf16 bits [B, len(heads), N, d]) and W_proj (bf16 bits [d, d]).

    ``heads`` selects a subset of the H heads (default: all); a head's bytes do
    not depend on which other heads are generated.
    """
    hs = list(range(H)) if heads is None else list(heads)
    q = _tensor(seed, 0, B, hs, N, d, dist, grid, outliers, False)
    k = _tensor(seed, 1, B, hs, N, d, dist, grid, outliers, True)
    v = _tensor(seed, 2, B, hs, N, d, dist, grid, False, False)
    w = _rng(seed, (3,)).standard_normal((d, d), dtype=np.float32) * np.float32(1.0 / math.sqrt(d))
    return {"q": q, "k": k, "v": v, "proj": f32_to_bf16_bits(w)}


def make_workload(w: Workload, heads: list | None = None) -> dict:
    """Inputs of a named workload (optionally a subset of its heads)."""
    return make_inputs(w.B, w.H, w.N, w.d, w.seed, w.dist, w.grid, w.outliers, heads)
