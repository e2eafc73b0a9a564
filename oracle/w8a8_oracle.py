"""CPU oracle for the W8A8 block-quantised linear layer.  TEST INFRASTRUCTURE
ONLY: imported by the tests and the benchmark's CPU-baseline leg, never by
the library, and sharing no code with the CUDA sources.

Sources.
  "Turbo Diffusion：秒级生成与高清保真的视频扩散技术突破" (lanhy.cn), section
  三(四) item 1: weights and activations of the linear layers in 8 bits,
  quantisation parameters per independent 128x128 block of the weight
  matrix (1), activations quantised dynamically at inference time with
  clipping of extreme values (2).
  chooseai.net news page ("TuroDiffusion：为高质量视频'系统性提速'"), the
  linear-layer acceleration paragraph: parameters AND activations are
  quantised in 8 bits with 128x128 block granularity.

Readings (the pages give no formula):
  * A linear layer computes Y = X . W^T + bias (X [M, K] activations, W [N, K]
    weights in the out_features x in_features layout, optional bias [N]); all
    inputs are bf16.
  * Both X and W are cut into blocks of 128 rows x 128 columns (the last
    row / column block may be partial); each block has one float32 scale
    s = float32(max|x| / 127) over its valid elements and codes
    clamp(round_half_even(float32(x / s)), -127, 127) (IEEE division; the
    same rule as the attention quantiser); an all-zero block has s = 0 and
    codes 0.  "Clipping of extreme values" is read as this saturation to
    +-127.  X's scales are computed from the X of the call (dynamic).
  * Y[m, n] = sum over column blocks kb of P_kb[m, n] * sx[m // 128, kb] *
    sw[n // 128, kb] (+ bias[n]), where P_kb = sum_{k in kb} Xq[m, k] Wq[n, k]
    is an exact integer: the int8 products are summed exactly within a block
    and the block sums are weighted by the two scales.  Here in float64; the
    CUDA path accumulates in float32 in the order of kb and returns bf16
    (round to nearest even) or float32.

Parity: every function is pinned by tests/test_w8a8_oracle.py (brute force
with exact rationals, library matmuls in other libraries, closed forms, the
attention quantiser on one-column-block matrices).
"""

from __future__ import annotations

import numpy as np

BLOCK = 128


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32)


def nblocks(n: int) -> int:
    return (n + BLOCK - 1) // BLOCK


def quantize_2d(x_bits: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """bf16 [R, K] -> (codes int8 [R, K], scales float32 [ceil(R/128), ceil(K/128)])."""
    x = bf16_to_f32(x_bits)
    R, K = x.shape
    codes = np.zeros((R, K), dtype=np.int8)
    scales = np.zeros((nblocks(R), nblocks(K)), dtype=np.float32)
    for rb in range(nblocks(R)):
        for kb in range(nblocks(K)):
            blk = x[rb * BLOCK:(rb + 1) * BLOCK, kb * BLOCK:(kb + 1) * BLOCK]
            m = np.float32(np.max(np.abs(blk)))
            s = np.float32(m / np.float32(127.0))              # IEEE float32 division
            scales[rb, kb] = s
            if s > 0:
                qf = (blk / s).astype(np.float32)               # float32 quotient
                codes[rb * BLOCK:(rb + 1) * BLOCK, kb * BLOCK:(kb + 1) * BLOCK] = \
                    np.clip(np.rint(qf), -127, 127).astype(np.int8)
    return codes, scales


def gemm(xq: np.ndarray, sx: np.ndarray, wq: np.ndarray, sw: np.ndarray, bias_bits=None, rows=None):
    """Y = sum_kb P_kb * sx * sw (+ bias) in float64 for the rows `rows` of X
    (default: all).  Returns (y [len(rows), N], a [len(rows), N]) where
    a = sum_kb |P_kb * sx * sw| + |bias| is the magnitude the float32
    accumulation error is bounded against."""
    rows = np.arange(xq.shape[0]) if rows is None else np.asarray(rows, dtype=np.int64)
    K = xq.shape[1]
    N = wq.shape[0]
    y = np.zeros((len(rows), N))
    a = np.zeros((len(rows), N))
    mb = rows // BLOCK
    nb = np.arange(N) // BLOCK
    for kb in range(nblocks(K)):
        cols = slice(kb * BLOCK, (kb + 1) * BLOCK)
        # exact integers: every product and partial sum is an integer of
        # magnitude <= 128 * 127^2 < 2^53, so the float64 matmul is exact
        P = xq[rows, cols].astype(np.float64) @ wq[:, cols].astype(np.float64).T
        s = sx[mb, kb].astype(np.float64)[:, None] * sw[nb, kb].astype(np.float64)[None, :]
        t = P * s
        y += t
        a += np.abs(t)
    if bias_bits is not None:
        b = bf16_to_f32(bias_bits).astype(np.float64)
        y += b[None, :]
        a += np.abs(b)[None, :]
    return y, a


def linear(x_bits, w_bits, bias_bits=None, rows=None) -> dict:
    """The whole layer: quantise X (dynamic) and W, then the block-scaled GEMM."""
    xq, sx = quantize_2d(x_bits)
    wq, sw = quantize_2d(w_bits)
    y, a = gemm(xq, sx, wq, sw, bias_bits, rows)
    return {"y": y, "abs": a, "xq": xq, "sx": sx, "wq": wq, "sw": sw}


def f32_error_bound(a: np.ndarray, K: int) -> np.ndarray:
    """Bound on |float32 result - y|: the float32 path rounds each scale
    product (sx*sw), each term (an exact integer times it, or one fused
    multiply-add) and each of the nkb + 1 additions (bias last), so the error
    is at most (nkb + 3) u a with u = 2^-24 (first order; the factor 1.001
    covers the second-order terms for nkb < 10^5)."""
    return 1.001 * (nblocks(K) + 3) * 2.0 ** -24 * a
