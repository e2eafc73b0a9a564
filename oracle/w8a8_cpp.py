"""The plain C++ W8A8 oracle (w8a8_oracle.cpp) behind the same Python
functions as the numpy statement (w8a8_oracle.py).  TEST INFRASTRUCTURE ONLY:
imported by the tests and the benchmark's CPU leg.

The C++ file restates the layer independently of the numpy one (plain loops,
exact int32 block sums, float64 weighting in column-block order); the two
agree bit for bit (tests/test_w8a8_oracle.py), and the numpy statement's pins
run against both.  This module only marshals numpy arrays.
"""

from __future__ import annotations

import ctypes

import numpy as np

from .cpp_oracle import lib as _base_lib, threads

BLOCK = 128
_ready = False


def lib() -> ctypes.CDLL:
    global _ready
    L = _base_lib()
    if not _ready:
        vp, i = ctypes.c_void_p, ctypes.c_int
        L.ora_w8a8_quantize.argtypes = [vp, i, i, vp, vp]
        L.ora_w8a8_gemm.argtypes = [vp, vp, vp, vp, vp, i, i, vp, i, i, vp, vp]
        _ready = True
    return L


def _p(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def nblocks(n: int) -> int:
    return (n + BLOCK - 1) // BLOCK


def quantize_2d(x_bits):
    """bf16 [R, K] -> (codes int8 [R, K], scales float32 [ceil(R/128), ceil(K/128)])."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    R, K = x.shape
    codes = np.empty((R, K), dtype=np.int8)
    scales = np.empty((nblocks(R), nblocks(K)), dtype=np.float32)
    lib().ora_w8a8_quantize(_p(x), R, K, _p(codes), _p(scales))
    return codes, scales


def gemm(xq, sx, wq, sw, bias_bits=None, rows=None):
    """(y, a) for the rows `rows` of X (default: all); see w8a8_oracle.gemm."""
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    wq = np.ascontiguousarray(wq, dtype=np.int8)
    sx = np.ascontiguousarray(sx, dtype=np.float32)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    M, K = xq.shape
    N = wq.shape[0]
    assert wq.shape[1] == K and sx.shape == (nblocks(M), nblocks(K)) and sw.shape == (nblocks(N), nblocks(K))
    r = np.arange(M, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    assert r.size == 0 or (r.min() >= 0 and r.max() < M)
    b = None if bias_bits is None else np.ascontiguousarray(bias_bits, dtype=np.uint16)
    assert b is None or b.shape == (N,)
    y = np.empty((len(r), N))
    a = np.empty((len(r), N))
    lib().ora_w8a8_gemm(_p(xq), _p(sx), _p(wq), _p(sw), _p(b), N, K, _p(r), len(r), threads(), _p(y), _p(a))
    return y, a


def linear(x_bits, w_bits, bias_bits=None, rows=None) -> dict:
    """The whole layer: quantise X (dynamic) and W, then the block-scaled GEMM."""
    xq, sx = quantize_2d(x_bits)
    wq, sw = quantize_2d(w_bits)
    y, a = gemm(xq, sx, wq, sw, bias_bits, rows)
    return {"y": y, "abs": a, "xq": xq, "sx": sx, "wq": wq, "sw": sw}
