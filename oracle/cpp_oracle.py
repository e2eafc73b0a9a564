"""The plain C++ CPU oracle (sla_oracle.cpp) behind the same Python functions
as the numpy statement (sla_oracle.py).  TEST INFRASTRUCTURE ONLY: imported
by the tests, the package's smoke check and the benchmark's CPU-baseline leg.

The C++ file restates the method independently of the numpy one (plain loops,
float64, exact integer sums, std::thread workers over query blocks); both are
pinned by tests/test_oracle_pins.py and checked against each other by
tests/test_oracle_cpp.py.  This module only marshals numpy arrays to the C
functions and assembles the same result dictionaries as sla_oracle.py.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import LIB, build

NEAR_TIE_REL = 1e-9

_lib = None


def threads() -> int:
    """Worker threads: every core this process may run on."""
    return len(os.sched_getaffinity(0))


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(LIB)
        vp, i, f, ll = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_longlong
        L.ora_round_bf16.argtypes = [vp, ll, vp]
        L.ora_channel_mean.argtypes = [vp, i, i, i, i, vp]
        L.ora_quantize_blocks.argtypes = [vp, i, i, i, i, i, i, vp, vp]
        L.ora_smooth_k.argtypes = [vp, vp, i, i, i, vp]
        L.ora_block_means.argtypes = [vp, i, i, i, i, i, vp]
        L.ora_block_probs.argtypes = [vp, vp, i, i, i, i, vp]
        L.ora_select_topk.argtypes = [vp, ll, i, i, i, vp, vp]
        L.ora_topk_count.argtypes = [i, f]
        L.ora_topk_count.restype = i
        L.ora_skip_count.argtypes = [i, i, f]
        L.ora_skip_count.restype = i
        L.ora_block_classes.argtypes = [vp, ll, i, ll, i, vp, vp, i, vp, vp]
        L.ora_sla_rows.argtypes = [vp] * 4 + [i] * 5 + [vp] * 6 + [i] * 4 + [vp, i, i] + [vp] * 3
        L.ora_sla_rows.restype = i
        _lib = L
    return _lib


def _p(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- number formats

def round_bf16(x: np.ndarray) -> np.ndarray:
    x = _c(x, np.float64)
    y = np.empty_like(x)
    lib().ora_round_bf16(_p(x), x.size, _p(y))
    return y


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return bf16_to_f32(bits).astype(np.float64)


def topk_count(nblk: int, topk_frac: float) -> int:
    kc = lib().ora_topk_count(int(nblk), float(topk_frac))
    if kc < 0:
        raise ValueError("topk_frac must be in (0, 1]")
    return kc


# ---------------------------------------------------------------- smoothing and quantisation

def channel_mean(k_bits: np.ndarray) -> np.ndarray:
    k = _c(k_bits, np.uint16)
    B, H, N, d = k.shape
    mu = np.empty((B, H, d), dtype=np.float32)
    lib().ora_channel_mean(_p(k), B * H, N, d, threads(), _p(mu))
    return mu


def smooth_k(k_bits: np.ndarray, mu: np.ndarray) -> np.ndarray:
    k = _c(k_bits, np.uint16)
    B, H, N, d = k.shape
    out = np.empty((B, H, N, d), dtype=np.float32)
    lib().ora_smooth_k(_p(k), _p(_c(mu, np.float32)), B * H, N, d, _p(out))
    return out


def quantize_groups(x32: np.ndarray, block: int, gran: int):
    if block % gran:
        raise ValueError("gran must divide block")
    x = _c(x32, np.float32)
    B, H, N, d = x.shape
    nblk = (N + block - 1) // block
    codes = np.empty((B, H, nblk * block, d), dtype=np.int8)
    scales = np.empty((B, H, nblk * block // gran), dtype=np.float32)
    lib().ora_quantize_blocks(_p(x), B * H, N, d, block, gran, threads(), _p(codes), _p(scales))
    return codes, scales


def quantize_blocks(x32: np.ndarray, block: int):
    return quantize_groups(x32, block, block)


def quantize(q_bits: np.ndarray, k_bits: np.ndarray, block: int, gran=None) -> dict:
    mu = channel_mean(k_bits)
    g = block if gran is None else gran
    qi8, sq = quantize_groups(bf16_to_f32(q_bits), block, g)
    ki8, sk = quantize_groups(smooth_k(k_bits, mu), block, g)
    return {"mu": mu, "q_i8": qi8, "q_scale": sq, "k_i8": ki8, "k_scale": sk}


# ---------------------------------------------------------------- block mask

def block_means(x_bits: np.ndarray, block: int) -> np.ndarray:
    x = _c(x_bits, np.uint16)
    B, H, N, d = x.shape
    nblk = (N + block - 1) // block
    out = np.empty((B, H, nblk, d), dtype=np.float64)
    lib().ora_block_means(_p(x), B * H, N, d, block, threads(), _p(out))
    return out


def block_probs(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    qb, kb = _c(qbar, np.float64), _c(kbar, np.float64)
    shp = qb.shape[:-2]
    nblk, d = qb.shape[-2], qb.shape[-1]
    BH = int(np.prod(shp)) if shp else 1
    p = np.empty(shp + (nblk, nblk), dtype=np.float64)
    lib().ora_block_probs(_p(qb), _p(kb), BH, nblk, d, threads(), _p(p))
    return p


def select_topk(p: np.ndarray, kc: int):
    pp = _c(p, np.float64)
    shp = pp.shape[:-1]
    n = pp.shape[-1]
    rows = int(np.prod(shp)) if shp else 1
    idx = np.empty(shp + (kc,), dtype=np.int32)
    tie = np.empty(shp, dtype=np.uint8)
    lib().ora_select_topk(_p(pp), rows, n, kc, threads(), _p(idx), _p(tie))
    return idx, tie.astype(bool)


def block_mask(q_bits: np.ndarray, k_bits: np.ndarray, block: int, topk_frac: float) -> dict:
    p = block_probs(block_means(q_bits, block), block_means(k_bits, block))
    kc = topk_count(p.shape[-1], topk_frac)
    idx, tie = select_topk(p, kc)
    return {"idx": idx, "near_tie": tie, "probs": p, "kc": kc}


def bitmap_of(idx: np.ndarray, nblk: int) -> np.ndarray:
    out = np.zeros(idx.shape[:-1] + (nblk,), dtype=np.uint8)
    np.put_along_axis(out, idx.astype(np.int64), 1, axis=-1)
    return out


# ---------------------------------------------------------------- three classes, per-head counts

CLS_NEGLIGIBLE, CLS_LINEAR, CLS_CRITICAL = 0, 1, 2


def skip_count(nblk: int, kc: int, skip_frac: float) -> int:
    kn = lib().ora_skip_count(int(nblk), int(kc), float(skip_frac))
    if kn < 0:
        raise ValueError("skip_frac must be in [0, 1)")
    return kn


def head_counts(nblk: int, H: int, topk_frac, skip_frac=None):
    tf = np.broadcast_to(np.asarray(topk_frac, dtype=np.float64), (H,))
    sf = np.broadcast_to(np.asarray(0.0 if skip_frac is None else skip_frac, dtype=np.float64), (H,))
    kc = np.array([topk_count(nblk, float(t)) for t in tf], dtype=np.int64)
    kn = np.array([skip_count(nblk, int(c), float(x)) for c, x in zip(kc, sf)], dtype=np.int64)
    return kc, kn


def _classes(p, rows_per_head, kc, kn):
    pp = _c(p, np.float64)
    n = pp.shape[-1]
    rows = pp.size // n
    cls = np.empty(pp.shape, dtype=np.uint8)
    tie = np.empty(pp.shape[:-1], dtype=np.uint8)
    kca = _c(kc, np.int32)
    kna = _c(kn, np.int32)
    lib().ora_block_classes(_p(pp), rows, n, rows_per_head, len(kca), _p(kca), _p(kna), threads(), _p(cls), _p(tie))
    return cls, tie.astype(bool)


def block_classes(p: np.ndarray, kc: int, kn: int):
    n = p.shape[-1]
    return _classes(p, max(1, np.asarray(p).size // n), [kc], [kn])


def block_mask_classes(q_bits, k_bits, block: int, topk_frac, skip_frac=None) -> dict:
    p = block_probs(block_means(q_bits, block), block_means(k_bits, block))
    B, H, nblk, _ = p.shape
    kc, kn = head_counts(nblk, H, topk_frac, skip_frac)
    cls, tie = _classes(p, nblk, kc, kn)
    idx = np.full((B, H, nblk, int(kc.max())), -1, dtype=np.int32)
    for h in range(H):
        crit = np.nonzero(cls[:, h] == CLS_CRITICAL)   # row-major: ascending j within each (b, i)
        idx[:, h, :, :kc[h]] = crit[2].reshape(B, nblk, int(kc[h]))
    return {"cls": cls, "idx": idx, "kc": kc, "kn": kn, "near_tie": tie, "probs": p}


# ---------------------------------------------------------------- the whole operator

def sla_attention(q_bits, k_bits, v_bits, w_bits, block: int, topk_frac, *,
                  items=None, quant=True, pcast=True, smooth=True, idx_override=None, skip_frac=None,
                  gran=None):
    """Same arguments and result as sla_oracle.sla_attention: {"out",
    "o_sparse", "o_lin" (before the projection): {(b, h, i): float64 rows},
    "mask", "quant"}."""
    q = _c(q_bits, np.uint16)
    k = _c(k_bits, np.uint16)
    v = _c(v_bits, np.uint16)
    w = _c(w_bits, np.uint16)
    B, H, N, d = q.shape
    nblk = (N + block - 1) // block
    classes = skip_frac is not None or np.ndim(topk_frac) > 0
    if classes:
        mask = block_mask_classes(q, k, block, topk_frac, skip_frac)
        cls = np.array(mask["cls"], dtype=np.uint8, copy=True)
        for (b, h, i), row in (idx_override or {}).items():
            cls[b, h, i] = np.asarray(row, dtype=np.uint8)
    else:
        mask = block_mask(q, k, block, topk_frac)
        cls = np.ones((B, H, nblk, nblk), dtype=np.uint8)
        np.put_along_axis(cls, mask["idx"].astype(np.int64), CLS_CRITICAL, axis=-1)
        for (b, h, i), lst in (idx_override or {}).items():
            cls[b, h, i] = CLS_LINEAR
            cls[b, h, i, np.asarray(lst, dtype=np.int64)] = CLS_CRITICAL
    qz = quantize(q, k, block, gran) if quant else None
    mu = qz["mu"] if quant else channel_mean(k)
    if items is None:
        items = [(b, h, i) for b in range(B) for h in range(H) for i in range(nblk)]
    items = [tuple(int(t) for t in it) for it in items]
    it = np.array(items, dtype=np.int32).reshape(-1, 3)
    n = len(items)
    out = np.empty((n, block, d))
    osp = np.empty((n, block, d))
    olin = np.empty((n, block, d))
    if quant:
        ptrs = [_p(qz["q_i8"]), _p(qz["k_i8"]), _p(qz["q_scale"]), _p(qz["k_scale"])]
    else:
        ptrs = [None, None, None, None]
    rc = lib().ora_sla_rows(_p(q), _p(k), _p(v), _p(w), B, H, N, d, block, _p(cls),
                            _p(_c(mu, np.float32)), *ptrs, block if gran is None else gran, 1 if quant else 0,
                            1 if pcast else 0,
                            1 if smooth else 0, _p(it), n, threads(), _p(out), _p(osp), _p(olin))
    if rc != 0:
        raise RuntimeError(f"ora_sla_rows failed ({rc})")
    res = {"out": {}, "o_sparse": {}, "o_lin": {}, "mask": mask, "quant": qz}
    for t, (b, h, i) in enumerate(items):
        rows = min(N, (i + 1) * block) - i * block
        res["out"][(b, h, i)] = out[t, :rows]
        res["o_sparse"][(b, h, i)] = osp[t, :rows]
        res["o_lin"][(b, h, i)] = olin[t, :rows]
    return res
