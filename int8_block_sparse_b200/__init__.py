"""SageSLA attention for NVIDIA B200 (sm_100a) -- Python binding.

This module only marshals arguments: every step of the operator runs in the
CUDA kernels of ``libsla.so`` (built from ``csrc/`` by ``build.py``), called
through its C interface (``include/sla.h``).  PyTorch supplies device memory
and streams.  There is no CPU fallback: if the library is missing, importing
the binding's functions raises.
"""

from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsla.so")

SLA_OK = 0
STATUS_NAMES = {0: "SLA_OK", 1: "SLA_ERR_INVALID_ARG", 2: "SLA_ERR_UNSUPPORTED", 3: "SLA_ERR_CUDA",
                4: "SLA_ERR_OOM", 5: "SLA_ERR_TIMEOUT", 7: "SLA_ERR_SCRATCH_LIMIT",
                8: "SLA_ERR_SMEM_LAYOUT"}

EXPORTS = ("sla_topk_count", "sla_quant", "sla_mask", "sla_attn", "sla_attn_ex", "sla_attn_host",
           "sla_get_error", "sla_status_string", "sla_profile_enable", "sla_profile_read",
           "sla_mask_noalloc", "sla_selftest_wait_timeout", "sla_head_counts", "sla_mask_classes",
           "sla_attn_classes", "sla_attn_classes_host", "sla_w8a8_quant", "sla_w8a8_gemm", "sla_w8a8_linear",
           "sla_quant_gran", "sla_attn_gran")

KERNEL_KINDS = ("stats", "mean", "quant", "mask", "attn", "lingemm", "quant2d", "w8a8")

OUT_BF16, OUT_F32 = 0, 1


class SlaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({status_string(status)})")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libsla.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with `python -m int8_block_sparse_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        L.sla_topk_count.argtypes = [i, i, f]
        L.sla_quant.argtypes = [vp] * 7 + [i] * 5 + [vp]
        L.sla_mask.argtypes = [vp] * 4 + [i] * 5 + [f, vp]
        L.sla_mask_noalloc.argtypes = [vp] * 4 + [i] * 5 + [f, vp]
        L.sla_selftest_wait_timeout.argtypes = [vp]
        L.sla_attn.argtypes = [vp] * 5 + [i] * 5 + [f, vp]
        L.sla_attn_ex.argtypes = [vp] * 5 + [i] + [vp] * 2 + [i] * 5 + [f, vp]
        L.sla_attn_host.argtypes = [vp] * 5 + [i] * 5 + [f]
        L.sla_head_counts.argtypes = [i, i, i, vp, vp, vp, vp]
        L.sla_mask_classes.argtypes = [vp] * 4 + [i] * 5 + [vp, vp, vp]
        L.sla_attn_classes.argtypes = [vp] * 5 + [i] + [vp] * 2 + [i] * 5 + [vp, vp, vp]
        L.sla_attn_classes_host.argtypes = [vp] * 5 + [i] * 5 + [vp, vp]
        L.sla_w8a8_quant.argtypes = [vp, i, i, vp, vp, vp]
        L.sla_quant_gran.argtypes = [vp] * 7 + [i] * 6 + [vp]
        L.sla_attn_gran.argtypes = [vp] * 5 + [i] + [vp] * 2 + [i] * 5 + [f, i, vp]
        L.sla_w8a8_gemm.argtypes = [vp] * 6 + [i] * 4 + [vp]
        L.sla_w8a8_linear.argtypes = [vp] * 5 + [i] * 4 + [vp]
        L.sla_get_error.argtypes = [vp]
        L.sla_status_string.argtypes = [i]
        L.sla_status_string.restype = ctypes.c_char_p
        L.sla_profile_enable.argtypes = [i]
        L.sla_profile_read.argtypes = [vp, vp, i]
        for name in EXPORTS:
            if name != "sla_status_string":
                getattr(L, name).restype = i
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().sla_status_string(int(status)).decode()


def _check(rc: int, where: str) -> None:
    if rc != SLA_OK:
        raise SlaError(rc, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch

    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _shape(q):
    if q.dim() != 4:
        raise ValueError("q must be [B, H, N, d]")
    return tuple(int(x) for x in q.shape)


def topk_count(N: int, block: int, topk_frac: float) -> int:
    kc = lib().sla_topk_count(int(N), int(block), float(topk_frac))
    if kc < 0:
        raise SlaError(-kc, "sla_topk_count")
    return kc


def nblk(N: int, block: int) -> int:
    return (N + block - 1) // block


def _after(check: bool, stream, where: str) -> None:
    """With check=True, wait for the call and raise on a device-side status
    (a timed-out wait, a shared-memory layout failure); without it, such a
    status is only seen by a later get_error()."""
    if check:
        _check(get_error(stream), where)


def sla_quant(q, k, block: int, stream=None, check: bool = False, gran=None):
    """Smoothing + INT8 quantisation.  Returns (q_i8, k_i8, q_scale, k_scale, k_mean);
    one scale per block, or per ``gran`` tokens ([B, H, nblk * block / gran])."""
    import torch

    B, H, N, d = _shape(q)
    nb = nblk(N, block)
    dev = q.device
    g = block if gran is None else int(gran)
    qi8 = torch.empty((B, H, nb * block, d), dtype=torch.int8, device=dev)
    ki8 = torch.empty_like(qi8)
    sq = torch.empty((B, H, nb * block // g), dtype=torch.float32, device=dev)
    sk = torch.empty_like(sq)
    mu = torch.empty((B, H, d), dtype=torch.float32, device=dev)
    if gran is None:
        rc = lib().sla_quant(_ptr(q), _ptr(k), _ptr(qi8), _ptr(ki8), _ptr(sq), _ptr(sk), _ptr(mu),
                             B, H, N, d, block, _stream(stream))
    else:
        rc = lib().sla_quant_gran(_ptr(q), _ptr(k), _ptr(qi8), _ptr(ki8), _ptr(sq), _ptr(sk), _ptr(mu),
                                  B, H, N, d, block, g, _stream(stream))
    _check(rc, "sla_quant")
    _after(check, stream, "sla_quant")
    return qi8, ki8, sq, sk, mu


def sla_mask(q, k, block: int, topk_frac: float, bitmap: bool = False, stream=None, check: bool = False):
    """Pooled top-k block mask.  Returns idx [B,H,nblk,kc] int32 (and the uint8 bitmap)."""
    import torch

    B, H, N, d = _shape(q)
    nb = nblk(N, block)
    kc = topk_count(N, block, topk_frac)
    idx = torch.empty((B, H, nb, kc), dtype=torch.int32, device=q.device)
    bm = torch.empty((B, H, nb, nb), dtype=torch.uint8, device=q.device) if bitmap else None
    _check(lib().sla_mask(_ptr(q), _ptr(k), _ptr(idx), _ptr(bm), B, H, N, d, block, float(topk_frac),
                          _stream(stream)), "sla_mask")
    _after(check, stream, "sla_mask")
    return (idx, bm) if bitmap else idx


def sla_attn(q, k, v, proj, block: int = 128, topk_frac: float = 0.1, out=None, out_dtype=None,
             o_sparse=None, o_lin=None, stream=None, check: bool = False, gran=None):
    """SageSLA attention; q, k, v bf16 [B,H,N,d], proj bf16 [d,d] on the GPU.

    Returns out [B,H,N,d], bf16 by default (out_dtype=torch.float32, or a
    float32 `out`, for the unrounded result).  o_sparse / o_lin (float32,
    optional) receive the two parts, O_sparse and O_lin . W_proj.  gran: tokens
    per quantisation scale (32, 64 or 128; default one scale per block)."""
    import torch

    B, H, N, d = _shape(q)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=out_dtype or torch.bfloat16, device=q.device)
    if out.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out must be bf16 or float32")
    if gran is not None:
        kind = OUT_F32 if out.dtype == torch.float32 else OUT_BF16
        rc = lib().sla_attn_gran(_ptr(q), _ptr(k), _ptr(v), _ptr(proj), _ptr(out), kind, _ptr(o_sparse),
                                 _ptr(o_lin), B, H, N, d, block, float(topk_frac), int(gran), _stream(stream))
    elif out.dtype == torch.bfloat16 and o_sparse is None and o_lin is None:
        rc = lib().sla_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(proj), _ptr(out), B, H, N, d, block,
                            float(topk_frac), _stream(stream))
    else:
        kind = OUT_F32 if out.dtype == torch.float32 else OUT_BF16
        rc = lib().sla_attn_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(proj), _ptr(out), kind, _ptr(o_sparse),
                               _ptr(o_lin), B, H, N, d, block, float(topk_frac), _stream(stream))
    _check(rc, "sla_attn")
    _after(check, stream, "sla_attn")
    return out


def _head_fracs(H: int, topk_frac, skip_frac):
    """HOST float32 arrays of one topk_frac and one skip_frac (or None) per head."""
    tf = (ctypes.c_float * H)(*[float(x) for x in _per_head(topk_frac, H)])
    sf = None if skip_frac is None else (ctypes.c_float * H)(*[float(x) for x in _per_head(skip_frac, H)])
    return tf, sf


def _per_head(x, H: int):
    try:
        vals = [float(t) for t in x]
    except TypeError:
        vals = [float(x)] * H
    if len(vals) != H:
        raise ValueError(f"expected one fraction per head ({H})")
    return vals


def _cptr(arr):
    return None if arr is None else ctypes.cast(arr, ctypes.c_void_p)


def head_counts(N: int, block: int, H: int, topk_frac, skip_frac=None):
    """(kc per head, kn per head, list pitch) of the three-class mask."""
    tf, sf = _head_fracs(H, topk_frac, skip_frac)
    kc = (ctypes.c_int * H)()
    kn = (ctypes.c_int * H)()
    kcp = lib().sla_head_counts(int(N), int(block), int(H), _cptr(tf), _cptr(sf), _cptr(kc), _cptr(kn))
    if kcp < 0:
        raise SlaError(-kcp, "sla_head_counts")
    return list(kc), list(kn), kcp


def sla_mask_classes(q, k, block: int, topk_frac, skip_frac=None, classes: bool = False, stream=None,
                     check: bool = False):
    """Three-class block mask with per-head fractions.  Returns idx [B,H,nblk,kcp]
    int32 (kept blocks ascending, then -1) and, with classes=True, the uint8
    class map [B,H,nblk,nblk] (2 kept, 1 linear branch, 0 left out)."""
    import torch

    B, H, N, d = _shape(q)
    nb = nblk(N, block)
    tf, sf = _head_fracs(H, topk_frac, skip_frac)
    _, _, kcp = head_counts(N, block, H, topk_frac, skip_frac)
    idx = torch.empty((B, H, nb, kcp), dtype=torch.int32, device=q.device)
    cm = torch.empty((B, H, nb, nb), dtype=torch.uint8, device=q.device) if classes else None
    _check(lib().sla_mask_classes(_ptr(q), _ptr(k), _ptr(idx), _ptr(cm), B, H, N, d, block, _cptr(tf), _cptr(sf),
                                  _stream(stream)), "sla_mask_classes")
    _after(check, stream, "sla_mask_classes")
    return (idx, cm) if classes else idx


def sla_attn_classes(q, k, v, proj, block: int = 128, topk_frac=0.1, skip_frac=None, out=None, out_dtype=None,
                     o_sparse=None, o_lin=None, stream=None, check: bool = False):
    """SageSLA attention with per-head fractions and an optional third block
    class left out of the linear branch (skip_frac per head or scalar)."""
    import torch

    B, H, N, d = _shape(q)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=out_dtype or torch.bfloat16, device=q.device)
    if out.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out must be bf16 or float32")
    tf, sf = _head_fracs(H, topk_frac, skip_frac)
    kind = OUT_F32 if out.dtype == torch.float32 else OUT_BF16
    _check(lib().sla_attn_classes(_ptr(q), _ptr(k), _ptr(v), _ptr(proj), _ptr(out), kind, _ptr(o_sparse),
                                  _ptr(o_lin), B, H, N, d, block, _cptr(tf), _cptr(sf), _stream(stream)),
           "sla_attn_classes")
    _after(check, stream, "sla_attn_classes")
    return out


def sla_attn_host(q, k, v, proj, out, block: int = 128, topk_frac: float = 0.1) -> None:
    """SageSLA attention on host (CPU) tensors (out: bf16); copies in and out inside the call."""
    B, H, N, d = _shape(q)
    _check(lib().sla_attn_host(_ptr(q), _ptr(k), _ptr(v), _ptr(proj), _ptr(out), B, H, N, d, block,
                               float(topk_frac)), "sla_attn_host")


def sla_attn_classes_host(q, k, v, proj, out, block: int = 128, topk_frac=0.1, skip_frac=None) -> None:
    """sla_attn_classes on host (CPU) tensors (out: bf16); copies in and out inside the call."""
    B, H, N, d = _shape(q)
    tf, sf = _head_fracs(H, topk_frac, skip_frac)
    _check(lib().sla_attn_classes_host(_ptr(q), _ptr(k), _ptr(v), _ptr(proj), _ptr(out), B, H, N, d, block,
                                       _cptr(tf), _cptr(sf)), "sla_attn_classes_host")


def w8a8_quant(x, stream=None, check: bool = False):
    """128x128 block quantisation of a bf16 [R, K] matrix: (codes int8 [R, K], scales [ceil(R/128), ceil(K/128)])."""
    import torch

    if x.dim() != 2:
        raise ValueError("x must be [R, K]")
    R, K = (int(t) for t in x.shape)
    codes = torch.empty((R, K), dtype=torch.int8, device=x.device)
    scales = torch.empty(((R + 127) // 128, (K + 127) // 128), dtype=torch.float32, device=x.device)
    _check(lib().sla_w8a8_quant(_ptr(x), R, K, _ptr(codes), _ptr(scales), _stream(stream)), "sla_w8a8_quant")
    _after(check, stream, "sla_w8a8_quant")
    return codes, scales


def _y_for(M, N, out, out_dtype, device):
    import torch

    if out is None:
        out = torch.empty((M, N), dtype=out_dtype or torch.bfloat16, device=device)
    if out.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out must be bf16 or float32")
    return out, (OUT_F32 if out.dtype == torch.float32 else OUT_BF16)


def w8a8_gemm(xq, sx, wq, sw, bias=None, out=None, out_dtype=None, stream=None, check: bool = False):
    """Y = X . W^T + bias from the codes and scales of X [M, K] and W [N, K]."""
    M, K = (int(t) for t in xq.shape)
    N = int(wq.shape[0])
    y, kind = _y_for(M, N, out, out_dtype, xq.device)
    _check(lib().sla_w8a8_gemm(_ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), _ptr(bias), _ptr(y), kind, M, N, K,
                               _stream(stream)), "sla_w8a8_gemm")
    _after(check, stream, "sla_w8a8_gemm")
    return y


def w8a8_linear(x, wq, sw, bias=None, out=None, out_dtype=None, stream=None, check: bool = False):
    """The W8A8 layer on bf16 activations x [M, K] (quantised in the call) and
    pre-quantised weights (wq [N, K], sw from w8a8_quant)."""
    M, K = (int(t) for t in x.shape)
    N = int(wq.shape[0])
    y, kind = _y_for(M, N, out, out_dtype, x.device)
    _check(lib().sla_w8a8_linear(_ptr(x), _ptr(wq), _ptr(sw), _ptr(bias), _ptr(y), kind, M, N, K, _stream(stream)),
           "sla_w8a8_linear")
    _after(check, stream, "sla_w8a8_linear")
    return y


def profile_enable(on: bool = True) -> None:
    """Bracket every library kernel launch with CUDA events (see sla_profile_read)."""
    lib().sla_profile_enable(1 if on else 0)


def profile_read() -> dict:
    """{kernel kind: (summed device ms, launches)} since the last read; clears them."""
    n = len(KERNEL_KINDS)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_longlong * n)()
    _check(lib().sla_profile_read(ctypes.cast(ms, ctypes.c_void_p), ctypes.cast(cnt, ctypes.c_void_p), n),
           "sla_profile_read")
    return {k: (ms[i], cnt[i]) for i, k in enumerate(KERNEL_KINDS)}


def get_error(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device error status."""
    return lib().sla_get_error(_stream(stream))
