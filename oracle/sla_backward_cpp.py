"""The plain C++ oracle of the SLA fine-tune path (sla_backward_oracle.cpp)
behind the same Python functions as the numpy statement
(sla_backward_oracle.py).  TEST INFRASTRUCTURE ONLY: imported by the tests.

The C++ file restates the forward and its gradient with plain loops; the
numpy statement's finite-difference and autograd pins run against both, and
the two agree to float64 rounding (tests/test_backward_oracle.py).  This
module only marshals numpy arrays.
"""

from __future__ import annotations

import ctypes

import numpy as np

from .cpp_oracle import lib as _base_lib

_ready = False


def lib() -> ctypes.CDLL:
    global _ready
    L = _base_lib()
    if not _ready:
        vp, i = ctypes.c_void_p, ctypes.c_int
        L.ora_sla_train_forward.argtypes = [vp] * 5 + [i] * 3 + [vp]
        L.ora_sla_train_backward.argtypes = [vp] * 5 + [i] * 3 + [vp] * 5
        _ready = True
    return L


def _p(a):
    return ctypes.c_void_p(a.ctypes.data)


def _prep(q, k, v, w, crit_lists, block):
    q, k, v, w = (np.ascontiguousarray(a, dtype=np.float64) for a in (q, k, v, w))
    N, d = q.shape
    assert k.shape == v.shape == (N, d) and w.shape == (d, d)
    nblk = (N + block - 1) // block
    assert len(crit_lists) == nblk
    kept = np.zeros((nblk, nblk), dtype=np.uint8)
    for i, lst in enumerate(crit_lists):
        lst = np.asarray(lst, dtype=np.int64)
        assert lst.size > 0 and lst.min() >= 0 and lst.max() < nblk
        kept[i, lst] = 1
    return q, k, v, w, kept, N, d


def forward(q, k, v, w, crit_lists, block):
    """{"out": [N, d]} of one head for fixed kept-block lists (float64)."""
    q, k, v, w, kept, N, d = _prep(q, k, v, w, crit_lists, block)
    out = np.empty((N, d))
    lib().ora_sla_train_forward(_p(q), _p(k), _p(v), _p(w), _p(kept), N, d, block, _p(out))
    return {"out": out}


def backward(q, k, v, w, crit_lists, block, g):
    """Gradients of L = sum(out * g): {"dq", "dk", "dv", "dw"}."""
    q, k, v, w, kept, N, d = _prep(q, k, v, w, crit_lists, block)
    g = np.ascontiguousarray(g, dtype=np.float64)
    assert g.shape == (N, d)
    dq, dk, dv = (np.empty((N, d)) for _ in range(3))
    dw = np.empty((d, d))
    lib().ora_sla_train_backward(_p(q), _p(k), _p(v), _p(w), _p(kept), N, d, block, _p(g), _p(dq), _p(dk), _p(dv),
                                 _p(dw))
    return {"dq": dq, "dk": dk, "dv": dv, "dw": dw}
