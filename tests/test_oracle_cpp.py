"""The plain C++ oracle against the numpy statement of the same method, on
small seeded cases that span several blocks, ragged tails, d = 64 and 128,
both block sizes, B > 1 and every block kept.  The two are written
independently (plain loops and exact integer sums in C++; numpy and BLAS in
Python) and both are pinned by tests/test_oracle_pins.py; here they must
agree bit for bit on the INT8 codes, scales, channel means and block lists
(up to rows the oracle marks as near ties) and to float64 rounding on the
outputs.  No GPU needed."""

import numpy as np
import pytest

import oracle as NP
from oracle import cpp_oracle as C
from synth import make_inputs

CASES = [
    # (B, H, N, d, block, frac, dist, seed)
    (1, 2, 1024, 64, 64, 0.25, "iid", 0),
    (1, 1, 1000, 128, 128, 0.25, "iid", 11),
    (2, 3, 640, 128, 128, 0.4, "iid", 12),
    (1, 2, 129, 128, 128, 0.5, "iid", 13),
    (1, 1, 1, 128, 128, 0.1, "iid", 14),
    (1, 2, 777, 64, 128, 0.3, "iid", 15),
    (1, 2, 700, 128, 64, 0.2, "iid", 16),
    (1, 1, 1024, 128, 128, 1.0, "iid", 17),
    (1, 2, 4096, 64, 128, 0.1, "field", 18),
]


@pytest.mark.parametrize("B,H,N,d,block,frac,dist,seed", CASES)
def test_cpp_oracle_agrees_with_numpy_oracle(B, H, N, d, block, frac, dist, seed):
    grid = (4, 32, 32) if dist == "field" else None
    x = make_inputs(B, H, N, d, seed, dist, grid)
    a = NP.sla_attention(x["q"], x["k"], x["v"], x["proj"], block, frac)
    b = C.sla_attention(x["q"], x["k"], x["v"], x["proj"], block, frac)
    for key in ("mu", "q_i8", "k_i8", "q_scale", "k_scale"):
        assert np.array_equal(a["quant"][key], b["quant"][key]), key
    diff = np.any(a["mask"]["idx"] != b["mask"]["idx"], axis=-1)
    assert not np.any(diff & ~a["mask"]["near_tie"])
    assert np.array_equal(a["mask"]["near_tie"], b["mask"]["near_tie"])
    assert np.allclose(a["mask"]["probs"], b["mask"]["probs"], rtol=1e-13, atol=0)
    for part in ("out", "o_sparse", "o_lin"):
        for key in a[part]:
            if diff[key]:
                continue
            assert np.max(np.abs(a[part][key] - b[part][key])) <= 1e-12, (part, key)


def test_cpp_oracle_modes_agree_with_numpy_oracle():
    """The invariant modes (quantisation off, P cast off, smoothing off)."""
    x = make_inputs(1, 2, 320, 32, 5)
    for kw in ({"quant": False}, {"pcast": False}, {"quant": False, "pcast": False, "smooth": False}):
        a = NP.sla_attention(x["q"], x["k"], x["v"], x["proj"], 64, 0.4, **kw)
        b = C.sla_attention(x["q"], x["k"], x["v"], x["proj"], 64, 0.4, **kw)
        for key in a["out"]:
            assert np.max(np.abs(a["out"][key] - b["out"][key])) <= 1e-12, kw


@pytest.mark.parametrize("N,d,block,fr,sk,seed", [
    (1000, 64, 64, [0.1, 0.3, 0.5], [0.5, 0.2, 0.0], 21),
    (777, 128, 128, [0.25, 1.0, 0.05], [0.7, 0.0, 0.9], 22),
])
def test_cpp_oracle_three_classes_agree_with_numpy_oracle(N, d, block, fr, sk, seed):
    x = make_inputs(2, 3, N, d, seed, "iid", None)
    a = NP.sla_attention(x["q"], x["k"], x["v"], x["proj"], block, fr, skip_frac=sk)
    b = C.sla_attention(x["q"], x["k"], x["v"], x["proj"], block, fr, skip_frac=sk)
    assert np.array_equal(a["mask"]["kc"], b["mask"]["kc"]) and np.array_equal(a["mask"]["kn"], b["mask"]["kn"])
    assert np.array_equal(a["mask"]["near_tie"], b["mask"]["near_tie"])
    diff = np.any(a["mask"]["cls"] != b["mask"]["cls"], axis=-1)
    assert not np.any(diff & ~a["mask"]["near_tie"])
    assert np.array_equal(a["mask"]["idx"][~diff], b["mask"]["idx"][~diff])
    for part in ("out", "o_sparse", "o_lin"):
        for key in a[part]:
            if diff[key]:
                continue
            assert np.max(np.abs(a[part][key] - b[part][key])) <= 1e-12, (part, key)
