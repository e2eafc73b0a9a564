"""Pins of the W8A8 linear-layer oracles (the numpy statement
oracle/w8a8_oracle.py and the plain C++ one behind oracle/w8a8_cpp.py)
against things other than themselves: exact rational arithmetic on tiny
cases, integer matmuls of another library, closed forms, and the attention
quantiser (itself pinned in test_oracle_pins.py) on matrices of one column
block; tests taking the `impl` fixture run against both.  The two oracles
must also agree bit for bit.  No GPU needed."""

from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as A
from oracle import w8a8_cpp as WC
from oracle import w8a8_oracle as W
from synth.linear import make_linear
from synth.workloads import f32_to_bf16_bits


@pytest.fixture(params=["numpy", "cpp"])
def impl(request):
    return W if request.param == "numpy" else WC


def bits(x):
    x = np.asarray(x, dtype=np.float32)
    b = f32_to_bf16_bits(x)
    assert np.array_equal(W.bf16_to_f32(b), x), "test values must be exact in bf16"
    return b


def test_quant_ties_round_half_to_even(impl):
    """A block whose maximum is 127 * 2^-3 has scale exactly 2^-3; x = 2.5 and
    3.5 and -2.5 steps quantise to 2, 4, -2 (half to even)."""
    x = np.zeros((130, 200), dtype=np.float32)
    x[0, 0] = 127 * 0.125
    x[1, 1], x[2, 2], x[3, 3], x[4, 4] = 2.5 * 0.125, 3.5 * 0.125, -2.5 * 0.125, 0.5 * 0.125
    codes, scales = impl.quantize_2d(bits(x))
    assert scales[0, 0] == np.float32(0.125)
    assert [codes[1, 1], codes[2, 2], codes[3, 3], codes[4, 4]] == [2, 4, -2, 0]


def test_quant_blocks_are_128_by_128_and_partial_at_the_edges(impl):
    """Each scale is the maximum over exactly its 128 x 128 tile (brute force),
    and changing an element outside a tile changes neither its scale nor its
    codes."""
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((300, 270)) * np.exp(rng.standard_normal((300, 270)))).astype(np.float32)
    xb = f32_to_bf16_bits(x)
    xf = W.bf16_to_f32(xb)
    codes, scales = impl.quantize_2d(xb)
    assert scales.shape == (3, 3) and codes.shape == (300, 270)
    for rb in range(3):
        for kb in range(3):
            m = 0.0
            for r in range(rb * 128, min(300, rb * 128 + 128)):
                for c in range(kb * 128, min(270, kb * 128 + 128)):
                    m = max(m, abs(float(xf[r, c])))
            assert scales[rb, kb] == np.float32(np.float32(m) / np.float32(127))
    y = xb.copy()
    y[0, 200] = f32_to_bf16_bits(np.array([1e4], dtype=np.float32))[0]       # tile (0, 1)
    c2, s2 = impl.quantize_2d(y)
    assert np.array_equal(s2[:, 0], scales[:, 0]) and np.array_equal(c2[:, :128], codes[:, :128])
    assert s2[0, 1] != scales[0, 1]


def test_quant_round_trip_and_zero_block(impl):
    rng = np.random.default_rng(2)
    ints = rng.integers(-127, 128, size=(256, 256))
    ints[0, 0] = 127
    ints[0, 128] = -127
    ints[128, 0] = 127
    ints[128:, 128:] = 0                                           # a zero tile
    x = ints.astype(np.float32) * np.float32(2.0 ** -5)
    codes, scales = impl.quantize_2d(bits(x))
    assert scales.tolist() == [[2.0 ** -5, 2.0 ** -5], [2.0 ** -5, 0.0]]
    assert np.array_equal(codes.astype(np.int64), ints)


def test_quant_equals_the_attention_quantiser_on_one_column_block(impl):
    """With K = 128 there is one column block, so the 128 x 128 tiles are the
    attention quantiser's blocks of 128 rows x d = 128 channels."""
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((1, 1, 1000, 128)) * 3).astype(np.float32)
    xb = f32_to_bf16_bits(x)
    codes_a, scales_a = A.quantize_blocks(A.bf16_to_f32(xb), 128)
    codes, scales = impl.quantize_2d(xb[0, 0])
    assert np.array_equal(codes, codes_a[0, 0, :1000])
    assert np.array_equal(scales[:, 0], scales_a[0, 0])


def test_gemm_exact_rationals_on_a_tiny_case(impl):
    """Y from exact rational arithmetic over the codes and scales (three
    column blocks, two row blocks of W, a bias)."""
    d = make_linear(3, 130, 300, seed=4)
    lin = impl.linear(d["x"], d["w"], d["bias"])
    xq, sx, wq, sw = lin["xq"], lin["sx"], lin["wq"], lin["sw"]
    b = W.bf16_to_f32(d["bias"])
    for m in range(3):
        for n in (0, 1, 127, 128, 129):
            acc = Fraction(0)
            for k in range(300):
                kb = k // 128
                acc += Fraction(int(xq[m, k]) * int(wq[n, k])) * Fraction(float(sx[0, kb])) * \
                    Fraction(float(sw[n // 128, kb]))
            acc += Fraction(float(b[n]))
            assert lin["y"][m, n] == pytest.approx(float(acc), rel=1e-14, abs=1e-300)


def test_gemm_is_x_times_w_transposed(impl):
    """Unit scales (every tile's maximum is 127) and integer inputs: Y is the
    integer product X W^T exactly (torch int64), and not X W."""
    rng = np.random.default_rng(5)
    x = rng.integers(-127, 128, size=(128, 128))
    w = rng.integers(-127, 128, size=(128, 128))
    x[0, 0] = w[0, 0] = 127
    lin = impl.linear(bits(x), bits(w))
    assert lin["sx"].tolist() == [[1.0]] and lin["sw"].tolist() == [[1.0]]
    ref = (torch.from_numpy(x) @ torch.from_numpy(w).T).numpy()
    assert np.array_equal(lin["y"], ref.astype(np.float64))
    assert not np.array_equal(lin["y"], (x @ w).astype(np.float64))


def test_gemm_equals_the_product_of_the_dequantised_matrices(impl):
    """sum_kb P_kb sx sw = (Xq * sx) (Wq * sw)^T with the scales spread over
    their tiles (torch float64 matmul), up to float64 rounding."""
    d = make_linear(300, 260, 400, seed=6, bias=False)
    lin = impl.linear(d["x"], d["w"])
    ex = np.kron(lin["sx"].astype(np.float64), np.ones((128, 128)))[:300, :400]
    ew = np.kron(lin["sw"].astype(np.float64), np.ones((128, 128)))[:260, :400]
    deq = torch.from_numpy(lin["xq"] * ex) @ torch.from_numpy(lin["wq"] * ew).T
    assert np.allclose(lin["y"], deq.numpy(), rtol=1e-12, atol=1e-12)


def test_linear_is_close_to_the_unquantised_layer_within_the_quantisation_bound(impl):
    """|Y - (X W^T + b)| <= sum_k (|x| e_w + |w| e_x + e_x e_w) with e = s/2 plus
    the float32 rounding of the quotient (one unit in x/s): a closed-form
    bound of block quantisation."""
    d = make_linear(200, 150, 384, seed=7)
    lin = impl.linear(d["x"], d["w"], d["bias"])
    x = W.bf16_to_f32(d["x"]).astype(np.float64)
    w = W.bf16_to_f32(d["w"]).astype(np.float64)
    b = W.bf16_to_f32(d["bias"]).astype(np.float64)
    ex = np.kron(lin["sx"].astype(np.float64), np.ones((128, 128)))[:200, :384] * (0.5 + 2.0 ** -16)
    ew = np.kron(lin["sw"].astype(np.float64), np.ones((128, 128)))[:150, :384] * (0.5 + 2.0 ** -16)
    bound = np.abs(x) @ ew.T + ex @ np.abs(w).T + ex @ ew.T
    err = np.abs(lin["y"] - (x @ w.T + b))
    assert np.all(err <= bound * (1 + 1e-12) + 1e-12)
    assert err.max() > 0


def test_rows_subset_matches_the_full_product(impl):
    d = make_linear(400, 130, 256, seed=8)
    full = impl.linear(d["x"], d["w"], d["bias"])
    part = impl.linear(d["x"], d["w"], d["bias"], rows=[0, 129, 399])
    assert np.array_equal(part["y"], full["y"][[0, 129, 399]])


def test_f32_error_bound_covers_a_float32_accumulation():
    """The stated bound holds for a float32 evaluation in the CUDA path's order
    (scale product rounded, one fused multiply-add per column block, bias last)."""
    d = make_linear(64, 64, 1024, seed=9)
    lin = W.linear(d["x"], d["w"], d["bias"])
    xq, sx, wq, sw = lin["xq"], lin["sx"], lin["wq"], lin["sw"]
    acc = np.zeros((64, 64), dtype=np.float32)
    for kb in range(8):
        cols = slice(kb * 128, kb * 128 + 128)
        P = (xq[:, cols].astype(np.int64) @ wq[:, cols].astype(np.int64).T).astype(np.float32)
        s = np.float32(sx[0, kb] * sw[0, kb])
        acc = (P.astype(np.float64) * np.float64(s) + acc.astype(np.float64)).astype(np.float32)   # fma
    acc = (acc + W.bf16_to_f32(d["bias"])[None, :]).astype(np.float32)
    err = np.abs(acc.astype(np.float64) - lin["y"])
    assert np.all(err <= W.f32_error_bound(lin["abs"], 1024))


@pytest.mark.parametrize("M,N,K,bias,seed", [
    (300, 260, 400, True, 10),
    (1, 1, 1, True, 11),
    (129, 17, 1000, False, 12),
    (256, 384, 128, True, 13),
])
def test_cpp_and_numpy_oracles_agree_bit_for_bit(M, N, K, bias, seed):
    d = make_linear(M, N, K, seed=seed, bias=bias)
    rows = sorted({0, M - 1, M // 2})
    for r in (None, rows):
        a = W.linear(d["x"], d["w"], d["bias"], rows=r)
        b = WC.linear(d["x"], d["w"], d["bias"], rows=r)
        for key in ("xq", "sx", "wq", "sw", "y", "abs"):
            assert a[key].dtype == b[key].dtype and np.array_equal(a[key], b[key]), key
