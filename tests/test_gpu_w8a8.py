"""The W8A8 linear layer's CUDA path against its CPU oracle
(oracle/w8a8_oracle.py), through the C interface.

The codes and scales must be bit-exact.  The float32 result must be within
the bound the float32 arithmetic allows (f32_error_bound: (nkb + 3) units of
2^-24 of the sum of the magnitudes of the terms) of the oracle's float64
value, element by element; the bf16 result must be exactly the float32
result rounded to nearest even.
"""

import numpy as np
import pytest

from oracle import cpp_oracle as C
from oracle import w8a8_oracle as W
from synth.linear import LINEAR_CONFIGS, make_linear, make_linear_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    import torch

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import int8_block_sparse_b200 as S
    from int8_block_sparse_b200.build import build

    build()
    S.lib()
    return S


def dev(bits):
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def check_quant(S, bits):
    codes, scales = S.w8a8_quant(dev(bits))
    assert S.get_error() == 0
    rc, rs = W.quantize_2d(bits)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    got = codes.cpu().numpy()
    assert np.array_equal(got, rc), int(np.sum(got != rc))
    return codes, scales


def check_linear(S, d, rows=None, case="?"):
    import torch

    x, w, b = dev(d["x"]), dev(d["w"]), (None if d["bias"] is None else dev(d["bias"]))
    wq, sw = check_quant(S, d["w"])
    y32 = S.w8a8_linear(x, wq, sw, b, out_dtype=torch.float32)
    y16 = S.w8a8_linear(x, wq, sw, b)
    assert S.get_error() == 0
    M, K = d["x"].shape
    xq_ref, sx_ref = W.quantize_2d(d["x"]) if rows is None else (None, None)
    if rows is None:
        xq, sx = check_quant(S, d["x"])
        ref_xq, ref_sx = xq_ref, sx_ref
        rows = np.arange(M)
    else:
        # the rows' 128-row blocks are quantised in full by the oracle
        blocks = sorted({int(r) // 128 for r in rows})
        ref_xq = np.zeros((M, K), dtype=np.int8)
        ref_sx = np.zeros(((M + 127) // 128, (K + 127) // 128), dtype=np.float32)
        xs = x.view(torch.int16).cpu().numpy().view(np.uint16)
        for rb in blocks:
            c, s = W.quantize_2d(xs[rb * 128:(rb + 1) * 128])
            ref_xq[rb * 128:rb * 128 + len(c)] = c
            ref_sx[rb] = s[0]
        xq, sx = S.w8a8_quant(x)
        for rb in blocks:
            assert np.array_equal(sx[rb].cpu().numpy(), ref_sx[rb])
            assert np.array_equal(xq[rb * 128:(rb + 1) * 128].cpu().numpy(), ref_xq[rb * 128:(rb + 1) * 128])
    y, a = W.gemm(ref_xq, ref_sx, wq.cpu().numpy(), sw.cpu().numpy(), d["bias"], rows)
    g32 = y32[torch.as_tensor(rows, device="cuda")].cpu().numpy().astype(np.float64)
    g16 = y16[torch.as_tensor(rows, device="cuda")].float().cpu().numpy().astype(np.float64)
    err = np.abs(g32 - y)
    bound = W.f32_error_bound(a, K)
    assert np.all(err <= bound), (case, float((err / np.maximum(bound, 1e-300)).max()))
    assert np.array_equal(g16, C.round_bf16(g32)), case
    rel = float(np.max(err / np.maximum(a, 1e-30)))
    print(f'{{"case": "{case}", "rows": {len(rows)}, "max_err_over_bound": '
          f'{float(np.max(err / np.maximum(bound, 1e-300))):.3f}, "max_rel_to_abs_sum": {rel:.3e}}}')


SHAPES = [
    # (M, N, K, bias, seed)
    (1000, 528, 656, True, 1),       # no dimension a multiple of 128; the last N tile has 16 columns
    (128, 256, 128, False, 2),       # one tile, one k-block
    (1, 16, 16, True, 3),            # the smallest layer
    (300, 1024, 4096, True, 4),      # 32 k-blocks
    (2000, 272, 1536, False, 5),     # N = 256 + 16
    (129, 384, 2048, True, 6),       # a one-row second M block
]


@pytest.mark.parametrize("M,N,K,bias,seed", SHAPES)
def test_w8a8_small(S, M, N, K, bias, seed):
    check_linear(S, make_linear(M, N, K, seed, bias), case=f"{M}x{N}x{K}")


def test_w8a8_gemm_entry_matches_linear(S):
    import torch

    d = make_linear(700, 512, 1024, 7)
    x, w, b = dev(d["x"]), dev(d["w"]), dev(d["bias"])
    wq, sw = S.w8a8_quant(w)
    xq, sx = S.w8a8_quant(x)
    a = S.w8a8_gemm(xq, sx, wq, sw, b)
    c = S.w8a8_linear(x, wq, sw, b)
    assert torch.equal(a, c)


def test_w8a8_zero_blocks_and_outliers(S):
    """An all-zero 128x128 block of X (scale 0) and a column block with one
    huge value: codes and outputs still match."""
    d = make_linear(256, 256, 384, 8)
    x = d["x"].copy()
    x[:128, 128:256] = 0
    from synth.workloads import f32_to_bf16_bits

    x[200, 300] = f32_to_bf16_bits(np.array([3.0e4], dtype=np.float32))[0]
    d["x"] = x
    check_linear(S, d, case="zero-block")


@pytest.mark.parametrize("name", ["w8a8_small", "w8a8_14b_ffn", "w8a8_14b_proj", "w8a8_1b3_ffn"])
def test_w8a8_workloads(S, name):
    w = LINEAR_CONFIGS[name]
    d = make_linear_workload(w)
    rng = np.random.default_rng(w.seed)
    rows = None if w.M <= 2048 else np.unique(np.concatenate([[0, 127, 128, w.M - 1],
                                                               rng.integers(0, w.M, 60)]))
    check_linear(S, d, rows=rows, case=name)
