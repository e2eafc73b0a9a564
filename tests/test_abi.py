"""The C interface without a GPU: the library loads, exports every entry point
include/sla.h declares, and refuses invalid arguments before any CUDA call."""

import ctypes
import os
import re

import pytest

import int8_block_sparse_b200 as S

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "sla.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sla_[a-z_0-9]+)\s*\(", text)))


def test_library_exports_every_declared_function():
    names = declared_functions()
    assert len(names) >= 12
    lib = S.lib()
    for n in names:
        assert hasattr(lib, n), n
        assert n in S.EXPORTS, n


def test_status_strings():
    header = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    declared = {int(v): n for n, v in re.findall(r"\b(SLA_(?:OK|ERR_[A-Z_]+))\s*=\s*(\d+)", header)}
    assert declared == S.STATUS_NAMES
    for code in declared:
        assert S.status_string(code) and S.status_string(code) != "unknown status", code
    assert S.status_string(99) == "unknown status"


@pytest.mark.parametrize("N,block,frac,kc", [(32768, 128, 0.1, 26), (75600, 128, 0.1, 60), (1024, 64, 0.25, 4),
                                             (1, 128, 0.5, 1), (129, 64, 1.0, 3)])
def test_topk_count_matches_oracle_rule(N, block, frac, kc):
    import oracle as O

    assert S.topk_count(N, block, frac) == kc == O.topk_count((N + block - 1) // block, frac)


def test_invalid_arguments_are_refused_without_a_gpu():
    L = S.lib()
    f = ctypes.c_float
    dummy = 4096                      # 16-byte aligned, never dereferenced
    # null pointers
    assert L.sla_attn(None, dummy, dummy, dummy, dummy, 1, 1, 128, 128, 128, f(0.1), None) == 1
    assert L.sla_quant(dummy, None, dummy, dummy, dummy, dummy, None, 1, 1, 128, 128, 128, None) == 1
    assert L.sla_mask(dummy, dummy, None, None, 1, 1, 128, 128, 128, f(0.1), None) == 1
    # misaligned pointer
    assert L.sla_attn(dummy + 2, dummy, dummy, dummy, dummy, 1, 1, 128, 128, 128, f(0.1), None) == 1
    # shapes
    assert L.sla_attn(dummy, dummy, dummy, dummy, dummy, 0, 1, 128, 128, 128, f(0.1), None) == 1
    assert L.sla_attn(dummy, dummy, dummy, dummy, dummy, 1, 1, 0, 128, 128, f(0.1), None) == 1
    assert L.sla_attn(dummy, dummy, dummy, dummy, dummy, 1, 1, 128, 96, 128, f(0.1), None) == 2
    assert L.sla_attn(dummy, dummy, dummy, dummy, dummy, 1, 1, 128, 128, 32, f(0.1), None) == 2
    assert L.sla_attn(dummy, dummy, dummy, dummy, dummy, 1, 70000, 128, 128, 128, f(0.1), None) == 2
    # top-k fraction
    for bad in (0.0, -0.5, 1.5, float("nan")):
        assert L.sla_attn(dummy, dummy, dummy, dummy, dummy, 1, 1, 128, 128, 128, f(bad), None) == 1
        assert L.sla_mask(dummy, dummy, dummy, None, 1, 1, 128, 128, 128, f(bad), None) == 1
    assert L.sla_topk_count(0, 128, f(0.1)) == -1
    assert L.sla_topk_count(10, 128, f(0.0)) == -1
    # the allocation-free mask refuses problems beyond its fixed buffer
    assert L.sla_mask_noalloc(dummy, dummy, dummy, None, 1, 40, 75600, 128, 128, f(0.1), None) == 7


def test_head_counts_match_the_oracle_rules():
    import oracle as O

    fr, sk = [0.1, 0.05, 0.4, 1.0], [0.5, 0.9, 0.0, 0.3]
    kc, kn, kcp = S.head_counts(32768, 128, 4, fr, sk)
    okc, okn = O.head_counts(256, 4, fr, sk)
    assert kc == okc.tolist() and kn == okn.tolist() and kcp == max(kc)
    kc, kn, kcp = S.head_counts(1000, 64, 3, 0.25)           # scalar, no skip
    assert kc == [4, 4, 4] and kn == [0, 0, 0] and kcp == 4


def test_class_entry_points_refuse_invalid_arguments_without_a_gpu():
    L = S.lib()
    dummy = 4096
    arr = lambda *v: ctypes.cast((ctypes.c_float * len(v))(*v), ctypes.c_void_p)
    good = arr(0.1, 0.2)
    for bad in (arr(0.1, 0.0), arr(1.5, 0.1), arr(float("nan"), 0.1)):
        assert L.sla_attn_classes(dummy, dummy, dummy, dummy, dummy, 0, None, None, 1, 2, 128, 128, 128, bad,
                                  None, None) == 1
        assert L.sla_mask_classes(dummy, dummy, dummy, None, 1, 2, 128, 128, 128, bad, None, None) == 1
    for bad in (arr(0.0, 1.0), arr(-0.1, 0.0)):
        assert L.sla_attn_classes(dummy, dummy, dummy, dummy, dummy, 0, None, None, 1, 2, 128, 128, 128, good,
                                  bad, None) == 1
    assert L.sla_attn_classes(dummy, dummy, dummy, dummy, dummy, 0, None, None, 1, 2, 128, 128, 128, None,
                              None, None) == 1
    many = (ctypes.c_float * 600)(*([0.1] * 600))
    assert L.sla_attn_classes(dummy, dummy, dummy, dummy, dummy, 0, None, None, 1, 600, 128, 128, 128,
                              ctypes.cast(many, ctypes.c_void_p), None, None) == 2
    assert L.sla_head_counts(128, 128, 2, None, None, None, None) == -1


def test_binding_marshals_the_class_entry_points(monkeypatch):
    """The binding's argument marshalling for the class entry points, against a
    stand-in for the library that records each call (no GPU: CPU tensors and
    a stream object with a null handle)."""
    import torch

    calls = []

    class FakeFn:
        def __init__(self, name):
            self.name = name

        def __call__(self, *a):
            calls.append((self.name, a))
            if self.name == "sla_head_counts":
                kc = ctypes.cast(a[5], ctypes.POINTER(ctypes.c_int))
                kn = ctypes.cast(a[6], ctypes.POINTER(ctypes.c_int))
                for h in range(a[2]):
                    kc[h], kn[h] = 3 + h, 1
                return 3 + a[2] - 1
            return 0

    class FakeLib:
        def __getattr__(self, name):
            return FakeFn(name)

    class FakeStream:
        cuda_stream = 0

    monkeypatch.setattr(S, "_lib", FakeLib())
    q = torch.zeros((1, 2, 256, 64), dtype=torch.bfloat16)
    idx, cm = S.sla_mask_classes(q, q, 64, [0.1, 0.5], 0.25, classes=True, stream=FakeStream())
    assert idx.shape == (1, 2, 4, 4) and cm.shape == (1, 2, 4, 4)
    out = S.sla_attn_classes(q, q, q, torch.zeros((64, 64), dtype=torch.bfloat16), block=64, topk_frac=[0.1, 0.5],
                             skip_frac=[0.25, 0.0], out_dtype=torch.float32, stream=FakeStream())
    assert out.dtype == torch.float32 and out.shape == q.shape
    S.sla_attn_classes_host(q, q, q, q[0, 0, :64], out.bfloat16(), block=64, topk_frac=0.3)
    names = [c[0] for c in calls]
    assert names == ["sla_head_counts", "sla_mask_classes", "sla_attn_classes", "sla_attn_classes_host"]
    fr = ctypes.cast(calls[2][1][13], ctypes.POINTER(ctypes.c_float))
    sk = ctypes.cast(calls[2][1][14], ctypes.POINTER(ctypes.c_float))
    assert [fr[0], fr[1]] == [pytest.approx(0.1), 0.5] and [sk[0], sk[1]] == [0.25, 0.0]
    assert calls[2][1][5] == S.OUT_F32
    assert calls[3][1][11] is None                  # no skip fractions: NULL
    with pytest.raises(ValueError):
        S.sla_attn_classes(q, q, q, q, topk_frac=[0.1, 0.2, 0.3], stream=FakeStream())


def test_w8a8_entry_points_refuse_invalid_arguments_without_a_gpu():
    L = S.lib()
    dummy = 4096
    # shapes: K and N multiples of 16, every dimension >= 1
    assert L.sla_w8a8_linear(dummy, dummy, dummy, None, dummy, 0, 128, 128, 100, None) == 2
    assert L.sla_w8a8_linear(dummy, dummy, dummy, None, dummy, 0, 128, 100, 128, None) == 2
    assert L.sla_w8a8_linear(dummy, dummy, dummy, None, dummy, 0, 0, 128, 128, None) == 1
    assert L.sla_w8a8_gemm(dummy, dummy, dummy, dummy, None, dummy, 0, 128, 128, 0, None) == 1
    assert L.sla_w8a8_quant(dummy, 10, 24, dummy, dummy, None) == 2
    # null and misaligned pointers, bad output type
    assert L.sla_w8a8_linear(None, dummy, dummy, None, dummy, 0, 128, 128, 128, None) == 1
    assert L.sla_w8a8_linear(dummy, dummy, dummy, dummy + 8, dummy, 0, 128, 128, 128, None) == 1
    assert L.sla_w8a8_gemm(dummy, dummy, dummy + 4, dummy, None, dummy, 0, 128, 128, 128, None) == 1
    assert L.sla_w8a8_gemm(dummy, dummy, dummy, dummy, None, dummy, 5, 128, 128, 128, None) == 1
    assert L.sla_w8a8_quant(dummy, 128, 128, None, dummy, None) == 1


def test_binding_marshals_the_w8a8_entry_points(monkeypatch):
    import torch

    calls = []

    class FakeLib:
        def __getattr__(self, name):
            return lambda *a: calls.append((name, a)) or 0

    class FakeStream:
        cuda_stream = 0

    monkeypatch.setattr(S, "_lib", FakeLib())
    x = torch.zeros((300, 256), dtype=torch.bfloat16)
    codes, scales = S.w8a8_quant(x, stream=FakeStream())
    assert codes.shape == (300, 256) and codes.dtype == torch.int8 and scales.shape == (3, 2)
    wq = torch.zeros((512, 256), dtype=torch.int8)
    y = S.w8a8_linear(x, wq, scales, None, out_dtype=torch.float32, stream=FakeStream())
    assert y.shape == (300, 512) and y.dtype == torch.float32
    y = S.w8a8_gemm(codes, scales, wq, scales, stream=FakeStream())
    assert y.shape == (300, 512) and y.dtype == torch.bfloat16
    assert [c[0] for c in calls] == ["sla_w8a8_quant", "sla_w8a8_linear", "sla_w8a8_gemm"]
    assert calls[1][1][5:9] == (S.OUT_F32, 300, 512, 256)
    assert calls[2][1][6:10] == (S.OUT_BF16, 300, 512, 256)


def test_granularity_entry_points_refuse_invalid_arguments_without_a_gpu():
    L = S.lib()
    f = ctypes.c_float
    dummy = 4096
    for bad in (0, 16, 48, 256):
        assert L.sla_attn_gran(dummy, dummy, dummy, dummy, dummy, 0, None, None, 1, 1, 128, 128, 128, f(0.1), bad,
                               None) == 2
        assert L.sla_quant_gran(dummy, dummy, dummy, dummy, dummy, dummy, None, 1, 1, 128, 128, 128, bad, None) == 2
    # a group larger than the block
    assert L.sla_attn_gran(dummy, dummy, dummy, dummy, dummy, 0, None, None, 1, 1, 128, 128, 64, f(0.1), 128,
                           None) == 2
    assert L.sla_attn_gran(dummy, dummy, dummy, dummy, dummy, 3, None, None, 1, 1, 128, 128, 64, f(0.1), 32,
                           None) == 1


def test_product_path_has_no_cpu_fallback(monkeypatch, tmp_path):
    """Without libsla.so the binding raises instead of computing anything, and
    no product source imports, loads or names the CPU oracle."""
    import pathlib

    import int8_block_sparse_b200 as S

    monkeypatch.setattr(S, "_lib", None)
    monkeypatch.setattr(S, "LIB_PATH", str(tmp_path / "missing" / "libsla.so"))
    with pytest.raises(ImportError, match="missing"):
        S.lib()
    with pytest.raises(ImportError):
        S.topk_count(1024, 128, 0.1)
    root = pathlib.Path(S.__file__).parent
    for f in list(root.rglob("*.py")) + list(root.rglob("*.cu")) + list(root.rglob("*.cuh")) + \
            list((root.parent / "include").glob("*.h")):
        text = f.read_text()
        assert "oracle" not in text, f
