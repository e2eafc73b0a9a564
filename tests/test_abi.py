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
