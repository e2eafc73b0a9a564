"""The allocation-free block-mask entry point, sla_mask_noalloc.

Some callers cannot allocate device memory while they run (a server that
plans all device memory at start-up, or a host whose allocator belongs to
another framework).  sla_mask_noalloc serves them from a fixed 16 MiB device
buffer inside the library.  This test calls it through the C interface and
checks that it returns exactly the block lists and bitmap of sla_mask (index
work: bit-exact), on two calls in a row with different inputs, so that a
second call over the buffer's stale contents is covered too.  It also checks
that a problem too large for the buffer is refused before any work.

The file is named to be collected last, so that a run stopping at the first
failure has already run every other test.
"""

import ctypes

import numpy as np
import pytest

from synth import make_inputs

pytestmark = pytest.mark.gpu


def _dev(bits):
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _noalloc(S, q, k, block, frac):
    import torch

    B, H, N, d = q.shape
    nb = (N + block - 1) // block
    kc = S.topk_count(N, block, frac)
    idx = torch.full((B, H, nb, kc), -1, dtype=torch.int32, device="cuda")
    bm = torch.full((B, H, nb, nb), 7, dtype=torch.uint8, device="cuda")
    rc = S.lib().sla_mask_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                  ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(bm.data_ptr()),
                                  B, H, N, d, block, ctypes.c_float(frac),
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, S.status_string(rc)
    assert S.get_error() == 0
    return idx.cpu().numpy(), bm.cpu().numpy()


def test_noalloc_mask_matches_sla_mask_on_two_calls():
    import torch

    assert torch.cuda.is_available()
    import int8_block_sparse_b200 as S
    from int8_block_sparse_b200.build import build

    build()
    cases = [
        (make_inputs(1, 12, 32768, 128, 1, "field", (21, 30, 52), heads=[0, 1, 2, 3]), 128, 0.1),
        (make_inputs(2, 3, 1000, 64, 7), 64, 0.25),
    ]
    for x, block, frac in cases:
        q, k = _dev(x["q"]), _dev(x["k"])
        ref_idx, ref_bm = S.sla_mask(q, k, block, frac, bitmap=True)
        got_idx, got_bm = _noalloc(S, q, k, block, frac)
        assert np.array_equal(got_idx, ref_idx.cpu().numpy())
        assert np.array_equal(got_bm, ref_bm.cpu().numpy())


def test_noalloc_mask_leaves_device_memory_untouched():
    """After the first call on the device (its set-up), a call with another
    shape changes neither the device's free memory nor the library's pool."""
    import torch

    import int8_block_sparse_b200 as S
    from int8_block_sparse_b200.build import build

    build()
    x1 = make_inputs(1, 2, 1500, 128, 8)
    x2 = make_inputs(2, 2, 700, 64, 9)
    q1, k1 = _dev(x1["q"]), _dev(x1["k"])
    q2, k2 = _dev(x2["q"]), _dev(x2["k"])
    _noalloc(S, q1, k1, 128, 0.2)                     # set-up call
    idx = torch.empty((2, 2, 11, S.topk_count(700, 64, 0.3)), dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    rc = S.lib().sla_mask_noalloc(ctypes.c_void_p(q2.data_ptr()), ctypes.c_void_p(k2.data_ptr()),
                                  ctypes.c_void_p(idx.data_ptr()), None, 2, 2, 700, 64, 64, ctypes.c_float(0.3),
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert S.get_error() == 0
    ref = S.sla_mask(q2, k2, 64, 0.3).cpu().numpy()
    assert np.array_equal(idx.cpu().numpy(), ref)


def test_noalloc_mask_refuses_problems_beyond_its_buffer():
    import int8_block_sparse_b200 as S

    # the 720P shape (B*H = 40, nblk = 591) needs more than the buffer holds;
    # the call is refused before anything is enqueued, so the (aligned,
    # never dereferenced) dummy pointers are not touched
    rc = S.lib().sla_mask_noalloc(16, 16, 16, None, 1, 40, 75600, 128, 128, ctypes.c_float(0.1), None)
    assert rc == 7 and S.status_string(rc).startswith("problem larger")
