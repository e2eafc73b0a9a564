"""CUDA path vs the CPU oracle, element by element, through the C interface.

The oracle here is the plain C++ one (oracle/sla_oracle.cpp, through
oracle/cpp_oracle.py), pinned by tests/test_oracle_pins.py together with the
numpy statement it restates.

Integer work (INT8 codes, scales, the channel mean, the block lists) must be
bit-exact; a block list may differ only on a row the oracle marks as a near
tie, and then the oracle is re-run with the GPU's list for that row.  The
float32 output must be within max-abs 2e-2, mean-abs 2e-3 and cosine 0.9999
of the oracle's float64 output.
"""

import json

import numpy as np
import pytest

from oracle import cpp_oracle as O
from oracle import sla_oracle as NP
from synth import CONFIGS, make_inputs, make_workload
from tests.parity import (MAX_ABS, MEAN_ABS, MIN_COS, assert_out_ok, compare_out, mask_mismatch,
                          mask_record, sample_items, to_dev)

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


def run_quant(S, x, block, gran=None):
    q, k = to_dev(x["q"]), to_dev(x["k"])
    qi8, ki8, sq, sk, mu = S.sla_quant(q, k, block, gran=gran)
    assert S.get_error() == 0
    return {"q_i8": qi8.cpu().numpy(), "k_i8": ki8.cpu().numpy(), "q_scale": sq.cpu().numpy(),
            "k_scale": sk.cpu().numpy(), "mu": mu.cpu().numpy()}


def check_quant(got, ref):
    for key in ("mu", "q_scale", "k_scale"):
        assert np.array_equal(got[key].view(np.uint32), ref[key].view(np.uint32)), key
    for key in ("q_i8", "k_i8"):
        assert np.array_equal(got[key], ref[key]), (key, int(np.sum(got[key] != ref[key])))


def run_attn(S, x, block, frac, gran=None):
    """The operator through the C interface: float32 out with both parts
    (sla_attn_ex), the default bf16 out (sla_attn) and the block lists."""
    import torch

    q, k, v, w = (to_dev(x[t]) for t in ("q", "k", "v", "proj"))
    B, H, N, d = x["q"].shape

    def f32():
        return torch.full((B, H, N, d), float("nan"), dtype=torch.float32, device="cuda")

    out, osp, olin = f32(), f32(), f32()
    S.sla_attn(q, k, v, w, block=block, topk_frac=frac, out=out, o_sparse=osp, o_lin=olin, gran=gran)
    ob = S.sla_attn(q, k, v, w, block=block, topk_frac=frac, gran=gran)
    assert ob.dtype == torch.bfloat16
    idx = S.sla_mask(q, k, block, frac)
    assert S.get_error() == 0
    got = {"out": out, "o_sparse": osp, "o_lin": olin, "out_bf16": ob.float()}
    return {key: t.cpu().numpy().astype(np.float64) for key, t in got.items()}, idx.cpu().numpy()


def check_attn(x, block, frac, items=None, case="?", gran=None):
    """Full comparison (items None) or on sampled query blocks.

    Returns (out stats, o_sparse stats, mask record).  The mask record counts
    the query rows the oracle marks as near ties and the rows whose GPU list
    differs from the oracle's; every differing row must be a near tie, and
    near ties must stay rare (at most 1% of the rows), else the bit-exact
    mask comparison would mean little.  The float32 output and its two parts
    (O_sparse; O_lin . W_proj) are held to the output tolerance against the
    oracle's float64 values; the bf16 output must be the float32 output rounded
    to bf16, and within the tolerance of the oracle's rounded output (see
    check_bf16)."""
    import int8_block_sparse_b200 as S

    got, gidx = run_attn(S, x, block, frac, gran)
    B, H, N, d = x["q"].shape
    ref_mask = O.block_mask(x["q"], x["k"], block, frac)
    diff, bad = mask_mismatch(gidx, ref_mask["idx"], ref_mask["near_tie"])
    rec = mask_record(case, ref_mask["near_tie"], diff, bad)
    print(json.dumps(rec))
    assert not bad.any(), f"{int(bad.sum())} block lists differ off near ties"
    assert rec["near_tie_rows"] <= 0.01 * rec["rows"], rec
    override = {tuple(int(t) for t in ix): gidx[tuple(ix)] for ix in np.argwhere(diff)}
    res = O.sla_attention(x["q"], x["k"], x["v"], x["proj"], block, frac, items=items,
                          idx_override=override or None, gran=gran)
    w64 = O.bf16_to_f64(x["proj"])
    parts = {"out": [], "o_sparse": [], "o_lin": [], "out_bf16": []}
    refs = {"out": [], "o_sparse": [], "o_lin": []}
    for (b, h, i), o in res["out"].items():
        lo, hi = i * block, min(N, (i + 1) * block)
        for key in parts:
            parts[key].append(got[key][b, h, lo:hi])
        refs["out"].append(o)
        refs["o_sparse"].append(res["o_sparse"][(b, h, i)])
        refs["o_lin"].append(res["o_lin"][(b, h, i)] @ w64)
    cat = {key: np.concatenate(v) for key, v in parts.items()}
    ref = {key: np.concatenate(v) for key, v in refs.items()}
    st = compare_out(cat["out"], ref["out"])
    st_sp = compare_out(cat["o_sparse"], ref["o_sparse"])
    st_lin = compare_out(cat["o_lin"], ref["o_lin"]) if np.any(ref["o_lin"]) else None
    assert_out_ok(st_sp, "o_sparse")
    if st_lin is not None:
        assert_out_ok(st_lin, "o_lin")
    else:
        assert not np.any(cat["o_lin"]), "no linear part, yet o_lin is not zero"
    assert_out_ok(st, "out")
    st_b = check_bf16(cat["out_bf16"], cat["out"], ref["out"])
    print(json.dumps({"case": case, "out": st, "o_sparse": st_sp, "o_lin": st_lin, "out_bf16": st_b}))
    return st, st_sp, rec


def check_bf16(got_b, got_f32, ref):
    """The bf16 output: exactly the float32 result of the same operator rounded
    to bf16 (round to nearest even; both outputs come from the same kernel,
    which differs only in the store), and close to the oracle's float64 output
    rounded to bf16 the same way: mean-abs and cosine within the output
    tolerance, and per element within the max-abs tolerance or one bf16 step
    of the rounded value, whichever is larger (where the float32 error
    straddles a rounding boundary the two roundings land one step apart, and a
    step is 2^-5 already at |out| >= 4)."""
    assert np.array_equal(got_b, O.round_bf16(got_f32)), "bf16 out is not the rounded float32 out"
    ref_b = O.round_bf16(ref)
    st = compare_out(got_b, ref_b)
    assert st["mean_abs"] <= MEAN_ABS and st["cos"] >= MIN_COS, ("out_bf16", st)
    mag = np.maximum(np.abs(ref_b), 2.0 ** -126)
    step = np.exp2(np.floor(np.log2(mag)) - 7)
    assert np.all(np.abs(got_b - ref_b) <= np.maximum(MAX_ABS, step)), ("out_bf16", st)
    st["equal_to_rounded_oracle"] = float(np.mean(got_b == ref_b))
    return st


# ---------------------------------------------------------------- small cases

SMALL = [
    # (B, H, N, d, block, frac, dist, seed)
    (1, 2, 1024, 64, 64, 0.25, "iid", 0),        # the tiny configuration
    (1, 1, 1000, 128, 128, 0.25, "iid", 11),     # ragged tail (1000 = 7*128 + 104)
    (2, 3, 640, 128, 128, 0.4, "iid", 12),       # several heads, B > 1
    (1, 2, 129, 128, 128, 0.5, "iid", 13),       # last block has one row
    (1, 1, 1, 128, 128, 0.1, "iid", 14),         # a single token
    (1, 2, 777, 64, 128, 0.3, "iid", 15),        # d = 64 with 128-token blocks
    (1, 2, 700, 128, 64, 0.2, "iid", 16),        # 64-token blocks with d = 128
    (1, 2, 2048, 128, 128, 1.0, "iid", 17),      # every block kept: no linear branch
    (1, 2, 4096, 128, 128, 0.1, "field", 18),    # field inputs, many blocks
]


@pytest.mark.parametrize("B,H,N,d,block,frac,dist,seed", SMALL)
def test_quant_bitexact_small(S, B, H, N, d, block, frac, dist, seed):
    grid = (4, 32, 32) if dist == "field" else None
    x = make_inputs(B, H, N, d, seed, dist, grid)
    check_quant(run_quant(S, x, block), O.quantize(x["q"], x["k"], block))


@pytest.mark.parametrize("B,H,N,d,block,frac,dist,seed", SMALL)
def test_attention_small(S, B, H, N, d, block, frac, dist, seed):
    grid = (4, 32, 32) if dist == "field" else None
    x = make_inputs(B, H, N, d, seed, dist, grid)
    check_attn(x, block, frac, case=f"small-{seed}")


def test_mask_bitmap_and_list_agree(S):
    x = make_inputs(1, 2, 1500, 128, 3)
    q, k = to_dev(x["q"]), to_dev(x["k"])
    idx, bm = S.sla_mask(q, k, 128, 0.3, bitmap=True)
    idx, bm = idx.cpu().numpy(), bm.cpu().numpy()
    assert np.array_equal(bm, O.bitmap_of(idx, bm.shape[-1]))
    assert np.all(np.diff(idx, axis=-1) > 0)


def test_mask_exact_ties_go_to_the_lower_block(S):
    """Seven identical key blocks share the top score of every query row and
    kc = 4: the kept list must be the four lowest of them, exactly as the
    oracle's tie rule says (exact ties are not exempt here)."""
    from synth.workloads import f32_to_bf16_bits

    B, H, N, d, block, frac = 1, 1, 1024, 64, 64, 0.25   # nblk 16, kc 4
    rng = np.random.default_rng(21)
    k = rng.standard_normal((B, H, N, d)).astype(np.float32)
    q = rng.standard_normal((B, H, N, d)).astype(np.float32) * 0.1
    k[..., 64:128, 0] += 6.0                 # key block 1: large channel-0 mean
    for j in (3, 5, 7, 9, 11, 13):           # six exact copies of key block 1
        k[..., j * 64:(j + 1) * 64, :] = k[..., 64:128, :]
    q[..., 0] += 1.0                          # every query block prefers channel 0
    qb, kb = f32_to_bf16_bits(q), f32_to_bf16_bits(k)
    ref = O.block_mask(qb, kb, block, frac)
    assert ref["kc"] == 4
    assert np.all(ref["idx"] == np.array([1, 3, 5, 7], dtype=ref["idx"].dtype))
    idx = S.sla_mask(to_dev(qb), to_dev(kb), block, frac).cpu().numpy()
    assert S.get_error() == 0
    assert np.array_equal(idx, ref["idx"])


def test_host_buffers_match_device_path(S):
    import torch

    x = make_inputs(1, 2, 900, 128, 4)
    dev = [to_dev(x[t]) for t in ("q", "k", "v", "proj")]
    out_dev = S.sla_attn(*dev, block=128, topk_frac=0.25)
    host = [t.cpu().pin_memory() for t in dev]
    out_host = torch.empty(host[0].shape, dtype=torch.bfloat16).pin_memory()
    S.sla_attn_host(*host, out_host, block=128, topk_frac=0.25)
    assert torch.equal(out_host, out_dev.cpu())


def test_call_captured_in_a_cuda_graph_matches_eager(S):
    """The operator's two-stream sequence can be captured in a CUDA graph (the
    second stream joins the capture through its events) and replayed."""
    import torch

    x = make_inputs(1, 2, 1500, 128, 7)
    dev = [to_dev(x[t]) for t in ("q", "k", "v", "proj")]
    eager = S.sla_attn(*dev, block=128, topk_frac=0.2)
    out = torch.empty_like(eager)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):            # warm-up outside the capture
        S.sla_attn(*dev, block=128, topk_frac=0.2, out=out, stream=side)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        S.sla_attn(*dev, block=128, topk_frac=0.2, out=out)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert S.get_error() == 0
    assert torch.equal(out, eager)


def test_repeated_calls_are_deterministic(S):
    import torch

    x = make_inputs(1, 3, 2000, 128, 5, "field", (2, 25, 40))
    dev = [to_dev(x[t]) for t in ("q", "k", "v", "proj")]
    a = S.sla_attn(*dev, block=128, topk_frac=0.2)
    b = S.sla_attn(*dev, block=128, topk_frac=0.2)
    assert torch.equal(a, b)


# ---------------------------------------------------------------- finer quantisation groups

GRAN_CASES = [
    # (B, H, N, d, block, frac, gran, dist, seed)
    (1, 2, 1000, 128, 128, 0.25, 32, "iid", 41),    # ragged tail: a partial group and one wholly past N
    (1, 2, 777, 64, 128, 0.3, 32, "iid", 42),       # d = 64
    (1, 2, 700, 128, 64, 0.2, 32, "iid", 43),       # 64-token blocks, two groups each
    (1, 2, 2048, 128, 128, 0.2, 64, "field", 44),   # 64-token groups
    (2, 2, 640, 128, 128, 1.0, 32, "iid", 45),      # every block kept
]


@pytest.mark.parametrize("B,H,N,d,block,frac,gran,dist,seed", GRAN_CASES)
def test_quant_and_attention_with_finer_groups(S, B, H, N, d, block, frac, gran, dist, seed):
    grid = (N // 1024, 32, 32) if dist == "field" else None
    x = make_inputs(B, H, N, d, seed, dist, grid)
    check_quant(run_quant(S, x, block, gran), O.quantize(x["q"], x["k"], block, gran))
    check_attn(x, block, frac, case=f"gran{gran}-{seed}", gran=gran)


def test_finer_groups_lossless_inputs(S):
    """Rows scaled by a different power of two per 32 tokens: with 32-token
    groups the GPU codes are the integers and its output matches the oracle's."""
    from synth.workloads import f32_to_bf16_bits

    rng = np.random.default_rng(46)
    N, d, block, gran = 512, 128, 128, 32
    qi = rng.integers(-127, 128, size=(1, 1, N, d)).astype(np.float32)
    ki = rng.integers(-127, 128, size=(1, 1, N, d)).astype(np.float32)
    pw = np.repeat(2.0 ** -(4 + np.arange(N // gran) % 6), gran).astype(np.float32)
    x = {"q": f32_to_bf16_bits(qi * pw[None, None, :, None]), "k": f32_to_bf16_bits(ki * pw[None, None, :, None]),
         "v": f32_to_bf16_bits(rng.standard_normal((1, 1, N, d)).astype(np.float32)),
         "proj": f32_to_bf16_bits((rng.standard_normal((d, d)) / np.sqrt(d)).astype(np.float32))}
    check_quant(run_quant(S, x, block, gran), O.quantize(x["q"], x["k"], block, gran))
    check_attn(x, block, 0.5, case="gran32-lossless", gran=gran)


# ---------------------------------------------------------------- three classes, per-head fractions

def run_attn_classes(S, x, block, fr, sk):
    import torch

    q, k, v, w = (to_dev(x[t]) for t in ("q", "k", "v", "proj"))
    B, H, N, d = x["q"].shape

    def f32():
        return torch.full((B, H, N, d), float("nan"), dtype=torch.float32, device="cuda")

    out, osp, olin = f32(), f32(), f32()
    S.sla_attn_classes(q, k, v, w, block=block, topk_frac=fr, skip_frac=sk, out=out, o_sparse=osp, o_lin=olin)
    ob = S.sla_attn_classes(q, k, v, w, block=block, topk_frac=fr, skip_frac=sk)
    idx, cls = S.sla_mask_classes(q, k, block, fr, sk, classes=True)
    assert S.get_error() == 0
    got = {"out": out, "o_sparse": osp, "o_lin": olin, "out_bf16": ob.float()}
    return ({key: t.cpu().numpy().astype(np.float64) for key, t in got.items()}, idx.cpu().numpy(),
            cls.cpu().numpy())


def check_attn_classes(x, block, fr, sk, items=None, case="?"):
    """check_attn for the three-class mask with per-head fractions: the class
    map and the padded block lists bit-exact off near-tie rows (a differing
    row is re-run in the oracle with the GPU's classes), the outputs as in
    check_attn."""
    import int8_block_sparse_b200 as S

    got, gidx, gcls = run_attn_classes(S, x, block, fr, sk)
    B, H, N, d = x["q"].shape
    ref_mask = O.block_mask_classes(x["q"], x["k"], block, fr, sk)
    diff = np.any(gcls != ref_mask["cls"], axis=-1)
    bad = diff & ~ref_mask["near_tie"]
    rec = mask_record(case, ref_mask["near_tie"], diff, bad)
    print(json.dumps(rec))
    assert not bad.any(), f"{int(bad.sum())} class rows differ off near ties"
    assert rec["near_tie_rows"] <= 0.01 * rec["rows"], rec
    assert np.array_equal(gidx[~diff], ref_mask["idx"][~diff])
    for b in range(B):                      # the lists are the kept classes, ascending, then -1
        for h in range(H):
            kc = int(ref_mask["kc"][h])
            assert (gidx[b, h, :, kc:] == -1).all()
            kept = np.argwhere(gcls[b, h] == 2)
            assert np.array_equal(gidx[b, h, :, :kc].reshape(-1), kept[:, 1])
    override = {tuple(int(t) for t in ix): gcls[tuple(ix)] for ix in np.argwhere(diff)}
    res = O.sla_attention(x["q"], x["k"], x["v"], x["proj"], block, fr, skip_frac=sk, items=items,
                          idx_override=override or None)
    w64 = O.bf16_to_f64(x["proj"])
    parts = {"out": [], "o_sparse": [], "o_lin": [], "out_bf16": []}
    refs = {"out": [], "o_sparse": [], "o_lin": []}
    for (b, h, i), o in res["out"].items():
        lo, hi = i * block, min(N, (i + 1) * block)
        for key in parts:
            parts[key].append(got[key][b, h, lo:hi])
        refs["out"].append(o)
        refs["o_sparse"].append(res["o_sparse"][(b, h, i)])
        refs["o_lin"].append(res["o_lin"][(b, h, i)] @ w64)
    cat = {key: np.concatenate(v) for key, v in parts.items()}
    ref = {key: np.concatenate(v) for key, v in refs.items()}
    st = compare_out(cat["out"], ref["out"])
    st_sp = compare_out(cat["o_sparse"], ref["o_sparse"])
    assert_out_ok(st_sp, "o_sparse")
    # rows without a linear part must have exactly zero O_lin
    zero_rows = ~np.any(ref["o_lin"], axis=-1)
    assert not np.any(cat["o_lin"][zero_rows])
    st_lin = compare_out(cat["o_lin"], ref["o_lin"]) if np.any(ref["o_lin"]) else None
    if st_lin is not None:
        assert_out_ok(st_lin, "o_lin")
    assert_out_ok(st, "out")
    st_b = check_bf16(cat["out_bf16"], cat["out"], ref["out"])
    print(json.dumps({"case": case, "out": st, "o_sparse": st_sp, "o_lin": st_lin, "out_bf16": st_b}))
    return st, st_sp, rec


CLASS_CASES = [
    # (B, H, N, d, block, topk_frac per head, skip_frac per head or None, dist, seed)
    (1, 3, 1000, 64, 64, [0.1, 0.3, 0.5], [0.5, 0.2, 0.0], "iid", 31),
    (2, 3, 777, 128, 128, [0.25, 1.0, 0.05], [0.7, 0.0, 0.9], "iid", 32),   # a dense head; ragged tail
    (1, 4, 4096, 128, 128, [0.05, 0.1, 0.15, 0.2], [0.5] * 4, "field", 33),
    (1, 2, 2048, 128, 64, [0.1, 0.2], None, "iid", 34),                    # per-head fractions only
    (1, 2, 1024, 128, 128, [0.25, 0.5], [0.75, 0.5], "iid", 35),            # no linear block at all
]


@pytest.mark.parametrize("B,H,N,d,block,fr,sk,dist,seed", CLASS_CASES)
def test_attention_classes_small(S, B, H, N, d, block, fr, sk, dist, seed):
    grid = (4, 32, 32) if dist == "field" else None
    x = make_inputs(B, H, N, d, seed, dist, grid)
    check_attn_classes(x, block, fr, sk, case=f"classes-{seed}")


def test_classes_host_buffers_match_device_path(S):
    import torch

    x = make_inputs(2, 3, 900, 128, 37)
    fr, sk = [0.1, 0.25, 0.5], [0.5, 0.0, 0.25]
    dev = [to_dev(x[t]) for t in ("q", "k", "v", "proj")]
    out_dev = S.sla_attn_classes(*dev, block=128, topk_frac=fr, skip_frac=sk)
    host = [t.cpu().pin_memory() for t in dev]
    out_host = torch.empty(host[0].shape, dtype=torch.bfloat16).pin_memory()
    S.sla_attn_classes_host(*host, out_host, block=128, topk_frac=fr, skip_frac=sk)
    assert torch.equal(out_host, out_dev.cpu())


def test_classes_with_uniform_fractions_equal_the_two_class_operator(S):
    import torch

    x = make_inputs(1, 3, 1500, 128, 36)
    dev = [to_dev(x[t]) for t in ("q", "k", "v", "proj")]
    a = S.sla_attn(*dev, block=128, topk_frac=0.2)
    b = S.sla_attn_classes(*dev, block=128, topk_frac=[0.2] * 3, skip_frac=[0.0] * 3)
    assert torch.equal(a, b)
    ia = S.sla_mask(dev[0], dev[1], 128, 0.2)
    ib = S.sla_mask_classes(dev[0], dev[1], 128, 0.2)
    assert torch.equal(ia, ib)


# ---------------------------------------------------------------- full-size configurations

def _full_case(S, name, per_head):
    w = CONFIGS[name]
    x = make_workload(w)
    check_quant(run_quant(S, x, w.block, w.gran), O.quantize(x["q"], x["k"], w.block, w.gran))
    items = sample_items(w.B, w.H, w.nblk, per_head=per_head, seed=w.seed)
    if w.classes:
        st, st_sp, rec = check_attn_classes(x, w.block, w.fracs, w.skip_frac, items=items, case=name)
    else:
        st, st_sp, rec = check_attn(x, w.block, w.topk_frac, items=items, case=name, gran=w.gran)
    print(json.dumps({"case": name, "out": st, "o_sparse": st_sp}))


def test_full_tiny(S):
    _full_case(S, "tiny", per_head=16)


def test_full_480p(S):
    _full_case(S, "480p", per_head=4)


def test_full_dense(S):
    _full_case(S, "dense", per_head=2)


@pytest.mark.parametrize("name", ["sweep0.05", "sweep0.10", "sweep0.20", "sweep0.40"])
def test_full_sweep(S, name):
    _full_case(S, name, per_head=2)


def test_full_720p(S):
    _full_case(S, "720p", per_head=2)


def test_full_480p_classes(S):
    _full_case(S, "480p_classes", per_head=4)


def test_full_480p_gran32(S):
    _full_case(S, "480p_gran32", per_head=4)


def _wide_exponent_inputs(N, d, seed):
    """K whose channels span more exponents than a float64 sum holds exactly:
    the channel mean must still be the exact mean rounded once to float32."""
    from synth.workloads import f32_to_bf16_bits

    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, 1, N, d)).astype(np.float32)
    k = rng.standard_normal((1, 1, N, d)).astype(np.float32) + 3.0
    # channel 0: 2^100, 1, -2^100 among zeros (exact sum 1)
    k[..., :, 0] = 0.0
    k[..., 5, 0], k[..., N // 2, 0], k[..., N - 1, 0] = 2.0 ** 100, 1.0, -(2.0 ** 100)
    # channel 1: magnitudes near 8 and near 2^-30, random signs
    mag = np.where(rng.random(N) < 0.5, 8.0, 2.0 ** -30) * rng.uniform(1.0, 2.0, N)
    k[0, 0, :, 1] = mag * rng.choice([-1.0, 1.0], N)
    # channel 2: near the largest bf16 value, alternating signs, and tiny values
    k[0, 0, :, 2] = np.where(np.arange(N) % 3 == 0, 1e-30, 3.0e38) * np.where(np.arange(N) % 2, -1.0, 1.0)
    kb = f32_to_bf16_bits(k)
    # channel 3: bf16 subnormals (raw patterns) with a few values of 1
    sub = rng.integers(1, 128, N).astype(np.uint16) | (rng.integers(0, 2, N).astype(np.uint16) << 15)
    sub[:: max(1, N // 7)] = 0x3F80
    kb[0, 0, :, 3] = sub
    # channel 4: every value is -0.0
    kb[0, 0, :, 4] = 0x8000
    return f32_to_bf16_bits(q), kb


@pytest.mark.parametrize("N,d,block", [(32768, 128, 128), (1000, 64, 64), (777, 128, 128)])
def test_channel_mean_exact_for_wide_exponent_spans(S, N, d, block):
    qb, kb = _wide_exponent_inputs(N, d, seed=N)
    got = run_quant(S, {"q": qb, "k": kb}, block)
    ref = O.quantize(qb, kb, block)
    check_quant(got, ref)
    # channel 0 sums to exactly 1, so its mean is 1/N rounded once
    assert got["mu"][0, 0, 0] == np.float32(NP.round_rational_to_f32(1, N))


def test_bounded_wait_reports_timeout_and_context_survives(S):
    """A kernel whose barrier is never completed gives up after its bounded wait,
    records SLA_ERR_TIMEOUT and returns; the context stays usable."""
    import ctypes

    import torch

    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert S.lib().sla_selftest_wait_timeout(st) == 0
    assert S.get_error() == 5
    assert S.get_error() == 0            # the error word was cleared
    x = make_inputs(1, 1, 256, 128, 6)
    check_attn(x, 128, 0.5, case="after-timeout")   # the device still computes correctly
