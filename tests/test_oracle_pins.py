"""Pins of the CPU oracle against things other than itself.

Each test checks one oracle function against a closed form, a library
routine, a brute force or a hand-derived case (tests/golden/), chosen so that
a dropped term, a wrong sign or index, or a transposed operand fails one of
them.  Tests taking the `impl` fixture run against both oracles, the numpy
statement (oracle/sla_oracle.py) and the plain C++ one (oracle/sla_oracle.cpp);
the rest pin helpers only the numpy statement has.  No GPU needed.
"""

import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import torch

import oracle as O
from oracle import cpp_oracle as C
from synth import make_inputs
from synth.workloads import f32_to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

IMPLS = {"numpy": O, "cpp": C}


@pytest.fixture(params=sorted(IMPLS))
def impl(request):
    """The oracle under test: the numpy statement or the plain C++ one."""
    return IMPLS[request.param]


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def bits(x):
    """float values that bf16 holds exactly -> bf16 bits (asserts exactness)."""
    x32 = np.asarray(x, dtype=np.float32)
    b = f32_to_bf16_bits(x32)
    assert np.array_equal(O.bf16_to_f32(b), x32), "test value not representable in bf16"
    return b


# --- number formats --------------------------------------------------------

def test_round_bf16_special_values(impl):
    e = 2.0 ** -8
    cases = {
        1.0: 1.0,
        1.0 + e: 1.0,                     # tie, even neighbour is 1.0
        1.0 + 3 * e: 1.0 + 4 * e,         # tie, even neighbour is 1 + 2**-6
        -(1.0 + e): -1.0,
        1.0 + 1.5 * e: 1.0 + 2 * e,       # above the tie
        2.0 ** -130: 2.0 ** -130,         # bf16 subnormal, exact
        3 * 2.0 ** -135: 2.0 ** -133,     # 0.75 of the subnormal spacing
        0.0: 0.0,
    }
    for x, y in cases.items():
        assert impl.round_bf16(np.array([x]))[0] == y, x


def test_round_bf16_matches_torch_on_float32_inputs(impl):
    rng = np.random.default_rng(5)
    x = (rng.standard_normal(200000) * np.exp(rng.uniform(-20, 20, 200000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(impl.round_bf16(x.astype(np.float64)), ref)


def _nearest_f32_bruteforce(fr: Fraction) -> float:
    f = np.float32(float(fr))
    best = None
    for c in (np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))):
        err = abs(Fraction(float(c)) - fr)
        key = (err, int(np.array(c, dtype=np.float32).view(np.uint32)) & 1)
        if best is None or key < best[0]:
            best = (key, float(c))
    return best[1]


def test_round_rational_to_f32_bruteforce():
    rng = np.random.default_rng(7)
    for _ in range(3000):
        num = int(rng.integers(-2**62, 2**62)) * (1 << int(rng.integers(0, 40)))
        den = int(rng.integers(1, 2**40))
        assert O.round_rational_to_f32(num, den) == _nearest_f32_bruteforce(Fraction(num, den))
    # exact ties between two float32 values: (1 + 2**-24) is halfway between 1 and 1 + 2**-23
    assert O.round_rational_to_f32((1 << 24) + 1, 1 << 24) == 1.0
    assert O.round_rational_to_f32((1 << 24) + 3, 1 << 24) == 1.0 + 2.0 ** -22


# --- smoothing -------------------------------------------------------------

def test_channel_mean_is_exact_where_float64_summation_is_not(impl):
    # per channel: 2**100, 1, -2**100  -> exact sum 1; a float64 running sum gives 0
    k = np.zeros((1, 1, 3, 2), dtype=np.float32)
    k[0, 0, :, 0] = [2.0 ** 100, 1.0, -(2.0 ** 100)]
    k[0, 0, :, 1] = [3.0, -1.0, 2.0 ** -60]
    mu = impl.channel_mean(bits(k))
    assert mu[0, 0, 0] == np.float32(1.0 / 3.0)
    assert mu[0, 0, 1] == _nearest_f32_bruteforce((Fraction(2) + Fraction(2) ** -60) / 3)


def test_channel_mean_matches_exact_rationals(impl):
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((2, 1, 37, 3)) * np.exp(rng.uniform(-30, 30, (2, 1, 37, 3)))).astype(np.float32)
    b = f32_to_bf16_bits(x)
    vals = O.bf16_to_f64(b)
    mu = impl.channel_mean(b)
    for i in range(2):
        for c in range(3):
            ex = sum(Fraction(float(t)) for t in vals[i, 0, :, c]) / 37
            assert mu[i, 0, c] == _nearest_f32_bruteforce(ex)


# --- quantisation ----------------------------------------------------------

def test_quant_ties_golden(impl):
    g = golden("quant_ties.json")
    x = np.array(g["x"], dtype=np.float32).reshape(1, 1, -1, 1)
    codes, scales = impl.quantize_blocks(x, g["block"])
    assert scales[0, 0, 0] == g["scale"]
    assert codes[0, 0, :, 0].tolist() == g["codes"]


def test_quant_round_trip_of_representable_blocks(impl):
    rng = np.random.default_rng(3)
    block, d, nblk = 16, 8, 5
    m = rng.integers(-127, 128, size=(1, 1, nblk * block, d))
    for r in range(nblk):           # force max |m| = 127 in every block
        m[0, 0, r * block, 0] = 127 if r % 2 else -127
    s = 2.0 ** -np.arange(3, 3 + nblk)
    x = (m * np.repeat(s, block)[None, None, :, None]).astype(np.float32)
    codes, scales = impl.quantize_blocks(x, block)
    assert np.array_equal(codes.astype(np.int64), m)
    assert np.array_equal(scales[0, 0], s.astype(np.float32))


def test_quant_zero_block_partial_block_and_padding(impl):
    x = np.zeros((1, 1, 10, 4), dtype=np.float32)
    x[0, 0, 8:10] = [[1, -2, 3, 0.5], [0, 0, -3, 1]]
    codes, scales = impl.quantize_blocks(x, 4)            # blocks [0,4) [4,8) zero, [8,10) partial
    assert codes.shape == (1, 1, 12, 4)
    assert scales[0, 0].tolist() == [0.0, 0.0, np.float32(3.0) / np.float32(127.0)]
    assert not codes[0, 0, :8].any() and not codes[0, 0, 10:].any()
    assert codes[0, 0, 8].tolist() == [42, -85, 127, 21]     # x/s = 42.33, -84.67, 127, 21.17


# --- mask ------------------------------------------------------------------

def test_topk_counts_golden(impl):
    for c in golden("topk_counts.json")["cases"]:
        assert impl.topk_count(c["nblk"], c["frac"]) == c["kc"], c
    with pytest.raises(ValueError):
        impl.topk_count(10, 0.0)
    with pytest.raises(ValueError):
        impl.topk_count(10, 1.5)


def test_select_topk_bruteforce_over_all_subsets(impl):
    rng = np.random.default_rng(2)
    for trial in range(300):
        n = int(rng.integers(1, 9))
        kc = int(rng.integers(1, n + 1))
        p = rng.integers(0, 4, size=n).astype(np.float64)   # many exact ties
        idx, _ = impl.select_topk(p[None, :], kc)
        winners = []
        for sub in itertools.combinations(range(n), kc):
            rest = [j for j in range(n) if j not in sub]
            if all(p[a] > p[b] or (p[a] == p[b] and a < b) for a in sub for b in rest):
                winners.append(list(sub))
        assert len(winners) == 1
        assert idx[0].tolist() == winners[0]


def test_near_tie_flag(impl):
    p = np.array([[0.5, 0.3, 0.3 * (1 - 1e-12), 0.1], [0.5, 0.3, 0.29, 0.1]])
    _, tie = impl.select_topk(p, 2)
    assert tie.tolist() == [True, False]


def test_block_means_closed_form_with_partial_block(impl):
    N, block, d = 10, 4, 3
    x = np.zeros((1, 1, N, d), dtype=np.float32)
    for n in range(N):
        x[0, 0, n] = [n, -2 * n, 1.0]
    means = impl.block_means(bits(x), block)
    assert means[0, 0].tolist() == [[1.5, -3.0, 1.0], [5.5, -11.0, 1.0], [8.5, -17.0, 1.0]]


def test_block_probs_matches_scipy_softmax(impl):
    rng = np.random.default_rng(4)
    qb, kb = rng.standard_normal((2, 3, 7, 16)), rng.standard_normal((2, 3, 7, 16))
    ref = scipy.special.softmax(np.einsum("bhic,bhjc->bhij", qb, kb) / 4.0, axis=-1)
    assert np.allclose(impl.block_probs(qb, kb), ref, rtol=0, atol=1e-15)


def test_mask_hand_case(impl):
    g = golden("linear_hand_case.json")
    q, k = bits(np.array(g["q"])[None, None]), bits(np.array(g["k"])[None, None])
    m = impl.block_mask(q, k, g["block"], g["topk_frac"])
    assert m["idx"][0, 0].tolist() == g["idx"]


# --- linear branch -----------------------------------------------------------

def test_phi_values():
    x = np.array([-2.0, -1.0, -1e-300, 0.0, 1e-300, 0.5, 3.0])
    assert np.allclose(O.phi(x), [math.exp(-2), math.exp(-1), 1.0, 1.0, 1.0, 1.5, 4.0], rtol=1e-15)


def test_linear_hand_case():
    g = golden("linear_hand_case.json")
    q = np.array(g["q"], dtype=np.float64)
    k = np.array(g["k"], dtype=np.float64)
    v = np.array(g["v"], dtype=np.float64)
    h, z = O.linear_states(k, v, g["block"])
    assert h.tolist() == g["h"] and z.tolist() == g["z"]
    e = math.e
    expect = np.array([[eval(s, {"e": e}) for s in row] for row in g["o_lin_expr"]])
    got = np.concatenate([O.linear_rows(q[0:2], h, z, g["idx"][0]),
                          O.linear_rows(q[2:4], h, z, g["idx"][1])])
    assert np.allclose(got, expect, rtol=1e-14, atol=0)


def test_linear_states_skip_rows_past_n():
    k = np.ones((5, 2))
    v = np.arange(10, dtype=np.float64).reshape(5, 2)
    h, z = O.linear_states(k, v, 4)           # second block has one valid row
    assert z.tolist() == [[8.0, 8.0], [2.0, 2.0]]
    assert h[1].tolist() == [[16.0, 18.0], [16.0, 18.0]]


def test_whole_operator_closed_form_q_k_zero(impl):
    """Q = K = 0: every score ties, so the lowest kc key blocks are kept; all
    codes are 0, so P = 1 on every kept key and phi = 1 elsewhere:
    out = mean(V over kept keys) + mean(V over the other keys) . W."""
    rng = np.random.default_rng(9)
    B, H, N, d, block, frac = 1, 2, 200, 8, 32, 0.3          # nblk 7 (last block 8 rows), kc 3
    v = rng.standard_normal((B, H, N, d)).astype(np.float32)
    w = rng.standard_normal((d, d)).astype(np.float32) / 4
    vb, wb = f32_to_bf16_bits(v), f32_to_bf16_bits(w)
    z = np.zeros((B, H, N, d), dtype=np.uint16)
    res = impl.sla_attention(z, z, vb, wb, block, frac)
    kc = impl.topk_count(7, frac)
    V, W = O.bf16_to_f64(vb), O.bf16_to_f64(wb)
    for h in range(H):
        assert (res["mask"]["idx"][0, h] == np.arange(kc)).all()
        expect = V[0, h, :kc * block].mean(0) + V[0, h, kc * block:].mean(0) @ W
        for i in range(7):
            rows = res["out"][(0, h, i)]
            assert np.allclose(rows, np.broadcast_to(expect, rows.shape), rtol=0, atol=1e-12)


def test_all_blocks_critical_means_no_linear_part(impl):
    x = make_inputs(1, 1, 96, 16, seed=1)
    res = impl.sla_attention(x["q"], x["k"], x["v"], x["proj"], 32, 1.0)
    for key, ol in res["o_lin"].items():
        assert not ol.any()
        assert np.array_equal(res["out"][key], res["o_sparse"][key])


# --- critical-block attention ----------------------------------------------------

def _sdpa64(q, k, v):
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None],
        torch.from_numpy(v)[None, None]).numpy()[0, 0]


@pytest.mark.parametrize("N,block", [(256, 64), (200, 64), (130, 32)])
def test_dense_unquantised_equals_library_attention(impl, N, block):
    x = make_inputs(1, 2, N, 32, seed=N)
    res = impl.sla_attention(x["q"], x["k"], x["v"], x["proj"], block, 1.0,
                          quant=False, pcast=False)
    Q, K, V = (O.bf16_to_f64(x[t]) for t in ("q", "k", "v"))
    for h in range(2):
        ref = _sdpa64(Q[0, h], K[0, h], V[0, h])
        got = np.concatenate([res["out"][(0, h, i)] for i in range((N + block - 1) // block)])
        assert np.max(np.abs(got - ref)) <= 1e-10


def test_smoothing_does_not_change_unquantised_output(impl):
    x = make_inputs(1, 2, 320, 32, seed=5)
    a = impl.sla_attention(x["q"], x["k"], x["v"], x["proj"], 64, 0.4, quant=False, pcast=False)
    b = impl.sla_attention(x["q"], x["k"], x["v"], x["proj"], 64, 0.4, quant=False, pcast=False,
                        smooth=False)
    assert np.array_equal(a["mask"]["idx"], b["mask"]["idx"])
    for key in a["out"]:
        assert np.max(np.abs(a["out"][key] - b["out"][key])) <= 1e-12


def test_quantised_path_on_losslessly_quantisable_inputs(impl):
    """Blocks of integers times 2**-6 with max |int| = 127 quantise without loss,
    and K rows in +- pairs have channel mean 0, so smoothing is the identity:
    the INT8 path then equals float64 attention up to float32 rounding of S."""
    rng = np.random.default_rng(12)
    N, d, block = 256, 32, 64
    qi = rng.integers(-127, 128, size=(1, 1, N, d))
    kh = rng.integers(-127, 128, size=(N // 2, d))
    for r in range(N // block):
        qi[0, 0, r * block, 0] = 127
    for r in range(N // 2 // block):
        kh[r * block, 1] = 127
    ki = np.concatenate([kh, -kh])[None, None]
    for r in range(N // block):
        assert np.abs(ki[0, 0, r * block:(r + 1) * block]).max() == 127
    qv = (qi * 2.0 ** -6).astype(np.float32)
    kv = (ki * 2.0 ** -6).astype(np.float32)
    v = rng.standard_normal((1, 1, N, d)).astype(np.float32)
    qb, kb, vb = bits(qv), bits(kv), f32_to_bf16_bits(v)
    wb = f32_to_bf16_bits(np.eye(d, dtype=np.float32))
    qz = impl.quantize(qb, kb, block)
    assert not qz["mu"].any()
    assert np.array_equal(qz["q_i8"].astype(np.int64), qi)
    assert np.array_equal(qz["k_i8"].astype(np.int64), ki)
    a = impl.sla_attention(qb, kb, vb, wb, block, 0.5, pcast=False)
    b = impl.sla_attention(qb, kb, vb, wb, block, 0.5, pcast=False, quant=False)
    for key in a["out"]:
        assert np.max(np.abs(a["o_sparse"][key] - b["o_sparse"][key])) <= 1e-5


def test_bf16_cast_of_p_error_bound(impl):
    """Rounding P to bf16 changes each P by at most 2**-9 of itself, so O moves by
    at most 2**-9 * max |V|."""
    x = make_inputs(1, 1, 512, 32, seed=8)
    a = impl.sla_attention(x["q"], x["k"], x["v"], x["proj"], 64, 0.25)
    b = impl.sla_attention(x["q"], x["k"], x["v"], x["proj"], 64, 0.25, pcast=False)
    vmax = np.abs(O.bf16_to_f64(x["v"])).max()
    worst = max(np.abs(a["o_sparse"][k] - b["o_sparse"][k]).max() for k in a["o_sparse"])
    assert 0 < worst <= 2.0 ** -9 * vmax


def test_projection_multiplies_on_the_right(impl):
    """W_proj = identity gives out = O_sparse + O_lin; W_proj = 0 gives O_sparse; a
    permutation matrix permutes the columns of O_lin."""
    x = make_inputs(1, 1, 256, 16, seed=21)
    d = 16
    eye = f32_to_bf16_bits(np.eye(d, dtype=np.float32))
    zero = np.zeros((d, d), dtype=np.uint16)
    perm = np.roll(np.eye(d, dtype=np.float32), 1, axis=1)          # e_a -> e_{a+1}
    a = impl.sla_attention(x["q"], x["k"], x["v"], eye, 32, 0.25)
    b = impl.sla_attention(x["q"], x["k"], x["v"], zero, 32, 0.25)
    c = impl.sla_attention(x["q"], x["k"], x["v"], f32_to_bf16_bits(perm), 32, 0.25)
    for key in a["out"]:
        assert np.array_equal(a["out"][key], a["o_sparse"][key] + a["o_lin"][key])
        assert np.array_equal(b["out"][key], b["o_sparse"][key])
        assert np.allclose(c["out"][key] - c["o_sparse"][key], np.roll(c["o_lin"][key], 1, axis=1),
                           rtol=0, atol=1e-15)


def test_quant_codes_match_exact_rational_division(impl):
    """Each code is the float32 nearest to x / s (exact rational arithmetic),
    rounded half to even; s is the float32 nearest to max|x| / 127."""
    rng = np.random.default_rng(17)
    x = (rng.standard_normal((1, 1, 64, 32)) * 3).astype(np.float32)
    x = O.bf16_to_f32(f32_to_bf16_bits(x))
    codes, scales = impl.quantize_blocks(x[:, :, :, :], 16)
    for r in range(4):
        blk = x[0, 0, r * 16:(r + 1) * 16]
        m = Fraction(float(np.abs(blk).max()))
        s = _nearest_f32_bruteforce(m / 127)
        assert scales[0, 0, r] == s
        for (n, c), val in np.ndenumerate(blk):
            qf = _nearest_f32_bruteforce(Fraction(float(val)) / Fraction(s))
            want = max(-127, min(127, int(np.rint(qf))))
            assert codes[0, 0, r * 16 + n, c] == want


def test_linear_hand_case_through_the_whole_operator(impl):
    """The hand-derived linear branch again, through the whole operator with
    W_proj = I (every value of the case is exact in bf16)."""
    g = golden("linear_hand_case.json")
    q = bits(np.array(g["q"])[None, None])
    k = bits(np.array(g["k"])[None, None])
    v = bits(np.array(g["v"])[None, None])
    w = bits(np.eye(g["d"]))
    res = impl.sla_attention(q, k, v, w, g["block"], g["topk_frac"])
    assert res["mask"]["idx"][0, 0].tolist() == g["idx"]
    e = math.e
    expect = np.array([[eval(s, {"e": e}) for s in row] for row in g["o_lin_expr"]])
    got = np.concatenate([res["o_lin"][(0, 0, i)] for i in range(2)])
    assert np.allclose(got, expect, rtol=1e-14, atol=0)


# ---------------------------------------------------------------- three classes, per-head fractions

def test_skip_counts_golden(impl):
    g = golden("skip_counts.json")
    for c in g["cases"]:
        assert impl.skip_count(c["nblk"], c["kc"], c["frac"]) == c["kn"], c
    with pytest.raises(ValueError):
        impl.skip_count(10, 1, 1.0)
    with pytest.raises(ValueError):
        impl.skip_count(10, 1, -0.1)


def test_block_classes_are_two_nested_top_k_selections(impl):
    """The ranking is a total order, so the critical blocks are the top kc and
    the blocks that are not negligible are the top nblk - kn; select_topk (pinned
    by brute force over all subsets above) gives both.  Rows with exact ties."""
    rng = np.random.default_rng(31)
    for n in (1, 2, 5, 9, 16):
        p = rng.integers(0, 4, size=(6, n)).astype(np.float64)   # many exact ties
        for kc in range(1, n + 1):
            for kn in range(0, n - kc + 1):
                cls, _ = impl.block_classes(p, kc, kn)
                for r in range(p.shape[0]):
                    top, _ = O.select_topk(p[r][None], kc)
                    keep, _ = O.select_topk(p[r][None], n - kn) if kn < n else (np.zeros((1, 0), int), None)
                    want = np.zeros(n, dtype=np.uint8)
                    want[keep[0]] = 1
                    want[top[0]] = 2
                    assert np.array_equal(cls[r], want), (n, kc, kn, r)


def test_block_classes_near_tie_at_either_boundary(impl):
    p = np.array([[0.5, 0.3, 0.2, 0.2 * (1 + 1e-12)],    # tie between ranks 2 and 3 only
                  [0.5, 0.5 * (1 - 1e-12), 0.1, 0.05]])   # tie between ranks 0 and 1 only
    _, t = impl.block_classes(p, 1, 1)     # boundaries after rank 0 and after rank 2
    assert t.tolist() == [True, True]
    _, t = impl.block_classes(p, 2, 0)     # boundary after rank 1 only
    assert t.tolist() == [False, False]


def test_three_classes_with_no_skip_equal_the_two_class_operator(impl):
    x = make_inputs(1, 2, 300, 16, seed=41)
    a = impl.sla_attention(x["q"], x["k"], x["v"], x["proj"], 32, 0.3)
    b = impl.sla_attention(x["q"], x["k"], x["v"], x["proj"], 32, [0.3, 0.3], skip_frac=0.0)
    assert np.array_equal(b["mask"]["idx"], a["mask"]["idx"])
    for key in a["out"]:
        assert np.array_equal(a["out"][key], b["out"][key])


def test_per_head_fractions_are_the_scalar_operator_head_by_head(impl):
    x = make_inputs(1, 3, 256, 16, seed=42)
    fr = [0.1, 0.25, 0.6]
    res = impl.sla_attention(x["q"], x["k"], x["v"], x["proj"], 32, fr, skip_frac=[0.0, 0.0, 0.0])
    for h, f in enumerate(fr):
        one = impl.sla_attention(x["q"][:, h:h + 1], x["k"][:, h:h + 1], x["v"][:, h:h + 1], x["proj"], 32, f)
        kc = impl.topk_count(8, f)
        assert res["mask"]["kc"][h] == kc
        assert np.array_equal(res["mask"]["idx"][0, h, :, :kc], one["mask"]["idx"][0, 0])
        assert (res["mask"]["idx"][0, h, :, kc:] == -1).all()
        for i in range(8):
            assert np.array_equal(res["out"][(0, h, i)], one["out"][(0, 0, i)])


def test_three_classes_closed_form_q_k_zero(impl):
    """Q = K = 0: every score ties, so the ranking is the block index: blocks
    [0, kc) critical, the last kn negligible, the rest linear; P = 1 on every
    kept key and phi = 1: out = mean(V over the critical keys) + mean(V over the
    linear keys) . W, per head with its own fractions."""
    rng = np.random.default_rng(43)
    B, H, N, d, block = 1, 3, 200, 8, 32                  # nblk 7, the last block 8 rows
    fr, sk = [0.3, 0.15, 0.5], [0.3, 0.6, 0.5]
    v = rng.standard_normal((B, H, N, d)).astype(np.float32)
    w = rng.standard_normal((d, d)).astype(np.float32) / 4
    vb, wb = f32_to_bf16_bits(v), f32_to_bf16_bits(w)
    z = np.zeros((B, H, N, d), dtype=np.uint16)
    res = impl.sla_attention(z, z, vb, wb, block, fr, skip_frac=sk)
    V, W = O.bf16_to_f64(vb), O.bf16_to_f64(wb)
    for h in range(H):
        kc = impl.topk_count(7, fr[h])
        kn = impl.skip_count(7, kc, sk[h])
        assert (kc, kn) == [(3, 2), (2, 4), (4, 3)][h]
        want = np.array([2] * kc + [1] * (7 - kc - kn) + [0] * kn, dtype=np.uint8)
        assert (res["mask"]["cls"][0, h] == want).all()
        lin_keys = V[0, h, kc * block:min(N, (7 - kn) * block)]
        expect = V[0, h, :kc * block].mean(0) + (lin_keys.mean(0) @ W if len(lin_keys) else 0.0)
        for i in range(7):
            rows = res["out"][(0, h, i)]
            assert np.allclose(rows, np.broadcast_to(expect, rows.shape), rtol=0, atol=1e-12)


def test_no_linear_class_means_no_linear_part(impl):
    """kc + kn = nblk leaves no block for the linear branch: O_lin = 0, out = O_sparse."""
    x = make_inputs(1, 1, 256, 16, seed=44)
    res = impl.sla_attention(x["q"], x["k"], x["v"], x["proj"], 32, 0.25, skip_frac=0.75)
    assert not (res["mask"]["cls"] == 1).any()
    for key in res["out"]:
        assert not res["o_lin"][key].any()
        assert np.array_equal(res["out"][key], res["o_sparse"][key])


# ---------------------------------------------------------------- finer quantisation groups

def test_scale_groups_are_the_maximum_over_exactly_their_tokens(impl):
    """Per 32-token group (brute force), with a ragged N inside the last block
    and a group wholly past N (scale 0, zero codes)."""
    rng = np.random.default_rng(51)
    N, d, block, gran = 200, 16, 128, 32            # nblk 2: groups 0..7, group 7 past N
    x = (rng.standard_normal((1, 2, N, d)) * np.exp(rng.standard_normal((1, 2, N, d)))).astype(np.float32)
    codes, scales = impl.quantize_groups(x, block, gran)
    assert scales.shape == (1, 2, 8) and codes.shape == (1, 2, 256, d)
    for h in range(2):
        for g in range(8):
            rows = [n for n in range(g * gran, (g + 1) * gran) if n < N]
            m = max((abs(float(x[0, h, n, c])) for n in rows for c in range(d)), default=0.0)
            assert scales[0, h, g] == np.float32(np.float32(m) / np.float32(127))
    assert not codes[:, :, N:].any()
    c2, s2 = O.quantize_blocks(x, gran)                  # the block quantiser with 32-token blocks
    assert np.array_equal(codes[:, :, :c2.shape[2]], c2) and np.array_equal(scales[:, :, :s2.shape[2]], s2)


def test_block_sized_groups_are_the_default_operator(impl):
    x = make_inputs(1, 2, 300, 16, seed=52)
    a = impl.sla_attention(x["q"], x["k"], x["v"], x["proj"], 64, 0.3)
    b = impl.sla_attention(x["q"], x["k"], x["v"], x["proj"], 64, 0.3, gran=64)
    for key in a["out"]:
        assert np.array_equal(a["out"][key], b["out"][key])


def test_32_token_groups_are_lossless_where_each_group_has_its_own_power_of_two(impl):
    """Integer-valued Q and K rows scaled by a different power of two per 32
    tokens (K rows in +- pairs inside each group, so mu = 0): with one scale
    per 32 tokens the codes are the integers and the INT8 path equals the
    float64 path up to float32 rounding of S; with one scale per 128-token
    block it is not lossless."""
    rng = np.random.default_rng(53)
    N, d, block, gran = 256, 32, 128, 32
    qi = rng.integers(-127, 128, size=(1, 1, N, d))
    kh = rng.integers(-127, 128, size=(1, 1, N // 2, d))
    ki = np.empty_like(qi)
    for g in range(N // gran):            # +- pairs within each group
        half = kh[0, 0, g * gran // 2:(g + 1) * gran // 2]
        ki[0, 0, g * gran:(g + 1) * gran] = np.concatenate([half, -half])
    for g in range(N // gran):
        qi[0, 0, g * gran, 0] = 127
        ki[0, 0, g * gran, 1], ki[0, 0, g * gran + gran // 2, 1] = 127, -127
    pw = 2.0 ** -np.arange(4, 4 + N // gran)             # one power of two per group
    qv = (qi * np.repeat(pw, gran)[None, None, :, None]).astype(np.float32)
    kv = (ki * np.repeat(pw, gran)[None, None, :, None]).astype(np.float32)
    v = rng.standard_normal((1, 1, N, d)).astype(np.float32)
    qb, kb, vb = bits(qv), bits(kv), f32_to_bf16_bits(v)
    wb = f32_to_bf16_bits(np.eye(d, dtype=np.float32))
    qz = impl.quantize(qb, kb, block, gran)
    assert not qz["mu"].any()
    assert np.array_equal(qz["q_i8"].astype(np.int64), qi) and np.array_equal(qz["k_i8"].astype(np.int64), ki)
    a = impl.sla_attention(qb, kb, vb, wb, block, 1.0, pcast=False, gran=gran)
    b = impl.sla_attention(qb, kb, vb, wb, block, 1.0, pcast=False, quant=False)
    c = impl.sla_attention(qb, kb, vb, wb, block, 1.0, pcast=False)
    for key in a["out"]:
        assert np.max(np.abs(a["o_sparse"][key] - b["o_sparse"][key])) <= 1e-5
    assert max(np.max(np.abs(c["o_sparse"][k] - b["o_sparse"][k])) for k in c["out"]) > 1e-4
