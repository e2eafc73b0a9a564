"""Pins of the SLA gradient oracles (the numpy statement
oracle/sla_backward_oracle.py and the plain C++ one behind
oracle/sla_backward_cpp.py) against things other than themselves: central
finite differences of the forward on every input element, torch autograd of
dense softmax attention, and the forward oracle (sla_oracle.sla_attention)
the fine-tune forward must agree with.  Tests taking the `impl` fixture run
against both; the two must also agree to float64 rounding.  No GPU needed."""

import math

import numpy as np
import pytest
import torch

import oracle as A
from oracle import sla_backward_cpp as BC
from oracle import sla_backward_oracle as BW
from synth import make_inputs


@pytest.fixture(params=["numpy", "cpp"])
def impl(request):
    return BW if request.param == "numpy" else BC


def _away_from_zero(x, eps=0.05):
    """phi = elu + 1 has a kink in its second derivative at 0; keep inputs
    clear of it so that central differences stay second-order accurate."""
    return np.where(np.abs(x) < eps, np.where(x < 0, -eps, eps), x)


def _case(N, d, seed):
    rng = np.random.default_rng(seed)
    q, k, v = (_away_from_zero(rng.standard_normal((N, d))) for _ in range(3))
    w = rng.standard_normal((d, d)) * 0.5
    g = rng.standard_normal((N, d))
    return q, k, v, w, g


def _loss(impl, q, k, v, w, crit, block, g):
    return float(np.sum(impl.forward(q, k, v, w, crit, block)["out"] * g))


@pytest.mark.parametrize("N,d,block,crit,seed", [
    # three blocks, the last one partial (3 rows); every row has a linear part
    (11, 4, 4, [[0], [1, 2], [2]], 1),
    # one block keeps everything (no linear part there), others keep one block
    (13, 6, 4, [[0, 1, 2, 3], [3], [0], [1, 3]], 2),
])
def test_gradient_matches_central_differences(impl, N, d, block, crit, seed):
    q, k, v, w, g = _case(N, d, seed)
    grads = impl.backward(q, k, v, w, crit, block, g)
    h = 1e-6
    args = {"q": q, "k": k, "v": v, "w": w}
    for name, x in args.items():
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + h
            lp = _loss(impl, args["q"], args["k"], args["v"], args["w"], crit, block, g)
            x[idx] = old - h
            lm = _loss(impl, args["q"], args["k"], args["v"], args["w"], crit, block, g)
            x[idx] = old
            num[idx] = (lp - lm) / (2 * h)
        got = grads["d" + name]
        assert np.allclose(got, num, rtol=1e-6, atol=1e-7), (name, np.max(np.abs(got - num)))
        assert np.max(np.abs(num)) > 1e-3, name    # the check is not vacuous


def test_every_block_kept_is_dense_attention(impl):
    """With every block kept there is no linear part: the gradient is that of
    softmax attention (torch autograd of scaled_dot_product_attention, float64)
    and dW_proj = 0."""
    N, d, block = 21, 8, 4
    q, k, v, w, g = _case(N, d, 3)
    nblk = (N + block - 1) // block
    crit = [list(range(nblk))] * nblk
    ours = impl.backward(q, k, v, w, crit, block, g)
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(tq[None, None], tk[None, None], tv[None, None])
    out.backward(torch.tensor(g)[None, None])
    for name, t in (("dq", tq), ("dk", tk), ("dv", tv)):
        assert np.allclose(ours[name], t.grad.numpy(), rtol=1e-10, atol=1e-12), name
    assert not np.any(ours["dw"])
    fw = impl.forward(q, k, v, w, crit, block)
    assert np.allclose(fw["out"], out.detach().numpy()[0, 0], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("N,d,block,frac,seed", [(300, 32, 64, 0.4, 4), (257, 16, 64, 0.25, 5)])
def test_forward_is_the_unquantised_operator(impl, N, d, block, frac, seed):
    """The fine-tune forward equals sla_attention with quantisation, the bf16
    cast of P and smoothing off, for the block lists that oracle picks."""
    x = make_inputs(1, 1, N, d, seed, "iid", None)
    ref = A.sla_attention(x["q"], x["k"], x["v"], x["proj"], block, frac, quant=False, pcast=False,
                          smooth=False)
    q, k, v, w = (A.bf16_to_f64(x[n][0, 0]) if n != "proj" else A.bf16_to_f64(x[n]) for n in ("q", "k", "v", "proj"))
    nblk = (N + block - 1) // block
    crit = [list(ref["mask"]["idx"][0, 0, i]) for i in range(nblk)]
    ours = impl.forward(q, k, v, w, crit, block)
    for i in range(nblk):
        rows = slice(i * block, min(N, (i + 1) * block))
        assert np.allclose(ours["out"][rows], ref["out"][(0, 0, i)], rtol=1e-12, atol=1e-13), i
        if "o_lin" in ours:
            assert np.allclose(ours["o_lin"][rows], ref["o_lin"][(0, 0, i)], rtol=1e-12, atol=1e-13), i


def test_linear_part_gradient_of_w_is_o_lin_transposed_times_g():
    """dW_proj = O_lin^T G: the projection is the last, linear step."""
    q, k, v, w, g = _case(17, 4, 6)
    crit = [[0], [1], [2], [3], [4]]
    fw = BW.forward(q, k, v, w, crit, 4)
    bw = BW.backward(q, k, v, w, crit, 4, g)
    assert np.allclose(bw["dw"], fw["o_lin"].T @ g, rtol=1e-13, atol=1e-14)
    assert math.isfinite(float(np.sum(bw["dq"])))


@pytest.mark.parametrize("N,d,block,seed", [(70, 8, 16, 7), (129, 16, 64, 8)])
def test_cpp_and_numpy_gradient_oracles_agree(N, d, block, seed):
    """Random kept-block lists (one to all blocks per query block)."""
    q, k, v, w, g = _case(N, d, seed)
    nblk = (N + block - 1) // block
    rng = np.random.default_rng(seed)
    crit = [sorted(rng.choice(nblk, size=rng.integers(1, nblk + 1), replace=False).tolist()) for _ in range(nblk)]
    a = BW.backward(q, k, v, w, crit, block, g)
    b = BC.backward(q, k, v, w, crit, block, g)
    for key in ("dq", "dk", "dv", "dw"):
        assert np.allclose(a[key], b[key], rtol=1e-11, atol=1e-12), key
    fa = BW.forward(q, k, v, w, crit, block)["out"]
    fb = BC.forward(q, k, v, w, crit, block)["out"]
    assert np.allclose(fa, fb, rtol=1e-12, atol=1e-13)
