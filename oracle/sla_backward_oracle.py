"""CPU oracle for the gradient of the SLA operator (the fine-tune path).

TEST INFRASTRUCTURE ONLY: imported by the tests, never by the library, and
sharing no code with the CUDA sources.  No CUDA kernel computes this yet; the
oracle is the first, pinned step of that path.

Sources.
  "Turbo Diffusion：秒级生成与高清保真的视频扩散技术突破" (lanhy.cn):
  section 三(二) SLA items 1-2 (the top-K blocks through softmax attention,
  the rest through an O(N) linear branch with a linear projection) and
  section 四 step 1 (SLA fine-tuning: dense attention is replaced by SLA and
  the attention layers are adapted by training, so gradients flow through
  the SLA operator).

Readings (the pages give no formula):
  * Training runs SLA without the INT8 step.  INT8 computation on the kept
    blocks is SageSLA's inference form; the training flow brings in
    quantisation only later, for the W8A8 linear layers.  So the forward is
    the unquantised operator in float64: S = Q K^T / sqrt(d) over the kept
    key blocks, softmax, P V; plus phi(q) H_i / (phi(q) . Z_i) times W_proj
    over the blocks not kept.  K smoothing is a per-row constant shift of S,
    which the softmax ignores, so it drops out here.
  * The block mask is a discrete choice from the pooled Q and K.  It is piecewise
    constant in the inputs, with gradient zero almost everywhere.  It is
    held fixed: the caller passes each query block's kept key blocks.
  * The gradient is that of L = sum(out * G) for a given upstream gradient G
    = dL/dout, with respect to Q, K, V (one head, [N, d]) and W_proj [d, d].

Notation as in sla_oracle: block i covers rows [i*block, min(N, (i+1)*block));
phi = elu + 1, phi'(x) = 1 for x > 0 and exp(x) otherwise; h_j = sum over the
rows m of block j of phi(k_m) v_m^T, z_j = sum phi(k_m).

Parity: pinned by tests/test_backward_oracle.py against central finite
differences of the forward (every input element of a small case), against
torch autograd of dense softmax attention (every block kept), and against the
forward oracle sla_oracle.sla_attention (unquantised, no bf16 cast of P).
"""

from __future__ import annotations

import math

import numpy as np


def phi(x):
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def dphi(x):
    """Derivative of elu + 1 (continuous at 0: both sides give 1)."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 0, 1.0, np.exp(np.minimum(x, 0.0)))


def _rows(i, block, N):
    return np.arange(i * block, min(N, (i + 1) * block))


def _keys(crit, block, N):
    return np.concatenate([_rows(j, block, N) for j in sorted(int(c) for c in crit)])


def _states(k, v, block):
    """h_j [nblk, d, d] and z_j [nblk, d] of one head (valid rows only)."""
    N, d = k.shape
    nblk = (N + block - 1) // block
    h = np.zeros((nblk, d, d))
    z = np.zeros((nblk, d))
    for j in range(nblk):
        r = _rows(j, block, N)
        f = phi(k[r])
        h[j] = f.T @ v[r]
        z[j] = f.sum(axis=0)
    return h, z


def forward(q, k, v, w, crit_lists, block):
    """out [N, d] of one head for fixed kept-block lists (float64).

    crit_lists[i] holds the key blocks query block i keeps; the others go
    through the linear branch (none: no linear part for that block).
    Returns {"out", "o_sparse", "o_lin"}, each [N, d].
    """
    q, k, v, w = (np.asarray(a, dtype=np.float64) for a in (q, k, v, w))
    N, d = q.shape
    nblk = (N + block - 1) // block
    h, z = _states(k, v, block)
    o_s = np.zeros((N, d))
    o_l = np.zeros((N, d))
    for i in range(nblk):
        r = _rows(i, block, N)
        keys = _keys(crit_lists[i], block, N)
        s = q[r] @ k[keys].T / math.sqrt(d)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        o_s[r] = p @ v[keys]
        rest = sorted(set(range(nblk)) - set(int(c) for c in crit_lists[i]))
        if rest:
            f = phi(q[r])
            o_l[r] = (f @ h[rest].sum(axis=0)) / (f @ z[rest].sum(axis=0))[:, None]
    return {"out": o_s + o_l @ w, "o_sparse": o_s, "o_lin": o_l}


def backward(q, k, v, w, crit_lists, block, g):
    """Gradients of L = sum(out * g) for one head: {"dq", "dk", "dv", "dw"}.

    Softmax part, per query block i over its kept keys (the standard
    attention gradient): dV += P^T g, dP = g V^T, D = rowsum(g * O_sparse),
    dS = P * (dP - D), dQ += dS K / sqrt(d), dK += dS^T Q / sqrt(d).

    Linear part, per query block i with the blocks it did not keep: with
    F = phi(Q_i), H_i = sum h_j, Z_i = sum z_j over those blocks, a = F H_i,
    b = F Z_i, O_lin = a / b and out = ... + O_lin W:
      dW += O_lin^T g,  dO_lin = g W^T,
      dA = dO_lin / b,  db = -rowsum(dO_lin * O_lin) / b,
      dF = dA H_i^T + db Z_i^T,  dQ_i += dF * phi'(Q_i),
      dH_i = F^T dA,  dZ_i = F^T db, added to dh_j, dz_j of every such j.
    Then per key block j with Phi = phi(K_j): h_j = Phi^T V_j and
    z_j = Phi^T 1 give dPhi = V_j dh_j^T + 1 dz_j^T, dK_j += dPhi * phi'(K_j),
    dV_j += Phi dh_j.
    """
    q, k, v, w, g = (np.asarray(a, dtype=np.float64) for a in (q, k, v, w, g))
    N, d = q.shape
    nblk = (N + block - 1) // block
    h, z = _states(k, v, block)
    dq = np.zeros((N, d))
    dk = np.zeros((N, d))
    dv = np.zeros((N, d))
    dw = np.zeros((d, d))
    dh = np.zeros((nblk, d, d))
    dz = np.zeros((nblk, d))
    sc = 1.0 / math.sqrt(d)
    for i in range(nblk):
        r = _rows(i, block, N)
        gi = g[r]
        # softmax attention over the kept keys
        keys = _keys(crit_lists[i], block, N)
        s = q[r] @ k[keys].T * sc
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        o_s = p @ v[keys]
        dv[keys] += p.T @ gi
        dp = gi @ v[keys].T
        D = np.sum(gi * o_s, axis=1, keepdims=True)
        ds = p * (dp - D)
        dq[r] += ds @ k[keys] * sc
        dk[keys] += ds.T @ q[r] * sc
        # linear branch over the blocks not kept
        rest = sorted(set(range(nblk)) - set(int(c) for c in crit_lists[i]))
        if not rest:
            continue
        f = phi(q[r])
        Hi = h[rest].sum(axis=0)
        Zi = z[rest].sum(axis=0)
        a = f @ Hi
        b = f @ Zi
        o_l = a / b[:, None]
        dw += o_l.T @ gi
        do_l = gi @ w.T
        dA = do_l / b[:, None]
        db = -np.sum(do_l * o_l, axis=1) / b
        dF = dA @ Hi.T + np.outer(db, Zi)
        dq[r] += dF * dphi(q[r])
        dH = f.T @ dA
        dZ = f.T @ db
        for j in rest:
            dh[j] += dH
            dz[j] += dZ
    for j in range(nblk):
        r = _rows(j, block, N)
        F = phi(k[r])
        dF = v[r] @ dh[j].T + dz[j][None, :]
        dk[r] += dF * dphi(k[r])
        dv[r] += F @ dh[j]
    return {"dq": dq, "dk": dk, "dv": dv, "dw": dw}
