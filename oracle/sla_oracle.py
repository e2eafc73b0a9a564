"""CPU oracle for SageSLA attention (INT8 block-quantised, top-k block-sparse
softmax attention plus a linear-attention branch for the blocks not picked).

TEST INFRASTRUCTURE ONLY.  This module is the slow, plain statement of what
the CUDA path computes.  Only the tests, the package's smoke check and the
benchmark's CPU-baseline leg may import it; the library itself never does,
and it shares no code with the CUDA sources.

Sources.  The pages describe the method only in prose:

[P1] "Turbo Diffusion：秒级生成与高清保真的视频扩散技术突破" (lanhy.cn),
     section 三(一) SageAttention2++ items 1-3 (outlier smoothing, per-sub-block
     quantisation parameters, 128x128 tensor-core tiles with a parallel
     softmax) and section 三(二) SLA items 1-3 (top-K 10% selection of the
     important regions, an O(N) linear branch with a linear projection, and
     SageSLA = SLA selection followed by INT8 computation on the kept part).
[P3] "TurboDiffusion技术指南：突破视频生成效率瓶颈的实践方案" (blog.gitcode.com),
     section "SageSLA：注意力机制的'瘦身'专家" and the T2V parameter list
     (``--sla_topk 0.1`` keeps 10%).
[P4] "TurboDiffusion: 即時AI影片生成的重大突破" (bonega.ai), section
     "SLA: 稀疏線性注意力" (sparse where full attention is not needed, near
     linear cost elsewhere).

The pages fix no formula, precision, layout or tie rule.  The precise
semantics below are the readings this project adopts (each stated where it is
used); every function says which passage it follows.

Notation: inputs are bf16 bit patterns, uint16 arrays Q, K, V [B, H, N, d] and
W_proj [d, d]; ``block`` tokens per block; nblk = ceil(N / block); block r
covers rows [r*block, min(N, (r+1)*block)).

The three-class mask (block_classes and its callers) is an extension: the
pages name two classes (top-K core blocks, the rest linear); a third class,
left out of both branches, is optional and off by default.

Parity status: every function here is pinned by a test in
tests/test_oracle_pins.py against a closed form, a library routine, a brute
force or a hand-derived case, except the choice of raw K (rather than
smoothed K) inside phi(K) for the linear branch, which no passage decides
("parity unpinned" for that choice; see the linear_states docstring).
"""

from __future__ import annotations

import math

import numpy as np

NEAR_TIE_REL = 1e-9


# ---------------------------------------------------------------------------
# number formats
# ---------------------------------------------------------------------------

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> exact float64 values."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> exact float32 values."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 value, ties to even.

    bf16 keeps 8 significant bits.  With x = m * 2**e, 0.5 <= |m| < 1
    (frexp), the spacing of bf16 values near x is 2**(e-8); below the
    smallest normal (2**-126) the spacing stays 2**-133.  Scaling by a power
    of two is exact, so rint (half to even) does the only rounding.
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    e = np.maximum(e, -125)
    y = np.ldexp(np.rint(np.ldexp(x, 8 - e)), e - 8)
    big = np.abs(y) > 3.3895313892515355e38  # beyond the largest finite bf16
    return np.where(big, np.copysign(np.inf, x), y)


def round_rational_to_f32(num: int, den: int) -> float:
    """The float32 nearest to num/den (exact integers, den > 0), ties to even."""
    if den <= 0:
        raise ValueError("den must be positive")
    if num == 0:
        return 0.0
    sign = -1.0 if num < 0 else 1.0
    a = abs(num)

    def split(e):
        if e >= 0:
            q, r = divmod(a, den << e)
            return q, r, den << e
        q, r = divmod(a << (-e), den)
        return q, r, den

    e = a.bit_length() - den.bit_length() - 24
    while True:
        q, r, dd = split(e)
        if q >= (1 << 24):
            e += 1
        elif q < (1 << 23) and e > -149:
            e -= 1
        else:
            break
    if e < -149:                        # subnormal float32: fixed spacing 2**-149
        e = -149
        q, r, dd = split(e)
    if 2 * r > dd or (2 * r == dd and (q & 1)):
        q += 1
    return sign * math.ldexp(q, e)


def topk_count(nblk: int, topk_frac: float) -> int:
    """Number of key blocks kept per query block: ceil(topk_frac * nblk) in [1, nblk].

    [P1] section 三(二) item 1 keeps the top K = 10% and [P3] reads
    ``--sla_topk 0.1`` as 10%.  Reading: the fraction is taken as the float32
    value the C interface receives, multiplied by nblk exactly (in float64),
    rounded up, and clamped to [1, nblk].
    """
    f = float(np.float32(topk_frac))
    if not (f > 0.0 and f <= 1.0):
        raise ValueError("topk_frac must be in (0, 1]")
    kc = math.ceil(f * nblk)
    return min(nblk, max(1, kc))


# ---------------------------------------------------------------------------
# smoothing and quantisation  ([P1] section 三(一) items 1 and 2)
# ---------------------------------------------------------------------------

def channel_mean(k_bits: np.ndarray) -> np.ndarray:
    """mu[b, h, c] = float32 nearest to the exact mean of K[b, h, :, c] over all N tokens.

    [P1] section 三(一) item 1 smooths outliers before quantising while keeping
    the overall distribution; the reading adopted is subtraction of the
    per-channel mean over tokens.  Reading: the mean is exact (the sum is
    formed without any rounding) and rounded once to float32, ties to even.

    A bf16 value is sig * 2**(E - 134) with an integer significand sig
    (|sig| < 256) and E = max(exponent field, 1).  Integer significands are
    accumulated per exponent (np.bincount; each partial sum is an integer of
    magnitude below 2**53, so its float64 accumulation is exact) and then
    combined as a Python integer multiple of 2**-133.
    """
    k = np.asarray(k_bits, dtype=np.uint16)
    B, H, N, d = k.shape
    mu = np.empty((B, H, d), dtype=np.float32)
    for b in range(B):
        for h in range(H):
            bits = k[b, h].astype(np.int64)
            expo = (bits >> 7) & 0xFF
            if np.any(expo == 0xFF):
                raise ValueError("K holds Inf/NaN")
            frac = bits & 0x7F
            sig = np.where(expo > 0, frac + 128, frac)
            sig = np.where((bits >> 15) & 1, -sig, sig)
            e = np.maximum(expo, 1)
            key = np.arange(d, dtype=np.int64)[None, :] * 256 + e
            counts = np.bincount(key.ravel(), weights=sig.ravel().astype(np.float64),
                                 minlength=d * 256).reshape(d, 256)
            for c in range(d):
                total = 0
                for ee in np.nonzero(counts[c])[0]:
                    total += int(counts[c, ee]) << (int(ee) - 1)   # units of 2**-133
                mu[b, h, c] = round_rational_to_f32(total, N << 133)
    return mu


def smooth_k(k_bits: np.ndarray, mu: np.ndarray) -> np.ndarray:
    """K_s = float32(K) - mu, one float32 rounding per element ([P1] 三(一) item 1).

    Q is not smoothed.  Reading: smoothing serves the quantisation only; the
    pooled mask and the linear branch use the raw K.
    """
    return bf16_to_f32(k_bits) - mu[:, :, None, :].astype(np.float32)


def quantize_blocks(x32: np.ndarray, block: int) -> tuple[np.ndarray, np.ndarray]:
    """Symmetric INT8 quantisation with one float32 scale per block of tokens.

    [P1] section 三(一) item 2: each sub-block gets its own quantisation
    parameters.  Readings: a block is ``block`` consecutive tokens by all d
    channels (the same blocks as the sparse mask); m = max |x| over the
    block's valid rows; scale s = float32(m / 127) (IEEE division);
    x_i8 = clamp(round_half_even(float32(x / s)), -127, 127); a block with
    m = 0 has s = 0 and all-zero codes.  Output rows past N (up to
    nblk * block) are zero.

    Returns (codes int8 [B, H, nblk*block, d], scales float32 [B, H, nblk]).
    """
    x32 = np.asarray(x32, dtype=np.float32)
    B, H, N, d = x32.shape
    nblk = (N + block - 1) // block
    codes = np.zeros((B, H, nblk * block, d), dtype=np.int8)
    scales = np.zeros((B, H, nblk), dtype=np.float32)
    for r in range(nblk):
        lo, hi = r * block, min(N, (r + 1) * block)
        xb = x32[:, :, lo:hi, :]
        m = np.max(np.abs(xb), axis=(2, 3))                      # float32, exact
        s = (m / np.float32(127.0)).astype(np.float32)           # IEEE float32 division
        scales[:, :, r] = s
        safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
        qf = (xb / safe[:, :, None, None]).astype(np.float32)    # float32 quotient
        qi = np.clip(np.rint(qf), -127, 127)                     # half to even
        qi = np.where(s[:, :, None, None] > 0, qi, 0)
        codes[:, :, lo:hi, :] = qi.astype(np.int8)
    return codes, scales


def quantize_groups(x32: np.ndarray, block: int, gran: int) -> tuple[np.ndarray, np.ndarray]:
    """quantize_blocks with one scale per ``gran`` tokens (gran divides block).

    [P1] section 三(一) item 2 names finer, "thread level" quantisation
    parameters than the attention tiles.  Reading: a scale group is ``gran``
    consecutive tokens by all d channels, inside the same blocks as the mask
    (block = gran is quantize_blocks itself).  It is quantize_blocks with
    block = gran, its codes padded with zero rows to nblk * block and its
    scales with zeros to nblk * block / gran (groups wholly past N).

    Returns (codes int8 [B, H, nblk*block, d], scales float32 [B, H, nblk*block/gran]).
    """
    if block % gran:
        raise ValueError("gran must divide block")
    B, H, N, d = np.shape(x32)
    nblk = (N + block - 1) // block
    codes_g, scales_g = quantize_blocks(x32, gran)
    codes = np.zeros((B, H, nblk * block, d), dtype=np.int8)
    codes[:, :, :codes_g.shape[2]] = codes_g
    scales = np.zeros((B, H, nblk * block // gran), dtype=np.float32)
    scales[:, :, :scales_g.shape[2]] = scales_g
    return codes, scales


def quantize(q_bits: np.ndarray, k_bits: np.ndarray, block: int, gran: int | None = None) -> dict:
    """Everything the quantisation entry point produces: mu, smoothed-K codes, Q codes, scales
    (one scale per block, or per ``gran`` tokens)."""
    mu = channel_mean(k_bits)
    g = block if gran is None else gran
    qi8, sq = quantize_groups(bf16_to_f32(q_bits), block, g)
    ki8, sk = quantize_groups(smooth_k(k_bits, mu), block, g)
    return {"mu": mu, "q_i8": qi8, "q_scale": sq, "k_i8": ki8, "k_scale": sk}


# ---------------------------------------------------------------------------
# block mask  ([P1] section 三(二) item 1; [P3] --sla_topk)
# ---------------------------------------------------------------------------

def block_means(x_bits: np.ndarray, block: int) -> np.ndarray:
    """Mean of each block's valid rows, per channel, in float64: [B, H, nblk, d].

    Reading: the block importance of [P1] 三(二) item 1 (a learnt predictor on
    the pages, which needs trained weights) is replaced by mean-pooled Q and
    K blocks; pooling uses the raw (unsmoothed) values; a partial last block
    is averaged over its valid rows only.
    """
    x = bf16_to_f64(x_bits)
    B, H, N, d = x.shape
    nblk = (N + block - 1) // block
    out = np.empty((B, H, nblk, d), dtype=np.float64)
    for r in range(nblk):
        lo, hi = r * block, min(N, (r + 1) * block)
        out[:, :, r, :] = x[:, :, lo:hi, :].sum(axis=2) / float(hi - lo)
    return out


def block_probs(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """Row-wise softmax over key blocks of qbar_i . kbar_j / sqrt(d), float64: [..., nblk, nblk]."""
    d = qbar.shape[-1]
    s = np.matmul(qbar, np.swapaxes(kbar, -1, -2)) / math.sqrt(d)
    e = np.exp(s - s.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def select_topk(p: np.ndarray, kc: int) -> tuple[np.ndarray, np.ndarray]:
    """Keep the kc largest entries of each row of p; equal values go to the lower index.

    Returns (indices int32 [..., kc] in ascending order, near_tie bool [...]).
    A row is a near tie when its kc-th and (kc+1)-th largest values differ by
    at most 1e-9 of the kc-th (then a different but equally valid choice is
    possible under any other rounding of the scores).
    """
    shp = p.shape[:-1]
    n = p.shape[-1]
    flat = p.reshape(-1, n)
    idx = np.empty((flat.shape[0], kc), dtype=np.int32)
    tie = np.zeros(flat.shape[0], dtype=bool)
    order_key = np.arange(n)
    for r in range(flat.shape[0]):
        row = flat[r]
        order = np.lexsort((order_key, -row))      # by value desc, then index asc
        idx[r] = np.sort(order[:kc])
        if kc < n:
            a, b = row[order[kc - 1]], row[order[kc]]
            tie[r] = (a - b) <= NEAR_TIE_REL * a
    return idx.reshape(shp + (kc,)), tie.reshape(shp)


def block_mask(q_bits: np.ndarray, k_bits: np.ndarray, block: int, topk_frac: float) -> dict:
    """The critical key blocks of every query block: {"idx", "near_tie", "probs", "kc"}."""
    qbar = block_means(q_bits, block)
    kbar = block_means(k_bits, block)
    p = block_probs(qbar, kbar)
    kc = topk_count(p.shape[-1], topk_frac)
    idx, tie = select_topk(p, kc)
    return {"idx": idx, "near_tie": tie, "probs": p, "kc": kc}


def bitmap_of(idx: np.ndarray, nblk: int) -> np.ndarray:
    """uint8 [..., nblk, nblk] with 1 at the kept (query block, key block) pairs."""
    out = np.zeros(idx.shape[:-1] + (nblk,), dtype=np.uint8)
    np.put_along_axis(out, idx.astype(np.int64), 1, axis=-1)
    return out


# ---------------------------------------------------------------------------
# three block classes and per-head fractions
# ---------------------------------------------------------------------------
# [P1] 三(二) items 1-2 split the key blocks of a query block into the top-K
# "core" blocks (exact attention) and the rest (the linear branch); [P4]
# "SLA: 稀疏線性注意力" replaces dense attention by cheaper substitutes where it
# is not needed.  Extension adopted here (the pages name no third class): the
# blocks at the bottom of the same ranking may be left out of the linear
# branch too ("negligible").  With skip_frac = 0 nothing is left out and the
# operator is exactly the two-class one above.  topk_frac and skip_frac may
# be given per head (the same value for every batch entry).

CLS_NEGLIGIBLE, CLS_LINEAR, CLS_CRITICAL = 0, 1, 2


def skip_count(nblk: int, kc: int, skip_frac: float) -> int:
    """Number of negligible key blocks per query block: floor(skip_frac * nblk), at most nblk - kc.

    Reading: like topk_frac, the fraction is the float32 value the C interface
    receives, multiplied by nblk exactly; it is rounded DOWN (a block is left
    out only when the whole fraction covers it) and capped so that the
    critical blocks stay.  skip_frac must be in [0, 1).
    """
    f = float(np.float32(skip_frac))
    if not (f >= 0.0 and f < 1.0):
        raise ValueError("skip_frac must be in [0, 1)")
    return min(math.floor(f * nblk), nblk - kc)


def head_counts(nblk: int, H: int, topk_frac, skip_frac=None) -> tuple[np.ndarray, np.ndarray]:
    """(kc [H], kn [H]) from a scalar or one fraction per head."""
    tf = np.broadcast_to(np.asarray(topk_frac, dtype=np.float64), (H,))
    sf = np.broadcast_to(np.asarray(0.0 if skip_frac is None else skip_frac, dtype=np.float64), (H,))
    kc = np.array([topk_count(nblk, float(t)) for t in tf], dtype=np.int64)
    kn = np.array([skip_count(nblk, int(c), float(f)) for c, f in zip(kc, sf)], dtype=np.int64)
    return kc, kn


def block_classes(p: np.ndarray, kc: int, kn: int) -> tuple[np.ndarray, np.ndarray]:
    """Class of every key block of every row of p: uint8 [..., n] and near_tie bool [...].

    The blocks are ranked by value, larger first, equal values by the lower
    index first (the same ranking as select_topk).  The first kc are critical
    (2), the last kn negligible (0), the rest go to the linear branch (1).  A
    row is a near tie when either boundary separates values that differ by at
    most 1e-9 of the larger.
    """
    shp = p.shape[:-1]
    n = p.shape[-1]
    flat = p.reshape(-1, n)
    cls = np.full(flat.shape, CLS_LINEAR, dtype=np.uint8)
    tie = np.zeros(flat.shape[0], dtype=bool)
    pos = np.arange(n)
    for r in range(flat.shape[0]):
        row = flat[r]
        order = np.lexsort((pos, -row))
        cls[r, order[:kc]] = CLS_CRITICAL
        if kn > 0:
            cls[r, order[n - kn:]] = CLS_NEGLIGIBLE
        for cut in (kc, n - kn):
            if 0 < cut < n:
                a, b = row[order[cut - 1]], row[order[cut]]
                tie[r] = tie[r] or bool((a - b) <= NEAR_TIE_REL * a)
    return cls.reshape(shp + (n,)), tie.reshape(shp)


def block_mask_classes(q_bits: np.ndarray, k_bits: np.ndarray, block: int, topk_frac, skip_frac=None) -> dict:
    """Three-class mask with per-head counts: {"cls" uint8 [B, H, nblk, nblk],
    "idx" int32 [B, H, nblk, max kc] (critical blocks ascending, then -1),
    "kc" [H], "kn" [H], "near_tie", "probs"}."""
    qbar = block_means(q_bits, block)
    kbar = block_means(k_bits, block)
    p = block_probs(qbar, kbar)
    B, H, nblk, _ = p.shape
    kc, kn = head_counts(nblk, H, topk_frac, skip_frac)
    cls = np.empty(p.shape, dtype=np.uint8)
    tie = np.empty(p.shape[:-1], dtype=bool)
    idx = np.full((B, H, nblk, int(kc.max())), -1, dtype=np.int32)
    for h in range(H):
        cls[:, h], tie[:, h] = block_classes(p[:, h], int(kc[h]), int(kn[h]))
        for b in range(B):
            for i in range(nblk):
                idx[b, h, i, :kc[h]] = np.flatnonzero(cls[b, h, i] == CLS_CRITICAL)
    return {"cls": cls, "idx": idx, "kc": kc, "kn": kn, "near_tie": tie, "probs": p}


# ---------------------------------------------------------------------------
# critical blocks: INT8 QK^T, softmax, bf16 P, PV  ([P1] 三(一) item 3, 三(二) item 3)
# ---------------------------------------------------------------------------

def critical_rows(qi8_blk, sq_rows, ki8, sk_keys, v64, crit, N, block, *, pcast=True,
                  q64_blk=None, ks64=None):
    """O_sparse for the rows of one query block over its critical key blocks (float64).

    Quantised mode (q64_blk is None), readings of [P1] 三(一) item 3 and
    三(二) item 3: S = float32(int32(Qi8 . Ki8^T)) * float32(sq_n * sk_m) *
    float32(1/sqrt(d)) in float32, sq_n the scale of query row n (sq_rows,
    [block]) and sk_m that of key m (sk_keys, one per padded key); keys at
    or past N are masked; softmax with
    the row maximum over all critical keys; P = exp(S - max) (float64 here);
    the normaliser l sums the unrounded P; P is rounded to bf16 when
    ``pcast``; O = (P . V) / l.

    The integer products are formed with a float64 matmul: every entry is an
    integer of magnitude at most d * 127**2 < 2**53, so it is exact.

    Unquantised mode (q64_blk, ks64 given): S = Q . K_s^T / sqrt(d) in float64.
    """
    d = v64.shape[-1]
    keys = np.concatenate([np.arange(j * block, (j + 1) * block) for j in crit])
    valid = keys < N
    if q64_blk is None:
        acc = np.matmul(qi8_blk.astype(np.float64), ki8[keys].astype(np.float64).T)
        c = (np.asarray(sq_rows, dtype=np.float32)[:, None] *
             np.asarray(sk_keys, dtype=np.float32)[keys][None, :]).astype(np.float32)
        S = (acc.astype(np.float32) * c).astype(np.float32)
        S = (S * np.float32(1.0 / math.sqrt(d))).astype(np.float32).astype(np.float64)
    else:
        kk = np.zeros((len(keys), d))
        kk[valid] = ks64[keys[valid]]
        S = np.matmul(q64_blk, kk.T) / math.sqrt(d)
    S[:, ~valid] = -np.inf
    M = S.max(axis=1, keepdims=True)
    P = np.exp(S - M)
    ell = P.sum(axis=1, keepdims=True)
    Pb = round_bf16(P) if pcast else P
    vv = np.zeros((len(keys), d))
    vv[valid] = v64[keys[valid]]
    return np.matmul(Pb, vv) / ell


# ---------------------------------------------------------------------------
# linear branch  ([P1] 三(二) item 2; [P4] "SLA: 稀疏線性注意力")
# ---------------------------------------------------------------------------

def phi(x: np.ndarray) -> np.ndarray:
    """Feature map elu(x) + 1: x + 1 for x > 0, exp(x) otherwise (always positive)."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def linear_states(k64: np.ndarray, v64: np.ndarray, block: int) -> tuple[np.ndarray, np.ndarray]:
    """Per key block j of one head: h_j = sum_n phi(k_n) v_n^T [d, d], z_j = sum_n phi(k_n) [d].

    [P1] 三(二) item 2 gives the non-selected part an O(N) linear form; the
    reading adopted is phi = elu + 1 kernelised linear attention with
    per-block states.  Reading (parity unpinned: no passage decides it):
    phi is applied to the raw K, not the smoothed K.  Rows past N are left
    out of the sums.
    """
    N, d = k64.shape
    nblk = (N + block - 1) // block
    pk = np.zeros((nblk * block, d))
    pk[:N] = phi(k64)
    vv = np.zeros((nblk * block, d))
    vv[:N] = v64
    pk = pk.reshape(nblk, block, d)
    vv = vv.reshape(nblk, block, d)
    h = np.matmul(np.swapaxes(pk, 1, 2), vv)
    z = pk.sum(axis=1)
    return h, z


def linear_rows(q64_blk: np.ndarray, h: np.ndarray, z: np.ndarray, crit, lin=None) -> np.ndarray:
    """O_lin for the rows of one query block: phi(q) h_rest / (phi(q) . z_rest).

    h_rest and z_rest are summed directly over the key blocks NOT in ``crit``
    (the plain definition: every non-critical block goes through the linear
    branch), or, when ``lin`` (bool [nblk]) is given, over the blocks it
    marks (the linear class of the three-class mask).  With no block in the
    linear branch there is no linear part and O_lin = 0.
    """
    nblk, d, _ = h.shape
    if lin is not None:
        keep = np.asarray(lin, dtype=bool).copy()
    else:
        keep = np.ones(nblk, dtype=bool)
        keep[np.asarray(crit, dtype=np.int64)] = False
    if not keep.any():
        return np.zeros((q64_blk.shape[0], d))
    h_rest = h[keep].sum(axis=0)
    z_rest = z[keep].sum(axis=0)
    pq = phi(q64_blk)
    return np.matmul(pq, h_rest) / np.matmul(pq, z_rest)[:, None]


# ---------------------------------------------------------------------------
# the whole operator
# ---------------------------------------------------------------------------

def sla_attention(q_bits, k_bits, v_bits, w_bits, block: int, topk_frac, *,
                  items=None, quant=True, pcast=True, smooth=True, idx_override=None, skip_frac=None,
                  gran=None):
    """SageSLA attention: out = O_sparse + O_lin . W_proj.

    [P1] 三(二) item 3 (SLA selection, then INT8 computation on the selected
    blocks) and item 2 (the rest through the linear branch and a linear
    projection); [P3] "SageSLA" section.  Readings: W_proj multiplies O_lin on
    the right (row vectors); the result is float64 here (the CUDA path forms
    it in float32 and stores bf16, float32 on request).

    items: iterable of (b, h, i) query blocks to evaluate (default: all).
    quant/pcast/smooth: False switches off INT8 quantisation (float64 scores),
    the bf16 cast of P, or the K smoothing; all True is the operator itself.
    idx_override: optional {(b, h, i): key-block list} replacing the mask's
    choice for those rows (used where the mask is a near tie); with the
    three-class mask, {(b, h, i): class row uint8 [nblk]}.
    topk_frac may be one fraction per head, and skip_frac (scalar or per
    head) leaves the lowest-ranked blocks out of the linear branch; either
    one selects the three-class mask (block_mask_classes), whose "mask"
    entry is then that function's result.
    gran: tokens per quantisation scale (default: the block; see
    quantize_groups).

    Returns {"out": {(b,h,i): float64 [rows, d]}, "o_sparse", "o_lin",
    "mask": block_mask(...), "quant": quantize(...)}.
    """
    q_bits = np.asarray(q_bits, dtype=np.uint16)
    B, H, N, d = q_bits.shape
    nblk = (N + block - 1) // block
    classes = skip_frac is not None or np.ndim(topk_frac) > 0
    if classes:
        mask = block_mask_classes(q_bits, k_bits, block, topk_frac, skip_frac)
    else:
        mask = block_mask(q_bits, k_bits, block, topk_frac)
    qz = quantize(q_bits, k_bits, block, gran) if quant else None
    g = block if gran is None else gran
    mu = qz["mu"] if quant else channel_mean(k_bits)
    w64 = bf16_to_f64(w_bits)
    if items is None:
        items = [(b, h, i) for b in range(B) for h in range(H) for i in range(nblk)]
    by_head = {}
    for (b, h, i) in items:
        by_head.setdefault((b, h), []).append(i)
    res = {"out": {}, "o_sparse": {}, "o_lin": {}, "mask": mask, "quant": qz}
    for (b, h), rows in by_head.items():
        q64 = bf16_to_f64(q_bits[b, h])
        k64 = bf16_to_f64(k_bits[b, h])
        v64 = bf16_to_f64(v_bits[b, h])
        hst, zst = linear_states(k64, v64, block)
        ks64 = k64 - mu[b, h].astype(np.float64)[None, :] if smooth else k64
        for i in rows:
            lin = None
            if classes:
                row_cls = mask["cls"][b, h, i]
                if idx_override is not None and (b, h, i) in idx_override:
                    row_cls = np.asarray(idx_override[(b, h, i)], dtype=np.uint8)
                crit = np.flatnonzero(row_cls == CLS_CRITICAL).astype(np.int32)
                lin = row_cls == CLS_LINEAR
            else:
                crit = mask["idx"][b, h, i]
                if idx_override is not None and (b, h, i) in idx_override:
                    crit = np.asarray(idx_override[(b, h, i)], dtype=np.int32)
            lo, hi = i * block, min(N, (i + 1) * block)
            if quant:
                qi8_blk = qz["q_i8"][b, h, i * block:(i + 1) * block]
                sq_rows = np.repeat(qz["q_scale"][b, h], g)[i * block:(i + 1) * block]
                os_ = critical_rows(qi8_blk, sq_rows, qz["k_i8"][b, h],
                                    np.repeat(qz["k_scale"][b, h], g), v64, crit, N, block, pcast=pcast)
            else:
                qb = np.zeros((block, d))
                qb[:hi - lo] = q64[lo:hi]
                os_ = critical_rows(None, None, None, None, v64, crit, N, block, pcast=pcast,
                                    q64_blk=qb, ks64=ks64)
            os_ = os_[:hi - lo]
            ol = linear_rows(q64[lo:hi], hst, zst, crit, lin)
            out = os_ + np.matmul(ol, w64)
            res["o_sparse"][(b, h, i)] = os_
            res["o_lin"][(b, h, i)] = ol
            res["out"][(b, h, i)] = out
    return res
