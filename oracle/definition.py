"""fp64 definition of the post-RoPE Q/K transform with dynamic KV4 quantisation.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module.  The CUDA
library never does, and this module imports nothing from it.

What is computed, and where the pages state it:

* RoPE splits each head of d_h channels into d_h/2 fixed two-dimensional
  frequency pairs; pair k at position m is turned by the angle m * w_k
  (paper summary "When Local Variance Optimality Is Not Enough: RoPE-Aligned
  Q/K Rotations for Dynamic 4-Bit Quantisation", section "Problem statement";
  abstract of the same paper).  w_k = theta^(-2k/d_h) is the standard RoPE
  frequency; the pages leave it to the model, the workload gives theta.
* The transform acts on Q and K after RoPE (same summary, "Methodology";
  "LLM旋转量化笔记" §3.2.1, which writes Q~ = RoPE(Q) H_head, K~ = RoPE(K) H_head).
  Four mixings: the full-head normalised Hadamard x H_{d_h} / sqrt(d_h)
  ("Methodology" item 1; the normalisation 1/sqrt(K) is the one in
  "LLM旋转量化笔记" §2.2), the head-shared pairwise rotation inside each RoPE pair
  ("Methodology" item 2), pairwise followed by the Hadamard ("Methodology"
  item 3), and the block Hadamard of support b, I_{d_h/b} (x) H_b / sqrt(b)
  ("Core contributions", mixing support).
* K is quantised with the dynamic symmetric quantiser
  Q(x) = clip(round(x / s), -q_max, q_max) ("LLM旋转量化笔记" §1.2) whose step s
  is set from the tokenwise group range, s = max|x| / q_max ("Core
  contributions", objective mismatch), q_max = 7 for 4 bits.  Q is not
  quantised ("Estimation strategies": only K is quantised after the transform).
* Calibration: raw per-pair moment accumulators of the post-RoPE values pooled
  over heads; three estimators (pooled Q+K before centring, K only, equal
  weights for Q and K) ("Estimation strategies"); the head-shared angle phi*_k
  minimises the larger channel variance of the pair under that pooled
  covariance ("Optimisation objective").  The closed form used below is derived
  in ``solve_angles``.
* Measurement: the tokenwise group range of K~ and the relative quantisation
  error ("Core contributions", mixing support; "Results", support interpolation).

Readings taken where the pages are silent are listed in the repository's design
notes and repeated next to each function.  Everything here is float64 numpy,
written as the definition, with no blocking or reordering.
"""
from __future__ import annotations

import math

import numpy as np

QMAX = 7

MODES = {"hadamard": 0, "pairwise": 1, "pairwise_hadamard": 2, "block_hadamard": 3,
         "rope_only": 4}
ESTIMATORS = {"pooled": 0, "k_only": 1, "balanced": 2}
ROPE_STYLES = {"half": 0, "interleaved": 1}


# ---------------------------------------------------------------------------
# inputs
# ---------------------------------------------------------------------------

def bf16_bits_to_f64(h: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> exact float64 values."""
    u = np.asarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# RoPE
# ---------------------------------------------------------------------------

def inv_freq(d_h: int, theta: float) -> np.ndarray:
    """w_k = theta^(-2k/d_h), k = 0 .. d_h/2 - 1 (standard RoPE frequencies)."""
    k = np.arange(d_h // 2, dtype=np.float64)
    return np.array([theta ** (-(2.0 * kk) / d_h) for kk in k], dtype=np.float64)


def pair_channels(d_h: int, style: str = "half") -> tuple[np.ndarray, np.ndarray]:
    """Channels (first, second) of each RoPE frequency pair k.

    "half": (k, k + d_h/2), the rotate-half layout; "interleaved": (2k, 2k + 1).
    The pages only say that RoPE forms two-dimensional frequency pairs
    ("Problem statement"); both layouts are such pairs.
    """
    P = d_h // 2
    k = np.arange(P)
    if style == "half":
        return k, k + P
    if style == "interleaved":
        return 2 * k, 2 * k + 1
    raise ValueError(style)


def rotate_pairs(y: np.ndarray, cos: np.ndarray, sin: np.ndarray, style: str) -> np.ndarray:
    """(a, b) -> (a cos - b sin, a sin + b cos) on every frequency pair.

    ``cos``/``sin`` broadcast against y[..., pair]; returns a new array.
    """
    ia, ib = pair_channels(y.shape[-1], style)
    a, b = y[..., ia], y[..., ib]
    out = np.empty_like(y)
    out[..., ia] = a * cos - b * sin
    out[..., ib] = a * sin + b * cos
    return out


def rope(x: np.ndarray, pos: np.ndarray, theta: float, style: str = "half") -> np.ndarray:
    """RoPE of x [T, H, d_h] at positions pos [T], in float64."""
    d_h = x.shape[-1]
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv_freq(d_h, theta)[None, :]   # [T, P]
    return rotate_pairs(np.asarray(x, dtype=np.float64), np.cos(ang)[:, None, :],
                        np.sin(ang)[:, None, :], style)


# ---------------------------------------------------------------------------
# mixings
# ---------------------------------------------------------------------------

def sylvester_hadamard(n: int) -> np.ndarray:
    """Unnormalised Hadamard matrix of order n (power of two), natural (Sylvester)
    order: H[i, j] = (-1)^popcount(i & j)."""
    if n < 1 or n & (n - 1):
        raise ValueError("n must be a power of two")
    i = np.arange(n)
    bits = np.bitwise_and(i[:, None], i[None, :])
    pc = np.zeros_like(bits)
    while bits.any():
        pc += bits & 1
        bits >>= 1
    return np.where(pc % 2 == 0, 1.0, -1.0)


def block_hadamard(y: np.ndarray, b: int) -> np.ndarray:
    """y (row vectors) times I_{d_h/b} (x) H_b / sqrt(b): contiguous blocks of b channels.

    b = d_h is the full-head normalised Hadamard y H_{d_h} / sqrt(d_h).
    """
    d_h = y.shape[-1]
    if d_h % b:
        raise ValueError("b must divide d_h")
    H = sylvester_hadamard(b) / math.sqrt(b)
    yb = y.reshape(*y.shape[:-1], d_h // b, b)
    return (yb @ H).reshape(y.shape)


def value_transform(v: np.ndarray) -> np.ndarray:
    """Value rows turned by the full-head normalised Hadamard, V~ = V H_{d_h} / sqrt(d_h)
    ("LLM旋转量化笔记" §3.2.2: no RoPE on V; the rotation flattens the value cache and its
    H on the attention output, A V~ = (A V) H, folds into the output projection)."""
    v = np.asarray(v, dtype=np.float64)
    return block_hadamard(v, v.shape[-1])


def pairwise(y: np.ndarray, phi: np.ndarray, style: str = "half") -> np.ndarray:
    """Head-shared rotation of pair k by phi_k, the same convention as RoPE."""
    phi = np.asarray(phi, dtype=np.float64)
    return rotate_pairs(y, np.cos(phi), np.sin(phi), style)


def mix(y: np.ndarray, mode: str, b: int | None = None, phi: np.ndarray | None = None,
        style: str = "half") -> np.ndarray:
    """Apply one of the mixings to post-RoPE rows y [..., d_h]."""
    d_h = y.shape[-1]
    if mode == "rope_only":
        return np.array(y, dtype=np.float64)
    if mode == "hadamard":
        return block_hadamard(y, d_h)
    if mode == "pairwise":
        return pairwise(y, phi, style)
    if mode == "pairwise_hadamard":
        return block_hadamard(pairwise(y, phi, style), d_h)
    if mode == "block_hadamard":
        return block_hadamard(y, b)
    raise ValueError(mode)


def transform(x: np.ndarray, pos: np.ndarray, theta: float, mode: str, b: int | None = None,
              phi: np.ndarray | None = None, style: str = "half") -> np.ndarray:
    """x~ = mix(RoPE(x)) for rows x [T, H, d_h] (float64)."""
    return mix(rope(x, pos, theta, style), mode, b=b, phi=phi, style=style)


# ---------------------------------------------------------------------------
# dynamic symmetric 4-bit quantisation of K
# ---------------------------------------------------------------------------

def quantize(xt: np.ndarray, group: int) -> tuple[np.ndarray, np.ndarray]:
    """Per group of ``group`` contiguous channels: s = max|x| / 7,
    code = clip(round(x / s), -7, 7) with round-half-to-even.

    A group with max|x| = 0 gets codes 0 and s = 0 (reading: avoids 0/0).
    Returns (codes int8 [..., d_h], s float64 [..., d_h/group]).
    """
    d_h = xt.shape[-1]
    g = xt.reshape(*xt.shape[:-1], d_h // group, group)
    amax = np.max(np.abs(g), axis=-1)
    s = amax / QMAX
    safe = np.where(s > 0, s, 1.0)
    codes = np.clip(np.rint(g / safe[..., None]), -QMAX, QMAX)
    codes = np.where(s[..., None] > 0, codes, 0.0)
    return codes.reshape(xt.shape).astype(np.int8), s


def midpoint_distance(xt: np.ndarray, group: int) -> np.ndarray:
    """Per element, the distance of x / s to the nearest rounding midpoint n + 1/2, with
    s = max|x| / 7 of its group (the quotient the quantiser rounds); +inf in zero groups,
    whose codes do not depend on a rounding."""
    d_h = xt.shape[-1]
    g = np.asarray(xt, dtype=np.float64).reshape(*xt.shape[:-1], d_h // group, group)
    s = np.max(np.abs(g), axis=-1, keepdims=True) / QMAX
    with np.errstate(invalid="ignore", divide="ignore"):
        f = np.abs(g / s)
    dist = np.abs(f - np.floor(f) - 0.5)
    dist = np.where(s > 0, dist, np.inf)
    return dist.reshape(xt.shape)


def code_exceptions(codes: np.ndarray, xt: np.ndarray, group: int,
                    window: float = 1e-6) -> dict:
    """Compare quantiser codes with the definition's on the exact transformed values xt.

    The exception rule of the bit-exact contract: codes must equal ``quantize(xt)`` except
    for elements whose |x/s| lies within ``window`` of a rounding midpoint.  Returns the
    number of codes, how many differ, how many of those lie outside the window, how many
    differ by more than one step, and the largest midpoint distance among the differing."""
    ref, _ = quantize(xt, group)
    codes = np.asarray(codes, dtype=np.int8)
    bad = codes != ref
    dist = midpoint_distance(xt, group)
    return {"codes": int(codes.size), "differ": int(bad.sum()),
            "outside_window": int((bad & (dist >= window)).sum()),
            "off_by_more_than_one": int((np.abs(codes.astype(np.int16) - ref) > 1).sum()),
            "max_midpoint_distance": float(dist[bad].max()) if bad.any() else 0.0,
            "window": window}


def scale_to_f16_bits(s: np.ndarray) -> np.ndarray:
    """Stored scale: IEEE half, round to nearest even (numpy's conversion)."""
    return np.asarray(s, dtype=np.float64).astype(np.float16).view(np.uint16)


def pack_int4(codes: np.ndarray) -> np.ndarray:
    """Two codes per byte: byte j = (c[2j] & 0xF) | ((c[2j+1] & 0xF) << 4) (two's complement)."""
    c = np.asarray(codes, dtype=np.int8).astype(np.int16) & 0xF
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_int4(packed: np.ndarray) -> np.ndarray:
    """Inverse of ``pack_int4`` (sign-extends each nibble)."""
    p = np.asarray(packed, dtype=np.uint8).astype(np.int16)
    lo, hi = p & 0xF, (p >> 4) & 0xF
    lo = np.where(lo > 7, lo - 16, lo)
    hi = np.where(hi > 7, hi - 16, hi)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.int8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def dequantize(codes: np.ndarray, scale_f16_bits: np.ndarray, group: int) -> np.ndarray:
    """K^ = stored scale * code (float64)."""
    s = np.asarray(scale_f16_bits, dtype=np.uint16).view(np.float16).astype(np.float64)
    d_h = codes.shape[-1]
    c = codes.astype(np.float64).reshape(*codes.shape[:-1], d_h // group, group)
    return (c * s[..., None]).reshape(codes.shape)


# ---------------------------------------------------------------------------
# calibration: raw moments, estimators, closed-form angle
# ---------------------------------------------------------------------------

MOMENT_FIELDS = ("n", "Sa", "Sb", "Saa", "Sab", "Sbb")


def moments(yq: np.ndarray, yk: np.ndarray, style: str = "half") -> np.ndarray:
    """Raw (uncentred) accumulators per stream and frequency pair, pooled over
    heads and tokens: [2 (Q, K), P, 6] = (n, Sa, Sb, Saa, Sab, Sbb).

    ``yq``/``yk`` are post-RoPE, pre-mixing rows [T, H, d_h] (reading: the
    "position-averaged" surrogate averages over every calibration position of
    the rotated values).
    """
    d_h = yq.shape[-1]
    ia, ib = pair_channels(d_h, style)
    out = np.zeros((2, d_h // 2, 6), dtype=np.float64)
    for si, y in enumerate((yq, yk)):
        y = np.asarray(y, dtype=np.float64).reshape(-1, d_h)
        a, b = y[:, ia], y[:, ib]
        out[si, :, 0] = y.shape[0]
        out[si, :, 1] = a.sum(axis=0)
        out[si, :, 2] = b.sum(axis=0)
        out[si, :, 3] = (a * a).sum(axis=0)
        out[si, :, 4] = (a * b).sum(axis=0)
        out[si, :, 5] = (b * b).sum(axis=0)
    return out


def covariance(m: np.ndarray, estimator: str) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """2x2 covariance [[A, C], [C, D]] per pair under one of the three estimators.

    pooled   : add the Q and K raw accumulators, then centre once with the pooled mean.
    k_only   : K accumulators only.
    balanced : average the per-stream normalised uncentred moments with weight 1/2
               each, then centre.
    """
    Q, K = m[0], m[1]

    def norm(x):
        n = x[:, 0]
        return x[:, 1:3] / n[:, None], x[:, 3:6] / n[:, None]

    if estimator == "pooled":
        tot = Q + K
        m1, m2 = norm(tot)
    elif estimator == "k_only":
        m1, m2 = norm(K)
    elif estimator == "balanced":
        m1q, m2q = norm(Q)
        m1k, m2k = norm(K)
        m1, m2 = 0.5 * (m1q + m1k), 0.5 * (m2q + m2k)
    else:
        raise ValueError(estimator)
    A = m2[:, 0] - m1[:, 0] * m1[:, 0]
    C = m2[:, 1] - m1[:, 0] * m1[:, 1]
    D = m2[:, 2] - m1[:, 1] * m1[:, 1]
    return A, C, D


def channel_variances(A, C, D, phi):
    """Variances of the two channels of a pair after rotating by phi
    (y1 = a cos - b sin, y2 = a sin + b cos)."""
    c, s = np.cos(phi), np.sin(phi)
    v1 = A * c * c - 2.0 * C * s * c + D * s * s
    v2 = A * s * s + 2.0 * C * s * c + D * c * c
    return v1, v2


def empty_streams(m: np.ndarray, estimator: str = "pooled") -> np.ndarray:
    """Per pair: True where the estimator needs a stream that has no observations (n = 0):
    pooled needs Q and K together, k_only needs K, balanced needs each of Q and K.
    Reading (the pages are silent): such a pair has no covariance, so its angle is 0."""
    nq, nk = m[0, :, 0], m[1, :, 0]
    if estimator == "pooled":
        return ~(nq + nk > 0)
    if estimator == "k_only":
        return ~(nk > 0)
    if estimator == "balanced":
        return ~((nq > 0) & (nk > 0))
    raise ValueError(estimator)


def solve_angles(m: np.ndarray, estimator: str = "pooled") -> np.ndarray:
    """Closed-form head-shared angle phi*_k (float64, one per pair).

    With the rotation convention above,
        Var y1 = (A+D)/2 + ((A-D)/2) cos 2phi - C sin 2phi,
        Var y2 = (A+D)/2 - ((A-D)/2) cos 2phi + C sin 2phi,
    so max(Var y1, Var y2) = (A+D)/2 + |((A-D)/2) cos 2phi - C sin 2phi| >= tr/2,
    with equality iff tan 2phi = (A-D)/(2C), i.e. phi* = atan2(A-D, 2C)/2 (mod pi/2).
    The analytic minimum of the larger channel variance is tr/2.

    Tie-break (reading): phi* reduced into (-pi/4, pi/4]; a pair whose covariance is
    isotropic (|A-D| + 2|C| <= 1e-12 (A+D), or A+D <= 0) gets phi* = 0, and so does a pair
    whose estimator has an empty stream (``empty_streams``).
    """
    empty = empty_streams(m, estimator)
    with np.errstate(invalid="ignore", divide="ignore"):
        A, C, D = covariance(m, estimator)
    out = np.zeros(A.shape, dtype=np.float64)
    for k in range(A.shape[0]):
        if empty[k]:
            continue
        tr = A[k] + D[k]
        if not (tr > 0.0) or abs(A[k] - D[k]) + 2.0 * abs(C[k]) <= 1e-12 * tr:
            out[k] = 0.0
            continue
        phi = 0.5 * math.atan2(A[k] - D[k], 2.0 * C[k])
        if phi <= -math.pi / 4:
            phi += math.pi / 2
        elif phi > math.pi / 4:
            phi -= math.pi / 2
        out[k] = phi
    return out


# ---------------------------------------------------------------------------
# measurement
# ---------------------------------------------------------------------------

STAT_FIELDS = ("sum_err2", "sum_ref2", "sum_absmax", "sum_range", "max_absmax", "n_groups")


def dequant_stats(xt: np.ndarray, codes: np.ndarray, scale_f16_bits: np.ndarray,
                  group: int) -> np.ndarray:
    """[sum (x~ - K^)^2, sum x~^2, sum of group max|x~|, sum of group (max - min),
    max of group max|x~|, number of groups] over all (token, head, group).

    K range = sum_absmax / n_groups (the tokenwise group range that sets the
    quantiser's step); relative error = sqrt(sum_err2 / sum_ref2).
    """
    x = np.asarray(xt, dtype=np.float64)
    deq = dequantize(codes, scale_f16_bits, group)
    d_h = x.shape[-1]
    g = x.reshape(-1, d_h // group, group)
    amax = np.abs(g).max(axis=-1)
    rng = g.max(axis=-1) - g.min(axis=-1)
    return np.array([((x - deq) ** 2).sum(), (x * x).sum(), amax.sum(), rng.sum(),
                     amax.max() if amax.size else 0.0, float(amax.size)], dtype=np.float64)


def attention_scores(q_t_bits: np.ndarray, packed_codes: np.ndarray, scale_f16_bits: np.ndarray,
                     group: int) -> np.ndarray:
    """Attention logits of transformed queries against the int4 key cache, float64:
    S[tq, h, tk] = q~[tq, h] . K^[tk, h // (Hq / Hkv)] with K^ = stored scale * code.

    q_t_bits [Tq, Hq, d_h] bf16 bits, packed_codes [Tk, Hkv, d_h/2], scale_f16_bits
    [Tk, Hkv, d_h/group].  ("LLM旋转量化笔记" §3.2.1: the rotation cancels in Q~ K~^T, so the
    scores are taken against the quantised K~ directly; grouped-query heads share a key head.)
    """
    q = bf16_bits_to_f64(q_t_bits)
    khat = dequantize(unpack_int4(packed_codes), scale_f16_bits, group)   # [Tk, Hkv, d_h]
    Tq, Hq, d_h = q.shape
    Hkv = khat.shape[1]
    per = Hq // Hkv
    kh = np.repeat(khat, per, axis=1)                                     # [Tk, Hq, d_h]
    return np.einsum("qhc,khc->qhk", q, kh)


def k_range(stats: np.ndarray) -> float:
    return float(stats[2] / stats[5]) if stats[5] else 0.0


def rel_error(stats: np.ndarray) -> float:
    return float(math.sqrt(stats[0] / stats[1])) if stats[1] > 0 else 0.0
