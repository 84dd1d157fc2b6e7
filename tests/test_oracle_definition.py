"""Pins of the float64 oracle (oracle/definition.py) to what the pages and the
mathematics fix: closed forms, invariants, the worked example, hand-worked groups.

Each test names the passage it follows.  None of them re-types the oracle's own
formula: each checks a property that a dropped term, a wrong sign, a wrong index or
a transposed operand would break.
"""
import math
import os

import numpy as np
import pytest

from oracle import definition as D

RNG = np.random.default_rng(12345)


def _golden(golden_dir, name):
    with open(os.path.join(golden_dir, name), encoding="utf-8") as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.lstrip().startswith("#")]


# ---------------------------------------------------------------- RoPE ----------

def test_inv_freq_closed_form():
    # w_k = theta^(-2k/d_h): d_h = 8, theta = 1e4 gives 1, 0.1, 0.01, 0.001.
    np.testing.assert_allclose(D.inv_freq(8, 1e4), [1.0, 0.1, 0.01, 0.001], rtol=1e-15)
    # d_h = 4, theta = 100: 1, 0.1
    np.testing.assert_allclose(D.inv_freq(4, 100.0), [1.0, 0.1], rtol=1e-15)


@pytest.mark.parametrize("style", ["half", "interleaved"])
def test_rope_unit_vectors(style):
    """RoPE of unit vectors at m = 2, d_h = 4, theta = 100 (w = 1, 0.1): the first
    channel of pair k goes to (cos 2w_k, sin 2w_k), the second to (-sin, cos) —
    "Problem statement": every head splits into fixed 2-D frequency pairs."""
    ia, ib = D.pair_channels(4, style)
    pos = np.array([2])
    for k, wk in enumerate([1.0, 0.1]):
        e = np.zeros((1, 1, 4))
        e[0, 0, ia[k]] = 1.0
        y = D.rope(e, pos, 100.0, style)[0, 0]
        want = np.zeros(4)
        want[ia[k]], want[ib[k]] = math.cos(2 * wk), math.sin(2 * wk)
        np.testing.assert_allclose(y, want, atol=1e-15)
        e = np.zeros((1, 1, 4))
        e[0, 0, ib[k]] = 1.0
        y = D.rope(e, pos, 100.0, style)[0, 0]
        want = np.zeros(4)
        want[ia[k]], want[ib[k]] = -math.sin(2 * wk), math.cos(2 * wk)
        np.testing.assert_allclose(y, want, atol=1e-15)


def test_pair_layouts():
    ia, ib = D.pair_channels(8, "half")
    assert list(ia) == [0, 1, 2, 3] and list(ib) == [4, 5, 6, 7]
    ia, ib = D.pair_channels(8, "interleaved")
    assert list(ia) == [0, 2, 4, 6] and list(ib) == [1, 3, 5, 7]


@pytest.mark.parametrize("style", ["half", "interleaved"])
def test_rope_is_a_position_group_action(style):
    """RoPE at m1 then at m2 equals RoPE at m1 + m2; m = 0 is the identity."""
    x = RNG.standard_normal((5, 3, 16))
    m1, m2 = np.array([3, 7, 11, 0, 100]), np.array([5, 1, 0, 9, 23])
    np.testing.assert_allclose(D.rope(D.rope(x, m1, 1e4, style), m2, 1e4, style),
                               D.rope(x, m1 + m2, 1e4, style), atol=1e-12)
    np.testing.assert_allclose(D.rope(x, np.zeros(5, int), 1e4, style), x, atol=0)


# ----------------------------------------------------- commutation (converse) ----

@pytest.mark.parametrize("style", ["half", "interleaved"])
def test_pairwise_commutes_with_rope(style):
    """Per-pair rotations commute with RoPE at every position ("Theoretical
    characterisation"); the full-head Hadamard does not (negative control)."""
    x = RNG.standard_normal((64, 2, 32))
    pos = RNG.integers(0, 4096, size=64)
    phi = RNG.uniform(-math.pi / 4, math.pi / 4, size=16)
    a = D.pairwise(D.rope(x, pos, 5e5, style), phi, style)
    b = D.rope(D.pairwise(x, phi, style), pos, 5e5, style)
    np.testing.assert_allclose(a, b, atol=1e-12)
    h1 = D.block_hadamard(D.rope(x, pos, 5e5, style), 32)
    h2 = D.rope(D.block_hadamard(x, 32), pos, 5e5, style)
    assert np.abs(h1 - h2).max() > 1e-2


def test_generic_orthogonal_map_does_not_commute():
    """For distinct frequencies only in-pair planar rotations commute with RoPE
    ("Theoretical characterisation", converse result): a random orthogonal map
    mixing two pairs does not."""
    d = 8
    Qm, _ = np.linalg.qr(RNG.standard_normal((d, d)))
    x = RNG.standard_normal((20, 1, d))
    pos = RNG.integers(1, 500, size=20)
    lhs = D.rope(x, pos, 1e4) @ Qm
    rhs = D.rope(x @ Qm, pos, 1e4)
    assert np.abs(lhs - rhs).max() > 1e-2


def test_pairwise_rotation_direction():
    """phi = pi/2 sends (a, b) to (-b, a): the same sense as RoPE."""
    y = np.array([[1.0, 2.0, 3.0, 4.0]])   # half-split pairs (1, 3), (2, 4)
    out = D.pairwise(y, np.array([math.pi / 2, 0.0]), "half")
    np.testing.assert_allclose(out, [[-3.0, 2.0, 1.0, 4.0]], atol=1e-15)


# -------------------------------------------------------------- Hadamard --------

def test_sylvester_h4_golden(golden_dir):
    rows = _golden(golden_dir, "hadamard_h4.txt")
    H4 = np.array([[float(v) for v in r.split()] for r in rows])
    np.testing.assert_array_equal(D.sylvester_hadamard(4), H4)


@pytest.mark.parametrize("n", [2, 4, 8, 16, 32, 64, 128])
def test_hadamard_orthogonal(n):
    H = D.sylvester_hadamard(n)
    np.testing.assert_array_equal(H @ H.T, n * np.eye(n))
    # Sylvester recursion H_2n = [[H_n, H_n], [H_n, -H_n]]
    if n >= 4:
        h = D.sylvester_hadamard(n // 2)
        np.testing.assert_array_equal(H, np.block([[h, h], [h, -h]]))


def test_worked_example_outlier(golden_dir):
    """"LLM旋转量化笔记" §2.2: one outlier of 10.0 among K = 4096 channels of 0.1 is
    spread to about 10/sqrt(K) = 10/64 ~ 0.156 by the normalised Hadamard."""
    g = dict(r.split() for r in _golden(golden_dir, "worked_example_outlier.txt"))
    K, base, out = int(g["K"]), float(g["base"]), float(g["outlier"])
    assert math.isqrt(K) == int(g["page_sqrt_K"])
    x = np.full((1, K), base)
    x[0, -1] = out
    y = D.block_hadamard(x, K)[0]
    # exact: entry 0 = (0.1 * 4095 + 10)/64, every other entry = +-(10 - 0.1)/64
    assert y[0] == pytest.approx((base * (K - 1) + out) / 64, rel=1e-12)
    np.testing.assert_allclose(np.abs(y[1:]), (out - base) / 64, rtol=1e-12)
    # the outlier alone: every entry is +-10/64 = +-0.15625, the page's ~0.156
    e = np.zeros((1, K))
    e[0, -1] = out
    ye = D.block_hadamard(e, K)[0]
    np.testing.assert_allclose(np.abs(ye), out / 64, rtol=1e-12)
    assert abs(out / 64 - float(g["page_approx_value"])) < 1e-3
    assert np.linalg.norm(y) == pytest.approx(np.linalg.norm(x), rel=1e-12)


@pytest.mark.parametrize("b", [2, 4, 8, 16, 32, 64, 128])
def test_block_hadamard_acts_per_block(b):
    """I_{d_h/b} (x) H_b / sqrt(b): a change inside block j moves only block j, by
    H_b / sqrt(b) times the change ("Core contributions", mixing support b)."""
    d = 128
    y = RNG.standard_normal((1, d))
    j = (d // b) - 1
    dy = np.zeros((1, d))
    dy[0, j * b:(j + 1) * b] = RNG.standard_normal(b)
    diff = D.block_hadamard(y + dy, b) - D.block_hadamard(y, b)
    assert np.abs(diff[0, :j * b]).max(initial=0.0) < 1e-12
    np.testing.assert_allclose(diff[0, j * b:], dy[0, j * b:] @ D.sylvester_hadamard(b) / math.sqrt(b),
                               atol=1e-12)


def test_block_b_equals_full_head():
    """b = d_h reproduces the full-head Hadamard ("Results", support interpolation
    reaches the full-head baseline at b = d_h)."""
    y = RNG.standard_normal((7, 3, 64))
    np.testing.assert_array_equal(D.mix(y, "block_hadamard", b=64), D.mix(y, "hadamard"))


# ------------------------------------------------- invariants of every mode -----

MODES = [("hadamard", None), ("pairwise", None), ("pairwise_hadamard", None),
         ("block_hadamard", 2), ("block_hadamard", 8), ("block_hadamard", 64), ("rope_only", None)]


@pytest.mark.parametrize("mode,b", MODES)
@pytest.mark.parametrize("style", ["half", "interleaved"])
def test_qk_scores_preserved(mode, b, style):
    """Q~ K~^T = RoPE(Q) R R^T RoPE(K)^T = RoPE(Q) RoPE(K)^T ("LLM旋转量化笔记" §3.2.1)."""
    d = 64
    Tq, Tk = 6, 9
    q = RNG.standard_normal((Tq, 1, d))
    k = RNG.standard_normal((Tk, 1, d))
    pq, pk = RNG.integers(0, 8192, Tq), RNG.integers(0, 8192, Tk)
    phi = RNG.uniform(-math.pi / 4, math.pi / 4, d // 2)
    qt = D.transform(q, pq, 5e5, mode, b=b, phi=phi, style=style)[:, 0]
    kt = D.transform(k, pk, 5e5, mode, b=b, phi=phi, style=style)[:, 0]
    ref = D.rope(q, pq, 5e5, style)[:, 0] @ D.rope(k, pk, 5e5, style)[:, 0].T
    np.testing.assert_allclose(qt @ kt.T, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


@pytest.mark.parametrize("mode,b", MODES)
def test_norm_preserved(mode, b):
    """||x R||_2 = ||x||_2 ("LLM旋转量化笔记" §2.2) after RoPE and every mixing."""
    x = RNG.standard_normal((10, 4, 128)) * 3
    pos = RNG.integers(0, 131072, 10)
    phi = RNG.uniform(-1, 1, 64)
    y = D.transform(x, pos, 5e5, mode, b=b, phi=phi)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-12)


# ------------------------------------------------------------- quantiser --------

def _parse_groups(golden_dir):
    out = []
    for r in _golden(golden_dir, "quantizer_groups.txt"):
        xs, cs, bs, sc = [p.split() for p in r.split("|")]
        out.append((np.array([float(v) for v in xs]), np.array([int(v) for v in cs]),
                    np.array([int(v, 16) for v in bs], dtype=np.uint8), int(sc[0], 16)))
    return out


def test_quantizer_hand_groups(golden_dir):
    groups = _parse_groups(golden_dir)
    x = np.stack([g[0] for g in groups])[:, None, :]          # [5, 1, 8]
    codes, s = D.quantize(x, 8)
    np.testing.assert_array_equal(codes[:, 0], np.stack([g[1] for g in groups]))
    np.testing.assert_array_equal(D.pack_int4(codes)[:, 0], np.stack([g[2] for g in groups]))
    np.testing.assert_array_equal(D.scale_to_f16_bits(s)[:, 0, 0], [g[3] for g in groups])


def test_quantizer_invariants():
    """|code| <= 7; the group maximum maps to +-7; per-element error <= s/2
    ("LLM旋转量化笔记" §1.2: the rounding error is about s/2)."""
    x = RNG.standard_normal((50, 4, 128)) * np.exp(RNG.standard_normal((50, 4, 1)))
    for g in (32, 64, 128):
        codes, s = D.quantize(x, g)
        assert np.abs(codes).max() <= 7
        xg = x.reshape(50, 4, 128 // g, g)
        cg = codes.reshape(xg.shape)
        i = np.abs(xg).argmax(axis=-1)
        top = np.take_along_axis(cg, i[..., None], -1)[..., 0]
        np.testing.assert_array_equal(np.abs(top), 7)
        err = np.abs(xg - cg * s[..., None])
        assert (err <= s[..., None] / 2 * (1 + 1e-12)).all()


def test_pack_roundtrip():
    c = RNG.integers(-7, 8, size=(3, 5, 64)).astype(np.int8)
    np.testing.assert_array_equal(D.unpack_int4(D.pack_int4(c)), c)


def test_dequant_stats_hand():
    """Statistics of two groups of 4 worked by hand."""
    xt = np.array([[[7.0, -3.5, 1.0, 0.0, 2.0, -2.0, 1.2, 0.5]]])
    codes, s = D.quantize(xt, 4)          # group 1: s = 1 -> 7,-4,1,0 ; group 2: s = 2/7
    scl = D.scale_to_f16_bits(s)
    st = D.dequant_stats(xt, codes, scl, 4)
    s2 = float(np.float16(2.0 / 7.0))
    c2 = np.rint(np.array([2.0, -2.0, 1.2, 0.5]) / (2.0 / 7.0))   # 7, -7, 4 (4.2), 2 (1.75)
    assert list(c2) == [7, -7, 4, 2]
    err = 0.5 ** 2 + sum((v - s2 * c) ** 2 for v, c in zip([2.0, -2.0, 1.2, 0.5], c2))
    ref = 49 + 12.25 + 1 + 4 + 4 + 1.44 + 0.25
    assert st[0] == pytest.approx(err, rel=1e-12)
    assert st[1] == pytest.approx(ref, rel=1e-15)
    assert st[2] == pytest.approx(7.0 + 2.0)
    assert st[3] == pytest.approx((7.0 + 3.5) + (2.0 + 2.0))
    assert st[4] == 7.0 and st[5] == 2.0
    assert D.k_range(st) == pytest.approx(4.5)


def test_code_exceptions_hand_group():
    """The exception count of the bit-exact contract on a hand-built group (group max 7, so
    s = 1 and x/s = x): codes that differ from round(x/s) are counted, and split by whether
    x/s lies within the window of a rounding midpoint n + 1/2."""
    x = np.array([[7.0, 2.5 + 4e-7, 1.3, -0.5 - 2e-6, 0.0, 3.0, -6.9, 4.2]])
    ref, s = D.quantize(x, 8)
    assert s[0, 0] == 1.0
    np.testing.assert_array_equal(ref[0], [7, 3, 1, -1, 0, 3, -7, 4])
    codes = ref.copy()
    codes[0, 1] = 2          # 2.5000004 -> 3; 2 differs within 1e-6 of the midpoint 2.5
    codes[0, 2] = 2          # 1.3 -> 1; 2 differs far from a midpoint
    codes[0, 3] = 0          # -0.500002 -> -1; 0 differs 2e-6 from the midpoint: outside
    codes[0, 7] = 6          # off by two steps
    ex = D.code_exceptions(codes, x, 8)
    assert ex["codes"] == 8 and ex["differ"] == 4
    assert ex["outside_window"] == 3 and ex["off_by_more_than_one"] == 1
    assert ex["max_midpoint_distance"] == pytest.approx(0.3)
    dist = D.midpoint_distance(x, 8)
    assert dist[0, 1] == pytest.approx(4e-7, abs=1e-12)
    # a zero group decides nothing by rounding
    z = np.zeros((1, 8))
    assert np.isinf(D.midpoint_distance(z, 8)).all()
    assert D.code_exceptions(np.zeros((1, 8), np.int8), z, 8)["differ"] == 0
