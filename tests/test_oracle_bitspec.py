"""Pins of the oracle's fp32 operation sequence (oracle/bitspec.c).

It must (a) reproduce the float64 definition within an error bound derived from
fp32 rounding, (b) take the same 4-bit decisions as the definition everywhere
except within that bound of a rounding midpoint, (c) convert number formats
exactly as the IEEE / bfloat16 round-to-nearest-even rules (checked against
numpy's and torch's conversions), and (d) keep the exact structural facts the
pages fix (b = d_h is the full head; the worked example of "LLM旋转量化笔记" §2.2).
"""
import functools
import math

import numpy as np
import pytest

import synth
from oracle import bitspec as B
from oracle import definition as D

RNG = np.random.default_rng(2024)
EPS = 2.0 ** -24


# ------------------------------------------------------------ formats -----------

def _edge_floats():
    r = np.random.default_rng(5)
    bits = r.integers(0, 2 ** 32, size=20000, dtype=np.uint64).astype(np.uint32)
    v = bits.view(np.float32)
    v = v[np.isfinite(v)]
    extra = np.array([0.0, -0.0, 1.0, -1.0, 65504.0, 65519.99, 65520.0, 65536.0, 1e-8, 6e-8,
                      5.9604645e-08, 2.9802322e-08, 2.98e-8, 3e-8, 6.1035156e-05, 6.1e-5,
                      1.0009765625, 1.00048828125, 1.00146484375, 3.4e38, 1e-40,
                      1.0 + 2 ** -8, 1.0 + 2 ** -9, 1.0 + 3 * 2 ** -9], dtype=np.float32)
    scaled = (r.standard_normal(20000) * np.exp(r.uniform(-25, 12, 20000))).astype(np.float32)
    return np.concatenate([v, extra, -extra, scaled])


def test_f16_conversion_matches_ieee():
    x = _edge_floats()
    got = B.f32_to_f16(x)
    with np.errstate(over="ignore"):  # the edge values include ones that overflow fp16 on purpose
        want = x.astype(np.float16).view(np.uint16)
    np.testing.assert_array_equal(got, want)


def test_bf16_conversion_matches_torch():
    torch = pytest.importorskip("torch")
    x = _edge_floats()
    got = B.f32_to_bf16(x)
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(got, want)


# ------------------------------------------------------------ table -------------

def test_rope_table_closed_form():
    """table[m, k] = fp32(cos(m * theta^(-2k/d_h))), sin likewise."""
    c, s = B.rope_table(4096, 128, 5e5)
    assert (c[0] == 1.0).all() and (s[0] == 0.0).all()
    for m, k in [(1, 0), (4095, 0), (17, 5), (3000, 63), (2048, 31)]:
        ang = m * (5e5 ** (-(2.0 * k) / 128))
        assert c[m, k] == np.float32(math.cos(ang))
        assert s[m, k] == np.float32(math.sin(ang))


# ------------------------------------------------------------ FWHT --------------

@pytest.mark.parametrize("n", [2, 4, 8, 16, 32, 64, 128])
def test_fwht_matches_dense_matrix(n):
    x = RNG.standard_normal((20, n)).astype(np.float32)
    H = D.sylvester_hadamard(n)
    for row in x:
        y = B.fwht(row)
        ref = row.astype(np.float64) @ H
        bound = math.log2(n) * EPS * np.abs(row).sum() + 1e-30
        assert np.abs(y - ref).max() <= bound


def test_fwht_worked_example():
    """"LLM旋转量化笔记" §2.2: an outlier of 10 among K = 4096 channels becomes
    +-10/64 = +-0.15625 everywhere after the normalised Hadamard (exact in fp32)."""
    e = np.zeros(4096, dtype=np.float32)
    e[-1] = 10.0
    y = B.fwht(e) * np.float32(1.0 / 64.0)
    np.testing.assert_array_equal(np.abs(y), np.float32(0.15625))


# ------------------------------------------------- sequence vs definition --------

CASES = [("hadamard", None), ("pairwise", None), ("pairwise_hadamard", None),
         ("block_hadamard", 2), ("block_hadamard", 4), ("block_hadamard", 8),
         ("block_hadamard", 16), ("block_hadamard", 32), ("block_hadamard", 64),
         ("block_hadamard", 128), ("rope_only", None)]

# (workload, tokens, group): the tiny shape (d_h 64, Gaussian with x20 outlier channels),
# the 8B heads (d_h 128, Student-t with anisotropic pairs and x30 outliers) and the 3B heads
# (d_h 128, the Gaussian family with a log-normal per-token magnitude), at every group size
# the workloads use; positions spread over each workload's range
SHAPES = [("tiny", 96, 64), ("llama31_8b_128k", 40, 128), ("llama31_8b_128k", 40, 32),
          ("llama32_3b", 40, 128), ("llama32_3b", 40, 32)]


def _row_bound(x64_rows, n_mix):
    """fp32 error bound per row: RoPE and pair rotation (a few ulps of the pair
    norm, carried through an orthogonal map) plus log2(n) butterfly stages and the
    final scale (each at most one rounding of a value bounded by ||row||_2 sqrt(n)
    before the 1/sqrt(n) scale)."""
    nrm = np.linalg.norm(x64_rows, axis=-1, keepdims=True)
    stages = math.log2(n_mix) if n_mix > 1 else 0.0
    return (8.0 + 2.0 * stages) * EPS * nrm * 2.0


@functools.lru_cache(maxsize=None)
def _tables(wname, split):
    """The oracle's fp32 RoPE tables of a workload (one row per position, or split)."""
    w = synth.WORKLOADS[wname]
    return (B.rope_table_split if split else B.rope_table)(w.max_pos, w.d_h, w.theta)


def _spread_positions(w, T):
    """T positions spread over the workload's whole range (large angles included)."""
    return np.linspace(0, w.max_pos - 1, T).astype(np.int32)


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"{s[0]}-g{s[2]}")
@pytest.mark.parametrize("mode,b", CASES)
@pytest.mark.parametrize("style", ["half", "interleaved"])
@pytest.mark.parametrize("split", [False, True])
def test_sequence_matches_definition(shape, mode, b, style, split):
    """The fp32 sequence (RoPE, then the pair rotation as its own rounded step, then the
    butterflies) against the float64 definition on the same bf16 inputs.
    split: the RoPE entry composed from the split tables (a few more roundings in c and s,
    well inside the row bound)."""
    wname, T, g = shape
    w = synth.WORKLOADS[wname]
    if b is not None and b > w.d_h:
        pytest.skip("support above d_h")
    inp = synth.make_inputs(wname, T=T)
    pos = inp["pos"] if wname == "tiny" else _spread_positions(w, T)
    inp = dict(inp, pos=pos)
    phi = RNG.uniform(-math.pi / 4, math.pi / 4, w.P).astype(np.float32)
    ct, st = _tables(wname, split)
    out = B.transform_quantize(inp["q"], inp["k"], inp["pos"], w.d_h, cos_t=ct, sin_t=st,
                               mode=mode, b=b, group=g, phi=phi, style=style, want_f32=True,
                               split=split, max_pos=w.max_pos)
    assert out["status"] == 0
    q64 = D.bf16_bits_to_f64(inp["q"])
    k64 = D.bf16_bits_to_f64(inp["k"])
    n_mix = {"hadamard": w.d_h, "pairwise_hadamard": w.d_h, "block_hadamard": b or 1}.get(mode, 1)
    for x64, got in ((q64, out["q_f32"]), (k64, out["k_f32"])):
        ref = D.transform(x64, inp["pos"], w.theta, mode, b=b, phi=phi.astype(np.float64),
                          style=style)
        assert (np.abs(got - ref) <= _row_bound(x64, n_mix)).all()
    # Q is stored as bf16 of the fp32 row
    np.testing.assert_array_equal(out["q_out"], B.f32_to_bf16(out["q_f32"]))
    # K codes: the same decisions as the float64 definition except within the
    # error bound of a rounding midpoint
    kref = D.transform(k64, inp["pos"], w.theta, mode, b=b, phi=phi.astype(np.float64),
                       style=style)
    codes_ref, s_ref = D.quantize(kref, g)
    codes = D.unpack_int4(out["k_codes"])
    bound = _row_bound(k64, n_mix)                                     # [T, H, 1]
    amax = s_ref * 7.0
    grp = np.repeat(amax, g, axis=-1)
    delta = bound * 7.0 / grp * 2.0 + 8.0 * EPS * 7.0                  # in units of x/s
    frac = np.abs(kref / np.repeat(s_ref, g, axis=-1))
    near_mid = np.abs(frac - np.floor(frac) - 0.5) < delta
    bad = codes != codes_ref
    assert (np.abs(codes.astype(int) - codes_ref) <= 1).all()
    assert not (bad & ~near_mid).any()
    assert bad.sum() <= max(2, codes.size // 1000)
    # scales: fp16 of the fp32 step vs fp16 of the exact step: equal or adjacent
    scl = out["k_scales"].view(np.float16).astype(np.float64)
    np.testing.assert_allclose(scl, s_ref, rtol=2e-3)


# ------------------------------------------------ split (two-level) RoPE tables -----

def test_split_table_rows_are_plain_table_rows():
    """Low row l is the plain table's row l; high row h is the plain row 64 h (the same
    fp64 angle (64 h) * w_k), bit for bit."""
    max_pos = 1000
    c, s = B.rope_table(max_pos, 64, 5e5)
    sc, ss = B.rope_table_split(max_pos, 64, 5e5)
    assert sc.shape == (64 + 16, 32)
    np.testing.assert_array_equal(sc[:64], c[:64])
    np.testing.assert_array_equal(ss[:64], s[:64])
    np.testing.assert_array_equal(sc[64:], c[::64])
    np.testing.assert_array_equal(ss[64:], s[::64])


def _rope_coefficients(pos, d_h, theta, split):
    """(c, s) per position and pair, read back through the fp32 sequence: a half-style
    row (1, ..., 1, 0, ..., 0) leaves RoPE as a' = fma(1, c, -(0*s)) = c, b' = s."""
    T = len(pos)
    row = np.concatenate([np.full(d_h // 2, 0x3F80, np.uint16), np.zeros(d_h // 2, np.uint16)])
    x = np.broadcast_to(row, (T, 1, d_h)).copy()
    out = B.transform_quantize(x, x, np.asarray(pos, np.int32), d_h, theta=theta,
                               mode="rope_only", group=d_h, want_f32=True, split=split,
                               max_pos=int(max(pos)) + 1)
    kf = out["k_f32"][:, 0]
    return kf[:, : d_h // 2], kf[:, d_h // 2:]


def test_split_composition_is_exact_where_a_row_is_the_identity():
    """At positions 64 h the low row is (1, 0), and below 64 the high row is (1, 0): the
    composition is then exact and equals the plain table entry."""
    pos = np.concatenate([np.arange(0, 131072, 64 * 97), np.arange(64)])
    c1, s1 = _rope_coefficients(pos, 128, 5e5, split=True)
    c0, s0 = _rope_coefficients(pos, 128, 5e5, split=False)
    np.testing.assert_array_equal(c1, c0)
    np.testing.assert_array_equal(s1, s0)


def test_split_coefficients_within_rounding_bound_of_fp64():
    """|c - cos(m w_k)| and |s - sin(m w_k)| stay below (2 sqrt 2 + 2) * 2^-25: four table
    entries each within half an ulp (<= 2^-25, magnitudes <= 1), one rounded product and
    the fused multiply-add's rounding.  Checked over positions up to 131071."""
    d_h, theta = 128, 5e5
    pos = np.unique(np.concatenate([RNG.integers(0, 131072, 3000), [63, 64, 65, 131071]]))
    c, s = _rope_coefficients(pos, d_h, theta, split=True)
    w = theta ** (-(2.0 * np.arange(d_h // 2)) / d_h)
    ang = pos[:, None].astype(np.float64) * w[None, :]
    bound = (2 * math.sqrt(2) + 2) * 2.0 ** -25
    assert np.abs(c - np.cos(ang)).max() <= bound
    assert np.abs(s - np.sin(ang)).max() <= bound
    # and the composition is not a no-op: it differs from the plain table somewhere
    c0, _ = _rope_coefficients(pos, d_h, theta, split=False)
    assert (c != c0).any()


def test_block_b_equals_full_head_bit_exact():
    """b = d_h is the full-head Hadamard, bit for bit in the fp32 sequence."""
    for name in ("tiny", "llama32_3b"):
        w = synth.WORKLOADS[name]
        inp = synth.make_inputs(name, T=32)
        a = B.transform_quantize(inp["q"], inp["k"], inp["pos"], w.d_h, theta=w.theta,
                                 mode="hadamard", group=w.group, want_f32=True)
        c = B.transform_quantize(inp["q"], inp["k"], inp["pos"], w.d_h, theta=w.theta,
                                 mode="block_hadamard", b=w.d_h, group=w.group, want_f32=True)
        for key in ("q_out", "k_codes", "k_scales", "k_f32", "q_f32"):
            np.testing.assert_array_equal(a[key], c[key])


def test_pairwise_zero_angle_is_rope_only():
    w = synth.WORKLOADS["tiny"]
    inp = synth.make_inputs("tiny", T=16)
    a = B.transform_quantize(inp["q"], inp["k"], inp["pos"], w.d_h, theta=w.theta,
                             mode="pairwise", phi=np.zeros(w.P, np.float32), group=w.group,
                             want_f32=True)
    c = B.transform_quantize(inp["q"], inp["k"], inp["pos"], w.d_h, theta=w.theta,
                             mode="rope_only", group=w.group, want_f32=True)
    np.testing.assert_array_equal(a["k_f32"], c["k_f32"])
    np.testing.assert_array_equal(a["q_out"], c["q_out"])


def test_quantizer_hand_groups_fp32(golden_dir):
    """The hand-worked groups of "LLM旋转量化笔记" §1.2, through the fp32 sequence
    (mode rope_only at position 0 leaves the row unchanged)."""
    import os
    rows = []
    with open(os.path.join(golden_dir, "quantizer_groups.txt"), encoding="utf-8") as f:
        for ln in f:
            if ln.strip() and not ln.lstrip().startswith("#"):
                rows.append(ln)
    for r in rows:
        xs, cs, bs, sc = [p.split() for p in r.split("|")]
        x = np.array([float(v) for v in xs], dtype=np.float32)
        k = synth.f32_to_bf16_bits(np.tile(x, 4)).reshape(1, 1, 32)   # d_h = 32, 4 groups of 8
        xb = synth.bf16_bits_to_f32(k).ravel()[:8]
        if not (xb == x).all():
            # values not exact in bf16 (in G3, G5): rounding them moves no x/s across
            # a rounding midpoint, so the hand-worked codes still hold
            moved = xb != x
            assert np.abs(xb).max() == np.abs(x).max()
            v = np.abs(xb.astype(np.float64) * 7.0 / np.abs(x).max())[moved]
            assert (np.abs(v - np.floor(v) - 0.5) > 0.02).all()
        q = np.zeros((1, 1, 32), np.uint16)
        out = B.transform_quantize(q, k, np.array([0], np.int32), 32, theta=1e4,
                                   mode="rope_only", group=8, max_pos=1)
        np.testing.assert_array_equal(D.unpack_int4(out["k_codes"])[0, 0, :8],
                                      [int(v) for v in cs])
        np.testing.assert_array_equal(out["k_codes"][0, 0, :4], [int(v, 16) for v in bs])
        assert out["k_scales"][0, 0, 0] == int(sc[0], 16)


# ------------------------------------------------------------ status bits -------

def test_status_bits():
    w = synth.WORKLOADS["tiny"]
    inp = synth.make_inputs("tiny", T=8)
    k = inp["k"].copy()
    k[3, 1, 5] = 0x7FC0                                     # NaN
    out = B.transform_quantize(inp["q"], k, inp["pos"], w.d_h, theta=w.theta, group=w.group)
    assert out["status"] & 1
    k = inp["k"].copy()
    k[2, 0, :] = synth.f32_to_bf16_bits(np.full(w.d_h, 5.0e5, np.float32))   # s > 65504
    out = B.transform_quantize(inp["q"], k, inp["pos"], w.d_h, theta=w.theta, group=w.group,
                               mode="rope_only")
    assert out["status"] == 2
    pos = inp["pos"].copy()
    pos[4] = 10_000
    cos_t, sin_t = B.rope_table(256, w.d_h, w.theta)
    out = B.transform_quantize(inp["q"], inp["k"], pos, w.d_h, cos_t=cos_t, sin_t=sin_t,
                               group=w.group)
    assert out["status"] == 4
    pos2 = pos.copy()
    pos2[4] = 255                                            # clamped row
    ref = B.transform_quantize(inp["q"], inp["k"], pos2, w.d_h, cos_t=cos_t, sin_t=sin_t,
                               group=w.group)
    np.testing.assert_array_equal(out["k_codes"], ref["k_codes"])


def test_zero_and_tiny_groups():
    d = 64
    k = np.zeros((2, 1, d), np.uint16)
    k[1, 0, 7] = synth.f32_to_bf16_bits(np.array([1e-39], np.float32))[0]  # subnormal bf16
    q = np.zeros((2, 1, d), np.uint16)
    out = B.transform_quantize(q, k, np.array([0, 0], np.int32), d, theta=1e4, mode="rope_only",
                               group=32, max_pos=1)
    assert (out["k_codes"] == 0).all() and (out["k_scales"] == 0).all()
    assert out["status"] == 0


# ---------------------------------------- the order of the steps, one rounding each -----

def _fma32(a, b, c):
    """fp32 fused multiply-add, emulated exactly: a*b is exact in float64 for fp32 a and b;
    the sum with c is split error-free (two-sum) and rounded once to fp32, the float64
    part's own rounding undone where it lands on an fp32 midpoint."""
    a, b, c = (np.asarray(v, dtype=np.float32).astype(np.float64) for v in (a, b, c))
    p = a * b
    s = p + c
    bb = s - p
    err = (p - (s - bb)) + (c - bb)
    r = s.astype(np.float32)
    # s is an fp32 midpoint iff both neighbours are equally far; then err decides
    up = np.nextafter(r, np.float32(np.inf)).astype(np.float64)
    dn = np.nextafter(r, np.float32(-np.inf)).astype(np.float64)
    r64 = r.astype(np.float64)
    lo = np.where(s >= r64, r64, dn)
    hi = np.where(s >= r64, up, r64)
    mid = (s - lo) == (hi - s)
    pick_hi = np.where(mid & (err != 0), err > 0, s - lo > hi - s)
    out = np.where(mid & (err == 0), r64, np.where(pick_hi, hi, lo))
    return out.astype(np.float32)


def test_fma32_emulation():
    """The emulation against exact rational arithmetic on random and tie-breaking cases."""
    from fractions import Fraction
    r = np.random.default_rng(11)
    a = r.standard_normal(2000).astype(np.float32)
    b = r.standard_normal(2000).astype(np.float32)
    c = (r.standard_normal(2000) * np.exp(r.uniform(-20, 5, 2000))).astype(np.float32)
    # products that cancel against c almost exactly
    c[:500] = -(a[:500].astype(np.float64) * b[:500]).astype(np.float32)
    got = _fma32(a, b, c)
    for i in range(2000):
        exact = Fraction(float(a[i])) * Fraction(float(b[i])) + Fraction(float(c[i]))
        x = np.float32(float(exact))
        cand = [np.nextafter(x, np.float32(-np.inf)), x, np.nextafter(x, np.float32(np.inf))]
        d = [abs(Fraction(float(v)) - exact) for v in cand]
        best = min(d)
        ok = [v for v, dd in zip(cand, d) if dd == best]
        if len(ok) == 2:  # tie: even mantissa
            ok = [v for v in ok if (int(np.float32(v).view(np.uint32)) & 1) == 0]
        assert got[i] == ok[0], i


def _rotate32(rows, c, s, style):
    """The pair rotation a' = fma(a, c, -(b*s)), b' = fma(a, s, b*c) on fp32 rows."""
    d_h = rows.shape[-1]
    ia, ib = D.pair_channels(d_h, style)
    a, b = rows[..., ia], rows[..., ib]
    bs = (b * s).astype(np.float32)
    bc = (b * c).astype(np.float32)
    out = rows.copy()
    out[..., ia] = _fma32(a, c, -bs)
    out[..., ib] = _fma32(a, s, bc)
    return out


@pytest.mark.parametrize("style", ["half", "interleaved"])
@pytest.mark.parametrize("wname", ["tiny", "llama31_8b_128k"])
def test_pairwise_is_rope_then_pair_rotation(style, wname):
    """The pairwise modes take RoPE and the pair rotation in the method's order, each as
    its own rounded step ("Methodology" items 2 and 3 of the paper summary): the pairwise
    output equals the RoPE-only output turned by phi with the rotation's fp32 steps, and
    pairwise + Hadamard equals the fast Walsh-Hadamard transform of that, times
    fp32(1/sqrt(d_h)) — bit for bit."""
    w = synth.WORKLOADS[wname]
    inp = synth.make_inputs(wname, T=24)
    pos = _spread_positions(w, 24) if wname != "tiny" else inp["pos"][:24]
    phi = RNG.uniform(-math.pi / 4, math.pi / 4, w.P).astype(np.float32)
    ct, st = _tables(wname, False)
    run = lambda mode: B.transform_quantize(inp["q"], inp["k"], pos, w.d_h, cos_t=ct, sin_t=st,
                                            mode=mode, group=w.d_h, phi=phi, style=style,
                                            want_f32=True)
    rope, pw, pwh = run("rope_only"), run("pairwise"), run("pairwise_hadamard")
    cphi = np.cos(phi.astype(np.float64)).astype(np.float32)
    sphi = np.sin(phi.astype(np.float64)).astype(np.float32)
    kappa = np.float32(1.0 / math.sqrt(w.d_h))
    for key in ("q_f32", "k_f32"):
        turned = _rotate32(rope[key], cphi, sphi, style)
        np.testing.assert_array_equal(pw[key].view(np.uint32), turned.view(np.uint32))
        mixed = np.stack([B.fwht(r) for r in turned.reshape(-1, w.d_h)]).reshape(turned.shape)
        np.testing.assert_array_equal(pwh[key].view(np.uint32),
                                      (mixed * kappa).astype(np.float32).view(np.uint32))
