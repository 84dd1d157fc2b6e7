"""GPU parity of the calibration side path (qkq_accumulate_moments, qkq_solve_angles)
and of the measurement path (qkq_dequant_error, qkq_dequant_error_recompute) with the
oracle.

Moments: the kernel and the oracle sum the same fp32 post-RoPE values in fp64 (products
exact), so they agree to summation-order rounding (rtol 1e-12).  Angles: within 1e-5
rad modulo pi/2 (phi and phi + pi/2 are equally optimal); for near-isotropic pairs
(|A - D| + 2|C| < 1e-3 tr) the attained objective is compared instead.  Statistics:
the squared-error and reference sums (fp32 per lane and group) to
1.43e-6 relative, the group-range sums to 1e-10, the maximum and the group count exactly.
"""
import math

import numpy as np
import pytest

from tests import gpu_common as G

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import transform_rope_head_b200 as qkq  # noqa: E402
from oracle import bitspec as B  # noqa: E402
from oracle import definition as D  # noqa: E402

ESTS = ("pooled", "k_only", "balanced")


def oracle_post_rope(d: G.DevInputs, style: str, split: bool = False):
    """Post-RoPE, pre-mixing rows in fp32, from the oracle's fp32 sequence."""
    w = d.w
    table = B.rope_table_split if split else B.rope_table
    oc, os_ = table(d.max_pos, w.d_h, w.theta)
    r = B.transform_quantize(d.inp["q"], d.inp["k"], d.inp["pos"], w.d_h, cos_t=oc, sin_t=os_,
                             mode="rope_only", group=w.d_h, style=style, want_f32=True,
                             split=split, max_pos=d.max_pos)
    return r["q_f32"], r["k_f32"]


def circ(a, b):
    dd = (a - b) % (math.pi / 2)
    return np.minimum(dd, math.pi / 2 - dd)


def check_angles(phi_gpu, m_ref, est):
    phi_ref = D.solve_angles(m_ref, est)
    A, C, Dd = D.covariance(m_ref, est)
    tr = A + Dd
    well = np.abs(A - Dd) + 2 * np.abs(C) >= 1e-3 * tr
    assert (circ(phi_gpu[well].astype(np.float64), phi_ref[well]) < 1e-5).all()
    v1, v2 = D.channel_variances(A, C, Dd, phi_gpu.astype(np.float64))
    obj = np.maximum(v1, v2)
    np.testing.assert_allclose(obj[~well], tr[~well] / 2, rtol=1e-6)


@pytest.mark.parametrize("name,T,style", [("tiny", None, "half"), ("tiny", None, "interleaved"),
                                          ("llama32_1b", None, "half"),
                                          ("llama32_3b", 2000, "half"),
                                          ("llama32_3b", 777, "interleaved"),
                                          ("mistral7b_decode", None, "half")])
def test_moments_match_oracle(name, T, style):
    d = G.DevInputs(G.draw(name, T=T))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    m = qkq.accumulate_moments(d.q, d.k, d.pos, d.cos, d.sin, rope_style=style, status=st)
    got = m.cpu().numpy()
    qf, kf = oracle_post_rope(d, style)
    ref = D.moments(qf, kf, style)
    np.testing.assert_array_equal(got[:, :, 0], ref[:, :, 0])
    scale = np.abs(ref).max(axis=(0, 1), keepdims=True)
    assert (np.abs(got - ref) <= 1e-12 * scale + 1e-12 * np.abs(ref)).all()
    assert int(st.item()) == 0
    # accumulators are ADDED TO: a second call doubles them
    qkq.accumulate_moments(d.q, d.k, d.pos, d.cos, d.sin, m, rope_style=style)
    np.testing.assert_allclose(m.cpu().numpy(), 2 * got, rtol=1e-14)


@pytest.mark.parametrize("name,T,style", [("tiny", None, "interleaved"),
                                          ("llama32_3b", 1200, "half"),
                                          ("mistral7b_decode", None, "half")])
def test_moments_split_table_match_oracle(name, T, style):
    d = G.DevInputs(G.draw(name, T=T))
    ct, st_, kw = d.tables(True)
    m = qkq.accumulate_moments(d.q, d.k, d.pos, ct, st_, rope_style=style, **kw)
    got = m.cpu().numpy()
    qf, kf = oracle_post_rope(d, style, split=True)
    ref = D.moments(qf, kf, style)
    np.testing.assert_array_equal(got[:, :, 0], ref[:, :, 0])
    scale = np.abs(ref).max(axis=(0, 1), keepdims=True)
    assert (np.abs(got - ref) <= 1e-12 * scale + 1e-12 * np.abs(ref)).all()


def test_moments_calibration_batches_add_up():
    """The 1B calibration set drawn in 4 batches of 2 x 2048 tokens equals one big call."""
    inp = G.draw("llama32_1b", T=4 * 4096, seed=1102)
    d = G.DevInputs(inp)
    whole = qkq.accumulate_moments(d.q, d.k, d.pos, d.cos, d.sin).cpu().numpy()
    acc = None
    for i in range(4):
        s = slice(i * 4096, (i + 1) * 4096)
        acc = qkq.accumulate_moments(d.q[s], d.k[s], d.pos[s], d.cos, d.sin, acc)
    np.testing.assert_allclose(acc.cpu().numpy(), whole, rtol=1e-12)


@pytest.mark.parametrize("est", ESTS)
@pytest.mark.parametrize("name", ["tiny", "llama32_1b", "mistral7b_decode"])
def test_solve_on_oracle_moments(name, est):
    d = G.DevInputs(G.draw(name))
    qf, kf = oracle_post_rope(d, "half")
    m_ref = D.moments(qf, kf)
    mm = torch.empty(d.w.P, dtype=torch.float64, device="cuda")
    phi = qkq.solve_angles(torch.from_numpy(m_ref).cuda(), est, min_maxvar=mm).cpu().numpy()
    assert ((phi > -math.pi / 4) & (phi <= math.pi / 4 + 1e-7)).all()
    check_angles(phi, m_ref, est)
    A, C, Dd = D.covariance(m_ref, est)
    np.testing.assert_allclose(mm.cpu().numpy(), (A + Dd) / 2, rtol=1e-9)


@pytest.mark.parametrize("est", ESTS)
def test_end_to_end_calibration(est):
    """GPU moments -> GPU angles vs oracle moments -> oracle angles (1B shape)."""
    d = G.DevInputs(G.draw("llama32_1b"))
    m = qkq.accumulate_moments(d.q, d.k, d.pos, d.cos, d.sin)
    phi = qkq.solve_angles(m, est).cpu().numpy()
    qf, kf = oracle_post_rope(d, "half")
    check_angles(phi, D.moments(qf, kf), est)


def test_estimators_differ_on_anisotropic_data():
    d = G.DevInputs(G.draw("llama32_1b"))
    m = qkq.accumulate_moments(d.q, d.k, d.pos, d.cos, d.sin)
    ph = [qkq.solve_angles(m, e).cpu().numpy() for e in ESTS]
    assert np.abs(ph[0] - ph[1]).max() > 1e-3 and np.abs(ph[0] - ph[2]).max() > 1e-3


@pytest.mark.parametrize("est", ESTS)
def test_solve_reports_empty_streams(est):
    """Pairs whose estimator needs a stream without observations get phi = 0 and the
    empty-stream status bit, as the oracle's reading says; the other pairs are solved as
    usual and a call without such pairs leaves the status at 0."""
    d = G.DevInputs(G.draw("tiny"))
    qf, kf = oracle_post_rope(d, "half")
    m = D.moments(qf, kf)
    m[0, :8] = 0.0     # pairs 0-7: no Q observations
    m[1, 8:16] = 0.0   # pairs 8-15: no K observations
    m[:, 16:20] = 0.0  # pairs 16-19: neither
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    mm = torch.empty(d.w.P, dtype=torch.float64, device="cuda")
    phi = qkq.solve_angles(torch.from_numpy(m).cuda(), est, min_maxvar=mm,
                           status=status).cpu().numpy()
    empty = D.empty_streams(m, est)
    assert empty.any()
    assert int(status.item()) == qkq.STATUS_BITS["empty_stream"]
    np.testing.assert_array_equal(phi[empty], 0.0)
    assert np.isnan(mm.cpu().numpy()[empty]).all()
    ok = ~empty
    ref = D.solve_angles(m, est)
    dphi = np.abs(phi[ok].astype(np.float64) - ref[ok]) % (math.pi / 2)
    assert np.minimum(dphi, math.pi / 2 - dphi).max() < 1e-5
    status.zero_()
    qkq.solve_angles(torch.from_numpy(D.moments(qf, kf)).cuda(), est, status=status)
    assert int(status.item()) == 0


def test_solve_special_cases():
    """C = 0, A > D -> pi/4; A = D -> 0; isotropic -> 0 (both streams identical)."""
    P = 32
    m = np.zeros((2, P, 6))
    for s in range(2):
        m[s, :, 0] = 100.0
        m[s, 0, 3], m[s, 0, 5] = 300.0, 100.0           # A = 3, D = 1, C = 0
        m[s, 1, 3], m[s, 1, 4], m[s, 1, 5] = 200.0, 70.0, 200.0  # A = D
        m[s, 2, 3], m[s, 2, 5] = 100.0, 100.0           # isotropic
        m[s, 3:, 3], m[s, 3:, 5] = 100.0, 200.0
    phi = qkq.solve_angles(torch.from_numpy(m).cuda(), "pooled").cpu().numpy()
    assert phi[0] == np.float32(math.pi / 4)
    assert phi[1] == 0.0 and phi[2] == 0.0


# ------------------------------------------------------------ measurement ---------

@pytest.mark.parametrize("name,T,mode,b,group,style", [
    ("tiny", None, "hadamard", 0, 64, "half"),
    ("tiny", None, "pairwise", 0, 32, "interleaved"),
    ("llama32_3b", 1500, "pairwise_hadamard", 0, 128, "half"),
    ("llama32_3b", 1500, "block_hadamard", 8, 32, "half"),
    ("mistral7b_decode", None, "block_hadamard", 2, 128, "half"),
    ("mistral7b_decode", None, "block_hadamard", 128, 128, "half"),
    ("llama31_8b_128k", 3000, "rope_only", 0, 64, "half"),
])
def test_dequant_error_matches_oracle(name, T, mode, b, group, style):
    d = G.DevInputs(G.draw(name, T=T))
    phi = G.random_phi(d.w.P, seed=21) if "pairwise" in mode else None
    phi_d = None if phi is None else torch.from_numpy(phi).cuda()
    _, codes, scales, _ = qkq.transform_quantize(d.q, d.k, d.pos, d.cos, d.sin, mode=mode, b=b,
                                                 group=group, phi=phi_d, rope_style=style)
    st = qkq.dequant_error_recompute(d.k, d.pos, d.cos, d.sin, codes, scales, mode=mode, b=b, group=group,
                           phi=phi_d, rope_style=style).cpu().numpy()
    w = d.w
    oc, os_ = B.rope_table(d.max_pos, w.d_h, w.theta)
    r = B.transform_quantize(d.inp["q"], d.inp["k"], d.inp["pos"], w.d_h, cos_t=oc, sin_t=os_,
                             mode=mode, b=b or None, group=group, phi=phi, style=style,
                             want_f32=True)
    ref = D.dequant_stats(r["k_f32"], D.unpack_int4(r["k_codes"]), r["k_scales"], group)
    # sum (x~ - K^)^2 and sum x~^2: fp32 sums of at most 16 non-negative terms per lane and
    # group (d_h 128), each term carrying up to 6 roundings, then 2 more before the fp64
    # total: relative error below (16 + 8) * 2^-24 = 1.43e-6
    np.testing.assert_allclose(st[[0, 1]], ref[[0, 1]], rtol=24 * 2.0 ** -24)
    # group max|x~| and max - min: fp32 values added in fp64
    np.testing.assert_allclose(st[[2, 3]], ref[[2, 3]], rtol=1e-10)
    assert st[4] == ref[4] and st[5] == ref[5]
    assert 0.0 < qkq.rel_error(st) < 0.5


@pytest.mark.parametrize("mode,b,style", [("pairwise_hadamard", 0, "half"),
                                          ("block_hadamard", 16, "interleaved")])
def test_dequant_error_split_table(mode, b, style):
    d = G.DevInputs(G.draw("llama32_3b", T=900))
    ct, st_, kw = d.tables(True)
    phi = G.random_phi(d.w.P, seed=23) if "pairwise" in mode else None
    phi_d = None if phi is None else torch.from_numpy(phi).cuda()
    _, codes, scales, _ = qkq.transform_quantize(d.q, d.k, d.pos, ct, st_, mode=mode, b=b,
                                                 group=32, phi=phi_d, rope_style=style, **kw)
    st = qkq.dequant_error_recompute(d.k, d.pos, ct, st_, codes, scales, mode=mode, b=b, group=32,
                           phi=phi_d, rope_style=style, **kw).cpu().numpy()
    w = d.w
    oc, os_ = B.rope_table_split(d.max_pos, w.d_h, w.theta)
    r = B.transform_quantize(d.inp["q"], d.inp["k"], d.inp["pos"], w.d_h, cos_t=oc, sin_t=os_,
                             mode=mode, b=b or None, group=32, phi=phi, style=style,
                             want_f32=True, split=True, max_pos=d.max_pos)
    ref = D.dequant_stats(r["k_f32"], D.unpack_int4(r["k_codes"]), r["k_scales"], 32)
    np.testing.assert_allclose(st[[0, 1]], ref[[0, 1]], rtol=24 * 2.0 ** -24)
    np.testing.assert_allclose(st[[2, 3]], ref[[2, 3]], rtol=1e-10)
    assert st[4] == ref[4] and st[5] == ref[5]


def test_support_sweep_k_range_falls_with_b():
    """Mixing support interpolation on the decode shape: K range at b = d_h is below
    b = 2 ("Results": K range falls as the support grows; reported, with the
    full sweep, by the benchmark)."""
    d = G.DevInputs(G.draw("mistral7b_decode"))
    kr = {}
    for b in (2, 128):
        _, codes, scales, _ = qkq.transform_quantize(d.q, d.k, d.pos, d.cos, d.sin,
                                                     mode="block_hadamard", b=b)
        st = qkq.dequant_error_recompute(d.k, d.pos, d.cos, d.sin, codes, scales, mode="block_hadamard",
                               b=b)
        kr[b] = qkq.k_range(st)
    assert kr[128] < kr[2]


@pytest.mark.parametrize("mode,group", [("rope_only", 32), ("pairwise_hadamard", 128)])
def test_dequant_error_edge_groups(mode, group):
    """Planted key rows at the corners of the per-group normalisation: a zero row (zero
    groups, scale 0), rows scaled to 1e-30 and 1e-6 (scales that underflow fp16 to 0 or
    to a subnormal while the codes are nonzero) and a row scaled by 100 (large scales)."""
    import synth
    inp = G.draw("llama32_3b", T=24)
    k = inp["k"].copy()
    base = synth.bf16_bits_to_f32(k)
    k[3] = 0
    for t, f in ((5, 1e-30), (9, 1e-6), (13, 1e2)):
        k[t] = synth.f32_to_bf16_bits((base[t] * np.float32(f)).astype(np.float32))
    inp = dict(inp, k=k)
    d = G.DevInputs(inp)
    phi = G.random_phi(d.w.P, seed=5) if "pairwise" in mode else None
    phi_d = None if phi is None else torch.from_numpy(phi).cuda()
    _, codes, scales, _ = qkq.transform_quantize(d.q, d.k, d.pos, d.cos, d.sin, mode=mode,
                                                 group=group, phi=phi_d)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = qkq.dequant_error_recompute(d.k, d.pos, d.cos, d.sin, codes, scales, mode=mode, group=group,
                           phi=phi_d, status=status).cpu().numpy()
    assert int(status.item()) == 0
    w = d.w
    oc, os_ = B.rope_table(d.max_pos, w.d_h, w.theta)
    r = B.transform_quantize(inp["q"], inp["k"], inp["pos"], w.d_h, cos_t=oc, sin_t=os_,
                             mode=mode, group=group, phi=phi, want_f32=True)
    assert (r["k_scales"][5] == 0).all() and (D.unpack_int4(r["k_codes"][5]) != 0).any()
    ref = D.dequant_stats(r["k_f32"], D.unpack_int4(r["k_codes"]), r["k_scales"], group)
    np.testing.assert_allclose(st[[0, 1]], ref[[0, 1]], rtol=24 * 2.0 ** -24)
    np.testing.assert_allclose(st[[2, 3]], ref[[2, 3]], rtol=1e-10)
    assert st[4] == ref[4] and st[5] == ref[5]


def test_dequant_error_flags_overflowed_scales():
    """A group whose scale overflows fp16 dequantises to inf / NaN: the squared error is
    then non-finite on both sides and the measurement reports ST_NONFINITE."""
    import synth
    inp = G.draw("llama32_3b", T=8)
    k = inp["k"].copy()
    k[2, 0, :] = synth.f32_to_bf16_bits(np.full(128, 5.0e5, np.float32))
    inp = dict(inp, k=k)
    d = G.DevInputs(inp)
    st_t = torch.zeros(1, dtype=torch.int32, device="cuda")
    _, codes, scales, _ = qkq.transform_quantize(d.q, d.k, d.pos, d.cos, d.sin, mode="hadamard",
                                                 status=st_t)
    assert int(st_t.item()) == 2
    st_m = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = qkq.dequant_error_recompute(d.k, d.pos, d.cos, d.sin, codes, scales, mode="hadamard",
                           status=st_m).cpu().numpy()
    assert int(st_m.item()) == 1 and not np.isfinite(st[0])
    w = d.w
    oc, os_ = B.rope_table(d.max_pos, w.d_h, w.theta)
    r = B.transform_quantize(inp["q"], inp["k"], inp["pos"], w.d_h, cos_t=oc, sin_t=os_,
                             mode="hadamard", want_f32=True)
    with np.errstate(all="ignore"):
        ref = D.dequant_stats(r["k_f32"], D.unpack_int4(r["k_codes"]), r["k_scales"], w.d_h)
    assert not np.isfinite(ref[0])


# ------------------------------------- measurement of a given fp32 K~ (qkq_dequant_error) --

def _stats_bar(st, ref):
    """The measurement's bar (see test_dequant_error_matches_oracle)."""
    np.testing.assert_allclose(st[[0, 1]], ref[[0, 1]], rtol=24 * 2.0 ** -24)
    np.testing.assert_allclose(st[[2, 3]], ref[[2, 3]], rtol=1e-10)
    assert st[4] == ref[4] and st[5] == ref[5]


@pytest.mark.parametrize("name,T,mode,b,group", [
    ("tiny", None, "pairwise", 0, 32),
    ("llama32_3b", 1501, "pairwise_hadamard", 0, 128),
    ("llama32_3b", 1501, "block_hadamard", 8, 32),
    ("llama31_8b_128k", 2999, "hadamard", 0, 64),
    ("mistral7b_decode", None, "block_hadamard", 2, 128),
])
def test_dequant_error_given_k_matches_definition(name, T, mode, b, group):
    """qkq_dequant_error on the butterfly transform's fp32 K~ and codes: the statistics of the
    fp64 definition (oracle.definition.dequant_stats) on the same K~, codes and scales, within
    the measurement's bar; and the recomputing call agrees within it too."""
    d = G.DevInputs(G.draw(name, T=T))
    phi = G.random_phi(d.w.P, seed=31) if "pairwise" in mode else None
    phi_d = None if phi is None else torch.from_numpy(phi).cuda()
    _, codes, scales, kf = qkq.transform_quantize(d.q, d.k, d.pos, d.cos, d.sin, mode=mode, b=b,
                                                  group=group, phi=phi_d, want_k_f32=True)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = qkq.dequant_error(kf, codes, scales, status=status).cpu().numpy()
    assert int(status.item()) == 0
    ref = D.dequant_stats(kf.cpu().numpy(), D.unpack_int4(codes.cpu().numpy()),
                          G.bits16(scales), group)
    _stats_bar(st, ref)
    again = qkq.dequant_error_recompute(d.k, d.pos, d.cos, d.sin, codes, scales, mode=mode, b=b,
                                        group=group, phi=phi_d).cpu().numpy()
    _stats_bar(again, ref)
    summ = qkq.dequant_summary(st)
    assert summ["k_range"] == pytest.approx(D.k_range(ref), rel=1e-10)
    assert summ["rel_error"] == pytest.approx(D.rel_error(ref), rel=2e-6)


@pytest.mark.parametrize("mode,b", [("hadamard", 0), ("pairwise_hadamard", 0),
                                    ("block_hadamard", 16)])
def test_dequant_error_measures_tensor_core_codes(mode, b):
    """The codes of the tensor-core variant, measured against its own fp32 K~ (which the
    recomputing call cannot reproduce: its K~ is not the butterfly's)."""
    d = G.DevInputs(G.draw("llama32_3b", T=700))
    phi = G.random_phi(d.w.P, seed=33) if "pairwise" in mode else None
    phi_d = None if phi is None else torch.from_numpy(phi).cuda()
    _, codes, scales, kf = qkq.transform_quantize_tc(d.q, d.k, d.pos, d.cos, d.sin, mode=mode,
                                                     b=b, group=32, phi=phi_d, want_k_f32=True)
    st = qkq.dequant_error(kf, codes, scales).cpu().numpy()
    ref = D.dequant_stats(kf.cpu().numpy(), D.unpack_int4(codes.cpu().numpy()),
                          G.bits16(scales), 32)
    _stats_bar(st, ref)


def test_dequant_error_measures_value_rows():
    """Value rows of the fused Q/K/V launch: their codes against their fp32 V~."""
    inp = G.draw("llama32_3b", T=600)
    d = G.DevInputs(inp)
    v = G.to_dev_bf16(np.ascontiguousarray(inp["k"][::-1]))   # a second block of rows
    out = qkq.transform_quantize_qkv(d.q, d.k, v, d.pos, d.cos, d.sin, mode="hadamard",
                                     group=64, want_f32=True)
    v_codes, v_scales, vf = out[3], out[4], out[6]
    st = qkq.dequant_error(vf, v_codes, v_scales).cpu().numpy()
    ref = D.dequant_stats(vf.cpu().numpy(), D.unpack_int4(v_codes.cpu().numpy()),
                          G.bits16(v_scales), 64)
    _stats_bar(st, ref)


def test_dequant_error_given_k_empty_and_workspace():
    kf = torch.zeros((0, 8, 128), dtype=torch.float32, device="cuda")
    codes = torch.zeros((0, 8, 64), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((0, 8, 1), dtype=torch.float16, device="cuda")
    st = qkq.dequant_error(kf, codes, scales).cpu().numpy()
    np.testing.assert_array_equal(st, np.zeros(6))
    kf = torch.zeros((5, 8, 128), dtype=torch.float32, device="cuda")
    codes = torch.zeros((5, 8, 64), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((5, 8, 1), dtype=torch.float16, device="cuda")
    with pytest.raises(qkq.QKQError):
        qkq.dequant_error(kf, codes, scales, workspace=torch.zeros(8, dtype=torch.uint8,
                                                                   device="cuda"))
    # all-zero keys: zero groups, no error, no NaN
    st = qkq.dequant_error(kf, codes, scales).cpu().numpy()
    np.testing.assert_array_equal(st, [0, 0, 0, 0, 0, 40])


# ------------------------------------------------ statistics fused into the transform --

@pytest.mark.parametrize("name,T,mode,b,group,style,split", [
    ("tiny", None, "pairwise_hadamard", 0, 32, "interleaved", False),
    ("llama32_3b", 1500, "pairwise_hadamard", 0, 128, "half", False),
    ("llama32_3b", 1500, "block_hadamard", 8, 32, "half", True),
    ("mistral7b_decode", None, "hadamard", 0, 64, "half", False),
    ("llama31_8b_128k", 3000, "rope_only", 0, 128, "half", False),
])
def test_transform_stats_match_oracle_and_standalone(name, T, mode, b, group, style, split):
    """qkq_transform_quantize_stats: outputs equal the plain launch bit for bit; the fused
    statistics equal the oracle's within the measurement's bar and agree with
    qkq_dequant_error's (same definitions, another summation order)."""
    d = G.DevInputs(G.draw(name, T=T))
    ct, sn, kw = d.tables(split)
    phi = G.random_phi(d.w.P, seed=61) if "pairwise" in mode else None
    phi_d = None if phi is None else torch.from_numpy(phi).cuda()
    st_f = torch.zeros(1, dtype=torch.int32, device="cuda")
    q1, c1, s1, stats = qkq.transform_quantize_stats(d.q, d.k, d.pos, ct, sn, mode=mode, b=b,
                                                     group=group, phi=phi_d, rope_style=style,
                                                     status=st_f, **kw)
    q0, c0, s0, _ = qkq.transform_quantize(d.q, d.k, d.pos, ct, sn, mode=mode, b=b, group=group,
                                           phi=phi_d, rope_style=style, **kw)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(G.bits16(q1), G.bits16(q0))
    np.testing.assert_array_equal(c1.cpu().numpy(), c0.cpu().numpy())
    np.testing.assert_array_equal(G.bits16(s1), G.bits16(s0))
    assert int(st_f.item()) == 0
    got = stats.cpu().numpy()
    alone = qkq.dequant_error_recompute(d.k, d.pos, ct, sn, c0, s0, mode=mode, b=b, group=group, phi=phi_d,
                              rope_style=style, **kw).cpu().numpy()
    w = d.w
    tab = B.rope_table_split if split else B.rope_table
    oc, os_ = tab(d.max_pos, w.d_h, w.theta)
    r = B.transform_quantize(d.inp["q"], d.inp["k"], d.inp["pos"], w.d_h, cos_t=oc, sin_t=os_,
                             mode=mode, b=b or None, group=group, phi=phi, style=style,
                             want_f32=True, split=split, max_pos=d.max_pos)
    ref = D.dequant_stats(r["k_f32"], D.unpack_int4(r["k_codes"]), r["k_scales"], group)
    for st in (got, alone):
        np.testing.assert_allclose(st[[0, 1]], ref[[0, 1]], rtol=24 * 2.0 ** -24)
        np.testing.assert_allclose(st[[2, 3]], ref[[2, 3]], rtol=1e-10)
        assert st[4] == ref[4] and st[5] == ref[5]


def test_transform_stats_empty_and_workspace_checks():
    d = G.DevInputs(G.draw("tiny", T=8))
    e = d.q[:0]
    out = qkq.transform_quantize_stats(e, d.k[:0], d.pos[:0], d.cos, d.sin)
    torch.cuda.synchronize()
    assert (out[3].cpu().numpy() == 0).all()
    with pytest.raises(qkq.QKQError):
        qkq.transform_quantize_stats(d.q, d.k, d.pos, d.cos, d.sin,
                                     workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))


@pytest.mark.parametrize("factor", [1e-39, 1e-20, 1e30])
def test_moments_extreme_magnitudes(factor):
    """Rows scaled into the fp32 subnormal range, near its bottom, and large: the fp64 sums
    of exact products still match the oracle (both channels of every pair, including the
    second, which the kernel widens with integer operations)."""
    import synth
    inp = G.draw("llama32_3b", T=64)
    base_q = synth.bf16_bits_to_f32(inp["q"])
    base_k = synth.bf16_bits_to_f32(inp["k"])
    inp = dict(inp, q=synth.f32_to_bf16_bits((base_q * np.float32(factor)).astype(np.float32)),
               k=synth.f32_to_bf16_bits((base_k * np.float32(factor)).astype(np.float32)))
    d = G.DevInputs(inp)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    m = qkq.accumulate_moments(d.q, d.k, d.pos, d.cos, d.sin, status=st).cpu().numpy()
    qf, kf = oracle_post_rope(d, "half")
    ref = D.moments(qf, kf, "half")
    scale = np.abs(ref).max(axis=(0, 1), keepdims=True)
    assert (np.abs(m - ref) <= 1e-12 * scale + 1e-12 * np.abs(ref)).all()
    assert int(st.item()) == 0


def test_moments_flag_nonfinite_second_channels():
    """A NaN in a pair's second channel is reported."""
    import synth
    inp = G.draw("tiny", T=8)
    k = inp["k"].copy()
    k[0, 0, 40] = 0x7FC0           # bf16 NaN in a second channel (k = 8 + 32), position 0
    inp = dict(inp, k=k)
    d = G.DevInputs(inp)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    qkq.accumulate_moments(d.q, d.k, d.pos, d.cos, d.sin, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & 1


# ------------------------------------------------ failure detection -------------------

def test_bounded_wait_reports_timeout_and_the_context_survives():
    """A wait with nothing to wait for gives up by its clock and reports
    QKQ_STATUS_TIMEOUT; the next calls run normally."""
    import ctypes
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert qkq.lib().qkq_selftest_bounded_wait(2_000_000, ctypes.c_void_p(st.data_ptr()), s) == 0
    torch.cuda.synchronize()
    assert int(st.item()) == qkq.STATUS_BITS["timeout"]
    # the context is fine: a real call afterwards matches the oracle
    d = G.DevInputs(G.draw("tiny", T=16))
    m = qkq.accumulate_moments(d.q, d.k, d.pos, d.cos, d.sin).cpu().numpy()
    qf, kf = oracle_post_rope(d, "half")
    ref = D.moments(qf, kf, "half")
    scale = np.abs(ref).max(axis=(0, 1), keepdims=True)
    assert (np.abs(m - ref) <= 1e-12 * scale + 1e-12 * np.abs(ref)).all()


# ------------------------------------------------ the calibrating transform -------------

@pytest.mark.parametrize("name,T,mode,b,group,style,split", [
    ("tiny", None, "pairwise_hadamard", 0, 32, "half", False),
    ("tiny", None, "block_hadamard", 8, 64, "interleaved", False),
    ("llama32_1b", None, "hadamard", 0, 64, "half", False),
    ("llama32_3b", 1777, "pairwise_hadamard", 0, 128, "half", False),
    ("llama32_3b", 901, "pairwise", 0, 32, "interleaved", True),
    ("mistral7b_decode", None, "rope_only", 0, 128, "half", False),
])
def test_calibrating_transform(name, T, mode, b, group, style, split):
    """qkq_transform_quantize_calibrate: Q~, codes and scales equal the plain launch bit for
    bit, and the moments equal the oracle's (and accumulate_moments') to the calibration bar."""
    d = G.DevInputs(G.draw(name, T=T))
    ct, sn, kw = d.tables(split)
    phi = G.random_phi(d.w.P, seed=81) if "pairwise" in mode else None
    phi_d = None if phi is None else torch.from_numpy(phi).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q1, c1, s1, m = qkq.transform_quantize_calibrate(d.q, d.k, d.pos, ct, sn, mode=mode, b=b,
                                                     group=group, phi=phi_d, rope_style=style,
                                                     status=st, **kw)
    q0, c0, s0, _ = qkq.transform_quantize(d.q, d.k, d.pos, ct, sn, mode=mode, b=b, group=group,
                                           phi=phi_d, rope_style=style, **kw)
    m_alone = qkq.accumulate_moments(d.q, d.k, d.pos, ct, sn, rope_style=style, **kw)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(G.bits16(q1), G.bits16(q0))
    np.testing.assert_array_equal(c1.cpu().numpy(), c0.cpu().numpy())
    np.testing.assert_array_equal(G.bits16(s1), G.bits16(s0))
    assert int(st.item()) == 0
    got = m.cpu().numpy()
    qf, kf = oracle_post_rope(d, style, split=split)
    ref = D.moments(qf, kf, style)
    np.testing.assert_array_equal(got[:, :, 0], ref[:, :, 0])
    scale = np.abs(ref).max(axis=(0, 1), keepdims=True)
    assert (np.abs(got - ref) <= 1e-12 * scale + 1e-12 * np.abs(ref)).all()
    np.testing.assert_allclose(got, m_alone.cpu().numpy(), rtol=1e-12, atol=1e-9)


def test_calibrating_transform_accumulates_and_checks():
    d = G.DevInputs(G.draw("llama32_3b", T=300))
    phi = torch.from_numpy(G.random_phi(64, seed=82)).cuda()
    _, _, _, m = qkq.transform_quantize_calibrate(d.q, d.k, d.pos, d.cos, d.sin,
                                                  mode="pairwise_hadamard", phi=phi)
    once = m.cpu().numpy().copy()
    qkq.transform_quantize_calibrate(d.q, d.k, d.pos, d.cos, d.sin, m, mode="pairwise_hadamard",
                                     phi=phi)
    np.testing.assert_allclose(m.cpu().numpy(), 2 * once, rtol=1e-14)
    with pytest.raises(qkq.QKQError):          # in place is refused
        qkq.transform_quantize_calibrate(d.q, d.k, d.pos, d.cos, d.sin, mode="hadamard", q_out=d.q)
    e = d.q[:0]
    out = qkq.transform_quantize_calibrate(e, d.k[:0], d.pos[:0], d.cos, d.sin)
    torch.cuda.synchronize()
    assert (out[3].cpu().numpy() == 0).all()
