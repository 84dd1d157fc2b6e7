"""Pins of the value-row path of the oracle (V~ = V H_head / sqrt(d_h), then the K
quantiser; "LLM旋转量化笔记" §3.2.2): the fp64 definition against the properties the page
states, and the fp32 sequence against the fp64 definition and against the oracle's own
K path, which reaches the same arithmetic by another route.
"""
import math
import os

import numpy as np
import pytest

import synth
from oracle import bitspec as B
from oracle import definition as D

RNG = np.random.default_rng(777)
EPS = 2.0 ** -24


def test_value_rotation_is_its_own_inverse_and_keeps_norms():
    v = RNG.standard_normal((50, 128))
    t = D.value_transform(v)
    np.testing.assert_allclose(D.value_transform(t), v, rtol=0, atol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(t, axis=-1), np.linalg.norm(v, axis=-1), rtol=1e-12)


def test_attention_output_carries_the_rotation():
    """A V~ = (A V) H_head / sqrt(d_h): the rotation moves to the attention output, where the
    page folds it into the output projection (W_O <- W_O H_head)."""
    A = RNG.random((7, 50))
    A /= A.sum(axis=1, keepdims=True)           # softmax-like rows
    v = RNG.standard_normal((50, 64))
    lhs = A @ D.value_transform(v)
    rhs = D.value_transform(A @ v)
    np.testing.assert_allclose(lhs, rhs, rtol=0, atol=1e-12)
    # and folding it back recovers the plain output
    np.testing.assert_allclose(D.value_transform(lhs), A @ v, rtol=0, atol=1e-12)


def test_value_outlier_is_spread(golden_dir):
    """The worked example of "LLM旋转量化笔记" §2.2 on a value row: one 10.0 among K channels
    becomes +-10/sqrt(K) everywhere."""
    g = {}
    with open(os.path.join(golden_dir, "worked_example_outlier.txt"), encoding="utf-8") as f:
        for ln in f:
            if ln.strip() and not ln.lstrip().startswith("#"):
                key, val = ln.split()
                g[key] = val
    K, out = int(g["K"]), float(g["outlier"])
    e = np.zeros((1, K))
    e[0, 0] = out
    y = D.value_transform(e)[0]
    np.testing.assert_allclose(y, out / math.sqrt(K), rtol=1e-12)    # row 0 of H is all +1
    e2 = np.zeros((1, K))
    e2[0, -1] = out
    np.testing.assert_allclose(np.abs(D.value_transform(e2)[0]), out / 64, rtol=1e-12)


@pytest.mark.parametrize("name,group", [("tiny", 64), ("tiny", 32), ("llama32_3b", 128),
                                        ("llama32_3b", 32)])
def test_value_sequence_is_the_key_path_at_position_zero(name, group):
    """RoPE at position 0 is the identity in the fp32 sequence (a' = fma(a, 1, -(b*0)) = a,
    b' = fma(a, 0, b*1) = b), so value rows through the value path and the same rows as keys
    at position 0 through the Hadamard mode agree bit for bit."""
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(name, T=48)
    v = inp["k"]
    out = B.value_quantize(v, group, want_f32=True)
    ref = B.transform_quantize(inp["q"], v, np.zeros(48, np.int32), w.d_h, theta=w.theta,
                               mode="hadamard", group=group, want_f32=True, max_pos=1)
    np.testing.assert_array_equal(out["v_codes"], ref["k_codes"])
    np.testing.assert_array_equal(out["v_scales"], ref["k_scales"])
    np.testing.assert_array_equal(out["v_f32"].view(np.uint32), ref["k_f32"].view(np.uint32))
    assert out["status"] == ref["status"]


@pytest.mark.parametrize("name", ["tiny", "llama32_3b"])
def test_value_sequence_matches_definition(name):
    """fp32 sequence within log2(d_h) + 2 roundings of ||row|| of the fp64 rotation; codes
    equal to the fp64 quantiser's except within that bound of a rounding midpoint."""
    w = synth.WORKLOADS[name]
    v = synth.make_inputs(name, T=64)["k"]
    out = B.value_quantize(v, w.d_h, want_f32=True)
    v64 = D.bf16_bits_to_f64(v)
    ref = D.value_transform(v64)
    nrm = np.linalg.norm(v64, axis=-1, keepdims=True)
    bound = (math.log2(w.d_h) + 2) * EPS * nrm * 2
    assert (np.abs(out["v_f32"] - ref) <= bound).all()
    codes_ref, s_ref = D.quantize(ref, w.d_h)
    codes = D.unpack_int4(out["v_codes"])
    frac = np.abs(ref / np.repeat(s_ref, w.d_h, axis=-1))
    delta = bound * 7.0 / np.repeat(s_ref * 7.0, w.d_h, axis=-1) * 2.0 + 8.0 * EPS * 7.0
    near_mid = np.abs(frac - np.floor(frac) - 0.5) < delta
    assert not ((codes != codes_ref) & ~near_mid).any()
    assert (np.abs(codes.astype(int) - codes_ref) <= 1).all()


def test_value_rejects_bad_sizes():
    with pytest.raises(ValueError):
        B.value_quantize(np.zeros((2, 96), np.uint16), 32)          # not a power of two
    with pytest.raises(ValueError):
        B.value_quantize(np.zeros((2, 64), np.uint16), 48)          # group does not divide
