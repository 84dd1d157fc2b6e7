"""Pins of the KV4 consumer's definition (attention logits against the int4 key cache,
oracle/definition.attention_scores): closed forms, the grouped-query head mapping, and the
pages' identity Q~ K~^T = RoPE(Q) RoPE(K)^T ("LLM旋转量化笔记" §3.2.1) carried through the
quantised cache within the Cauchy-Schwarz bound of the quantisation error.
"""
import numpy as np
import pytest

import synth
from oracle import bitspec as B
from oracle import definition as D

RNG = np.random.default_rng(4242)


def _bits(x):
    return synth.f32_to_bf16_bits(np.asarray(x, np.float32))


def test_score_of_a_row_with_itself_is_its_squared_norm():
    """q of small integers, keys = the same integers as codes with scale 1: S = sum q^2."""
    d_h, g = 64, 32
    q = RNG.integers(-7, 8, size=(1, 1, d_h)).astype(np.float64)
    codes = D.pack_int4(q[0].astype(np.int8))[None]                       # [Tk=1, Hkv=1, d_h/2]
    scales = np.full((1, 1, d_h // g), np.float16(1.0)).view(np.uint16)
    s = D.attention_scores(_bits(q), codes, scales, g)
    assert s.shape == (1, 1, 1) and s[0, 0, 0] == (q ** 2).sum()
    # a group's scale multiplies only its own channels' contribution
    scales2 = scales.copy()
    scales2[0, 0, 1] = np.float16(2.0).view(np.uint16)
    s2 = D.attention_scores(_bits(q), codes, scales2, g)
    assert s2[0, 0, 0] == (q[..., :g] ** 2).sum() + 2 * (q[..., g:] ** 2).sum()


def test_grouped_query_heads_share_their_key_head():
    """Hq = 8, Hkv = 2: query heads 0-3 read key head 0, heads 4-7 key head 1."""
    d_h, g, Tk = 64, 64, 5
    q = _bits(RNG.standard_normal((2, 8, d_h)))
    codes = RNG.integers(0, 256, size=(Tk, 2, d_h // 2)).astype(np.uint8)
    codes[:, 1] = 0                                                        # key head 1: zero
    scales = np.full((Tk, 2, 1), np.float16(0.5)).view(np.uint16)
    s = D.attention_scores(q, codes, scales, g)
    assert (s[:, 4:] == 0).all() and (np.abs(s[:, :4]) > 0).all()


@pytest.mark.parametrize("mode", ["hadamard", "pairwise_hadamard", "block_hadamard", "rope_only"])
def test_scores_carry_rope_q_rope_k_through_the_int4_cache(mode):
    """|S - RoPE(Q) RoPE(K)^T| <= ||q~ - q~_bf16|| ||K^|| + ||q~|| ||K~ - K^|| per score
    (Cauchy-Schwarz on the two substitutions), with the exact products from the fp64
    definition and the codes from the fp32 sequence."""
    name = "llama32_3b"
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(name, T=24)
    phi = RNG.uniform(-np.pi / 4, np.pi / 4, w.P).astype(np.float32)
    b = 16 if mode == "block_hadamard" else None
    r = B.transform_quantize(inp["q"], inp["k"], inp["pos"], w.d_h, theta=w.theta, mode=mode,
                             b=b, group=32, phi=phi, want_f32=True)
    q64 = D.rope(D.bf16_bits_to_f64(inp["q"]), inp["pos"], w.theta)
    k64 = D.rope(D.bf16_bits_to_f64(inp["k"]), inp["pos"], w.theta)
    exact = np.einsum("qhc,khc->qhk", q64, np.repeat(k64, w.Hq // w.Hkv, axis=1))
    s = D.attention_scores(r["q_out"], r["k_codes"], r["k_scales"], 32)
    qt = D.mix(q64, mode, b=b, phi=phi.astype(np.float64))
    kt = D.mix(k64, mode, b=b, phi=phi.astype(np.float64))
    khat = D.dequantize(D.unpack_int4(r["k_codes"]), r["k_scales"], 32)
    dq = np.linalg.norm(D.bf16_bits_to_f64(r["q_out"]) - qt, axis=-1)     # [Tq, Hq]
    dk = np.linalg.norm(kt - khat, axis=-1)                               # [Tk, Hkv]
    nq = np.linalg.norm(qt, axis=-1)
    nkh = np.linalg.norm(khat, axis=-1)
    per = w.Hq // w.Hkv
    bound = (dq[:, :, None] * np.repeat(nkh, per, axis=1).T[None]
             + nq[:, :, None] * np.repeat(dk, per, axis=1).T[None])
    assert (np.abs(s - exact) <= bound * (1 + 1e-9) + 1e-9).all()
    # and the cache is informative: scores track the exact logits closely
    assert np.corrcoef(s.ravel(), exact.ravel())[0, 1] > 0.99
