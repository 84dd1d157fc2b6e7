"""GPU parity of the KV4 consumers (qkq_attention_scores, and qkq_attention_scores_tc on the
tensor cores) with the oracle's definition.

Bar: every score within (d_h + d_h/group + 2) * 2^-24 * sum_c |q~_c| |scale * code_c| of the
float64 score of the same bf16 queries and codes (the fp32 sums' rounding bound), twice that
for the tensor-core entry (its adder tree may truncate: up to one ulp per addition); and,
end to end from the GPU transform, within the Cauchy-Schwarz bound of RoPE(Q) RoPE(K)^T
("LLM旋转量化笔记" §3.2.1: the rotation cancels in the score product).
"""
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


def oracle_cache(name, Tk, group, mode="pairwise_hadamard", seed=None):
    """Transformed queries and the int4 cache from the oracle's fp32 sequence."""
    inp = G.draw(name, T=Tk, seed=seed)
    w = inp["workload"]
    phi = G.random_phi(w.P, seed=51)
    r = B.transform_quantize(inp["q"], inp["k"], inp["pos"], w.d_h, theta=w.theta, mode=mode,
                             group=group, phi=phi if "pairwise" in mode else None,
                             max_pos=w.max_pos)
    return inp, r


def check(q_bits, codes, scales, group, tc=False):
    qd = torch.from_numpy(q_bits.view(np.int16)).cuda().view(torch.bfloat16)
    cd = torch.from_numpy(codes).cuda()
    sd = torch.from_numpy(scales.view(np.float16)).cuda()
    if tc:
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        s = qkq.attention_scores_tc(qd, cd, sd, status=st)
    else:
        s = qkq.attention_scores(qd, cd, sd)
    torch.cuda.synchronize()
    if tc:
        assert int(st.item()) == 0
    got = s.cpu().numpy()
    ref = D.attention_scores(q_bits, codes, scales, group)
    d_h = q_bits.shape[-1]
    q = np.abs(D.bf16_bits_to_f64(q_bits))
    kh = np.abs(D.dequantize(D.unpack_int4(codes), scales, group))
    per = q_bits.shape[1] // codes.shape[1]
    mag = np.einsum("qhc,khc->qhk", q, np.repeat(kh, per, axis=1))
    bound = (2 if tc else 1) * (d_h + d_h // group + 2) * 2.0 ** -24 * mag
    assert (np.abs(got - ref) <= bound).all()
    return got, ref


@pytest.mark.parametrize("name,Tk,Tq,group", [("tiny", 256, 3, 64), ("tiny", 77, 1, 32),
                                              ("llama32_1b", 1000, 2, 64),
                                              ("llama32_3b", 700, 4, 32),
                                              ("llama31_8b_128k", 1283, 2, 128),
                                              ("mistral7b_decode", 256, 5, 128)])
def test_scores_match_oracle(name, Tk, Tq, group):
    """Queries: the first Tq transformed tokens; keys: every cached token (ragged Tk)."""
    inp, r = oracle_cache(name, Tk, group)
    check(r["q_out"][:Tq], r["k_codes"], r["k_scales"], group)


@pytest.mark.parametrize("name,Tk,Tq,group", [("tiny", 256, 3, 64), ("tiny", 77, 1, 32),
                                              ("llama32_1b", 1000, 2, 64),
                                              ("llama32_3b", 700, 4, 32),
                                              ("llama31_8b_128k", 1283, 2, 128),
                                              ("llama31_8b_128k", 1283, 130, 128),
                                              ("llama31_8b_128k", 500, 40, 32),
                                              ("mistral7b_decode", 256, 5, 128),
                                              ("mistral7b_decode", 256, 256, 64)])
def test_tensor_core_scores_match_oracle(name, Tk, Tq, group):
    """The tensor-core entry on the same caches, ragged tiles of 128 cached tokens, and query
    blocks: 130 tokens of 4 query rows at group 128 take three launches (64 tokens each),
    40 tokens at group 32 (four accumulators) three launches of 16, 256 tokens at group 64
    (two accumulators) eight launches of 32."""
    inp, r = oracle_cache(name, Tk, group)
    check(r["q_out"][:Tq], r["k_codes"], r["k_scales"], group, tc=True)


def test_scores_query_heads_equal_key_heads():
    """Hq == Hkv (no grouping) and Hq == 8 Hkv, on synthetic codes."""
    rng = np.random.default_rng(3)
    for hq, hkv in ((4, 4), (16, 2), (12, 2)):
        q = (rng.integers(0, 1 << 16, size=(2, hq, 128)) & 0x7FFF).astype(np.uint16)
        q = (q & 0x807F) | 0x3C00                                         # modest magnitudes
        codes = rng.integers(0, 256, size=(300, hkv, 64)).astype(np.uint8)
        scales = rng.uniform(0.01, 2.0, size=(300, hkv, 2)).astype(np.float16).view(np.uint16)
        check(q, codes, scales, 64)
        check(q, codes, scales, 64, tc=True)


def test_end_to_end_from_the_gpu_transform():
    d = G.DevInputs(G.draw("llama31_8b_128k", T=600))
    w = d.w
    phi = torch.from_numpy(G.random_phi(64, seed=52)).cuda()
    q_out, codes, scales, _ = qkq.transform_quantize(d.q, d.k, d.pos, d.cos, d.sin,
                                                     mode="pairwise_hadamard", phi=phi)
    s = qkq.attention_scores(q_out[:3].contiguous(), codes, scales).cpu().numpy()
    q64 = D.rope(D.bf16_bits_to_f64(d.inp["q"]), d.inp["pos"], w.theta)
    k64 = D.rope(D.bf16_bits_to_f64(d.inp["k"]), d.inp["pos"], w.theta)
    exact = np.einsum("qhc,khc->qhk", q64[:3], np.repeat(k64, w.Hq // w.Hkv, axis=1))
    qt = D.mix(q64[:3], "pairwise_hadamard", phi=phi.cpu().numpy().astype(np.float64))
    kt = D.mix(k64, "pairwise_hadamard", phi=phi.cpu().numpy().astype(np.float64))
    khat = D.dequantize(D.unpack_int4(codes.cpu().numpy()), G.bits16(scales), 128)
    dq = np.linalg.norm(D.bf16_bits_to_f64(G.bits16(q_out[:3])) - qt, axis=-1)
    dk = np.linalg.norm(kt - khat, axis=-1)
    per = w.Hq // w.Hkv
    bound = (dq[:, :, None] * np.repeat(np.linalg.norm(khat, axis=-1), per, axis=1).T[None]
             + np.linalg.norm(qt, axis=-1)[:, :, None] * np.repeat(dk, per, axis=1).T[None])
    assert (np.abs(s - exact) <= bound * (1 + 1e-6) + 1e-4).all()
    assert np.corrcoef(s.ravel(), exact.ravel())[0, 1] > 0.98


def test_scores_empty_and_argument_checks():
    z = torch.zeros((0, 4, 64), dtype=torch.bfloat16, device="cuda")
    codes = torch.zeros((5, 2, 32), dtype=torch.uint8, device="cuda")
    scales = torch.ones((5, 2, 1), dtype=torch.float16, device="cuda")
    assert qkq.attention_scores(z, codes, scales).shape == (0, 4, 5)
    assert qkq.attention_scores_tc(z, codes, scales).shape == (0, 4, 5)
    q = torch.zeros((1, 5, 64), dtype=torch.bfloat16, device="cuda")   # 5 heads over 2
    with pytest.raises(qkq.QKQError):
        qkq.attention_scores(q, codes, scales)
    with pytest.raises(qkq.QKQError):
        qkq.attention_scores_tc(q, codes, scales)
    # an empty cache: nothing to compute, nothing written
    q = torch.ones((2, 4, 64), dtype=torch.bfloat16, device="cuda")
    for fn in (qkq.attention_scores, qkq.attention_scores_tc):
        assert fn(q, codes[:0], scales[:0]).shape == (2, 4, 0)
