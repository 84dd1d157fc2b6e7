"""GPU parity of the KV4 consumers (qkq_attention_scores; qkq_attention_scores_tc and
qkq_attention_scores_mma on the tensor cores) with the oracle's definition.

Bar: every score within (d_h + d_h/group + 2) * 2^-24 * sum_c |q~_c| |scale * code_c| of the
float64 score of the same bf16 queries and codes (the fp32 sums' rounding bound), twice that
for the tensor-core entries (their adder trees may truncate: up to one ulp per addition); and,
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


def run(kind, qd, cd, sd):
    """One consumer entry on device tensors: "cuda" (CUDA cores), "tc" (tcgen05), "mma"."""
    if kind == "tc":
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        s = qkq.attention_scores_tc(qd, cd, sd, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        return s
    s = (qkq.attention_scores_mma if kind == "mma" else qkq.attention_scores)(qd, cd, sd)
    torch.cuda.synchronize()
    return s


def bound_of(q_bits, codes, scales, group, kind):
    d_h = q_bits.shape[-1]
    q = np.abs(D.bf16_bits_to_f64(q_bits))
    kh = np.abs(D.dequantize(D.unpack_int4(codes), scales, group))
    per = q_bits.shape[1] // codes.shape[1]
    mag = np.einsum("qhc,khc->qhk", q, np.repeat(kh, per, axis=1))
    return (1 if kind == "cuda" else 2) * (d_h + d_h // group + 2) * 2.0 ** -24 * mag


def check(q_bits, codes, scales, group, tc=False, kind=None):
    kind = kind or ("tc" if tc else "cuda")
    qd = torch.from_numpy(q_bits.view(np.int16)).cuda().view(torch.bfloat16)
    cd = torch.from_numpy(codes).cuda()
    sd = torch.from_numpy(scales.view(np.float16)).cuda()
    got = run(kind, qd, cd, sd).cpu().numpy()
    ref = D.attention_scores(q_bits, codes, scales, group)
    assert (np.abs(got - ref) <= bound_of(q_bits, codes, scales, group, kind)).all()
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


@pytest.mark.parametrize("name,Tk,Tq,group", [("tiny", 256, 3, 64), ("tiny", 77, 1, 32),
                                              ("tiny", 9, 2, 64),
                                              ("llama32_1b", 1000, 1, 64),
                                              ("llama32_1b", 1000, 2, 32),
                                              ("llama32_3b", 700, 4, 32),
                                              ("llama31_8b_128k", 1283, 1, 128),
                                              ("llama31_8b_128k", 1283, 2, 128),
                                              ("llama31_8b_128k", 1283, 4, 64),
                                              ("llama31_8b_128k", 1283, 4, 128),
                                              ("llama31_8b_128k", 1283, 7, 128),
                                              ("llama31_8b_128k", 1283, 16, 128),
                                              ("llama31_8b_128k", 1283, 16, 32),
                                              ("llama31_8b_128k", 1283, 37, 128),
                                              ("mistral7b_decode", 256, 5, 128),
                                              ("mistral7b_decode", 256, 256, 64)])
def test_register_mma_scores_match_oracle(name, Tk, Tq, group):
    """The register-operand tensor-core entry: one, two, four and eight n-tiles of 8 query
    rows (1, 2, 4 (or 5 at 4 heads a key head: 20 rows) and 16 tokens), query blocks of 16
    tokens (37 and 256 tokens: several blocks, a ragged last one), ragged tiles of 16 cached
    tokens (1283, 77, 9), and every group size of both head dimensions."""
    inp, r = oracle_cache(name, Tk, group)
    check(r["q_out"][:Tq], r["k_codes"], r["k_scales"], group, kind="mma")


@pytest.mark.parametrize("Tq", [1, 16])
def test_register_mma_full_cache_sampled(Tq):
    """The Llama-3.1-8B cache of 131072 tokens (8 key heads, d_h 128, group 128) at the
    decode shapes the consumer is timed on, one and sixteen query tokens: every score of
    2048 sampled cached tokens (ragged positions included) against the definition."""
    rng = np.random.default_rng(17 + Tq)
    Tk, Hq, Hkv, d_h, group = 131072, 32, 8, 128, 128
    q = (rng.standard_normal((Tq, Hq, d_h)) * 0.5).astype(np.float32)
    q_bits = (q.view(np.uint32) >> 16).astype(np.uint16)
    codes = rng.integers(0, 256, size=(Tk, Hkv, d_h // 2), dtype=np.uint8)
    scales = rng.uniform(0.01, 1.0, size=(Tk, Hkv, 1)).astype(np.float16).view(np.uint16)
    qd = torch.from_numpy(q_bits.view(np.int16)).cuda().view(torch.bfloat16)
    got = run("mma", qd, torch.from_numpy(codes).cuda(),
              torch.from_numpy(scales.view(np.float16)).cuda()).cpu().numpy()
    idx = np.unique(np.concatenate([rng.integers(0, Tk, 2040), [0, 15, 16, Tk - 17, Tk - 16, Tk - 1]]))
    ref = D.attention_scores(q_bits, codes[idx], scales[idx], group)
    bound = bound_of(q_bits, codes[idx], scales[idx], group, "mma")
    assert (np.abs(got[:, :, idx] - ref) <= bound).all()


def test_scores_query_heads_equal_key_heads():
    """Hq == Hkv (no grouping), and 3, 6 and 8 query heads per key head, on synthetic codes."""
    rng = np.random.default_rng(3)
    for hq, hkv in ((4, 4), (16, 2), (12, 2), (6, 2), (24, 4)):
        q = (rng.integers(0, 1 << 16, size=(2, hq, 128)) & 0x7FFF).astype(np.uint16)
        q = (q & 0x807F) | 0x3C00                                         # modest magnitudes
        codes = rng.integers(0, 256, size=(300, hkv, 64)).astype(np.uint8)
        scales = rng.uniform(0.01, 2.0, size=(300, hkv, 2)).astype(np.float16).view(np.uint16)
        check(q, codes, scales, 64)
        check(q, codes, scales, 64, tc=True)
        check(q, codes, scales, 64, kind="mma")


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
    assert qkq.attention_scores_mma(z, codes, scales).shape == (0, 4, 5)
    q = torch.zeros((1, 5, 64), dtype=torch.bfloat16, device="cuda")   # 5 heads over 2
    for fn in (qkq.attention_scores, qkq.attention_scores_tc, qkq.attention_scores_mma):
        with pytest.raises(qkq.QKQError):
            fn(q, codes, scales)
    # the register-MMA entry indexes cache rows in 32 bits: Tk * Hkv >= 2^32 is refused on the
    # host, before any launch (the buffers passed are real but never read)
    L = qkq.lib()
    import ctypes
    v = ctypes.c_void_p
    q1 = torch.zeros((1, 8, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(16, dtype=torch.float32, device="cuda")
    assert L.qkq_attention_scores_mma(v(q1.data_ptr()), 1, v(codes.data_ptr()), v(scales.data_ptr()),
                                      1 << 29, 8, 8, 128, 128, v(out.data_ptr()), None) == -2
    # an empty cache: nothing to compute, nothing written
    q = torch.ones((2, 4, 64), dtype=torch.bfloat16, device="cuda")
    for fn in (qkq.attention_scores, qkq.attention_scores_tc, qkq.attention_scores_mma):
        assert fn(q, codes[:0], scales[:0]).shape == (2, 4, 0)
