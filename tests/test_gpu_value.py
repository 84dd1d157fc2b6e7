"""GPU parity of the fused Q/K/V launch (qkq_transform_quantize_qkv) with the oracle.

Bar: bit-exact, like the Q/K launch — Q~, K~, codes and scales equal the oracle's fp32
sequence, and the value rows (full-head Hadamard, no RoPE, the K quantiser) equal the
oracle's value path; the Q/K outputs equal those of the plain Q/K call.
"""
import numpy as np
import pytest

from tests import gpu_common as G

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import synth  # noqa: E402
import transform_rope_head_b200 as qkq  # noqa: E402
from oracle import bitspec as B  # noqa: E402


def draw_v(name, T, seed):
    """Value rows with the workload's key distribution, from their own seed."""
    return synth.make_inputs(name, T=T, seed=seed)["k"]


def run(d: G.DevInputs, v_np, mode, b, group, style, phi=None, split=False):
    w = d.w
    v = G.to_dev_bf16(v_np)
    phi_d = None if phi is None else torch.from_numpy(phi).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ct, sn, kw = d.tables(split)
    out = qkq.transform_quantize_qkv(d.q, d.k, v, d.pos, ct, sn, mode=mode, b=b, group=group,
                                     phi=phi_d, rope_style=style, want_f32=True, status=st, **kw)
    plain = qkq.transform_quantize(d.q, d.k, d.pos, ct, sn, mode=mode, b=b, group=group,
                                   phi=phi_d, rope_style=style, want_k_f32=True, **kw)
    torch.cuda.synchronize()
    q_out, kc, ks, vc, vs, kf, vf = out
    # Q/K identical to the plain launch
    np.testing.assert_array_equal(G.bits16(q_out), G.bits16(plain[0]))
    np.testing.assert_array_equal(kc.cpu().numpy(), plain[1].cpu().numpy())
    np.testing.assert_array_equal(G.bits16(ks), G.bits16(plain[2]))
    np.testing.assert_array_equal(G.bits32(kf), G.bits32(plain[3]))
    # Q/K against the oracle
    tab = B.rope_table_split if split else B.rope_table
    oc, os_ = tab(d.max_pos, w.d_h, w.theta)
    ref = B.transform_quantize(d.inp["q"], d.inp["k"], d.inp["pos"], w.d_h, cos_t=oc, sin_t=os_,
                               mode=mode, b=b or None, group=group, phi=phi, style=style,
                               want_f32=True, split=split, max_pos=d.max_pos)
    np.testing.assert_array_equal(G.bits16(q_out), ref["q_out"])
    np.testing.assert_array_equal(kc.cpu().numpy(), ref["k_codes"])
    # V against the oracle's value path
    vref = B.value_quantize(v_np, group, want_f32=True)
    np.testing.assert_array_equal(vc.cpu().numpy(), vref["v_codes"])
    np.testing.assert_array_equal(G.bits16(vs), vref["v_scales"])
    np.testing.assert_array_equal(G.bits32(vf), G.bits32(vref["v_f32"]))
    assert int(st.item()) == (ref["status"] | vref["status"])


@pytest.mark.parametrize("mode,b", [("hadamard", 0), ("pairwise_hadamard", 0), ("pairwise", 0),
                                    ("block_hadamard", 8), ("rope_only", 0)])
@pytest.mark.parametrize("style", ["half", "interleaved"])
def test_qkv_tiny(mode, b, style):
    d = G.DevInputs(G.draw("tiny"))
    phi = G.random_phi(32, seed=41) if "pairwise" in mode else None
    run(d, draw_v("tiny", None, 901), mode, b, 32, style, phi)


@pytest.mark.parametrize("mode,group", [("pairwise_hadamard", 128), ("hadamard", 32),
                                        ("block_hadamard", 64)])
def test_qkv_llama32_3b(mode, group):
    d = G.DevInputs(G.draw("llama32_3b", T=1001))
    phi = G.random_phi(64, seed=42) if "pairwise" in mode else None
    run(d, draw_v("llama32_3b", 1001, 902), mode, 16 if mode == "block_hadamard" else 0, group,
        "half", phi)


def test_qkv_split_table_and_decode_positions():
    d = G.DevInputs(G.draw("mistral7b_decode"))
    run(d, draw_v("mistral7b_decode", None, 903), "pairwise_hadamard", 0, 128, "half",
        G.random_phi(64, seed=43), split=True)


@pytest.mark.parametrize("T", [1, 5, 33])
def test_qkv_ragged(T):
    d = G.DevInputs(G.draw("llama31_8b_128k", T=T))
    run(d, draw_v("llama31_8b_128k", T, 904), "pairwise_hadamard", 0, 128, "half",
        G.random_phi(64, seed=44))


def test_qkv_value_status_bits():
    """A non-finite value row and an overflowing value scale are reported like K's (a
    non-finite group's codes are unspecified; every other row stays bit-exact)."""
    d = G.DevInputs(G.draw("tiny", T=16))
    v_np = draw_v("tiny", 16, 905).copy()
    v_np[3, 0, 5] = 0x7FC0                                # bf16 NaN
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = qkq.transform_quantize_qkv(d.q, d.k, G.to_dev_bf16(v_np), d.pos, d.cos, d.sin,
                                     mode="hadamard", status=st)
    torch.cuda.synchronize()
    vref = B.value_quantize(v_np, 64)
    assert int(st.item()) & 1 and vref["status"] & 1
    keep = np.ones((16, 2), bool)
    keep[3, 0] = False
    np.testing.assert_array_equal(out[3].cpu().numpy()[keep], vref["v_codes"][keep])
    v_np = draw_v("tiny", 16, 906).copy()
    v_np[4, 1, :] = synth.f32_to_bf16_bits(np.full(64, 5.0e5, np.float32))
    run(d, v_np, "hadamard", 0, 64, "half")


def test_qkv_requires_value_outputs():
    d = G.DevInputs(G.draw("tiny", T=8))
    v = torch.zeros_like(d.k)
    L = qkq.lib()
    import ctypes
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    q_out = torch.empty_like(d.q)
    codes = torch.empty((8, 2, 32), dtype=torch.uint8, device="cuda")
    sc = torch.empty((8, 2, 1), dtype=torch.float16, device="cuda")
    rc = L.qkq_transform_quantize_qkv(p(d.q), p(d.k), p(v), p(d.pos), 8, 4, 2, 64, 0, p(d.cos),
                                      p(d.sin), d.cos.shape[0], None, 0, 0, 64, p(q_out),
                                      p(codes), p(sc), None, p(sc), None, None, None, None)
    assert rc == -1
