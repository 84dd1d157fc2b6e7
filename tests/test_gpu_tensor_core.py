"""GPU checks of the tensor-core variant of the Hadamard modes (qkq_transform_quantize_tc).

The variant multiplies each post-RoPE row by (I (x) H_b) / sqrt(b) on the tensor cores with
the row split into two bf16 halves, so it is not the bit-exact fp32 sequence.  Its bar:

* every K~ value within 2^-14 * ||row||_2 of the fp64 product of the oracle's fp32
  post-RoPE row (then turned by phi in the pairwise mode) with the normalised block
  Hadamard — the split keeps 16 significant bits of each element (error <= 2^-17 |x|),
  and the fp32 accumulation of 2 b products adds at most 2 b 2^-24 ||x||_1 / sqrt(b);
* every Q~ value within that bound plus half a bf16 ulp (2^-8 of the value);
* the quantiser stage bit-exact: codes and fp16 scales equal the oracle's fp32 quantiser
  applied to the kernel's own K~.
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

BOUND = 2.0 ** -14


def reference(d: G.DevInputs, mode, b, style, phi):
    """fp64 mixing of the oracle's fp32 post-RoPE rows: (q~, k~) [T, H, d_h]."""
    w = d.w
    oc, os_ = B.rope_table(d.max_pos, w.d_h, w.theta)
    base = "pairwise" if mode == "pairwise_hadamard" else "rope_only"
    r = B.transform_quantize(d.inp["q"], d.inp["k"], d.inp["pos"], w.d_h, cos_t=oc, sin_t=os_,
                             mode=base, phi=phi, style=style, group=w.d_h, want_f32=True)
    n = b if mode == "block_hadamard" else w.d_h
    mix = [D.block_hadamard(r[key].astype(np.float64), n) for key in ("q_f32", "k_f32")]
    return mix[0], mix[1], r


def check(d: G.DevInputs, mode, b, group, style, phi=None):
    w = d.w
    phi_d = None if phi is None else torch.from_numpy(phi).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q_out, codes, scales, kf = qkq.transform_quantize_tc(
        d.q, d.k, d.pos, d.cos, d.sin, mode=mode, b=b, group=group, phi=phi_d, rope_style=style,
        want_k_f32=True, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    yq, yk, r = reference(d, mode, b, style, phi)
    kf = kf.cpu().numpy()
    nk = np.linalg.norm(r["k_f32"].astype(np.float64), axis=-1, keepdims=True)
    assert (np.abs(kf - yk) <= BOUND * nk).all()
    qo = D.bf16_bits_to_f64(G.bits16(q_out))
    nq = np.linalg.norm(r["q_f32"].astype(np.float64), axis=-1, keepdims=True)
    # bf16 keeps 8 significant bits: half an ulp is at most 2^-8 of the value
    assert (np.abs(qo - yq) <= 1.01 * BOUND * nq + 2.0 ** -8 * np.abs(yq)).all()
    rc, rs, _ = B.quantize_rows(kf, group)
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)
    np.testing.assert_array_equal(G.bits16(scales), rs)
    return codes, scales


@pytest.fixture(scope="module")
def tiny():
    return G.DevInputs(G.draw("tiny"))


@pytest.fixture(scope="module")
def l3b():
    return G.DevInputs(G.draw("llama32_3b", T=777))     # 18648 query rows: a ragged last tile


@pytest.mark.parametrize("mode,b", [("hadamard", 0), ("pairwise_hadamard", 0),
                                    ("block_hadamard", 2), ("block_hadamard", 16),
                                    ("block_hadamard", 64)])
@pytest.mark.parametrize("style", ["half", "interleaved"])
def test_tc_tiny_d64(tiny, mode, b, style):
    phi = G.random_phi(32, seed=31) if "pairwise" in mode else None
    check(tiny, mode, b, 32, style, phi)


@pytest.mark.parametrize("mode,b", [("hadamard", 0), ("pairwise_hadamard", 0),
                                    ("block_hadamard", 8), ("block_hadamard", 128)])
@pytest.mark.parametrize("group", [128, 32])
def test_tc_llama32_3b_d128(l3b, mode, b, group):
    phi = G.random_phi(64, seed=32) if "pairwise" in mode else None
    check(l3b, mode, b, group, "half", phi)


def test_tc_interleaved_d128(l3b):
    check(l3b, "pairwise_hadamard", 0, 64, "interleaved", G.random_phi(64, seed=33))


def test_tc_close_to_butterfly():
    """On the headline distribution, codes agree with the bit-exact butterfly path except
    where |x/s| sits within the bound of a rounding midpoint (a small fraction)."""
    d = G.DevInputs(G.draw("llama31_8b_128k", T=2000))
    phi = torch.from_numpy(G.random_phi(64, seed=34)).cuda()
    a = qkq.transform_quantize(d.q, d.k, d.pos, d.cos, d.sin, mode="pairwise_hadamard", phi=phi)
    t = qkq.transform_quantize_tc(d.q, d.k, d.pos, d.cos, d.sin, mode="pairwise_hadamard",
                                  phi=phi)
    ca = D.unpack_int4(a[1].cpu().numpy())
    ct = D.unpack_int4(t[1].cpu().numpy())
    assert (np.abs(ca.astype(int) - ct) <= 1).all()
    assert (ca != ct).mean() < 2e-3


def test_tc_rejects_other_modes_and_in_place(tiny):
    for mode in ("pairwise", "rope_only"):
        with pytest.raises(qkq.QKQError):
            qkq.transform_quantize_tc(tiny.q, tiny.k, tiny.pos, tiny.cos, tiny.sin, mode=mode,
                                      phi=torch.zeros(32, device="cuda"))
    with pytest.raises(qkq.QKQError):
        qkq.transform_quantize_tc(tiny.q, tiny.k, tiny.pos, tiny.cos, tiny.sin, mode="hadamard",
                                  q_out=tiny.q)


def test_tc_empty_input(tiny):
    e = tiny.q[:0]
    qkq.transform_quantize_tc(e, tiny.k[:0], tiny.pos[:0], tiny.cos, tiny.sin)
    torch.cuda.synchronize()
