"""GPU test of qkq_accumulate_moments_noalloc, the moment accumulation for callers that
cannot allocate device memory (an inference-runtime plugin whose enqueue step may not
allocate, an engine that keeps all free HBM in its own pool).  It must give what the
workspace-taking entry point gives, bit for bit (it launches the same grid, with its
partial sums in the library's fixed scratch), call after call, while allocating nothing
itself; and the oracle's moments within the calibration tolerance.

This file is collected last on purpose: if it fails, a run that stops at the first
failure has already run every other test.  It also passes alone in a fresh process,
where its first call performs the per-device set-up of the library's fixed scratch.
"""
import ctypes

import numpy as np
import pytest

from tests import gpu_common as G

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import transform_rope_head_b200 as qkq  # noqa: E402

RTOL = 1e-12   # the moment tolerance of the other calibration tests


def _noalloc_abi(d, moments, status, T=None, Hq=None, style=0):
    """Call the entry point through the C ABI directly (ctypes)."""
    w = d.w
    T = d.q.shape[0] if T is None else T
    v = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    return qkq.lib().qkq_accumulate_moments_noalloc(
        v(d.q), v(d.k), v(d.pos), T, w.Hq if Hq is None else Hq, w.Hkv, w.d_h, style, v(d.cos),
        v(d.sin), d.cos.shape[0], v(moments), v(status),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _same_bits(a, b):
    np.testing.assert_array_equal(a.cpu().numpy().view(np.uint64), b.cpu().numpy().view(np.uint64))


@pytest.mark.parametrize("name,T,style", [("llama32_1b", None, 0), ("llama32_3b", 3001, 0),
                                          ("llama32_3b", 3001, 1)])
def test_noalloc_matches_workspace_entry_point_two_calls(name, T, style):
    batches = [G.DevInputs(G.draw(name, T=T, seed=s)) for s in (501, 502)]
    P = batches[0].w.P
    ref = torch.zeros((2, P, 6), dtype=torch.float64, device="cuda")
    got = torch.zeros_like(ref)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rs = "half" if style == 0 else "interleaved"
    for d in batches:                       # two calls in a row, accumulating
        qkq.accumulate_moments(d.q, d.k, d.pos, d.cos, d.sin, ref, rope_style=rs)
        assert _noalloc_abi(d, got, status, style=style) == 0
        torch.cuda.synchronize()
        _same_bits(got, ref)                # same grid, same summation order
    assert int(status.item()) == 0


def test_noalloc_full_size_batch_fits_its_scratch():
    """The 8B/128K batch, two calls in a row: the variant's grid (the workspace entry point's
    largest) fits its fixed scratch, and the results equal the workspace entry point's bit
    for bit."""
    d = G.DevInputs(G.draw("llama31_8b_128k"))
    ref = torch.zeros((2, 64, 6), dtype=torch.float64, device="cuda")
    got = torch.zeros_like(ref)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        qkq.accumulate_moments(d.q, d.k, d.pos, d.cos, d.sin, ref)
        assert _noalloc_abi(d, got, status) == 0
        torch.cuda.synchronize()
        _same_bits(got, ref)
    assert int(status.item()) == 0


def test_noalloc_matches_oracle_moments():
    """Against the oracle: the fp64 definition's raw moments of the oracle's post-RoPE rows
    (the fp32 sequence's RoPE output), within the calibration tolerance."""
    from oracle import bitspec as B
    from oracle import definition as D
    d = G.DevInputs(G.draw("llama32_3b", T=777))
    w = d.w
    oc, os_ = B.rope_table(d.max_pos, w.d_h, w.theta)
    r = B.transform_quantize(d.inp["q"], d.inp["k"], d.inp["pos"], w.d_h, cos_t=oc, sin_t=os_,
                             mode="rope_only", want_f32=True)
    ref = D.moments(r["q_f32"], r["k_f32"])
    got = torch.zeros((2, w.P, 6), dtype=torch.float64, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert _noalloc_abi(d, got, status) == 0
    torch.cuda.synchronize()
    np.testing.assert_allclose(got.cpu().numpy(), ref, rtol=RTOL, atol=1e-9)


def test_noalloc_split_table():
    """The no-alloc entry point with the split RoPE tables."""
    d = G.DevInputs(G.draw("llama32_3b", T=1000))
    ct, st, kw = d.tables(True)
    ref = qkq.accumulate_moments(d.q, d.k, d.pos, ct, st, **kw)
    got = torch.zeros_like(ref)
    qkq.accumulate_moments_noalloc(d.q, d.k, d.pos, ct, st, got, **kw)
    torch.cuda.synchronize()
    _same_bits(got, ref)
