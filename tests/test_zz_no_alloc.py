"""GPU test of qkq_accumulate_moments_noalloc, the moment accumulation for callers that
cannot allocate device memory (an inference-runtime plugin whose enqueue step may not
allocate, an engine that keeps all free HBM in its own pool).  It must give what the
workspace-taking entry point gives, call after call, while allocating nothing itself.

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


def _noalloc_abi(d, moments, status, T=None, Hq=None):
    """Call the entry point through the C ABI directly (ctypes)."""
    w = d.w
    T = d.q.shape[0] if T is None else T
    v = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    return qkq.lib().qkq_accumulate_moments_noalloc(
        v(d.q), v(d.k), v(d.pos), T, w.Hq if Hq is None else Hq, w.Hkv, w.d_h, 0, v(d.cos),
        v(d.sin), d.cos.shape[0], v(moments), v(status),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("name,T", [("llama32_1b", None), ("llama32_3b", 3001)])
def test_noalloc_matches_workspace_entry_point_two_calls(name, T):
    batches = [G.DevInputs(G.draw(name, T=T, seed=s)) for s in (501, 502)]
    P = batches[0].w.P
    ref = torch.zeros((2, P, 6), dtype=torch.float64, device="cuda")
    got = torch.zeros_like(ref)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for d in batches:                       # two calls in a row, accumulating
        qkq.accumulate_moments(d.q, d.k, d.pos, d.cos, d.sin, ref)
        assert _noalloc_abi(d, got, status) == 0
        torch.cuda.synchronize()
        np.testing.assert_allclose(got.cpu().numpy(), ref.cpu().numpy(), rtol=RTOL, atol=0)
    assert int(status.item()) == 0


def test_noalloc_full_size_batch_fits_its_scratch():
    """The 8B/128K batch in one call: the variant's grid fits its fixed scratch, and the
    result equals the workspace entry point's within the calibration tolerance."""
    d = G.DevInputs(G.draw("llama31_8b_128k"))
    ref = torch.zeros((2, 64, 6), dtype=torch.float64, device="cuda")
    got = torch.zeros_like(ref)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    qkq.accumulate_moments(d.q, d.k, d.pos, d.cos, d.sin, ref)
    assert _noalloc_abi(d, got, status) == 0
    torch.cuda.synchronize()
    np.testing.assert_allclose(got.cpu().numpy(), ref.cpu().numpy(), rtol=RTOL, atol=0)
    assert int(status.item()) == 0


def test_noalloc_split_table():
    """The no-alloc entry point with the split RoPE tables."""
    d = G.DevInputs(G.draw("llama32_3b", T=1000))
    ct, st, kw = d.tables(True)
    ref = qkq.accumulate_moments(d.q, d.k, d.pos, ct, st, **kw)
    got = torch.zeros_like(ref)
    qkq.accumulate_moments_noalloc(d.q, d.k, d.pos, ct, st, got, **kw)
    torch.cuda.synchronize()
    np.testing.assert_allclose(got.cpu().numpy(), ref.cpu().numpy(), rtol=RTOL, atol=0)
