"""Python binding of libqkq — the post-RoPE Q/K transform with dynamic KV4 quantisation
on NVIDIA B200 (sm_100a).

Argument marshalling only: every function passes torch tensors' device pointers,
sizes and the current CUDA stream to the C ABI declared in ``include/qkq.h``; every
step of the computation runs in the library's CUDA kernels.  PyTorch provides device
memory and streams.  There is no CPU fallback: if ``libqkq.so`` is missing the import
fails, and every call on a non-sm_100 device returns an error.

Method: "When Local Variance Optimality Is Not Enough: RoPE-Aligned Q/K Rotations for
Dynamic 4-Bit Quantisation" (technical summary: "Methodology", "Optimisation
objective", "Estimation strategies", "Core contributions").
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "MODES", "ESTIMATORS", "ROPE_STYLES", "STATUS_BITS", "QKQError", "lib", "lib_path",
    "ROPE_SPLIT_TABLE", "rope_table", "rope_table_rows", "transform_quantize",
    "transform_quantize_tc", "transform_quantize_qkv", "transform_quantize_stats",
    "transform_quantize_calibrate",
    "attention_scores",
    "accumulate_moments", "accumulate_moments_noalloc",
    "solve_angles",
    "dequant_error", "dequant_error_recompute", "dequant_summary", "moments_workspace_bytes",
    "dequant_error_workspace_bytes", "status_string", "k_range", "rel_error",
]

MODES = {"hadamard": 0, "pairwise": 1, "pairwise_hadamard": 2, "block_hadamard": 3,
         "rope_only": 4}
ESTIMATORS = {"pooled": 0, "k_only": 1, "balanced": 2}
ROPE_STYLES = {"half": 0, "interleaved": 1}
ROPE_SPLIT_TABLE = 0x100  # flag OR-ed into the style: split (two-level) RoPE tables
STATUS_BITS = {"nonfinite": 1, "scale_overflow": 2, "pos_range": 4, "timeout": 8,
               "empty_stream": 16, "bounds": 32}

_HERE = os.path.dirname(os.path.abspath(__file__))
# QKQ_LIB_PATH selects another build of the library (e.g. a tuning variant)
_LIB_PATH = os.environ.get("QKQ_LIB_PATH") or os.path.join(_HERE, "_build", "libqkq.so")
SYMBOLS = ("qkq_version", "qkq_error_string", "qkq_status_string", "qkq_rope_table",
           "qkq_rope_table_split", "qkq_rope_table_rows",
           "qkq_transform_quantize", "qkq_transform_quantize_qkv", "qkq_transform_quantize_tc",
           "qkq_attention_scores", "qkq_attention_scores_tc", "qkq_attention_scores_mma", "qkq_transform_quantize_stats", "qkq_selftest_bounded_wait",
           "qkq_transform_quantize_calibrate",
           "qkq_moments_workspace_bytes", "qkq_accumulate_moments",
           "qkq_solve_angles", "qkq_dequant_error_workspace_bytes", "qkq_dequant_error",
           "qkq_dequant_error_recompute", "qkq_dequant_summary",
           "qkq_accumulate_moments_noalloc")


class QKQError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {_lib.qkq_error_string(code).decode()} (code {code})")


def lib_path() -> str:
    return _LIB_PATH


def _load() -> ctypes.CDLL:
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"libqkq.so is not built ({_LIB_PATH}); run "
                          "`python -c 'import __graft_entry__ as g; g.build()'` or "
                          "`python transform_rope_head_b200/build.py`")
    L = ctypes.CDLL(_LIB_PATH)
    P, I, I64, D, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double, ctypes.c_size_t
    L.qkq_version.argtypes, L.qkq_version.restype = [], I
    L.qkq_error_string.argtypes, L.qkq_error_string.restype = [I], ctypes.c_char_p
    L.qkq_status_string.argtypes, L.qkq_status_string.restype = [I], ctypes.c_char_p
    L.qkq_rope_table.argtypes, L.qkq_rope_table.restype = [P, P, I, I, D, P], I
    L.qkq_rope_table_split.argtypes, L.qkq_rope_table_split.restype = [P, P, I, I, D, P], I
    L.qkq_rope_table_rows.argtypes, L.qkq_rope_table_rows.restype = [I, I], SZ
    L.qkq_transform_quantize.argtypes = [P, P, P, I64, I, I, I, I, P, P, I, P, I, I, I, P, P, P,
                                         P, P, P]
    L.qkq_transform_quantize.restype = I
    L.qkq_transform_quantize_tc.argtypes = L.qkq_transform_quantize.argtypes
    L.qkq_transform_quantize_qkv.argtypes = [P, P, P, P, I64, I, I, I, I, P, P, I, P, I, I, I,
                                             P, P, P, P, P, P, P, P, P]
    L.qkq_transform_quantize_qkv.restype = I
    L.qkq_transform_quantize_stats.argtypes = [P, P, P, I64, I, I, I, I, P, P, I, P, I, I, I,
                                               P, P, P, P, P, SZ, P, P]
    L.qkq_transform_quantize_stats.restype = I
    L.qkq_transform_quantize_calibrate.argtypes = [P, P, P, I64, I, I, I, I, P, P, I, P, I, I, I,
                                                   P, P, P, P, P, SZ, P, P]
    L.qkq_transform_quantize_calibrate.restype = I
    L.qkq_selftest_bounded_wait.argtypes = [ctypes.c_ulonglong, P, P]
    L.qkq_selftest_bounded_wait.restype = I
    L.qkq_attention_scores.argtypes = [P, I64, P, P, I64, I, I, I, I, P, P]
    L.qkq_attention_scores.restype = I
    L.qkq_attention_scores_tc.argtypes = [P, I64, P, P, I64, I, I, I, I, P, P, P]
    L.qkq_attention_scores_tc.restype = I
    L.qkq_attention_scores_mma.argtypes = [P, I64, P, P, I64, I, I, I, I, P, P]
    L.qkq_attention_scores_mma.restype = I
    L.qkq_transform_quantize_tc.restype = I
    L.qkq_moments_workspace_bytes.argtypes = [I64, I, I, I]
    L.qkq_moments_workspace_bytes.restype = SZ
    L.qkq_accumulate_moments.argtypes = [P, P, P, I64, I, I, I, I, P, P, I, P, P, SZ, P, P]
    L.qkq_accumulate_moments.restype = I
    L.qkq_accumulate_moments_noalloc.argtypes = [P, P, P, I64, I, I, I, I, P, P, I, P, P, P]
    L.qkq_accumulate_moments_noalloc.restype = I
    L.qkq_solve_angles.argtypes, L.qkq_solve_angles.restype = [P, I, I, P, P, P, P], I
    L.qkq_dequant_error_workspace_bytes.argtypes = [I64, I, I, I]
    L.qkq_dequant_error_workspace_bytes.restype = SZ
    L.qkq_dequant_error.argtypes = [P, P, P, I64, I, I, I, P, P, SZ, P, P]
    L.qkq_dequant_error.restype = I
    L.qkq_dequant_error_recompute.argtypes = [P, P, I64, I, I, I, P, P, I, P, I, I, I, P, P, P,
                                              P, SZ, P, P]
    L.qkq_dequant_error_recompute.restype = I
    L.qkq_dequant_summary.argtypes = [P, P]
    L.qkq_dequant_summary.restype = I
    return L


_lib = _load()


def lib() -> ctypes.CDLL:
    return _lib


def _check(rc: int, where: str) -> None:
    if rc != 0:
        raise QKQError(rc, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def status_string(bits: int) -> str:
    return _lib.qkq_status_string(int(bits)).decode()


# ---------------------------------------------------------------- table -----------

def rope_table_rows(max_pos: int, split: bool = False) -> int:
    return int(_lib.qkq_rope_table_rows(int(max_pos), 1 if split else 0))


def rope_table(max_pos: int, d_h: int, theta: float, inv_freq=None, device="cuda",
               split: bool = False):
    """fp32 cos/sin tables (a model constant), built by the library on the host in fp64
    and copied to ``device``: [max_pos, d_h/2], or with split=True the split layout
    [64 + ceil(max_pos/64), d_h/2] (``qkq_rope_table_split``; pass split_table=True and
    max_pos to the calls that read it)."""
    import torch
    P = d_h // 2
    rows = rope_table_rows(max_pos, split)
    if rows == 0:
        raise QKQError(-2, "rope_table")
    c = torch.empty((rows, P), dtype=torch.float32, pin_memory=torch.cuda.is_available())
    s = torch.empty_like(c)
    inv = None
    if inv_freq is not None:
        inv = torch.as_tensor(inv_freq, dtype=torch.float64).contiguous()
    fn = _lib.qkq_rope_table_split if split else _lib.qkq_rope_table
    _check(fn(_ptr(c), _ptr(s), int(max_pos), int(d_h), float(theta), _ptr(inv)),
           "qkq_rope_table_split" if split else "qkq_rope_table")
    if device is None or str(device) == "cpu":
        return c, s
    return c.to(device, non_blocking=True), s.to(device, non_blocking=True)


def _rope_args(cos_tab, rope_style, split_table, max_pos):
    """(style argument, max_pos) of a call: one table row per position unless split."""
    style = ROPE_STYLES[rope_style]
    if split_table:
        if max_pos is None:
            raise ValueError("split_table=True needs max_pos (the positions' range)")
        if cos_tab.shape[0] != rope_table_rows(max_pos, True):
            raise ValueError("split tables must have 64 + ceil(max_pos/64) rows")
        return style | ROPE_SPLIT_TABLE, int(max_pos)
    return style, int(cos_tab.shape[0] if max_pos is None else max_pos)


# ---------------------------------------------------------------- hot path --------

def transform_quantize(q, k, pos, cos_tab, sin_tab, *, mode="hadamard", b=0, group=None,
                       phi=None, rope_style="half", q_out=None, k_codes=None, k_scales=None,
                       k_f32=None, want_k_f32=False, status=None, stream=None,
                       split_table=False, max_pos=None):
    """Fused transform + KV4 quantisation (``qkq_transform_quantize``).

    q [T, Hq, d_h] bf16, k [T, Hkv, d_h] bf16, pos [T] int32, tables [max_pos, d_h/2]
    fp32, phi [d_h/2] fp32 (pairwise modes) — all CUDA tensors.  Returns
    (q_out bf16, k_codes uint8 [T, Hkv, d_h/2], k_scales fp16 [T, Hkv, d_h/group],
    k_f32 or None).  Output tensors may be passed in to reuse memory.
    """
    return _transform(_lib.qkq_transform_quantize, "qkq_transform_quantize", q, k, pos, cos_tab,
                      sin_tab, mode, b, group, phi, rope_style, q_out, k_codes, k_scales, k_f32,
                      want_k_f32, status, stream, split_table, max_pos)


def transform_quantize_stats(q, k, pos, cos_tab, sin_tab, *, mode="hadamard", b=0, group=None,
                             phi=None, rope_style="half", q_out=None, k_codes=None,
                             k_scales=None, stats=None, workspace=None, status=None,
                             stream=None, split_table=False, max_pos=None):
    """transform_quantize with the K rows' measurement statistics (float64 [6], as
    dequant_error returns) computed in the same pass (``qkq_transform_quantize_stats``).
    Returns (q_out, k_codes, k_scales, stats)."""
    import torch
    T, Hq, d_h = q.shape
    Hkv = k.shape[1]
    group = d_h if group is None else int(group)
    dev = q.device
    if q_out is None:
        q_out = torch.empty_like(q)
    if k_codes is None:
        k_codes = torch.empty((T, Hkv, d_h // 2), dtype=torch.uint8, device=dev)
    if k_scales is None:
        k_scales = torch.empty((T, Hkv, d_h // group), dtype=torch.float16, device=dev)
    if stats is None:
        stats = torch.empty(6, dtype=torch.float64, device=dev)
    need = dequant_error_workspace_bytes(T, Hkv, d_h, group)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    for name, t in (("q", q), ("k", k), ("pos", pos), ("cos_tab", cos_tab), ("sin_tab", sin_tab)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    style, mp = _rope_args(cos_tab, rope_style, split_table, max_pos)
    _check(_lib.qkq_transform_quantize_stats(
        _ptr(q), _ptr(k), _ptr(pos), T, Hq, Hkv, d_h, style, _ptr(cos_tab), _ptr(sin_tab), mp,
        _ptr(phi), MODES[mode], int(b or 0), group, _ptr(q_out), _ptr(k_codes), _ptr(k_scales),
        _ptr(stats), _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(), _ptr(status),
        _stream(stream)), "qkq_transform_quantize_stats")
    return q_out, k_codes, k_scales, stats


def transform_quantize_calibrate(q, k, pos, cos_tab, sin_tab, moments=None, *, mode="hadamard",
                                 b=0, group=None, phi=None, rope_style="half", q_out=None,
                                 k_codes=None, k_scales=None, workspace=None, status=None,
                                 stream=None, split_table=False, max_pos=None):
    """transform_quantize plus accumulate_moments of the same tokens in one pass
    (``qkq_transform_quantize_calibrate``): the moments (float64 [2, d_h/2, 6], created
    zeroed when None, ADDED TO otherwise) are of the post-RoPE values, for the next solve.
    Returns (q_out, k_codes, k_scales, moments)."""
    import torch
    T, Hq, d_h = q.shape
    Hkv = k.shape[1]
    group = d_h if group is None else int(group)
    dev = q.device
    if q_out is None:
        q_out = torch.empty_like(q)
    if k_codes is None:
        k_codes = torch.empty((T, Hkv, d_h // 2), dtype=torch.uint8, device=dev)
    if k_scales is None:
        k_scales = torch.empty((T, Hkv, d_h // group), dtype=torch.float16, device=dev)
    if moments is None:
        moments = torch.zeros((2, d_h // 2, 6), dtype=torch.float64, device=dev)
    need = moments_workspace_bytes(T, Hq, Hkv, d_h)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    for name, t in (("q", q), ("k", k), ("pos", pos), ("cos_tab", cos_tab), ("sin_tab", sin_tab)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    style, mp = _rope_args(cos_tab, rope_style, split_table, max_pos)
    _check(_lib.qkq_transform_quantize_calibrate(
        _ptr(q), _ptr(k), _ptr(pos), T, Hq, Hkv, d_h, style, _ptr(cos_tab), _ptr(sin_tab), mp,
        _ptr(phi), MODES[mode], int(b or 0), group, _ptr(q_out), _ptr(k_codes), _ptr(k_scales),
        _ptr(moments), _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(), _ptr(status),
        _stream(stream)), "qkq_transform_quantize_calibrate")
    return q_out, k_codes, k_scales, moments


def transform_quantize_qkv(q, k, v, pos, cos_tab, sin_tab, *, mode="hadamard", b=0, group=None,
                           phi=None, rope_style="half", q_out=None, k_codes=None, k_scales=None,
                           v_codes=None, v_scales=None, want_f32=False, status=None,
                           stream=None, split_table=False, max_pos=None):
    """Q and K as transform_quantize, plus the value rows v [T, Hkv, d_h] bf16 in the same
    launch (``qkq_transform_quantize_qkv``: full-head Hadamard, no RoPE, then the K
    quantiser).  Returns (q_out, k_codes, k_scales, v_codes, v_scales, k_f32, v_f32); the
    fp32 copies are None unless want_f32."""
    import torch
    T, Hq, d_h = q.shape
    Hkv = k.shape[1]
    group = d_h if group is None else int(group)
    dev = q.device
    if tuple(v.shape) != tuple(k.shape) or not v.is_contiguous():
        raise ValueError("v must be a contiguous tensor shaped like k")
    if q_out is None:
        q_out = torch.empty_like(q)
    if k_codes is None:
        k_codes = torch.empty((T, Hkv, d_h // 2), dtype=torch.uint8, device=dev)
    if k_scales is None:
        k_scales = torch.empty((T, Hkv, d_h // group), dtype=torch.float16, device=dev)
    if v_codes is None:
        v_codes = torch.empty((T, Hkv, d_h // 2), dtype=torch.uint8, device=dev)
    if v_scales is None:
        v_scales = torch.empty((T, Hkv, d_h // group), dtype=torch.float16, device=dev)
    k_f32 = torch.empty((T, Hkv, d_h), dtype=torch.float32, device=dev) if want_f32 else None
    v_f32 = torch.empty((T, Hkv, d_h), dtype=torch.float32, device=dev) if want_f32 else None
    for name, t in (("q", q), ("k", k), ("pos", pos), ("cos_tab", cos_tab), ("sin_tab", sin_tab)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    style, mp = _rope_args(cos_tab, rope_style, split_table, max_pos)
    _check(_lib.qkq_transform_quantize_qkv(
        _ptr(q), _ptr(k), _ptr(v), _ptr(pos), T, Hq, Hkv, d_h, style, _ptr(cos_tab),
        _ptr(sin_tab), mp, _ptr(phi), MODES[mode], int(b or 0), group, _ptr(q_out),
        _ptr(k_codes), _ptr(k_scales), _ptr(v_codes), _ptr(v_scales), _ptr(k_f32), _ptr(v_f32),
        _ptr(status), _stream(stream)), "qkq_transform_quantize_qkv")
    return q_out, k_codes, k_scales, v_codes, v_scales, k_f32, v_f32


def transform_quantize_tc(q, k, pos, cos_tab, sin_tab, *, mode="hadamard", b=0, group=None,
                          phi=None, rope_style="half", q_out=None, k_codes=None, k_scales=None,
                          k_f32=None, want_k_f32=False, status=None, stream=None):
    """The Hadamard modes with the mixing on the tensor cores
    (``qkq_transform_quantize_tc``): same arguments and outputs as transform_quantize,
    within a stated bound of it rather than bit for bit; q_out must not alias q."""
    return _transform(_lib.qkq_transform_quantize_tc, "qkq_transform_quantize_tc", q, k, pos,
                      cos_tab, sin_tab, mode, b, group, phi, rope_style, q_out, k_codes,
                      k_scales, k_f32, want_k_f32, status, stream, False, None)


def _transform(fn, where, q, k, pos, cos_tab, sin_tab, mode, b, group, phi, rope_style, q_out,
               k_codes, k_scales, k_f32, want_k_f32, status, stream, split_table, max_pos):
    import torch
    T, Hq, d_h = q.shape
    Hkv = k.shape[1]
    group = d_h if group is None else int(group)
    dev = q.device
    if q_out is None:
        q_out = torch.empty_like(q)
    if k_codes is None:
        k_codes = torch.empty((T, Hkv, d_h // 2), dtype=torch.uint8, device=dev)
    if k_scales is None:
        k_scales = torch.empty((T, Hkv, d_h // group), dtype=torch.float16, device=dev)
    if k_f32 is None and want_k_f32:
        k_f32 = torch.empty((T, Hkv, d_h), dtype=torch.float32, device=dev)
    for name, t in (("q", q), ("k", k), ("pos", pos), ("cos_tab", cos_tab), ("sin_tab", sin_tab)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    style, mp = _rope_args(cos_tab, rope_style, split_table, max_pos)
    _check(fn(
        _ptr(q), _ptr(k), _ptr(pos), T, Hq, Hkv, d_h, style, _ptr(cos_tab),
        _ptr(sin_tab), mp, _ptr(phi), MODES[mode], int(b or 0), group,
        _ptr(q_out), _ptr(k_codes), _ptr(k_scales), _ptr(k_f32), _ptr(status), _stream(stream)),
        where)
    return q_out, k_codes, k_scales, k_f32


# ---------------------------------------------------------------- KV4 consumer ----

def _scores_args(q_t, k_codes, k_scales, scores):
    import torch
    Tq, Hq, d_h = q_t.shape
    Tk, hkv, half = k_codes.shape
    group = d_h // k_scales.shape[-1]
    if scores is None:
        scores = torch.empty((Tq, Hq, Tk), dtype=torch.float32, device=q_t.device)
    for name, t in (("q_t", q_t), ("k_codes", k_codes), ("k_scales", k_scales), ("scores", scores)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    return Tq, Hq, d_h, Tk, hkv, group, scores


def attention_scores(q_t, k_codes, k_scales, *, Hkv=None, scores=None, stream=None):
    """Attention logits of transformed queries q_t [Tq, Hq, d_h] (bf16) against the int4
    key cache (k_codes [Tk, Hkv, d_h/2] uint8, k_scales [Tk, Hkv, d_h/group] fp16):
    float32 [Tq, Hq, Tk] (``qkq_attention_scores``)."""
    Tq, Hq, d_h, Tk, hkv, group, scores = _scores_args(q_t, k_codes, k_scales, scores)
    _check(_lib.qkq_attention_scores(_ptr(q_t), Tq, _ptr(k_codes), _ptr(k_scales), Tk, Hq, hkv,
                                     d_h, group, _ptr(scores), _stream(stream)),
           "qkq_attention_scores")
    return scores


def attention_scores_tc(q_t, k_codes, k_scales, *, scores=None, status=None, stream=None):
    """The same logits with the per-group sums on the tensor cores
    (``qkq_attention_scores_tc``)."""
    Tq, Hq, d_h, Tk, hkv, group, scores = _scores_args(q_t, k_codes, k_scales, scores)
    _check(_lib.qkq_attention_scores_tc(_ptr(q_t), Tq, _ptr(k_codes), _ptr(k_scales), Tk, Hq,
                                        hkv, d_h, group, _ptr(scores), _ptr(status),
                                        _stream(stream)),
           "qkq_attention_scores_tc")
    return scores


def attention_scores_mma(q_t, k_codes, k_scales, *, scores=None, stream=None):
    """The same logits on the tensor cores with the codes unpacked into register operands,
    for decode-sized query blocks (``qkq_attention_scores_mma``)."""
    Tq, Hq, d_h, Tk, hkv, group, scores = _scores_args(q_t, k_codes, k_scales, scores)
    _check(_lib.qkq_attention_scores_mma(_ptr(q_t), Tq, _ptr(k_codes), _ptr(k_scales), Tk, Hq,
                                         hkv, d_h, group, _ptr(scores), _stream(stream)),
           "qkq_attention_scores_mma")
    return scores


# ---------------------------------------------------------------- calibration -----

def moments_workspace_bytes(T: int, Hq: int, Hkv: int, d_h: int) -> int:
    return int(_lib.qkq_moments_workspace_bytes(int(T), int(Hq), int(Hkv), int(d_h)))


def accumulate_moments(q, k, pos, cos_tab, sin_tab, moments=None, *, rope_style="half",
                       workspace=None, status=None, stream=None, split_table=False,
                       max_pos=None):
    """Add the raw per-pair accumulators of this batch into ``moments``
    (float64 [2, d_h/2, 6], created zeroed when None); returns it."""
    import torch
    T, Hq, d_h = q.shape
    Hkv = k.shape[1]
    if moments is None:
        moments = torch.zeros((2, d_h // 2, 6), dtype=torch.float64, device=q.device)
    need = moments_workspace_bytes(T, Hq, Hkv, d_h)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    style, mp = _rope_args(cos_tab, rope_style, split_table, max_pos)
    _check(_lib.qkq_accumulate_moments(
        _ptr(q), _ptr(k), _ptr(pos), T, Hq, Hkv, d_h, style, _ptr(cos_tab),
        _ptr(sin_tab), mp, _ptr(moments), _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(), _ptr(status),
        _stream(stream)), "qkq_accumulate_moments")
    return moments


def accumulate_moments_noalloc(q, k, pos, cos_tab, sin_tab, moments, *, rope_style="half",
                               status=None, stream=None, split_table=False, max_pos=None):
    """``accumulate_moments`` for callers that cannot allocate device memory: the
    library's fixed 5 MiB scratch replaces the workspace, so nothing is allocated here
    either (``moments`` must be passed in).  The scratch holds the partial sums of the
    workspace entry point's largest grid, so every batch fits and the results are the
    same bit for bit; calls that overlap on the GPU share the scratch and must be
    serialised."""
    T, Hq, d_h = q.shape
    Hkv = k.shape[1]
    style, mp = _rope_args(cos_tab, rope_style, split_table, max_pos)
    _check(_lib.qkq_accumulate_moments_noalloc(
        _ptr(q), _ptr(k), _ptr(pos), T, Hq, Hkv, d_h, style, _ptr(cos_tab),
        _ptr(sin_tab), mp, _ptr(moments), _ptr(status), _stream(stream)),
        "qkq_accumulate_moments_noalloc")
    return moments


def solve_angles(moments, estimator="pooled", *, phi=None, min_maxvar=None, status=None,
                 stream=None):
    """Closed-form head-shared angles phi*_k (float32 [d_h/2]) from the accumulators;
    status (int32 device tensor, nullable) receives the empty-stream bit."""
    import torch
    P = moments.shape[1]
    if phi is None:
        phi = torch.empty(P, dtype=torch.float32, device=moments.device)
    _check(_lib.qkq_solve_angles(_ptr(moments), 2 * P, ESTIMATORS[estimator], _ptr(phi),
                                 _ptr(min_maxvar), _ptr(status), _stream(stream)),
           "qkq_solve_angles")
    return phi


# ---------------------------------------------------------------- measurement -----

def dequant_error_workspace_bytes(T: int, Hkv: int, d_h: int, group: int) -> int:
    return int(_lib.qkq_dequant_error_workspace_bytes(int(T), int(Hkv), int(d_h), int(group)))


def dequant_error(k_f32, k_codes, k_scales, *, stats=None, workspace=None, status=None,
                  stream=None):
    """K range / relative quantisation error statistics (float64 [6], ``qkq_dequant_error``)
    of quantised keys against the fp32 K~ they came from: k_f32 [T, Hkv, d_h] float32,
    k_codes [T, Hkv, d_h/2] uint8, k_scales [T, Hkv, d_h/group] float16 (CUDA tensors)."""
    import torch
    T, Hkv, d_h = k_f32.shape
    group = d_h // k_scales.shape[-1]
    if stats is None:
        stats = torch.empty(6, dtype=torch.float64, device=k_f32.device)
    need = dequant_error_workspace_bytes(T, Hkv, d_h, group)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=k_f32.device)
    for name, t in (("k_f32", k_f32), ("k_codes", k_codes), ("k_scales", k_scales)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    _check(_lib.qkq_dequant_error(
        _ptr(k_f32), _ptr(k_codes), _ptr(k_scales), T, Hkv, d_h, group, _ptr(stats),
        _ptr(workspace), 0 if workspace is None else workspace.numel() * workspace.element_size(),
        _ptr(status), _stream(stream)), "qkq_dequant_error")
    return stats


def dequant_error_recompute(k, pos, cos_tab, sin_tab, k_codes, k_scales, *, mode="hadamard",
                            b=0, group=None, phi=None, rope_style="half", stats=None,
                            workspace=None, status=None, stream=None, split_table=False,
                            max_pos=None):
    """The same statistics for codes of ``transform_quantize``, K~ recomputed from the bf16
    keys with the transform's arguments (``qkq_dequant_error_recompute``)."""
    import torch
    T, Hkv, d_h = k.shape
    group = d_h if group is None else int(group)
    if stats is None:
        stats = torch.empty(6, dtype=torch.float64, device=k.device)
    need = dequant_error_workspace_bytes(T, Hkv, d_h, group)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=k.device)
    style, mp = _rope_args(cos_tab, rope_style, split_table, max_pos)
    _check(_lib.qkq_dequant_error_recompute(
        _ptr(k), _ptr(pos), T, Hkv, d_h, style, _ptr(cos_tab), _ptr(sin_tab),
        mp, _ptr(phi), MODES[mode], int(b or 0), group, _ptr(k_codes),
        _ptr(k_scales), _ptr(stats), _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(), _ptr(status),
        _stream(stream)), "qkq_dequant_error_recompute")
    return stats


def dequant_summary(stats) -> dict:
    """The library's summary of a stats[6] record (``qkq_dequant_summary``): K range, relative
    quantisation error, mean group range and the largest group max|K~|."""
    import numpy as np
    host = np.ascontiguousarray(
        stats.detach().cpu().numpy() if hasattr(stats, "detach") else stats, dtype=np.float64)
    out = np.zeros(4, dtype=np.float64)
    _check(_lib.qkq_dequant_summary(host.ctypes.data_as(ctypes.c_void_p),
                                    out.ctypes.data_as(ctypes.c_void_p)), "qkq_dequant_summary")
    return {"k_range": float(out[0]), "rel_error": float(out[1]),
            "mean_group_range": float(out[2]), "max_group_amax": float(out[3])}


def k_range(stats) -> float:
    """K range (mean over groups of max|K~|) of a stats[6] record, by the library."""
    return dequant_summary(stats)["k_range"]


def rel_error(stats) -> float:
    """Relative quantisation error ||K~ - K^||_F / ||K~||_F of a stats[6] record, by the
    library."""
    return dequant_summary(stats)["rel_error"]
