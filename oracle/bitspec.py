"""ctypes front end of the plain-C fp32 operation sequence (``oracle/bitspec.c``).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  The shared object is
compiled from ``bitspec.c`` by ``build()`` with gcc into ``oracle/_build/``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bitspec.c")
_OUT_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_OUT_DIR, "liborc_bitspec.so")

_CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
           "-fexcess-precision=standard", "-Wall", "-Wextra"]

_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle (gcc) if the shared object is missing or older than its source."""
    os.makedirs(_OUT_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P, I, I64, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        _lib.orc_rope_table.argtypes = [P, P, I, I, D, P]
        _lib.orc_rope_table.restype = I
        _lib.orc_rope_table_split.argtypes = [P, P, I, I, D, P]
        _lib.orc_rope_table_split.restype = I
        _lib.orc_fwht.argtypes = [P, I]
        _lib.orc_fwht.restype = None
        _lib.orc_f32_to_bf16.argtypes = [ctypes.c_float]
        _lib.orc_f32_to_bf16.restype = ctypes.c_uint16
        _lib.orc_f32_to_f16.argtypes = [ctypes.c_float]
        _lib.orc_f32_to_f16.restype = ctypes.c_uint16
        _lib.orc_f16_to_f32.argtypes = [ctypes.c_uint16]
        _lib.orc_f16_to_f32.restype = ctypes.c_float
        _lib.orc_transform_quantize.argtypes = [P, P, P, I64, I, I, I, I, P, P, I, P, I, I, I,
                                                P, P, P, P, P, P]
        _lib.orc_transform_quantize.restype = I
        _lib.orc_quantize_rows.argtypes = [P, I64, I, I, P, P]
        _lib.orc_quantize_rows.restype = I
        _lib.orc_value_quantize.argtypes = [P, I64, I, I, P, P, P]
        _lib.orc_value_quantize.restype = I
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


MODES = {"hadamard": 0, "pairwise": 1, "pairwise_hadamard": 2, "block_hadamard": 3,
         "rope_only": 4}
STYLES = {"half": 0, "interleaved": 1}


def rope_table(max_pos: int, d_h: int, theta: float, inv_freq=None):
    """fp32 cos/sin tables [max_pos, d_h/2] (fp32 of the fp64 libm values)."""
    P = d_h // 2
    c = np.empty((max_pos, P), dtype=np.float32)
    s = np.empty((max_pos, P), dtype=np.float32)
    inv = None if inv_freq is None else np.ascontiguousarray(inv_freq, dtype=np.float64)
    rc = lib().orc_rope_table(_ptr(c), _ptr(s), max_pos, d_h, float(theta), _ptr(inv))
    if rc:
        raise ValueError("orc_rope_table rejected its arguments")
    return c, s


def split_rows(max_pos: int) -> int:
    return 64 + (max_pos + 63) // 64


def rope_table_split(max_pos: int, d_h: int, theta: float, inv_freq=None):
    """Split fp32 cos/sin tables [64 + ceil(max_pos/64), d_h/2]: low rows l * w_k, then
    high rows 64 h * w_k (fp32 of the fp64 libm values)."""
    P = d_h // 2
    rows = split_rows(max_pos)
    c = np.empty((rows, P), dtype=np.float32)
    s = np.empty((rows, P), dtype=np.float32)
    inv = None if inv_freq is None else np.ascontiguousarray(inv_freq, dtype=np.float64)
    rc = lib().orc_rope_table_split(_ptr(c), _ptr(s), max_pos, d_h, float(theta), _ptr(inv))
    if rc != rows:
        raise ValueError("orc_rope_table_split rejected its arguments")
    return c, s


def quantize_rows(x: np.ndarray, group: int):
    """The fp32 quantiser on transformed rows x [..., d_h] (fp32): (packed codes, fp16 scale
    bits, status)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    d_h = x.shape[-1]
    rows = x.size // d_h
    codes = np.empty(x.shape[:-1] + (d_h // 2,), dtype=np.uint8)
    scales = np.empty(x.shape[:-1] + (d_h // group,), dtype=np.uint16)
    st = lib().orc_quantize_rows(_ptr(x), rows, d_h, group, _ptr(codes), _ptr(scales))
    if st < 0:
        raise ValueError("orc_quantize_rows rejected its arguments")
    return codes, scales, st


def value_quantize(v, group: int, want_f32: bool = False) -> dict:
    """Value rows v [..., d_h] (bf16 bits): full-head normalised Hadamard, then the K
    quantiser.  Returns v_codes, v_scales (fp16 bits), status and, with want_f32, v_f32."""
    v = np.ascontiguousarray(v, dtype=np.uint16)
    d_h = v.shape[-1]
    rows = v.size // d_h
    codes = np.empty(v.shape[:-1] + (d_h // 2,), dtype=np.uint8)
    scales = np.empty(v.shape[:-1] + (d_h // group,), dtype=np.uint16)
    f32 = np.empty(v.shape, dtype=np.float32) if want_f32 else None
    st = lib().orc_value_quantize(_ptr(v), rows, d_h, group, _ptr(codes), _ptr(scales), _ptr(f32))
    if st < 0:
        raise ValueError("orc_value_quantize rejected its arguments")
    out = {"v_codes": codes, "v_scales": scales, "status": st}
    if want_f32:
        out["v_f32"] = f32
    return out


def fwht(x: np.ndarray) -> np.ndarray:
    """Unnormalised fp32 FWHT of a 1-D power-of-two-length vector (strides 1, 2, ...)."""
    y = np.ascontiguousarray(x, dtype=np.float32).copy()
    lib().orc_fwht(_ptr(y), y.shape[0])
    return y


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    f = lib().orc_f32_to_bf16
    return np.array([f(float(v)) for v in np.asarray(x, dtype=np.float32).ravel()],
                    dtype=np.uint16).reshape(np.shape(x))


def f32_to_f16(x: np.ndarray) -> np.ndarray:
    f = lib().orc_f32_to_f16
    return np.array([f(float(v)) for v in np.asarray(x, dtype=np.float32).ravel()],
                    dtype=np.uint16).reshape(np.shape(x))


def transform_quantize(q, k, pos, d_h, theta=None, mode="hadamard", b=None, group=None,
                       phi=None, style="half", cos_t=None, sin_t=None, max_pos=None,
                       want_f32=False, split=False):
    """Run the fp32 sequence on bf16-bit inputs q [T, Hq, d_h], k [T, Hkv, d_h], pos [T].

    Either (cos_t, sin_t) or theta (+ max_pos) must be given; with split=True the tables
    are the split layout (rope_table_split) and max_pos is required when they are given.
    Returns a dict with
    q_out (bf16 bits), k_codes (packed uint8), k_scales (fp16 bits), status, and,
    with want_f32, the fp32 transformed rows q_f32 / k_f32.
    """
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    T, Hq, _ = q.shape
    Hkv = k.shape[1]
    group = d_h if group is None else group
    if cos_t is None:
        if max_pos is None:
            max_pos = int(pos.max()) + 1 if T else 1
        cos_t, sin_t = (rope_table_split if split else rope_table)(max_pos, d_h, theta)
    cos_t = np.ascontiguousarray(cos_t, dtype=np.float32)
    sin_t = np.ascontiguousarray(sin_t, dtype=np.float32)
    if split:
        if max_pos is None or cos_t.shape[0] != split_rows(max_pos):
            raise ValueError("split tables need max_pos with 64 + ceil(max_pos/64) rows")
    else:
        max_pos = cos_t.shape[0]
    phi_a = None if phi is None else np.ascontiguousarray(phi, dtype=np.float32)
    q_out = np.empty_like(q)
    codes = np.empty((T, Hkv, d_h // 2), dtype=np.uint8)
    scales = np.empty((T, Hkv, d_h // group), dtype=np.uint16)
    k_f32 = np.empty((T, Hkv, d_h), dtype=np.float32) if want_f32 else None
    q_f32 = np.empty((T, Hq, d_h), dtype=np.float32) if want_f32 else None
    status = ctypes.c_int(0)
    rc = lib().orc_transform_quantize(
        _ptr(q), _ptr(k), _ptr(pos), T, Hq, Hkv, d_h, STYLES[style] | (0x100 if split else 0),
        _ptr(cos_t), _ptr(sin_t),
        max_pos, _ptr(phi_a), MODES[mode], 0 if b is None else int(b), group, _ptr(q_out),
        _ptr(codes), _ptr(scales), _ptr(k_f32), _ptr(q_f32), ctypes.byref(status))
    if rc:
        raise ValueError("orc_transform_quantize rejected its arguments")
    out = {"q_out": q_out, "k_codes": codes, "k_scales": scales, "status": status.value}
    if want_f32:
        out["k_f32"] = k_f32
        out["q_f32"] = q_f32
    return out
