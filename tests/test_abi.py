"""CPU checks of the C ABI boundary (no GPU needed): the shared library loads,
exports every function include/qkq.h declares, rejects bad arguments on the host
before touching the device, and builds the RoPE table exactly as the oracle does.
"""
import ctypes
import math
import os
import re

import numpy as np
import pytest

from tests.conftest import ROOT

qkq = pytest.importorskip("transform_rope_head_b200")
from oracle import bitspec  # noqa: E402

HEADER = os.path.join(ROOT, "include", "qkq.h")


def _declared():
    with open(HEADER, encoding="utf-8") as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(qkq_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_abi():
    names = _declared()
    assert set(names) == set(qkq.SYMBOLS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(qkq.lib_path())
    for name in _declared():
        assert hasattr(lib, name), name
    assert lib.qkq_version() >= 100


def test_error_and_status_strings():
    L = qkq.lib()
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert L.qkq_error_string(code)
    assert qkq.status_string(0) == "ok"
    assert qkq.status_string(5) == "nonfinite|pos_range"
    assert qkq.status_string(16) == "empty_stream"
    assert qkq.status_string(31) == "nonfinite|scale_overflow|pos_range|timeout|empty_stream"
    assert qkq.status_string(32) == "bounds"
    assert qkq.status_string(64) == "unknown status bits"


def _tq(**over):
    """qkq_transform_quantize with plausible fake (never dereferenced) pointers."""
    a = dict(q=0x10000, k=0x20000, pos=0x30000, T=16, Hq=4, Hkv=2, d_h=64, style=0,
             cos=0x40000, sin=0x50000, max_pos=16, phi=0x60000, mode=0, b=0, group=64,
             q_out=0x70000, codes=0x80000, scales=0x90000, k_f32=None, status=None)
    a.update(over)
    L = qkq.lib()
    v = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    return L.qkq_transform_quantize(v(a["q"]), v(a["k"]), v(a["pos"]), a["T"], a["Hq"], a["Hkv"],
                                    a["d_h"], a["style"], v(a["cos"]), v(a["sin"]), a["max_pos"],
                                    v(a["phi"]), a["mode"], a["b"], a["group"], v(a["q_out"]),
                                    v(a["codes"]), v(a["scales"]), v(a["k_f32"]), v(a["status"]),
                                    None)


@pytest.mark.parametrize("over,code", [
    (dict(q=None), -1), (dict(codes=None), -1), (dict(mode=7), -1), (dict(style=2), -1),
    (dict(mode=1, phi=None), -1), (dict(mode=2, phi=None), -1),
    (dict(d_h=96), -2), (dict(d_h=256), -2), (dict(T=-1), -2), (dict(Hq=0), -2),
    (dict(Hkv=0), -2), (dict(max_pos=0), -2), (dict(group=16), -2), (dict(group=128), -2),
    (dict(mode=3, b=3), -2), (dict(mode=3, b=1), -2), (dict(mode=3, b=128), -2),
    (dict(q=0x10008), -3), (dict(cos=0x40004), -3), (dict(codes=0x80002), -3),
    (dict(scales=0x90001), -3), (dict(k_f32=0xA0008), -3),
    (dict(q_out=0x10000 + 64), -1),                       # partial overlap with q
    (dict(T=0), 0),                                        # empty: no-op, no device touched
])
def test_transform_argument_checks(over, code):
    assert _tq(**over) == code


def test_other_entry_points_reject_bad_arguments():
    L = qkq.lib()
    v = ctypes.c_void_p
    assert L.qkq_solve_angles(None, 64, 0, v(0x100), None, None, None) == -1
    assert L.qkq_solve_angles(v(0x100), 64, 5, v(0x200), None, None, None) == -1
    assert L.qkq_solve_angles(v(0x100), 96, 0, v(0x200), None, None, None) == -2
    assert L.qkq_solve_angles(v(0x100), 64, 0, v(0x200), None, v(0x302), None) == -3
    assert L.qkq_accumulate_moments(v(0x100), v(0x200), v(0x300), 8, 4, 2, 64, 0, v(0x400),
                                    v(0x500), 8, None, v(0x600), 1 << 20, None, None) == -1
    # too-small workspace is reported before any launch
    assert L.qkq_accumulate_moments(v(0x100), v(0x200), v(0x300), 8, 4, 2, 64, 0, v(0x400),
                                    v(0x500), 8, v(0x700), v(0x600), 1, None, None) == -6
    assert L.qkq_dequant_error_recompute(v(0x100), v(0x300), 8, 2, 64, 0, v(0x400), v(0x500), 8,
                                         None, 3, 5, 64, v(0x800), v(0x900), v(0xA00), v(0xB00),
                                         1 << 20, None, None) == -2


def test_noalloc_moments_rejects_bad_arguments():
    """qkq_accumulate_moments_noalloc refuses what qkq_accumulate_moments refuses, before
    anything touches the device (and T == 0 is a no-op)."""
    L = qkq.lib()
    v = ctypes.c_void_p
    ok = dict(q=v(0x1000), k=v(0x2000), pos=v(0x3000), T=8, Hq=4, Hkv=2, d=64, style=0,
              c=v(0x4000), s=v(0x5000), mp=8, m=v(0x6000), st=None)

    def call(**kw):
        a = dict(ok, **kw)
        return L.qkq_accumulate_moments_noalloc(a["q"], a["k"], a["pos"], a["T"], a["Hq"],
                                                a["Hkv"], a["d"], a["style"], a["c"], a["s"],
                                                a["mp"], a["m"], a["st"], None)
    assert call(style=2) == -1
    assert call(d=96) == -2
    assert call(T=-1) == -2
    assert call(Hq=0) == -2
    assert call(mp=0) == -2
    assert call(T=0, q=None) == 0          # nothing to do
    for name in ("q", "k", "pos", "c", "s", "m"):
        assert call(**{name: None}) == -1, name
    assert call(q=v(0x1008)) == -3
    assert call(c=v(0x4004)) == -3
    assert call(m=v(0x6004)) == -3
    assert call(st=v(0x7002)) == -3


def test_measurement_on_given_k_rejects_bad_arguments():
    """qkq_dequant_error (fp32 K~ given): sizes, null pointers and alignment are refused before
    anything touches the device."""
    L = qkq.lib()
    v = ctypes.c_void_p
    ok = dict(k=v(0x1000), c=v(0x2000), s=v(0x3000), T=8, H=2, d=64, g=64, st=v(0x4000),
              ws=v(0x5000), wsb=1 << 20)

    def call(**kw):
        a = dict(ok, **kw)
        return L.qkq_dequant_error(a["k"], a["c"], a["s"], a["T"], a["H"], a["d"], a["g"],
                                   a["st"], a["ws"], a["wsb"], None, None)
    assert call(d=96) == -2            # d_h outside {64, 128}
    assert call(g=48) == -2            # group outside {32, 64, 128}
    assert call(d=64, g=128) == -2     # group does not divide d_h
    assert call(T=-1) == -2
    assert call(H=0) == -2
    assert call(k=None) == -1
    assert call(c=None) == -1
    assert call(s=None) == -1
    assert call(st=None) == -1
    assert call(k=v(0x1004)) == -3     # K~ not 16-byte aligned
    assert call(c=v(0x2002)) == -3     # codes not 4-byte aligned
    assert call(s=v(0x3001)) == -3
    assert call(ws=v(0x5008)) == -3


def test_dequant_summary_host_arithmetic():
    """qkq_dequant_summary: K range = sum of group max|K~| / groups, relative error =
    sqrt(sum err^2 / sum K~^2), mean group range, largest group max; a hand-worked record and
    the degenerate ones."""
    L = qkq.lib()
    st = np.array([4.0, 100.0, 30.0, 45.0, 9.5, 6.0])
    out = np.zeros(4)
    P = ctypes.c_void_p
    assert L.qkq_dequant_summary(st.ctypes.data_as(P), out.ctypes.data_as(P)) == 0
    np.testing.assert_array_equal(out, [5.0, 0.2, 7.5, 9.5])
    st = np.zeros(6)
    assert L.qkq_dequant_summary(st.ctypes.data_as(P), out.ctypes.data_as(P)) == 0
    np.testing.assert_array_equal(out, [0.0, 0.0, 0.0, 0.0])
    st = np.array([1.0, 0.0, 0.0, 0.0, 0.0, 2.0])
    assert L.qkq_dequant_summary(st.ctypes.data_as(P), out.ctypes.data_as(P)) == 0
    assert math.isinf(out[1])
    assert L.qkq_dequant_summary(None, out.ctypes.data_as(P)) == -1
    assert L.qkq_dequant_summary(st.ctypes.data_as(P), None) == -1
    assert qkq.k_range(np.array([4.0, 100.0, 30.0, 45.0, 9.5, 6.0])) == 5.0
    assert qkq.rel_error(np.array([4.0, 100.0, 30.0, 45.0, 9.5, 6.0])) == 0.2


def test_tensor_core_entry_point_rejects_what_it_does_not_cover():
    L = qkq.lib()
    v = ctypes.c_void_p
    args = lambda mode, style: (v(0x10000), v(0x20000), v(0x30000), 8, 4, 2, 64, style,  # noqa: E731
                                v(0x40000), v(0x50000), 8, v(0x60000), mode, 0, 64, v(0x70000),
                                v(0x80000), v(0x90000), None, None, None)
    assert L.qkq_transform_quantize_tc(*args(1, 0)) == -5        # pairwise: no Hadamard to run
    assert L.qkq_transform_quantize_tc(*args(4, 0)) == -5        # RoPE only
    assert L.qkq_transform_quantize_tc(*args(0, 0x100)) == -5    # split RoPE tables
    assert L.qkq_transform_quantize_tc(*args(0, 2)) == -1        # bad pair layout


@pytest.mark.parametrize("entry", ["qkq_attention_scores", "qkq_attention_scores_tc",
                                   "qkq_attention_scores_mma"])
def test_consumer_entry_points_reject_bad_arguments(entry):
    """Host checks of the KV4 consumers, before any device is touched (the tcgen05 one also
    wants 16-byte aligned queries: it reads them 16 bytes at a time; the other two read them
    2 bytes at a time)."""
    L = qkq.lib()
    v = ctypes.c_void_p
    tc = entry.endswith("_tc")

    def call(q=0x10000, Tq=2, codes=0x20000, scales=0x30000, Tk=300, Hq=8, Hkv=2, d_h=128,
             group=64, scores=0x40000):
        args = [v(q) if q else None, Tq, v(codes) if codes else None, v(scales), Tk, Hq, Hkv,
                d_h, group, v(scores) if scores else None]
        if tc:
            args.append(None)
        return getattr(L, entry)(*args, None)

    assert call(q=None) == -1 and call(scores=None) == -1 and call(codes=None) == -1
    assert call(d_h=96) == -2 and call(group=16) == -2 and call(Hq=6, Hkv=4) == -2
    assert call(Tq=-1) == -2 and call(Tq=70000) == -2
    assert call(Hq=10, Hkv=2) == -5                          # 5 query heads per key head
    assert call(codes=0x20008) == -3 and call(scores=0x40002) == -3
    if tc:
        assert call(q=0x10008) == -3
    else:
        assert call(q=0x10001) == -3
    assert call(Tq=0) == 0 and call(Tk=0) == 0               # empty: no-op


def test_workspace_sizes():
    assert qkq.moments_workspace_bytes(0, 32, 8, 128) == 0
    # per-CTA partial sums (2 streams x d_h/2 pairs x 5 sums), at most 1024 CTAs
    assert qkq.moments_workspace_bytes(131072, 32, 8, 128) == 1024 * 2 * 64 * 5 * 8
    assert qkq.moments_workspace_bytes(256, 4, 2, 64) == 64 * 2 * 32 * 5 * 8
    assert qkq.dequant_error_workspace_bytes(256, 8, 128, 128) > 0


@pytest.mark.parametrize("d_h,theta,max_pos", [(64, 5e5, 300), (128, 5e5, 4096), (128, 1e6, 2000)])
def test_rope_table_matches_oracle_bit_exact(d_h, theta, max_pos):
    """The library's host table and the oracle's are two implementations of the same
    definition (fp32 of the fp64 cos/sin of m * theta^(-2k/d_h)); they agree bit for bit."""
    c, s = qkq.rope_table(max_pos, d_h, theta, device="cpu")
    oc, os_ = bitspec.rope_table(max_pos, d_h, theta)
    np.testing.assert_array_equal(c.numpy(), oc)
    np.testing.assert_array_equal(s.numpy(), os_)


@pytest.mark.parametrize("d_h,theta,max_pos", [(64, 5e5, 2048), (128, 1e6, 32768),
                                                (128, 5e5, 131072), (64, 5e5, 1)])
def test_split_rope_table_matches_oracle_bit_exact(d_h, theta, max_pos):
    c, s = qkq.rope_table(max_pos, d_h, theta, device="cpu", split=True)
    oc, os_ = bitspec.rope_table_split(max_pos, d_h, theta)
    np.testing.assert_array_equal(c.numpy(), oc)
    np.testing.assert_array_equal(s.numpy(), os_)


def test_rope_table_rows():
    rows = qkq.rope_table_rows
    assert rows(131072, True) == 64 + 2048 and rows(131072) == 131072
    assert rows(1, True) == 65 and rows(64, True) == 65 and rows(65, True) == 66
    assert rows(0, True) == 0 and rows(0) == 0


def test_rope_table_inv_freq_override():
    inv = np.array([1.0, 0.5, 0.25, 0.125])
    c, s = qkq.rope_table(10, 8, 1.0, inv_freq=inv, device="cpu")
    import math
    want_c = np.array([[math.cos(m * w) for w in inv] for m in range(10)], dtype=np.float32)
    want_s = np.array([[math.sin(m * w) for w in inv] for m in range(10)], dtype=np.float32)
    np.testing.assert_array_equal(c.numpy(), want_c)
    np.testing.assert_array_equal(s.numpy(), want_s)


def test_selftest_hook_argument_checks():
    L = qkq.lib()
    v = ctypes.c_void_p
    assert L.qkq_selftest_bounded_wait(1000, None, None) == -1
    assert L.qkq_selftest_bounded_wait(0, v(0x100), None) == -1
    assert L.qkq_selftest_bounded_wait(10 ** 9, v(0x100), None) == -1
    assert L.qkq_selftest_bounded_wait(1000, v(0x102), None) == -3
