"""Seeded synthetic Q/K activations for the post-RoPE Q/K transform.

This module is the one piece that both sides use: the CPU oracle (``oracle/``)
and the CUDA library (``transform_rope_head_b200``) read the same bytes it
writes. It therefore holds none of the transform's own arithmetic: no RoPE, no
Hadamard, no pair rotation, no quantiser. It only draws pre-RoPE activations
with the shapes and value distributions of the attention layers studied in
"When Local Variance Optimality Is Not Enough: RoPE-Aligned Q/K Rotations for
Dynamic 4-Bit Quantisation" (Methodology: Llama-3.2-1B, Llama-3.2-3B,
Llama-3.1-8B and Mistral-7B-v0.3), and rounds them to bfloat16.

Layouts (token-major, contiguous):
  q    uint16 [T, Hq,  d_h]   bfloat16 bit patterns
  k    uint16 [T, Hkv, d_h]   bfloat16 bit patterns
  pos  int32  [T]             RoPE position of each token

Three value distributions are used (named after the workloads that use them):

* ``gauss_outlier``: N(0, 1) per channel; in every head three distinct channels,
  drawn once per layer, are multiplied by 20.
* ``gauss_outlier_lognormal``: ``gauss_outlier`` times a per-token magnitude
  exp(N(0, 1)), one draw per token and per stream (Q and K separately).
* ``student_t_aniso``: per stream and per RoPE frequency pair k a random SPD
  covariance  S_k = R(a) diag(1, 1/c) R(a)^T,  a ~ U[0, pi), c ~ U[1, 50],
  shared by all heads of the stream; x = S_k^(1/2) z with z iid Student-t(4)/sqrt(2)
  (unit variance); 1 % of the (head, channel) slots are multiplied by 30.

The pairs used to shape ``student_t_aniso`` follow the RoPE pair layout the
workload names ("half": channels (k, k + d_h/2); "interleaved": (2k, 2k + 1)).

Everything is deterministic for a given (workload, seed, T): the per-layer
parameters come from ``layer_seed`` and the token draws from ``seed``; token
chunks use child seeds of ``numpy.random.SeedSequence`` so the bytes do not
depend on the number of threads.
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

__all__ = [
    "Workload",
    "WORKLOADS",
    "f32_to_bf16_bits",
    "bf16_bits_to_f32",
    "make_inputs",
    "make_positions",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape, RoPE base and value distribution of one synthetic attention layer."""

    name: str
    T: int                    # tokens (batch * seq) per call
    Hq: int                   # query heads
    Hkv: int                  # key/value heads
    d_h: int                  # head dimension
    theta: float              # RoPE base
    group: int                # K quantisation group size (channels)
    max_pos: int              # rows of the cos/sin table
    distribution: str         # see module docstring
    layer_seed: int           # per-layer parameters (outlier slots, covariances)
    seed: int                 # token draws
    positions: str            # "seq:<L>" (tokens are sequences of length L), "uniform"
    rope_style: str = "half"  # "half" or "interleaved"
    note: str = ""

    @property
    def P(self) -> int:
        return self.d_h // 2


# The five workloads of the build, sized like the pages' checkpoints.
WORKLOADS: dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny", T=256, Hq=4, Hkv=2, d_h=64, theta=5e5, group=64, max_pos=256,
                 distribution="gauss_outlier", layer_seed=1, seed=1001, positions="seq:256",
                 note="tiny correctness case"),
        Workload("llama32_1b", T=2048, Hq=32, Hkv=8, d_h=64, theta=5e5, group=64, max_pos=2048,
                 distribution="student_t_aniso", layer_seed=2, seed=1002, positions="seq:2048",
                 note="Llama-3.2-1B attention shape, one 2048-token sequence"),
        Workload("llama32_3b", T=8 * 4096, Hq=24, Hkv=8, d_h=128, theta=5e5, group=128,
                 max_pos=4096, distribution="gauss_outlier_lognormal", layer_seed=3, seed=1003,
                 positions="seq:4096", note="Llama-3.2-3B shape, batch 8 x 4096"),
        Workload("llama31_8b_128k", T=131072, Hq=32, Hkv=8, d_h=128, theta=5e5, group=128,
                 max_pos=131072, distribution="student_t_aniso", layer_seed=4, seed=1004,
                 positions="seq:131072",
                 note="Llama-3.1-8B shape, one 128K-token prefill"),
        Workload("mistral7b_decode", T=256, Hq=32, Hkv=8, d_h=128, theta=1e6, group=128,
                 max_pos=32768, distribution="student_t_aniso", layer_seed=5, seed=1005,
                 positions="uniform", note="Mistral-7B-v0.3 shape, 256 decode tokens"),
    ]
}

# Calibration set of the 1B shape: 128 sequences of 2048 tokens, its own token seed.
CALIBRATION = {"llama32_1b": dict(sequences=128, seq_len=2048, seed=1102)}


# ---------------------------------------------------------------------------
# bfloat16 bit patterns (input rounding of the synthetic data)
# ---------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); returns uint16 bits.

    Only finite inputs are produced by this module.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns (uint16) to float32 exactly."""
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---------------------------------------------------------------------------
# per-layer parameters
# ---------------------------------------------------------------------------

def _pair_channels(d_h: int, style: str) -> tuple[np.ndarray, np.ndarray]:
    P = d_h // 2
    k = np.arange(P)
    if style == "half":
        return k, k + P
    if style == "interleaved":
        return 2 * k, 2 * k + 1
    raise ValueError(f"unknown rope style {style!r}")


def _layer_params(w: Workload) -> dict:
    rng = np.random.default_rng(np.random.SeedSequence([w.layer_seed, 0x51A7]))
    out = {}
    for stream, H in (("q", w.Hq), ("k", w.Hkv)):
        p = {}
        if w.distribution.startswith("gauss_outlier"):
            # three distinct outlier channels per head
            p["outliers"] = np.stack([rng.choice(w.d_h, size=3, replace=False) for _ in range(H)])
        elif w.distribution == "student_t_aniso":
            a = rng.uniform(0.0, np.pi, size=w.P)
            c = rng.uniform(1.0, 50.0, size=w.P)
            # S^(1/2) = R(a) diag(1, 1/sqrt(c)) R(a)^T, per pair
            ca, sa = np.cos(a), np.sin(a)
            e1, e2 = np.ones_like(c), 1.0 / np.sqrt(c)
            m00 = ca * ca * e1 + sa * sa * e2
            m01 = ca * sa * (e1 - e2)
            m11 = sa * sa * e1 + ca * ca * e2
            p["sqrt_cov"] = np.stack([m00, m01, m11]).astype(np.float32)  # [3, P]
            n_slots = H * w.d_h
            n_out = max(1, int(round(0.01 * n_slots)))
            p["outlier_slots"] = rng.choice(n_slots, size=n_out, replace=False)
        else:
            raise ValueError(f"unknown distribution {w.distribution!r}")
        out[stream] = p
    return out


# ---------------------------------------------------------------------------
# token draws
# ---------------------------------------------------------------------------

_CHUNK = 4096  # tokens per independently seeded chunk


def _draw_chunk(w: Workload, params: dict, stream: str, H: int, seq: np.random.SeedSequence,
                n_tok: int) -> np.ndarray:
    rng = np.random.default_rng(seq)
    d = w.d_h
    if w.distribution.startswith("gauss_outlier"):
        x = rng.standard_normal((n_tok, H, d), dtype=np.float32)
        o = params["outliers"]                                   # [H, 3]
        x[:, np.arange(H)[:, None], o] *= np.float32(20.0)
        if w.distribution == "gauss_outlier_lognormal":
            mag = np.exp(rng.standard_normal(n_tok, dtype=np.float32))
            x *= mag[:, None, None]
        return x
    # student_t_aniso: z ~ t(4)/sqrt(2), via t = g / sqrt(chi2_4 / 4), chi2_4/4 = -ln(u1 u2)/2
    shape = (n_tok, H, d)
    g = rng.standard_normal(shape, dtype=np.float32)
    u1 = rng.random(shape, dtype=np.float32)
    u2 = rng.random(shape, dtype=np.float32)
    w2 = (np.float32(1.0) - u1) * (np.float32(1.0) - u2)
    z = g / np.sqrt(np.float32(-0.5) * np.log(w2)) * np.float32(1.0 / np.sqrt(2.0))
    del g, u1, u2, w2
    ia, ib = _pair_channels(d, w.rope_style)
    m00, m01, m11 = params["sqrt_cov"]
    za, zb = z[:, :, ia], z[:, :, ib]
    x = np.empty_like(z)
    x[:, :, ia] = m00 * za + m01 * zb
    x[:, :, ib] = m01 * za + m11 * zb
    xf = x.reshape(n_tok, H * d)
    xf[:, params["outlier_slots"]] *= np.float32(30.0)
    return x


def _draw_stream(w: Workload, params: dict, stream: str, H: int, T: int, seed: int,
                 threads: int) -> np.ndarray:
    out = np.empty((T, H, w.d_h), dtype=np.uint16)
    n_chunks = (T + _CHUNK - 1) // _CHUNK
    root = np.random.SeedSequence([seed, 0 if stream == "q" else 1])
    kids = root.spawn(n_chunks)

    def job(i: int) -> None:
        t0 = i * _CHUNK
        n = min(_CHUNK, T - t0)
        out[t0:t0 + n] = f32_to_bf16_bits(_draw_chunk(w, params, stream, H, kids[i], n))

    if threads <= 1 or n_chunks == 1:
        for i in range(n_chunks):
            job(i)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(job, range(n_chunks)))
    return out


def make_positions(w: Workload, T: int, seed: int) -> np.ndarray:
    """RoPE positions: consecutive within each sequence, or uniform in [0, max_pos)."""
    if w.positions.startswith("seq:"):
        L = int(w.positions.split(":")[1])
        return (np.arange(T, dtype=np.int64) % L).astype(np.int32)
    if w.positions == "uniform":
        rng = np.random.default_rng(np.random.SeedSequence([seed, 2]))
        return rng.integers(0, w.max_pos, size=T, dtype=np.int64).astype(np.int32)
    raise ValueError(w.positions)


def make_inputs(name: str | Workload, T: int | None = None, seed: int | None = None,
                threads: int | None = None, calibration: bool = False) -> dict:
    """Draw Q, K (bf16 bits) and positions for a workload.

    ``T`` overrides the token count (a prefix of the same sequence layout),
    ``seed`` the token seed; ``calibration=True`` draws the workload's
    calibration set instead (same layer parameters, its own seed).
    """
    w = WORKLOADS[name] if isinstance(name, str) else name
    if calibration:
        c = CALIBRATION[w.name]
        T = c["sequences"] * c["seq_len"] if T is None else T
        seed = c["seed"] if seed is None else seed
    T = w.T if T is None else int(T)
    seed = w.seed if seed is None else int(seed)
    threads = min(8, os.cpu_count() or 1) if threads is None else threads
    params = _layer_params(w)
    q = _draw_stream(w, params["q"], "q", w.Hq, T, seed, threads)
    k = _draw_stream(w, params["k"], "k", w.Hkv, T, seed, threads)
    pos = make_positions(w, T, seed)
    return {"q": q, "k": k, "pos": pos, "workload": w, "T": T, "seed": seed}
