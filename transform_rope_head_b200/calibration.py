"""Calibration artefacts on disk: per layer, the raw moment accumulators and the angles.

The only state the method keeps between calibration and inference is, per layer, the
head-shared pair angles phi [d_h/2] (fp32) that the pairwise modes apply ("Methodology" of
"When Local Variance Optimality Is Not Enough: RoPE-Aligned Q/K Rotations for Dynamic 4-Bit
Quantisation": the angles come from calibration statistics).  The raw accumulators
[2][d_h/2][6] (fp64: n, Sa, Sb, Saa, Sab, Sbb per stream and pair) are kept beside them:
``qkq_accumulate_moments`` adds into them, so a calibration resumes by loading them and
accumulating more batches, and the angles can be re-solved with another estimator.

One ``.npz`` file: ``moments`` [layers][2][d_h/2][6] float64, ``phi`` [layers][d_h/2]
float32, and ``meta`` (JSON: d_h, theta, rope_style, estimator, layer names, free-form
extras).  Values round-trip bit for bit.  Host code only (numpy); tensors on the device are
copied to the host to be saved, and loaded arrays can be moved back with torch.
"""
from __future__ import annotations

import json
import os

import numpy as np

FORMAT = "qkq-calibration-1"
ESTIMATORS = ("pooled", "k_only", "balanced")


def _host(a, dtype) -> np.ndarray:
    if hasattr(a, "detach"):  # a torch tensor, possibly on the device
        a = a.detach().cpu().numpy()
    a = np.asarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {np.dtype(dtype).name}, got {a.dtype}")
    return np.ascontiguousarray(a)


def save(path: str, moments, phi, *, d_h: int, theta: float, rope_style: str = "half",
         estimator: str = "pooled", layers=None, extra: dict | None = None) -> None:
    """Write the accumulators ``moments`` ([L][2][d_h/2][6] float64, or one layer's
    [2][d_h/2][6]) and the angles ``phi`` ([L][d_h/2] float32, or [d_h/2]) to ``path``
    (written to a temporary file first, then renamed into place)."""
    m = _host(moments, np.float64)
    p = _host(phi, np.float32)
    if m.ndim == 3:
        m = m[None]
    if p.ndim == 1:
        p = p[None]
    P = d_h // 2
    if d_h not in (64, 128) or m.shape[1:] != (2, P, 6) or p.shape != (m.shape[0], P):
        raise ValueError(f"shapes {m.shape} / {p.shape} do not match d_h = {d_h}")
    if rope_style not in ("half", "interleaved"):
        raise ValueError(f"rope_style {rope_style!r}")
    if estimator not in ESTIMATORS:
        raise ValueError(f"estimator {estimator!r}")
    names = [str(x) for x in (layers if layers is not None else range(m.shape[0]))]
    if len(names) != m.shape[0]:
        raise ValueError("one name per layer")
    meta = {"format": FORMAT, "d_h": int(d_h), "theta": float(theta), "rope_style": rope_style,
            "estimator": estimator, "layers": names, "extra": extra or {}}
    tmp = f"{path}.tmp{os.getpid()}.npz"
    np.savez(tmp, moments=m, phi=p, meta=np.frombuffer(json.dumps(meta).encode(), np.uint8))
    os.replace(tmp, path)


def load(path: str) -> dict:
    """The saved artefacts: ``moments`` [L][2][d_h/2][6] float64, ``phi`` [L][d_h/2] float32
    and the metadata keys (d_h, theta, rope_style, estimator, layers, extra)."""
    with np.load(path, allow_pickle=False) as z:
        meta = json.loads(bytes(z["meta"]).decode())
        if meta.get("format") != FORMAT:
            raise ValueError(f"{path}: not a calibration file of this format")
        out = dict(meta)
        out["moments"] = z["moments"].astype(np.float64, copy=True)
        out["phi"] = z["phi"].astype(np.float32, copy=True)
    P = out["d_h"] // 2
    L = len(out["layers"])
    if out["moments"].shape != (L, 2, P, 6) or out["phi"].shape != (L, P):
        raise ValueError(f"{path}: array shapes do not match the metadata")
    return out
