"""Helpers for the GPU parity tests: move the seeded synthetic inputs to the device,
run the library through its C ABI (the Python binding), run the oracle on the same
bytes, and compare."""
import numpy as np

import synth


def torch_mod():
    import torch
    return torch


def to_dev_bf16(a: np.ndarray):
    torch = torch_mod()
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def bits16(t) -> np.ndarray:
    """bf16 / fp16 device tensor -> uint16 numpy bit patterns."""
    torch = torch_mod()
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bits32(a) -> np.ndarray:
    if not isinstance(a, np.ndarray):
        a = a.contiguous().cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


class DevInputs:
    """Device copies of one synthetic draw plus the library's RoPE tables."""

    def __init__(self, inp: dict, max_pos: int | None = None):
        import transform_rope_head_b200 as qkq
        torch = torch_mod()
        w = inp["workload"]
        self.w = w
        self.inp = inp
        self.max_pos = w.max_pos if max_pos is None else max_pos
        self.q = to_dev_bf16(inp["q"])
        self.k = to_dev_bf16(inp["k"])
        self.pos = torch.from_numpy(inp["pos"]).cuda()
        self.cos, self.sin = qkq.rope_table(self.max_pos, w.d_h, w.theta)
        self._split = None

    def split_tables(self):
        """The split (two-level) RoPE tables for the same positions, built on first use."""
        import transform_rope_head_b200 as qkq
        if self._split is None:
            self._split = qkq.rope_table(self.max_pos, self.w.d_h, self.w.theta, split=True)
        return self._split

    def tables(self, split: bool):
        """(cos, sin, keyword arguments) for the library calls."""
        if split:
            c, s = self.split_tables()
            return c, s, {"split_table": True, "max_pos": self.max_pos}
        return self.cos, self.sin, {}


def random_phi(P: int, seed: int = 99) -> np.ndarray:
    r = np.random.default_rng(seed)
    return r.uniform(-np.pi / 4, np.pi / 4, P).astype(np.float32)


def draw(name: str, T: int | None = None, seed: int | None = None) -> dict:
    return synth.make_inputs(name, T=T, seed=seed)
