"""CPU oracle for the post-RoPE Q/K transform with dynamic KV4 quantisation.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import, call,
link or run anything under ``oracle/``.  The product package
``transform_rope_head_b200`` never imports it, and it imports nothing from the
product; the two share only the seeded input generators in ``synth/``.

Two layers:

* ``definition`` — the method in float64 numpy, written as its definition
  (dense Hadamard matrices, plain sums), pinned by ``tests/test_oracle_*.py``
  against closed forms, invariants, the pages' worked example and brute force.
* ``bitspec`` — the same transform as one fixed fp32 order of operations in
  plain C, because the 4-bit codes are integers decided by floating point and
  must be decided in the kernel's precision on both sides.  It is pinned to the
  float64 definition (tolerances derived from fp32 rounding) and to the same
  closed forms.

Every function is a parity reference; none is tuned for speed.
"""
from . import bitspec, definition  # noqa: F401

__all__ = ["bitspec", "definition"]
