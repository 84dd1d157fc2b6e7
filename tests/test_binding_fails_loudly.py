"""The product path has no CPU fallback: without its compiled library the binding refuses
to import (and never reaches for the oracle)."""
import os
import subprocess
import sys

from tests.conftest import ROOT


def test_import_fails_without_the_library(tmp_path):
    env = dict(os.environ, QKQ_LIB_PATH=str(tmp_path / "missing" / "libqkq.so"))
    r = subprocess.run([sys.executable, "-c", "import transform_rope_head_b200"], cwd=ROOT,
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode != 0
    assert "libqkq.so is not built" in r.stderr


def test_product_modules_do_not_import_the_oracle():
    for name in ("__init__.py", "distributed.py", "calibration.py"):
        with open(os.path.join(ROOT, "transform_rope_head_b200", name), encoding="utf-8") as f:
            src = f.read()
        assert "oracle" not in src.replace("# ", "")
