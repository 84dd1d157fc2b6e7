"""Build libqkq.so (sm_100a) in-tree from csrc/*.cu with nvcc.

The heavily templated kernels are compiled once per (d_h, RoPE layout) as separate
objects, in parallel; the CUDA runtime is linked statically, so the library uses
the process's primary CUDA context through the driver whatever runtime PyTorch
ships.  Output: transform_rope_head_b200/_build/libqkq.so.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
# QKQ_BUILD_DIR / QKQ_NVCC_EXTRA: build elsewhere / with extra nvcc flags (tuning variants)
OUT = os.environ.get("QKQ_BUILD_DIR") or os.path.join(HERE, "_build")
OBJ = os.path.join(OUT, "obj")
LIB = os.path.join(OUT, "libqkq.so")
# the bounds-checking debug library (-DQKQ_BOUNDS_CHECK: index checks that set a status bit)
CHECK_OUT = os.path.join(HERE, "_build_check")
CHECK_LIB = os.path.join(CHECK_OUT, "libqkq.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC",
              "-Xcompiler", "-Wall", f"-I{os.path.join(ROOT, 'include')}"]


def _units():
    units = [("api.cu", []), ("moments.cu", []), ("moments_noalloc.cu", []), ("solve.cu", []),
             ("dequant_f32.cu", []),
             ("attention_scores.cu", []), ("attention_scores_tc.cu", []),
             ("attention_scores_mma.cu", []), ("selftest.cu", [])]
    for dh in (64, 128):
        for st in (0, 1):
            d = [f"-DQKQ_DH={dh}", f"-DQKQ_STYLE={st}"]
            units.append(("transform_quant.cu", d))
            units.append(("transform_quant_tc.cu", d))
            units.append(("dequant_error.cu", d))
    return units


def _obj_name(src: str, defs: list[str]) -> str:
    tag = "".join(x.split("=")[1] if "=" in x else x for x in defs)
    return os.path.join(OBJ, os.path.splitext(src)[0] + (f"_{tag}" if tag else "") + ".o")


def _newest_input() -> float:
    files = glob.glob(os.path.join(CSRC, "*")) + [os.path.join(ROOT, "include", "qkq.h"),
                                                   os.path.abspath(__file__)]
    return max(os.path.getmtime(f) for f in files)


def nvcc() -> str:
    exe = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(exe):
        raise RuntimeError("nvcc not found: the CUDA toolkit is needed to build libqkq")
    return exe


def build(force: bool = False, jobs: int | None = None, verbose: bool = False,
          ptxas_info: bool = False, check: bool = False) -> str:
    """Compile (if stale) and link libqkq.so; returns its path.  check=True builds the
    bounds-checking debug library instead (transform_rope_head_b200/_build_check/)."""
    out, lib_path = (CHECK_OUT, CHECK_LIB) if check else (OUT, LIB)
    obj_dir = os.path.join(out, "obj")
    if not force and os.path.exists(lib_path) and os.path.getmtime(lib_path) >= _newest_input():
        return lib_path
    os.makedirs(obj_dir, exist_ok=True)
    exe = nvcc()
    extra = ["-Xptxas", "-v"] if ptxas_info else []
    if check:
        extra.append("-DQKQ_BOUNDS_CHECK")

    def compile_one(unit):
        src, defs = unit
        obj = _obj_name(src, defs).replace(OBJ, obj_dir)
        cmd = [exe, *NVCC_FLAGS, *extra, *os.environ.get("QKQ_NVCC_EXTRA", "").split(), *defs,
               "-c", os.path.join(CSRC, src), "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src} {defs}:\n{r.stdout}\n{r.stderr}")
        if verbose or ptxas_info:
            sys.stdout.write(r.stdout + r.stderr)
        return obj

    units = _units()
    with ThreadPoolExecutor(jobs or min(len(units), os.cpu_count() or 4)) as ex:
        objs = list(ex.map(compile_one, units))
    tmp = lib_path + f".tmp{os.getpid()}"
    cmd = [exe, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib_path)
    return lib_path


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                ptxas_info="--ptxas" in sys.argv, check="--check" in sys.argv))
