"""GPU run of the bounds-checking debug library (built with -DQKQ_BOUNDS_CHECK into
transform_rope_head_b200/_build_check/): the index checks on the pipeline's copies and the
transform's stores turn a failed check into a status bit and skip the access instead of
faulting.  On correct inputs it must report no failed check and give the normal library's
results bit for bit (the checks change no arithmetic).  It runs in a child process, which
loads the debug library in place of the normal one.
"""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import json, sys
import numpy as np, torch
sys.path.insert(0, ".")
import transform_rope_head_b200 as qkq
from oracle import bitspec as B
from tests import gpu_common as G
out = {"lib": qkq.lib_path(), "cases": []}
for name, T, mode, b, group, style in [
        ("tiny", None, "pairwise_hadamard", 0, 64, "half"),
        ("tiny", None, "block_hadamard", 8, 32, "interleaved"),
        ("llama32_3b", 333, "hadamard", 0, 32, "half"),
        ("mistral7b_decode", None, "pairwise", 0, 128, "half")]:   # row-split units
    d = G.DevInputs(G.draw(name, T=T))
    w = d.w
    phi = G.random_phi(w.P, seed=3) if "pairwise" in mode else None
    phi_d = None if phi is None else torch.from_numpy(phi).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q_out, codes, scales, kf = qkq.transform_quantize(
        d.q, d.k, d.pos, d.cos, d.sin, mode=mode, b=b, group=group, phi=phi_d, rope_style=style,
        want_k_f32=True, status=status)
    m = qkq.accumulate_moments(d.q, d.k, d.pos, d.cos, d.sin, rope_style=style, status=status)
    torch.cuda.synchronize()
    oc, os_ = B.rope_table(d.max_pos, w.d_h, w.theta)
    ref = B.transform_quantize(d.inp["q"], d.inp["k"], d.inp["pos"], w.d_h, cos_t=oc, sin_t=os_,
                               mode=mode, b=b or None, group=group, phi=phi, style=style,
                               want_f32=True)
    same = (np.array_equal(G.bits16(q_out), ref["q_out"])
            and np.array_equal(codes.cpu().numpy(), ref["k_codes"])
            and np.array_equal(G.bits16(scales), ref["k_scales"])
            and np.array_equal(G.bits32(kf), G.bits32(ref["k_f32"])))
    out["cases"].append({"case": f"{name}/{mode}", "status": int(status.item()), "same": bool(same)})
print(json.dumps(out))
'''


def test_bounds_checking_build_runs_clean():
    # (re)built when missing or older than the sources: the build is a no-op when fresh
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "qkq_build", os.path.join(ROOT, "transform_rope_head_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    lib = mod.build(check=True)
    env = dict(os.environ, QKQ_LIB_PATH=lib)
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    assert res["lib"].endswith(os.path.join("_build_check", "libqkq.so"))
    for c in res["cases"]:
        assert c["status"] == 0, c          # no failed index check (nor any other bit)
        assert c["same"], c                 # the oracle's bits, as the normal library gives
