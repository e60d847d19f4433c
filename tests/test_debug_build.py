"""The bounds-checked build (build.py --debug, -DMAGI_BCA_DEBUG).

Each attention kernel of that build first checks its work unit against the
problem's sizes and records MAGI_BCA_DEVICE_CHECK instead of touching memory
when a unit is out of range.  CPU: the checked kernels compile.  GPU: the
debug library, loaded through MAGI_BCA_LIBRARY in a fresh process, gives the
oracle's results with no check firing, forward and both backward paths, on
ragged, packed and global-block layouts."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_causal_attention_gqa_b200", "csrc")


def test_checked_kernels_compile(tmp_path):
    procs = []
    for f in ("bca_fwd.cu", "bca_bwd.cu", "bca_bwd_split.cu"):
        cmd = ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-c", "-DMAGI_BCA_DEBUG",
               "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"), "-o", str(tmp_path / (f + ".o")),
               os.path.join(CSRC, f)]
        procs.append(subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True))
    for p in procs:
        out, _ = p.communicate(timeout=600)
        assert p.returncode == 0, out[-2000:]


CHILD = r'''
import sys
sys.path.insert(0, sys.argv[1])
import numpy as np, torch
import block_causal_attention_gqa_b200 as bca, workloads
from oracle import bca_oracle as orc
from tests._helpers import assert_close, assert_lse_close, grad_bound, to_np
assert bca.library_path.endswith("libmagi_bca_debug.so"), bca.library_path
cases = [workloads.custom("ragged_d128", 2, [100, 333, 1000, 67], None, 4, 2, 128, seed=11),
         workloads.custom("packed_global_ragged", 2, [100, 333, 250, 67, 400, 190], None, 4, 2, 128, seed=52,
                          samples=[0, 2, 3, 6], n_global=1),
         workloads.custom("packed_global_r2_d64", 1, [256, 256, 256, 130, 126, 256, 256], None, 8, 2, 64, seed=53,
                          samples=[0, 3, 5, 7], n_global=1, kv_range=2)]
for w in cases:
    inp = workloads.make_inputs(w, with_grad_out=True)
    t = {x: inp[x].cuda() for x in ("q", "k", "v", "dout", "gamma_q", "gamma_k")}
    out, lse = bca.magi_bca_fwd(t["q"], t["k"], t["v"], w.q_offsets, w.kv_offsets, t["gamma_q"], t["gamma_k"], **w.mask_kw)
    g = bca.magi_bca_bwd(t["q"], t["k"], t["v"], out, t["dout"], lse, w.q_offsets, w.kv_offsets, t["gamma_q"],
                         t["gamma_k"], **w.mask_kw)
    gd = bca.magi_bca_bwd(t["q"], t["k"], t["v"], out, t["dout"], lse, w.q_offsets, w.kv_offsets, t["gamma_q"],
                          t["gamma_k"], deterministic=True, **w.mask_kw)
    torch.cuda.synchronize()
    st = bca.magi_bca_last_device_status()
    assert st == 0, (w.name, st)
    ref = orc.backward(inp["q"], inp["k"], inp["v"], inp["dout"], w.q_offsets, w.kv_offsets, inp["gamma_q"],
                       inp["gamma_k"], **w.mask_kw)
    assert_close(w.name + " out", to_np(out), ref["out"])
    assert_lse_close(w.name + " lse", to_np(lse), ref["lse"])
    for grads in (g, gd):
        for nm, got in zip(("dq", "dk", "dv"), grads[:3]):
            assert_close(w.name + " " + nm, to_np(got), ref[nm], max_abs=grad_bound(w.name))
    print(w.name, "ok")
print("DEBUG_BUILD_OK")
'''


@pytest.mark.gpu
def test_debug_build_matches_the_oracle_with_no_check_firing():
    sys.path.insert(0, ROOT)
    from block_causal_attention_gqa_b200 import build
    lib = build.build(debug=True)
    env = dict(os.environ, MAGI_BCA_LIBRARY=lib)
    out = subprocess.run([sys.executable, "-c", CHILD, ROOT], cwd=ROOT, env=env, capture_output=True, text=True,
                         timeout=900)
    assert out.returncode == 0 and "DEBUG_BUILD_OK" in out.stdout, (out.stdout[-2000:], out.stderr[-3000:])
