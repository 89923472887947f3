"""Host logic of the decode kernel's plan, checked on the CPU (no GPU).

tests/plan_check.cu includes the library's host code, builds the plan of
every workload shape (and small variants) and emulates the repack, the
producer's tile walk and the consumers' lane and thread mappings on the
streamed bytes in double precision: every weight element is copied exactly
once, every (row, column chunk) is read exactly once, and one layer's
q/k/v, gate/up, O, down and lane-mix products equal the canonical
matrix-vector products; and the named workloads' models and plans match the
keys of the shape-specialised kernel instances.  The kernel files are compiled
to PTX only (nothing runs on a GPU).
"""
import os
import subprocess

from decode_persistent_monokernel_b200 import build as kbuild

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def test_plan_mappings_cover_every_weight_once(tmp_path):
    exe = str(tmp_path / "plan_check")
    cmd = [kbuild.nvcc(), "-gencode", "arch=compute_100a,code=compute_100a", "-O1", "-std=c++17",
           "-I", os.path.join(ROOT, "include"), os.path.join(HERE, "plan_check.cu"),
           *[os.path.join(ROOT, "decode_persistent_monokernel_b200", "csrc", f)
             for f in ("monokernel.cu", "prefill_gemm.cu", "prefill.cu")],
           "-o", exe]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    res = subprocess.run([exe], capture_output=True, text=True, timeout=600)
    assert res.returncode == 0 and "ALL OK" in res.stdout, res.stdout[-3000:]
