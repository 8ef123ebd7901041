"""Host check of the kernels' shared-memory plans (no GPU needed): the
routing kernel's regions stay inside its plan for every expert count, and
every kernel's dynamic shared memory fits one CTA."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "ternary_moe_butterfly_b200", "csrc")


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="nvcc not found")
def test_shared_memory_plans_fit(tmp_path):
    exe = str(tmp_path / "check_smem_plans")
    src = os.path.join(ROOT, "tests", "host", "check_smem_plans.cu")
    subprocess.run(["nvcc", "-std=c++17", "-O1", "-x", "cu", "-I", CSRC, "-I", os.path.join(ROOT, "include"),
                    "-gencode", "arch=compute_100a,code=sm_100a", src, "-o", exe],
                   check=True, capture_output=True, timeout=300)
    out = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.strip().endswith("ok")
