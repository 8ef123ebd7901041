"""Host check of the kernels' shared table layouts (no GPU needed): the
consumption-order cos/sin table generators and their inverses are
bijections onto (stage, pair), and the slot order of the combine is a
permutation of the columns of a slice."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "ternary_moe_butterfly_b200", "csrc")


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="nvcc not found")
def test_table_layouts_are_bijections(tmp_path):
    exe = str(tmp_path / "check_tables")
    src = os.path.join(ROOT, "tests", "host", "check_tables.cu")
    subprocess.run(["nvcc", "-std=c++17", "-O1", "-x", "cu", "-I", CSRC, "-I", os.path.join(ROOT, "include"),
                    "-gencode", "arch=compute_100a,code=sm_100a", src, "-o", exe],
                   check=True, capture_output=True, timeout=300)
    out = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.strip().endswith("ok")
