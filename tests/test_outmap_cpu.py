"""The attention kernels' output map on the host: built from the same header
the kernels compile against, with g++, and run over many shapes (see
outmap_check.cpp). This is the index arithmetic of the fused output all-to-all
of Ulysses context parallelism (Causal-rCM section 3.2.1, "Parallelism")."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA_INC = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")


@pytest.mark.skipif(shutil.which("g++") is None or not os.path.isdir(CUDA_INC),
                    reason="needs g++ and the CUDA headers")
def test_output_map_is_a_bijection_onto_the_slices(tmp_path):
    exe = tmp_path / "outmap_check"
    subprocess.run(["g++", "-O1", "-std=c++17", "-I", os.path.join(ROOT, "masked_attention_jvp_b200", "csrc"),
                    "-I", CUDA_INC, os.path.join(ROOT, "tests", "outmap_check.cpp"), "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "mismatches 0" in r.stdout
