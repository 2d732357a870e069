"""The top-k selection list of the router epilogue and of the permutation's
warp merge (csrc/topk.cuh), compiled for the host with nvcc and checked
against a brute-force selection on random logits with ties, NaN and -inf
(tests/host/topk_check.cu).  No GPU needed."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"),
                    reason="nvcc not available")
def test_topk_list_matches_brute_force(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    exe = tmp_path / "topk_check"
    subprocess.run([nvcc, "-std=c++17", "-O2", "-x", "cu", "-Wno-deprecated-gpu-targets",
                    "-I", os.path.join(ROOT, "sparse_moe_transformer_router_b200", "csrc"),
                    os.path.join(ROOT, "tests", "host", "topk_check.cu"), "-o", str(exe)],
                   check=True, capture_output=True, timeout=300)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.startswith("OK"), r.stdout + r.stderr
