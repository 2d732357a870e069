"""Device-code helpers compiled for the host with nvcc and checked on the CPU
(no GPU needed):

- the top-k selection list of the router epilogue and of the permutation's
  warp merge (csrc/topk.cuh) against a brute-force selection on random
  logits with ties, NaN and -inf (tests/host/topk_check.cu);
- the grouped GEMM's tile schedule (tile_at, decode_tile) on random work
  lists: every tile decoded exactly once and inside its group
  (tests/host/schedule_check.cu);
- the workspace layout and split-K plan of the library's host code on random
  shapes, dtypes, k and token budgets: aligned, ordered segments large
  enough for any smaller batch, partial planes included
  (tests/host/layout_check.cu).
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
NVCC = shutil.which("nvcc") or ("/usr/local/cuda/bin/nvcc" if os.path.exists("/usr/local/cuda/bin/nvcc") else None)


def _build_and_run(src: str, exe, extra=("-O2",)):
    subprocess.run([NVCC, "-std=c++17", "-x", "cu", "--expt-relaxed-constexpr",
                    "-gencode", "arch=compute_100a,code=sm_100a", *extra,
                    "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(ROOT, "sparse_moe_transformer_router_b200", "csrc"),
                    os.path.join(ROOT, "tests", "host", src), "-o", str(exe)],
                   check=True, capture_output=True, timeout=600)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.startswith("OK"), r.stdout + r.stderr


@pytest.mark.skipif(NVCC is None, reason="nvcc not available")
def test_topk_list_matches_brute_force(tmp_path):
    _build_and_run("topk_check.cu", tmp_path / "topk_check")


@pytest.mark.skipif(NVCC is None, reason="nvcc not available")
def test_gemm_tile_schedule_covers_every_tile_once(tmp_path):
    _build_and_run("schedule_check.cu", tmp_path / "schedule_check")


@pytest.mark.skipif(NVCC is None, reason="nvcc not available")
def test_workspace_layout_holds_every_smaller_batch(tmp_path):
    _build_and_run("layout_check.cu", tmp_path / "layout_check", extra=("-O1",))
