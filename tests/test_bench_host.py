"""Host-side logic of bench.py that needs no GPU: the per-kernel FLOP split,
the parsing of committed ncu summaries, the weak-scaling value and the
oracle's timed CPU sample."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from sparse_moe_transformer_router_b200 import accounting  # noqa: E402
from sparse_moe_transformer_router_b200.workloads import CONFIGS, generate  # noqa: E402


@pytest.mark.parametrize("name", ["scout_prefill_bf16", "maverick_prefill_bf16", "maverick_fp8"])
def test_kernel_flops_add_up_to_the_layer(name):
    cfg = CONFIGS[name]
    counts = np.full(cfg.num_experts, cfg.T // cfg.num_experts)
    k = bench.kernel_flops_bytes(cfg, counts)
    total = sum(v["flops"] for v in k.values())
    assert total == accounting.layer_flops(cfg.T, cfg.d_model, cfg.num_experts, cfg.expert_ffn,
                                           cfg.shared_ffn)
    # the weights each GEMM streams: touched routed experts plus the shared one
    w = accounting.W_BYTES[cfg.dtype]
    assert k["gemm_down"]["bytes"] >= (cfg.num_experts * cfg.expert_ffn + cfg.shared_ffn) * cfg.d_model * w
    # a fused launch: the gate/up slot carries both contractions, the down slot the finish
    f = bench.kernel_flops_bytes(cfg, counts, plan={"fused": 1, "split_down": 3})
    assert f["gemm_gate_up"]["flops"] == k["gemm_gate_up"]["flops"] + k["gemm_down"]["flops"]
    assert f["gemm_gate_up"]["bytes"] == k["gemm_gate_up"]["bytes"] + k["gemm_down"]["bytes"]
    assert f["gemm_down"]["flops"] == 0 and sum(v["flops"] for v in f.values()) == total


def test_profile_traffic_needs_the_current_kernel_hash(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    path = tmp_path / "profiles" / "gemm_gate_up__w.md"
    sha = bench.kernel_sources_sha()
    path.write_text(f"# x\n\ndram_bytes_per_launch: 1234500000\nsources_sha256: {sha}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # the hash covers the kernel headers under ROOT: point it at the real ones
    monkeypatch.setattr(bench, "kernel_sources_sha", lambda kernel=None: sha)
    assert bench.profile_traffic("gemm_gate_up", "w") == 1234500000.0
    path.write_text("dram_bytes_per_launch: 1234500000\nsources_sha256: 0000000000000000\n")
    assert bench.profile_traffic("gemm_gate_up", "w") is None   # kernels changed since
    assert bench.profile_traffic("gemm_down", "w") is None      # no summary at all


def test_kernel_hash_covers_only_device_code():
    sha = bench.kernel_sources_sha()
    assert len(sha) == 16 and int(sha, 16) >= 0


def test_gemm_hash_covers_exactly_the_headers_the_gemm_includes():
    """A profiled kernel's hash lists its header and everything that header
    includes (so an edit there invalidates the committed counters), and no
    header the kernel does not include."""
    import re
    csrc = os.path.join(ROOT, "sparse_moe_transformer_router_b200", "csrc")

    def closure(name, seen):
        if name in seen:
            return seen
        seen.add(name)
        for inc in re.findall(r'#include "([^"]+)"', open(os.path.join(csrc, name)).read()):
            closure(inc, seen)
        return seen

    for kernel in ("gemm_gate_up", "gemm_down"):
        assert set(bench.KERNEL_HEADERS[kernel]) == closure("moe_gemm.cuh", set())
        assert bench.kernel_sources_sha(kernel) != bench.kernel_sources_sha()


def test_weak_scaling_value():
    # two ranks, 4096 tokens each, 10 steps in 20 ms on the slowest rank
    assert bench.replica_throughput(2, 4096, 10, 20.0) == pytest.approx(2 * 4096 * 10 / 0.020)


def test_cpu_baseline_times_the_oracle_on_a_bounded_sample():
    cfg = CONFIGS["tiny_f32"]
    inp = generate(cfg, seed=0)
    cb = bench.cpu_baseline(inp, budget_s=0.5)
    assert cb["kind"] == "oracle" and cb["unit"] == "tokens/s" and cb["value"] > 0
    assert cb["cores"] >= 1 and "of the 64 tokens" in cb["sample"]


def test_roofline_reports_measured_and_datasheet_fractions():
    # 1 TFLOP and 1 GB in 1 ms: tensor-bound at 1000 TFLOP/s against a 1600
    # measured / 2250 datasheet peak; HBM-bound when the bytes dominate
    r = bench.roofline_of(1e12, 1e9, 1e-3, 1600.0, 6500.0, 2250.0, 8000.0)
    assert r["bound"] == "tensor" and r["achieved"] == pytest.approx(1000.0)
    assert r["frac"] == pytest.approx(1000.0 / 1600.0)
    assert r["frac_of_datasheet"] == pytest.approx(1000.0 / 2250.0)
    r = bench.roofline_of(1e9, 5e9, 1e-3, 1600.0, 6500.0, 2250.0, 8000.0)
    assert r["bound"] == "hbm" and r["achieved"] == pytest.approx(5000.0)
    assert r["frac"] == pytest.approx(5000.0 / 6500.0)
    assert r["frac_of_datasheet"] == pytest.approx(5000.0 / 8000.0)


def test_extra_workloads_name_known_shapes():
    for name in bench.EXTRA_WORKLOADS:
        cfg = bench.workload_config(name)
        assert cfg.T > 0 and cfg.d_model > 0
    assert bench.workload_config("maverick_decode_bf16@T8").T == 8
    assert bench.DEFAULT_WORKLOAD not in bench.EXTRA_WORKLOADS
