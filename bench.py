"""Benchmark of the MoE feed-forward layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl b200|reference]

One step = one full forward of the layer (router, permutation, grouped
gate/up, grouped down) over one batch of T synthetic tokens already resident
in HBM.  The default workload is the Scout-shaped prefill layer (T = 4096,
d_model 5120, 16 experts, expert and shared SwiGLU width 8192, bf16).  The
metric is layer tokens/s; the JSON line also carries TFLOP/s on active FLOPs,
the layer's roofline fraction, the dominant kernel's roofline (its events
timed live on the launching stream), the end-to-end number through the
host-buffer C-ABI call (input copy in, output copy out, every step), the
oracle timed on the host cores, and the SM clocks sampled during the timed
region.

N > 1 (torchrun, one process per GPU): every rank runs its own replica on its
own batch (tokens are independent, so the layer shards by tokens with no data
exchange); value = all ranks' tokens / max-over-ranks time (weak scaling).

--impl reference times the CPU oracle, as it stands, on the host cores on a
bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_moe_transformer_router_b200 import accounting  # noqa: E402
from sparse_moe_transformer_router_b200.workloads import CODED, CONFIGS, generate, to_storage_numpy  # noqa: E402

DEFAULT_WORKLOAD = "scout_prefill_bf16"
METRIC = "moe_layer_tokens_per_s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), \
        int(os.environ.get("LOCAL_RANK", 0))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


def kernel_flops_bytes(cfg, counts, act8: bool = False, plan: dict | None = None):
    """Algorithmic FLOPs / bytes per launch of each kernel.  act8: the FP8
    activation mode (the contractions read 1-byte token and hidden rows; the
    hidden rows are written in bf16 and quantised by their own kernel).
    plan (the layer's launch plan): with a fused launch the gate/up timing
    slot covers both contractions and the down slot only the finish kernel
    (which reads the down's fp32 partials and writes the output)."""
    T, d, E, F, Fs = cfg.T, cfg.d_model, cfg.num_experts, cfg.expert_ffn, cfg.shared_ffn
    a = accounting.ACT_BYTES[cfg.dtype]
    w = accounting.W_BYTES[cfg.dtype]
    q = 1 if act8 else a  # bytes of a contraction's token-row element
    touched = int(np.count_nonzero(counts))
    out = {
        "router": {"flops": 2 * T * d * E, "bytes": T * d * a + d * E * a + T * 16},
        "permute": {"flops": 0, "bytes": T * 4 * 4},
        "row_copy": {"flops": 0, "bytes": T * d * a + 2 * T * d * q + T * 12},
        "gemm_gate_up": {"flops": 4 * T * d * (F + Fs),
                         "bytes": (touched * 2 * d * F + 2 * d * Fs) * w + 2 * T * d * q + T * (F + Fs) * a},
        "gemm_down": {"flops": 2 * T * d * (F + Fs),
                      "bytes": (touched * F * d + Fs * d) * w + T * (F + Fs) * q + T * d * a},
        "quant_hidden": {"flops": 0, "bytes": T * (F + Fs) * (a + 1) + 2 * T * 4},
    }
    if plan and plan.get("fused"):
        gu, dn = out["gemm_gate_up"], out["gemm_down"]
        out["gemm_gate_up"] = {"flops": gu["flops"] + dn["flops"], "bytes": gu["bytes"] + dn["bytes"]}
        out["gemm_down"] = {"flops": 0, "bytes": plan["split_down"] * 2 * T * d * 4 + T * d * a}
    return out


def profile_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary of this kernel,
    if the kernel sources are unchanged since it was taken (else None)."""
    path = os.path.join(ROOT, "profiles", f"{kernel}__{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_b = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    m_h = re.search(r"sources_sha256:\s*([0-9a-f]+)", text)
    if not m_b or not m_h or m_h.group(1) != kernel_sources_sha(kernel):
        return None
    return float(m_b.group(1))


# The headers each profiled kernel is compiled from (its own code and every
# header it includes); a committed ncu summary stays valid while they hash
# to the value it records.  Kernels not listed hash every device header.
KERNEL_HEADERS = {
    "gemm_gate_up": ("moe_gemm.cuh", "ptx.cuh", "schedule.cuh"),
    "gemm_down": ("moe_gemm.cuh", "ptx.cuh", "schedule.cuh"),
}


def kernel_sources_sha(kernel: str | None = None) -> str:
    """Hash of the device-code headers a kernel is built from (every kernel
    lives in a .cuh file); all of them when the kernel is not listed."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_moe_transformer_router_b200", "csrc")
    names = KERNEL_HEADERS.get(kernel) if kernel else None
    if names is None:
        names = [n for n in os.listdir(csrc) if n.endswith(".cuh")]
    for name in sorted(names):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


class HostLayer:
    """Host (storage-form) copies of one layer's inputs for the oracle,
    converted once per expert on first use."""

    def __init__(self, inp):
        self.inp = inp
        self.x = to_storage_numpy(inp.x)
        self.Wr = to_storage_numpy(inp.W_router)
        self.bias = None if inp.bias is None else inp.bias.cpu().numpy()
        self.Ws_gu = self._w(inp.Ws_gate_up)
        self.Ws_dn = self._w(inp.Ws_down)
        self.idx = None
        self._gu, self._dn, self._sgu, self._sdn = {}, {}, {}, {}

    def _w(self, t):
        """A weight in the oracle's storage form (packed int4 bytes viewed as
        the oracle's int4 type)."""
        a = to_storage_numpy(t)
        if self.inp.cfg.dtype == "int4":
            import oracle
            a = oracle.as_int4x2(a)
        return a

    def expert_args(self, need):
        inp, E = self.inp, self.inp.cfg.num_experts
        for e in need:
            if e not in self._gu:
                self._gu[e] = self._w(inp.W_gate_up[e])
                self._dn[e] = self._w(inp.W_down[e])
                if inp.cfg.dtype in CODED:
                    self._sgu[e] = inp.s_gate_up[e].cpu().numpy()
                    self._sdn[e] = inp.s_down[e].cpu().numpy()
        Wgu = [self._gu.get(e) if e in need else None for e in range(E)]
        Wdn = [self._dn.get(e) if e in need else None for e in range(E)]
        kw = {}
        if inp.cfg.dtype in CODED:
            kw = dict(s_gate_up=[self._sgu.get(e) if e in need else None for e in range(E)],
                      s_down=[self._sdn.get(e) if e in need else None for e in range(E)],
                      ss_gate_up=inp.ss_gate_up.cpu().numpy(), ss_down=inp.ss_down.cpu().numpy())
        return Wgu, Wdn, kw


def cpu_baseline(inp, budget_s: float = 15.0, host: HostLayer | None = None) -> dict:
    """The oracle, as it stands, on the host cores: full-layer outputs for a
    bounded sample of the workload's tokens; tokens/s."""
    import oracle
    cfg = inp.cfg
    threads = oracle.num_threads()
    h = host if host is not None else HostLayer(inp)
    if h.idx is None:
        h.idx, _, _ = oracle.route(h.x, h.Wr, h.bias)

    def run(n):
        sel = np.arange(n, dtype=np.int32) * max(1, cfg.T // max(n, 1))
        sel = sel[sel < cfg.T]
        need = set(int(e) for e in h.idx[sel]) if cfg.num_experts > 0 else set()
        Wgu, Wdn, kw = h.expert_args(need)
        t0 = time.perf_counter()
        oracle.forward(h.x, h.Wr, Wgu, Wdn, h.Ws_gu, h.Ws_dn, bias=h.bias, tokens=sel, **kw)
        return len(sel), time.perf_counter() - t0

    n, dt = run(max(1, threads))                      # calibration sample
    per_tok = dt / n
    n2 = int(max(1, min(cfg.T, budget_s / per_tok)))
    n2 = max(threads, (n2 // max(1, threads)) * threads) if n2 >= threads else n2
    n2 = min(n2, cfg.T)
    n2, dt2 = run(n2)
    return {"value": n2 / dt2, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"full-layer outputs (router + shared + routed SwiGLU, fp64) for {n2} of the "
                      f"{cfg.T} tokens, evenly spaced, {dt2:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    cfg = CONFIGS[args.workload]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = generate(cfg, seed=0, device=dev)
    host = HostLayer(inp)
    per_step_budget = max(1.0, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_baseline(inp, budget_s=per_step_budget / 4, host=host)
    vals, samples = [], []
    cb = None
    for _ in range(args.steps):
        cb = cpu_baseline(inp, budget_s=per_step_budget, host=host)
        vals.append(cb["value"])
        samples.append(cb["sample"])
    value = float(np.median(vals))
    ms = cfg.T / value * 1e3
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": config_dict(cfg, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cb["cores"], "kind": "oracle",
                             "sample": samples[-1] + "; value = median over steps; ms_per_step = T / value"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_dict(cfg, world):
    return {"workload": cfg.name, "T": cfg.T, "d_model": cfg.d_model, "experts": cfg.num_experts,
            "expert_ffn": cfg.expert_ffn, "shared_ffn": cfg.shared_ffn, "top_k": 1,
            "router": cfg.router, "parallelism": f"replicas{world}" if world > 1 else "single",
            "l2": "inputs larger than L2: every step streams all touched expert weights "
                  "(GBs) through a 126 MB L2; no explicit flush"}


def rank_barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def rank_max(v: float, world: int, device: str) -> float:
    """The slowest rank's time (every rank takes part, every rank gets it)."""
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(world: int, tokens_per_rank: int, steps: int, t_ms: float) -> float:
    """Weak scaling: every rank processed its own batch each step; the job's
    throughput is all ranks' tokens over the slowest rank's time."""
    return world * tokens_per_rank * steps / (t_ms / 1e3)


def free_port() -> int:
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def relaunch_ranks(n: int) -> int:
    """`--gpus N` without a launcher: start N ranks of this same command
    line under torch.distributed.run on this node (rendezvous on 127.0.0.1)
    and return its exit status.  The ranks find WORLD_SIZE set and run."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()),
           os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=None,
                    help="ranks (one per GPU); without torchrun, N > 1 relaunches this command "
                         "under torch.distributed.run")
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(CONFIGS))
    ap.add_argument("--tokens", type=int, default=0, help="override T (decode sweeps)")
    ap.add_argument("--experts", type=int, default=0,
                    help="override E (smaller profiling captures)")
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--act-fp8", action="store_true",
                    help="E4M3-weight workloads: run the FP8 activation mode")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="measure only --workload (skip the other shapes measured after it)")
    ap.add_argument("--e2e-steps", type=int, default=0)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.gpus is not None and args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(relaunch_ranks(args.gpus))
    rank, world, local = dist_env()
    if args.gpus is not None and world != args.gpus:
        raise SystemExit(f"bench.py: --gpus {args.gpus} but the launcher started {world} ranks")
    if world > 1:
        import datetime
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group("nccl" if args.impl == "b200" else "gloo",
                                timeout=datetime.timedelta(seconds=300))
    if args.tokens:
        CONFIGS[args.workload] = CONFIGS[args.workload].with_tokens(args.tokens)
    if args.experts:
        from dataclasses import replace
        c = CONFIGS[args.workload]
        CONFIGS[args.workload] = replace(c, num_experts=args.experts, name=f"{c.name}@E{args.experts}",
                                         n_dead=min(c.n_dead, args.experts // 4))
    if args.impl == "reference":
        run_reference(args, rank, world)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    run_b200(args, rank, world, local)


# Datasheet figures (NVIDIA B200: dense bf16 tensor throughput, HBM3e
# bandwidth), reported next to the fractions of the measured peaks.
DATASHEET = {"bf16_tflops": 2250.0, "hbm_gbs": 8000.0}
# dense E4M3 over dense bf16 tensor throughput, nominal (4.5 / 2.25 PFLOP/s)
FP8_OVER_BF16 = 2.0

# Workloads measured after the headline in the same run, each with its own
# timed region, roofline and clocks: the other shapes the layer is quoted on.
EXTRA_WORKLOADS = ("maverick_prefill_bf16", "maverick_decode_bf16@T1", "maverick_decode_bf16@T8",
                   "maverick_decode_bf16@T32", "maverick_decode_bf16@T128", "maverick_fp8",
                   "maverick_fp8+act8", "maverick_int8", "scout_prefill_int4", "maverick_dense_bf16",
                   "tiny_f32")


def workload_config(name: str):
    """A workload name: a config, optionally `@T<n>` (another token count)
    and `+act8` (the FP8 activation mode; see workload_act8)."""
    base, _, t = name.replace("+act8", "").partition("@T")
    cfg = CONFIGS[base]
    return cfg.with_tokens(int(t)) if t else cfg


def workload_act8(name: str) -> bool:
    return name.endswith("+act8")


def make_layer(cfg, rank, act8: bool = False):
    from sparse_moe_transformer_router_b200.binding import L4MoE
    inp = generate(cfg, seed=rank, device="cuda")
    layer = L4MoE(cfg.d_model, cfg.expert_ffn, cfg.shared_ffn, cfg.num_experts, cfg.dtype)
    if inp.bias is not None:
        layer.set_router_bias(inp.bias)
    if cfg.dtype in CODED:
        layer.set_weight_scales(inp.s_gate_up, inp.s_down, inp.ss_gate_up, inp.ss_down)
    if act8:
        layer.set_act_fp8(True)
    return inp, layer


def roofline_of(flops: float, nbytes: float, seconds: float, tensor_peak: float, hbm: float,
                tensor_sheet: float, hbm_sheet: float) -> dict:
    """The binding roof of work (flops, bytes) done in `seconds`: achieved
    rate and fraction of the measured peak and of the datasheet figure."""
    t_tensor = flops / (tensor_peak * 1e12) if flops else 0.0
    t_hbm = nbytes / (hbm * 1e9)
    if t_tensor >= t_hbm:
        achieved = flops / seconds / 1e12
        return {"bound": "tensor", "achieved": achieved, "peak": tensor_peak, "unit": "TFLOP/s",
                "frac": achieved / tensor_peak, "datasheet_peak": tensor_sheet,
                "frac_of_datasheet": achieved / tensor_sheet}
    achieved = nbytes / seconds / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
            "datasheet_peak": hbm_sheet, "frac_of_datasheet": achieved / hbm_sheet}


def measure(cfg, inp, layer, steps: int, warmup: int, world: int, local: int, act8: bool = False) -> dict:
    """Device-timed forwards of one workload: warm-up, a per-kernel
    breakdown pass, then `steps` forwards between two events on the
    launching stream (barrier + synchronize on both sides, max over ranks)
    with nvidia-smi clock samples during it -- the step time -- and a second
    region of the same `steps` forwards with the dominant kernel's own events
    around each of its launches -- its duration for the roofline.  (An event
    recorded between two launches ends the programmatic overlap of the
    second with the first, which the small-batch forwards rely on, so the
    step time is taken without them.)  Returns the measurement and roofline
    fields."""
    out = torch.empty((cfg.T, cfg.d_model), dtype=inp.x.dtype, device="cuda")
    fwd = lambda: layer.forward(inp.x, inp.W_router, inp.W_gate_up, inp.W_down,  # noqa: E731
                                inp.Ws_gate_up, inp.Ws_down, out=out)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        fwd()
    torch.cuda.synchronize()
    layer.check_device_status()
    counts = layer.routing()["counts"].cpu().numpy() if cfg.num_experts > 0 else np.zeros(0)
    layer.read_timing()  # drop anything recorded so far

    # per-kernel breakdown (a short pass of its own, every kernel timed): it
    # names the dominant kernel, the only one timed inside the timed region,
    # where every event pair would add to the step
    layer.set_timing(True)
    n_break = max(3, min(20, steps // 5))
    for _ in range(n_break):
        fwd()
    torch.cuda.synchronize()
    layer.set_timing(False)
    breakdown = layer.read_timing()
    dom = max((k for k in breakdown if breakdown[k][1]), key=lambda k: breakdown[k][0])

    sampler = ClockSampler(local)
    sampler.start()
    launches0 = layer.launch_count
    rank_barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fwd()
    e1.record(stream)
    torch.cuda.synchronize()
    rank_barrier(world)
    clocks = sampler.stop()
    launches = layer.launch_count - launches0
    t_ms = rank_max(e0.elapsed_time(e1), world, "cuda")
    # the dominant kernel's launches, event-timed over a region of the same steps
    layer.set_timing([dom])
    rank_barrier(world)
    torch.cuda.synchronize()
    for _ in range(steps):
        fwd()
    torch.cuda.synchronize()
    rank_barrier(world)
    layer.set_timing(False)
    ktimes = layer.read_timing()
    layer.check_device_status()
    ms_step = t_ms / steps

    peaks, peak_src = load_peaks()
    long_region = t_ms > 1000.0
    tensor_peak = peaks.get("bf16_tflops_sustained" if long_region else "bf16_tflops")
    tensor_sheet = DATASHEET["bf16_tflops"]
    if act8:  # E4M3 x E4M3: the measured bf16 peak times the nominal FP8 / bf16 ratio
        tensor_peak *= FP8_OVER_BF16
        tensor_sheet *= FP8_OVER_BF16
    hbm = peaks["hbm_gbs"]
    plan = layer.plan()
    kfb = kernel_flops_bytes(cfg, counts, act8, plan)
    per_kernel = {}
    for name, (ms, n) in breakdown.items():
        if n:
            avg = ms / n
            per_kernel[name] = {"avg_us": avg * 1e3, "share": None, "launches": n,
                                "tflops": kfb[name]["flops"] / (avg / 1e3) / 1e12,
                                "gbs": kfb[name]["bytes"] / (avg / 1e3) / 1e9}
    tot = sum(v["avg_us"] for v in per_kernel.values())
    for v in per_kernel.values():
        v["share"] = v["avg_us"] / tot if tot else None
    dom_ms, dom_n = ktimes[dom]
    f, b = kfb[dom]["flops"], kfb[dom]["bytes"]
    avg_s = dom_ms / dom_n / 1e3  # the dominant kernel's events inside the timed region
    roof = roofline_of(f, b, avg_s, tensor_peak, hbm, tensor_sheet, DATASHEET["hbm_gbs"])
    roof = {"kernel": dom, **roof, "traffic": profile_traffic(dom, cfg.name + ("+act8" if act8 else "")),
            "peak_source": (f"{peak_src} ({'sustained' if long_region else 'burst'})"
                            + (f" x {FP8_OVER_BF16:g} (nominal E4M3 / bf16 ratio)" if act8 else "")
                            if roof["bound"] == "tensor" else f"{peak_src} hbm_gbs"),
            "algorithmic_per_launch": {"flops": f, "bytes": b},
            "avg_us_timed_region": avg_s * 1e6, "launches_timed": dom_n,
            "timed_region": "a second region of the same steps right after the step-time region, "
                            "events around each launch of this kernel"}
    # whole layer against its own roof
    touched = accounting.experts_touched(counts)
    flops = accounting.layer_flops(cfg.T, cfg.d_model, cfg.num_experts, cfg.expert_ffn, cfg.shared_ffn)
    lbytes = accounting.layer_bytes(cfg.T, cfg.d_model, cfg.num_experts, cfg.expert_ffn, cfg.shared_ffn,
                                    cfg.dtype, touched)
    lr = roofline_of(flops, lbytes, ms_step / 1e3, tensor_peak, hbm, tensor_sheet, DATASHEET["hbm_gbs"])
    layer_roof = {"bound": lr["bound"], "frac": lr["frac"], "frac_of_datasheet": lr["frac_of_datasheet"],
                  "tflops_active": flops / (ms_step / 1e3) / 1e12,
                  "gbs_algorithmic": lbytes / (ms_step / 1e3) / 1e9,
                  "flops_per_step": flops, "bytes_per_step": lbytes}
    return {"ms_per_step": ms_step, "t_ms": t_ms, "steps": steps, "roofline": roof, "plan": plan,
            "layer_roofline": layer_roof, "kernels": per_kernel, "n_break": n_break, "dom": dom,
            "gpu_launches": launches, "clocks": clocks, "experts_touched": touched}


def run_extra_workloads(args, rank, world, local) -> dict:
    """The other workloads, one after another (each one's inputs freed before
    the next): tokens/s, ms/step, both rooflines and clocks for each."""
    res = {}
    for name in EXTRA_WORKLOADS:
        cfg = workload_config(name)
        act8 = workload_act8(name)
        inp, layer = make_layer(cfg, rank, act8)
        # a timed region of at least ~200 ms (and at least --steps forwards)
        out = torch.empty((cfg.T, cfg.d_model), dtype=inp.x.dtype, device="cuda")
        layer.forward(inp.x, inp.W_router, inp.W_gate_up, inp.W_down, inp.Ws_gate_up, inp.Ws_down, out=out)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        layer.forward(inp.x, inp.W_router, inp.W_gate_up, inp.W_down, inp.Ws_gate_up, inp.Ws_down, out=out)
        torch.cuda.synchronize()
        est_ms = (time.perf_counter() - t0) * 1e3
        steps = int(max(args.steps, min(400, 200.0 / max(est_ms, 1e-3))))
        m = measure(cfg, inp, layer, steps, args.warmup, world, local, act8)
        res[name] = {"tokens_per_s": replica_throughput(world, cfg.T, steps, m["t_ms"]),
                     "ms_per_step": m["ms_per_step"], "steps": steps, "T": cfg.T,
                     "experts": cfg.num_experts, "dtype": cfg.dtype, "router": cfg.router,
                     "layer_roofline": m["layer_roofline"], "roofline": m["roofline"],
                     "kernels": {k: round(v["avg_us"], 2) for k, v in m["kernels"].items()},
                     "gpu_launches": m["gpu_launches"], "clocks": m["clocks"], "plan": m["plan"],
                     "experts_touched": m["experts_touched"]}
        layer.close()
        del inp, layer, out
        torch.cuda.empty_cache()
    return res


def run_b200(args, rank, world, local):
    torch.cuda.set_device(local)
    cfg = CONFIGS[args.workload]
    inp, layer = make_layer(cfg, rank, args.act_fp8)
    m = measure(cfg, inp, layer, args.steps, args.warmup, world, local, args.act_fp8)
    value = replica_throughput(world, cfg.T, args.steps, m["t_ms"])

    # ------------------------------------------------------------- e2e (host buffers)
    stream = torch.cuda.current_stream()
    x_host = inp.x.cpu().pin_memory()
    out_host = torch.empty_like(x_host).pin_memory()
    e2e_steps = args.e2e_steps or args.steps  # same length as the device-timed region
    fwd_h = lambda: layer.forward_host(x_host, inp.W_router, inp.W_gate_up, inp.W_down,  # noqa: E731
                                       inp.Ws_gate_up, inp.Ws_down, out_host)
    for _ in range(2):
        fwd_h()
    torch.cuda.synchronize()
    rank_barrier(world)
    sampler = ClockSampler(local)
    sampler.start()
    h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0.record(stream)
    for _ in range(e2e_steps):
        fwd_h()
    layer.join_host(stream)  # the end event waits for the last output copy
    h1.record(stream)
    torch.cuda.synchronize()
    rank_barrier(world)
    e2e_clocks = sampler.stop()
    th_ms = rank_max(h0.elapsed_time(h1), world, "cuda")
    layer.check_device_status()
    io_bytes = cfg.T * cfg.d_model * inp.x.element_size()
    e2e = {"value": replica_throughput(world, cfg.T, e2e_steps, th_ms), "unit": "tokens/s",
           "h2d_bytes_per_step": io_bytes, "d2h_bytes_per_step": io_bytes,
           "ms_per_step": th_ms / e2e_steps, "clocks": e2e_clocks,
           "path": "l4moe_forward_host per step: pinned host x -> device (copy-in stream), layer "
                   "(caller stream), device -> pinned host out (copy-out stream); consecutive "
                   "steps overlap their copies with each other's compute; the timed region "
                   "ends after the last output copy"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(inp)
    layer.close()
    del inp, layer
    torch.cuda.empty_cache()
    extra = {} if args.no_workloads else run_extra_workloads(args, rank, world, local)

    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": m["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if cfg.dtype != "f32" else "f32",
            "data": "synthetic (seeded N(0,1) inputs, N(0,0.02) weights, random-init)",
            "config": config_dict(cfg, world), "roofline": m["roofline"],
            "layer_roofline": m["layer_roofline"], "kernels": m["kernels"],
            "kernels_note": f"every kernel event-timed over {m['n_break']} steps after the warm-up; the "
                            f"dominant kernel ({m['dom']}) again over a region of the timed steps; the "
                            f"step time itself is taken without per-kernel events",
            "e2e": e2e, "gpu_launches": m["gpu_launches"], "clocks": m["clocks"], "plan": m["plan"],
            "experts_touched": m["experts_touched"],
            "peaks_note": "frac: of the measured peak (peak_source); frac_of_datasheet: of NVIDIA's "
                          "dense bf16 2250 TFLOP/s or HBM3e 8000 GB/s"}
    if cfg.dtype in CODED:
        wname = {"fp8": "E4M3", "int8": "int8", "int4": "int4"}[cfg.dtype]
        line["dtype"] = f"f16 ({wname} weights widened exactly to f16, fp32 accumulate; bf16 in and out)"
    if args.act_fp8:
        line["dtype"] = "e4m3 (E4M3 weights and per-row E4M3 token / hidden rows, fp32 accumulate; bf16 in and out)"
        line["config"]["workload"] += "+act8"
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if extra:
        line["workloads"] = extra
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
