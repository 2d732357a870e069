"""Seeded synthetic layer inputs shared by the CUDA path's tests/benchmark and
by the oracle's tests.

This module draws random numbers and lays them out; it holds none of the
layer's arithmetic (no logits, no routing, no FFN).  Every tensor comes from
its own ``torch.Generator`` seeded from (seed, tensor name, expert), so any
subset of experts can be regenerated on its own and the draws do not depend
on the order of generation.  The same recipe runs on CPU or on a CUDA device;
the two devices' generators give different (equally distributed) numbers, so a
comparison always feeds one generated set to both sides.

Shapes follow the pages' Scout / Maverick configurations: d_model 5120, 16 or
128 experts, expert and shared SwiGLU width 8192 (KerasFormers "Llama 4" API
table; llm-architectures-explained "Llama 4 Maverick" field table).
"""
from __future__ import annotations

import functools
import math
import zlib
from dataclasses import dataclass, field, replace

import numpy as np
import torch

E4M3_MAX = 448.0
INT8_MAX = 127.0
INT4_MAX = 7.0
# layer dtypes whose weights are codes with per-output-column fp32 scales
CODED = ("fp8", "int8", "int4")


@dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int
    d_model: int
    num_experts: int
    expert_ffn: int
    shared_ffn: int
    dtype: str            # "f32" | "bf16" | "fp8" / "int8" / "int4" (coded weights, bf16 activations)
    router: str = "plain"  # "plain": no bias; "zipf": per-expert bias for Zipf loads
    x_std: float = 1.0
    w_std: float = 0.02
    wr_std: float = 0.02
    zipf_s: float = 1.1
    n_dead: int = 0

    def with_tokens(self, T: int) -> "LayerConfig":
        return replace(self, T=T, name=f"{self.name.split('@')[0]}@T{T}")


# The five workloads.  Sizes, dtypes and distributions: tiny fp32 layer; a
# Scout-shaped prefill layer (16 experts); a Maverick-shaped prefill layer
# (128 experts, Zipf(1.1) loads, 10 experts idle); Maverick-shaped decode
# (T in {1, 8, 32, 128}, uniform routing); Maverick with E4M3 weights.  Plus
# Maverick's dense feed-forward layer (no experts, width 16384).
CONFIGS = {
    "tiny_f32": LayerConfig("tiny_f32", 64, 128, 4, 256, 256, "f32", wr_std=0.1),
    "scout_prefill_bf16": LayerConfig("scout_prefill_bf16", 4096, 5120, 16, 8192, 8192, "bf16"),
    "maverick_prefill_bf16": LayerConfig("maverick_prefill_bf16", 8192, 5120, 128, 8192, 8192,
                                         "bf16", router="zipf", n_dead=10),
    "maverick_decode_bf16": LayerConfig("maverick_decode_bf16", 128, 5120, 128, 8192, 8192, "bf16"),
    "maverick_fp8": LayerConfig("maverick_fp8", 16384, 5120, 128, 8192, 8192, "fp8",
                                router="zipf", n_dead=10),
    # the layers without experts: one SwiGLU feed-forward of width 16384
    "maverick_dense_bf16": LayerConfig("maverick_dense_bf16", 8192, 5120, 0, 0, 16384, "bf16"),
    # weight-only int8 experts (per-output-column scales), Maverick-shaped
    "maverick_int8": LayerConfig("maverick_int8", 16384, 5120, 128, 8192, 8192, "int8",
                                 router="zipf", n_dead=10),
    # weight-only int4 experts, Scout-shaped (the glossary's Scout on one GPU in int4)
    "scout_prefill_int4": LayerConfig("scout_prefill_int4", 4096, 5120, 16, 8192, 8192, "int4"),
}
DECODE_TOKENS = (1, 8, 32, 128)


@dataclass
class LayerInputs:
    cfg: LayerConfig
    x: torch.Tensor                  # [T, d]      f32 or bf16
    W_router: torch.Tensor           # [d, E]      f32 or bf16
    bias: torch.Tensor | None        # [E]         f32
    W_gate_up: list                  # E x [d, 2F] f32 / bf16 / float8_e4m3fn (None = not made)
    W_down: list                     # E x [F, d]
    Ws_gate_up: torch.Tensor         # [d, 2Fs]
    Ws_down: torch.Tensor            # [Fs, d]
    s_gate_up: list | None = None    # E x [2F] f32 (fp8 only)
    s_down: list | None = None       # E x [d]  f32
    ss_gate_up: torch.Tensor | None = None
    ss_down: torch.Tensor | None = None
    extra: dict = field(default_factory=dict)


def _seed(seed: int, name: str, e: int = -1) -> int:
    return (seed * 1_000_003 + zlib.crc32(f"{name}/{e}".encode())) & 0x7FFF_FFFF_FFFF


def _normal(shape, std, seed, name, e, device) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(seed, name, e))
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    return t.mul_(std)


def quantize_e4m3_columns(w: torch.Tensor):
    """Per-output-column E4M3 quantisation of an fp32 [K, N] weight:
    scale[n] = max_k |w[k, n]| / 448, q = e4m3(w / scale) (round to nearest
    even, saturated to +-448).  Returns (q float8_e4m3fn [K, N], scale f32 [N])."""
    amax = w.abs().amax(dim=0)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    q = (w / scale).clamp_(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
    return q, scale.to(torch.float32)


def quantize_int8_columns(w: torch.Tensor):
    """Per-output-column symmetric int8 quantisation of an fp32 [K, N] weight:
    scale[n] = max_k |w[k, n]| / 127, q = round(w / scale) (to nearest even),
    clamped to [-127, 127].  Returns (q int8 [K, N], scale f32 [N])."""
    amax = w.abs().amax(dim=0)
    scale = torch.where(amax > 0, amax / INT8_MAX, torch.ones_like(amax))
    q = torch.round(w / scale).clamp_(-INT8_MAX, INT8_MAX).to(torch.int8)
    return q, scale.to(torch.float32)


def int4_codes_columns(w: torch.Tensor):
    """Per-output-column symmetric int4 codes of an fp32 [K, N] weight:
    scale[n] = max_k |w[k, n]| / 7, q = round(w / scale) (to nearest even),
    clamped to [-7, 7].  Returns (q int8 [K, N], scale f32 [N]), unpacked."""
    amax = w.abs().amax(dim=0)
    scale = torch.where(amax > 0, amax / INT4_MAX, torch.ones_like(amax))
    q = torch.round(w / scale).clamp_(-INT4_MAX, INT4_MAX).to(torch.int8)
    return q, scale.to(torch.float32)


def pack_int4(q: torch.Tensor) -> torch.Tensor:
    """int4 storage of integer codes q in [-8, 7], [K, N] with N even: two
    two's-complement nibbles per byte along the row, the even column in the
    low nibble.  Returns uint8 [K, N / 2]."""
    assert q.shape[-1] % 2 == 0
    n = (q.to(torch.int16) & 0xF).to(torch.uint8)
    return n[..., 0::2] | (n[..., 1::2] << 4)


def quantize_int4_columns(w: torch.Tensor):
    """int4_codes_columns, packed: (uint8 [K, N / 2], scale f32 [N])."""
    q, scale = int4_codes_columns(w)
    return pack_int4(q), scale


@functools.lru_cache(maxsize=16)
def zipf_router_bias(E: int, n_dead: int, s: float, logit_std: float, seed: int) -> np.ndarray:
    """Per-expert fp32 router bias whose expected expert loads follow Zipf(s).

    Model of the logits: each token's logit for expert e is b_e + sigma * Z_e
    with Z_e iid N(0, 1) (true for x ~ N(0, 1) and independent N(0, w^2)
    router columns, sigma = sqrt(d) * std(x) * std(w)).  Under that model the
    win probability of expert e is the integral over v of
    phi((v - b_e)/sigma)/sigma * prod_{j != e} Phi((v - b_j)/sigma); it is
    evaluated by quadrature, and b is fitted by the fixed-point update
    b <- b + eta * (log p_target - log p_model) for a fixed number of steps
    (deterministic; no sampling).  n_dead experts get b = -1e4 (no tokens).
    Zipf ranks are assigned to expert indices by a seeded permutation.
    """
    from scipy.special import log_ndtr

    n_live = E - n_dead
    ranks = np.arange(1, n_live + 1, dtype=np.float64)
    p = ranks ** (-s)
    p /= p.sum()
    sigma = float(logit_std)
    b = sigma * np.log(p)  # Gumbel-style start
    b -= b.mean()
    for _ in range(150):
        lo = b.min() - 7 * sigma
        hi = b.max() + 7 * sigma
        v = np.linspace(lo, hi, 3001)
        dv = v[1] - v[0]
        z = (v[None, :] - b[:, None]) / sigma                  # [E, V]
        log_cdf = log_ndtr(z)
        log_all = log_cdf.sum(axis=0)                          # [V]
        log_pdf = -0.5 * z * z - 0.5 * math.log(2 * math.pi) - math.log(sigma)
        dens = np.exp(log_pdf + log_all[None, :] - log_cdf)    # [E, V]
        pm = dens.sum(axis=1) * dv
        pm = np.maximum(pm / pm.sum(), 1e-300)
        b += 0.5 * sigma * (np.log(p) - np.log(pm))
        b -= b.mean()
    rng = np.random.default_rng(_seed(seed, "zipf_perm"))
    order = rng.permutation(E)
    bias = np.full(E, -1.0e4, dtype=np.float64)
    bias[order[:n_live]] = b
    bias = bias.astype(np.float32)
    bias.flags.writeable = False
    return bias


def generate(cfg: LayerConfig, seed: int = 0, device="cpu", experts=None) -> LayerInputs:
    """Draw one layer's inputs.  ``experts`` (iterable of indices) limits
    which routed experts' weights are materialised; the rest are None."""
    device = torch.device(device)
    T, d, E, F, Fs = cfg.T, cfg.d_model, cfg.num_experts, cfg.expert_ffn, cfg.shared_ffn
    act = torch.float32 if cfg.dtype == "f32" else torch.bfloat16
    x = _normal((T, d), cfg.x_std, seed, "x", -1, device).to(act)
    Wr = _normal((d, E), cfg.wr_std, seed, "W_router", -1, device).to(act)
    bias = None
    if cfg.router == "zipf":
        logit_std = math.sqrt(d) * cfg.x_std * cfg.wr_std
        bias = torch.tensor(zipf_router_bias(E, cfg.n_dead, cfg.zipf_s, logit_std, seed), device=device)
    want = set(range(E)) if experts is None else set(int(e) for e in experts)

    def weight(shape, name, e):
        w = _normal(shape, cfg.w_std, seed, name, e, device)
        if cfg.dtype == "fp8":
            return quantize_e4m3_columns(w)
        if cfg.dtype == "int8":
            return quantize_int8_columns(w)
        if cfg.dtype == "int4":
            return quantize_int4_columns(w)
        return w.to(act), None

    W_gu, W_dn, s_gu, s_dn = [], [], [], []
    for e in range(E):
        if e in want:
            a, sa = weight((d, 2 * F), "W_gate_up", e)
            b, sb = weight((F, d), "W_down", e)
        else:
            a = b = sa = sb = None
        W_gu.append(a)
        W_dn.append(b)
        s_gu.append(sa)
        s_dn.append(sb)
    Ws_gu, ss_gu = weight((d, 2 * Fs), "Ws_gate_up", -1)
    Ws_dn, ss_dn = weight((Fs, d), "Ws_down", -1)
    scaled = cfg.dtype in CODED
    return LayerInputs(cfg, x, Wr, bias, W_gu, W_dn, Ws_gu, Ws_dn,
                       s_gu if scaled else None, s_dn if scaled else None,
                       ss_gu if scaled else None, ss_dn if scaled else None)


# E4M3 code sets for layers that exercise the weight widening: every finite
# code (0x7F / 0xFF are NaN), and the zero and subnormal codes (exponent
# field 0) alone.
E4M3_FINITE_CODES = tuple(c for c in range(256) if c & 0x7F != 0x7F)
E4M3_SUBNORMAL_CODES = tuple(range(0x00, 0x08)) + tuple(range(0x80, 0x88))


INT8_CODES = tuple(range(-128, 128))


INT4_CODES = tuple(range(-8, 8))


def with_weight_codes(inp: LayerInputs, codes, scale: float, seed: int) -> LayerInputs:
    """Replace an E4M3, int8 or int4 layer's expert and shared weights by
    codes drawn uniformly (seeded) from ``codes`` and set every column scale
    to ``scale``."""
    assert inp.cfg.dtype in CODED
    ints = inp.cfg.dtype in ("int8", "int4")
    table = torch.tensor(codes, dtype=torch.int8 if ints else torch.uint8)

    def draw(w, name, e):
        if w is None:
            return None
        g = torch.Generator().manual_seed(_seed(seed, "codes:" + name, e))
        if inp.cfg.dtype == "int4":  # packed [K, N / 2] bytes: draw [K, N] codes, pack them
            i = torch.randint(0, table.numel(), (w.shape[0], 2 * w.shape[1]), generator=g)
            return pack_int4(table[i]).to(w.device)
        i = torch.randint(0, table.numel(), tuple(w.shape), generator=g)
        return (table[i] if ints else table[i].view(torch.float8_e4m3fn)).to(w.device)

    def full(s):
        return None if s is None else torch.full_like(s, scale)

    inp.W_gate_up = [draw(w, "W_gate_up", e) for e, w in enumerate(inp.W_gate_up)]
    inp.W_down = [draw(w, "W_down", e) for e, w in enumerate(inp.W_down)]
    inp.Ws_gate_up = draw(inp.Ws_gate_up, "Ws_gate_up", -1)
    inp.Ws_down = draw(inp.Ws_down, "Ws_down", -1)
    inp.s_gate_up = [full(s) for s in inp.s_gate_up]
    inp.s_down = [full(s) for s in inp.s_down]
    inp.ss_gate_up = full(inp.ss_gate_up)
    inp.ss_down = full(inp.ss_down)
    return inp


def to_storage_numpy(t: torch.Tensor | None) -> np.ndarray | None:
    """Host copy in storage form: float32 as is, bf16 as uint16 bit patterns,
    float8_e4m3fn as uint8 codes, int8 as int8, packed int4 bytes as uint8
    (marshalling only, no arithmetic)."""
    if t is None:
        return None
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.float32:
        return t.numpy()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    if t.dtype in (torch.int8, torch.uint8, torch.int32, torch.int64):
        return t.numpy()
    raise TypeError(f"no storage mapping for {t.dtype}")
