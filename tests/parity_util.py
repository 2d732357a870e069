"""Helpers shared by the GPU parity tests: run the CUDA path through the
C-ABI binding, run the oracle on the same seeded inputs, compare.

Acceptance (the layer's stated tolerances):
  * expert indices bit-exact on every token whose oracle top-2 fp32 logit
    margin is >= 1e-4 (closer tokens are excluded and counted);
  * per-expert counts equal the histogram of the indices, offsets/perm equal
    the oracle's stable permutation of the CUDA indices (exact);
  * outputs, two assertions (check_outputs):
    - the reading check: every output equals the oracle's exact evaluation
      of the stated roundings (hidden rows rounded to the activation type,
      bf16 -- f16 for 8-bit weight layers -- everything else exact) to
      within the output's own rounding and a small allowance for fp32
      accumulation order: |out - ref_h| <= halfulp(out) + READING_SLACK *
      rms(oracle), the slack covering hidden values whose fp32 value rounds
      to the neighbour of the exact value's rounding (see READING_SLACK).
      (fp32 layers multiply in TF32, which the oracle does not model: they
      take the plain bound below only.)
    - the stated bound max|out - oracle| <= tol * rms(oracle), tol = 2e-2
      (fp32, bf16) or 6e-2 (E4M3, int8 weights), asserted wherever every
      exact implementation of those roundings meets it: where the largest
      error such an implementation can make,
          max over elements of (halfulp(ref_h) + |ref_h - oracle|) / rms,
      plus READING_SLACK, is within tol.  Elsewhere the bound is out of
      reach of exact arithmetic itself (the bf16 rounding of the output
      alone can exceed 2e-2 * rms at the tails of small layers) and only the
      reading check applies; the plain max|err| / rms is reported either way.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from sparse_moe_transformer_router_b200.binding import L4MoE
from sparse_moe_transformer_router_b200.workloads import CODED, LayerInputs, to_storage_numpy

MARGIN_EXCLUDE = 1e-4
TOL = {"f32": 2e-2, "bf16": 2e-2, "fp8": 6e-2, "int8": 6e-2, "int4": 6e-2}
# the type the GPU holds the hidden rows in (None: fp32 layers, TF32 products)
HIDDEN = {"f32": None, "bf16": "bf16", "fp8": "f16", "int8": "f16", "int4": "f16"}
# Allowance, in units of rms(oracle), beyond the output's own rounding.  The
# GPU forms each hidden value in fp32 (tensor-core accumulation, fast exp)
# before rounding it to the hidden type; where that fp32 value and the exact
# one fall on either side of a rounding midpoint, the two round to adjacent
# values, and that one-spacing difference moves every output of the token
# by the spacing times the down-projection weights.  A relative 1e-6 to 1e-5
# error in the hidden values -- fp32 accumulation order -- is enough for a
# few such flips per token, and one flip of a large hidden value dominates:
# the CPU reproduction (tests/test_tolerance_floor.py) moves outputs by up to
# about 6e-3 * rms with bf16 hidden rows; f16 rows have an 8 times finer
# spacing.
READING_SLACK = {"bf16": 8e-3, "f16": 1.5e-3, "act8": 2.5e-2}
# The FP8 activation mode quantises each hidden row (held in bf16) to E4M3
# with the row's own scale.  A bf16 flip of an element whose two bf16
# neighbours straddle an E4M3 rounding midpoint moves that element by a whole
# E4M3 step (up to 1/8 of its value): rarer than a bf16 flip, 16 times
# larger, so the slack is the "act8" entry (pinned in
# tests/test_tolerance_floor.py by the same CPU reproduction).  A flip of the
# row's largest element changes the row's scale and so re-quantises the whole
# row; tokens where that can happen -- a near-largest hidden value within
# SCALE_MARGIN_EXCLUDE (relative) of a bf16 rounding midpoint, by the
# oracle's exact values -- are excluded and counted, like near-tie routings.
SCALE_MARGIN_EXCLUDE = 1e-5


def halfulp_bf16(v: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 numbers (8-bit significand) in the binade of
    each |v|: the largest rounding error a value that rounds to v can have
    had (for v a power of two, the larger spacing above it).  Zero for 0."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(e - 8), 0.0)


def round_out(v: np.ndarray, dtype: str) -> np.ndarray:
    """v rounded to the layer's output type (through fp32, as the GPU forms
    the output in fp32): a library conversion, not the oracle's."""
    f = torch.from_numpy(np.asarray(v, dtype=np.float64).astype(np.float32))
    if dtype == "f32":
        return f.double().numpy()
    return f.to(torch.bfloat16).double().numpy()


def make_layer(inp: LayerInputs) -> L4MoE:
    c = inp.cfg
    layer = L4MoE(c.d_model, c.expert_ffn, c.shared_ffn, c.num_experts, c.dtype)
    if inp.bias is not None:
        layer.set_router_bias(inp.bias)
    if c.dtype in CODED:
        layer.set_weight_scales(inp.s_gate_up, inp.s_down, inp.ss_gate_up, inp.ss_down)
    return layer


def run_gpu(layer: L4MoE, inp: LayerInputs, out=None):
    out = layer.forward(inp.x, inp.W_router, inp.W_gate_up, inp.W_down, inp.Ws_gate_up,
                        inp.Ws_down, out=out)
    torch.cuda.synchronize()
    layer.check_device_status()
    r = {k: v.clone() for k, v in layer.routing().items()}
    return out, r


def oracle_routing(inp: LayerInputs):
    x = to_storage_numpy(inp.x)
    Wr = to_storage_numpy(inp.W_router)
    b = None if inp.bias is None else inp.bias.detach().cpu().numpy()
    return oracle.route(x, Wr, b)


def check_routing(inp: LayerInputs, r: dict, ora=None) -> dict:
    """Compare the CUDA routing with the oracle's; returns a small report."""
    E = inp.cfg.num_experts
    T = inp.cfg.T
    o_idx, o_lmax, o_margin = ora if ora is not None else oracle_routing(inp)
    g_idx = r["idx"].cpu().numpy()
    keep = o_margin >= MARGIN_EXCLUDE
    mism = np.nonzero((g_idx != o_idx) & keep)[0]
    assert mism.size == 0, f"expert index mismatch on {mism.size} tokens, e.g. {mism[:8]}"
    assert np.all((g_idx >= 0) & (g_idx < E))
    # gate and winning logit where the routing agrees
    same = g_idx == o_idx
    g_lmax = r["lmax"].cpu().numpy()
    assert np.max(np.abs(g_lmax[same] - o_lmax[same]), initial=0.0) <= 1e-3 * max(1.0, np.max(np.abs(o_lmax[same]), initial=1.0))
    o_gate = 1.0 / (1.0 + np.exp(-o_lmax.astype(np.float64)))
    g_gate = r["gate"].cpu().numpy().astype(np.float64)
    assert np.max(np.abs(g_gate[same] - o_gate[same]), initial=0.0) <= 1e-5
    # histogram / scan / stable permutation of the CUDA indices (exact)
    counts, offsets, perm = oracle.permutation(g_idx, E)
    assert np.array_equal(r["counts"].cpu().numpy(), counts)
    assert np.array_equal(r["offsets"].cpu().numpy(), offsets)
    assert np.array_equal(r["perm"].cpu().numpy(), perm)
    assert counts.sum() == T
    o_counts = np.bincount(o_idx, minlength=E)
    flipped = int(np.count_nonzero(~same))
    if flipped == 0:
        assert np.array_equal(counts, o_counts)
    return {"excluded": int(np.count_nonzero(~keep)), "flipped": flipped,
            "counts": counts, "same": same, "o_idx": o_idx}


def check_routing_topk(inp: LayerInputs, r: dict, k: int) -> dict:
    """Top-k routing against the oracle's: the selected sets per token (the
    order of near-equal selected logits may differ from the oracle's fp64
    rounding, and the layer's output does not depend on it), each selected
    expert's gate, and the permutation of the CUDA entries (exact)."""
    E, T = inp.cfg.num_experts, inp.cfg.T
    x = to_storage_numpy(inp.x)
    Wr = to_storage_numpy(inp.W_router)
    b = None if inp.bias is None else inp.bias.detach().cpu().numpy()
    o_idx, o_lsel, o_margin = oracle.route_topk(x, Wr, k, b)
    g_idx = r["idx"].cpu().numpy().reshape(T, k)
    g_gate = r["gate"].cpu().numpy().reshape(T, k).astype(np.float64)
    keep = o_margin >= MARGIN_EXCLUDE
    same = np.all(np.sort(g_idx, axis=1) == np.sort(o_idx, axis=1), axis=1)
    bad = np.nonzero(~same & keep)[0]
    assert bad.size == 0, f"selected experts differ on {bad.size} tokens, e.g. {bad[:8]}"
    assert np.all((g_idx >= 0) & (g_idx < E))
    assert np.all(np.sort(g_idx, axis=1)[:, 1:] != np.sort(g_idx, axis=1)[:, :-1])  # distinct
    o_gate = 1.0 / (1.0 + np.exp(-o_lsel.astype(np.float64)))
    og = np.take_along_axis(o_gate, np.argsort(o_idx, axis=1), axis=1)
    gg = np.take_along_axis(g_gate, np.argsort(g_idx, axis=1), axis=1)
    assert np.max(np.abs(og[same] - gg[same]), initial=0.0) <= 1e-5
    counts, offsets, perm = oracle.permutation(g_idx.reshape(-1), E)
    assert np.array_equal(r["counts"].cpu().numpy(), counts)
    assert np.array_equal(r["offsets"].cpu().numpy(), offsets)
    assert np.array_equal(r["perm"].cpu().numpy(), perm)
    assert counts.sum() == T * k
    return {"excluded": int(np.count_nonzero(~keep)), "flipped": int(np.count_nonzero(~same)),
            "counts": counts, "same": same, "o_idx": o_idx}


def w_storage(t, dtype: str):
    """A weight in the oracle's storage form: packed int4 bytes are viewed as
    the oracle's int4 type, everything else as to_storage_numpy gives it."""
    a = to_storage_numpy(t)
    return oracle.as_int4x2(a) if dtype == "int4" and a is not None else a


def oracle_outputs(inp: LayerInputs, tokens: np.ndarray, o_idx=None, k: int = 1,
                   chunk_experts: int = 16):
    """The oracle's exact outputs and its evaluation of the stated roundings
    (None for fp32 layers) for `tokens`, in that order.  With the oracle's
    routing `o_idx` (top-1 layers), the tokens are evaluated in groups of at
    most `chunk_experts` experts, so that only those experts' weights are
    held on the host at a time (a full-size sample can touch all of them)."""
    ref, ref_h, _ = _oracle_eval(inp, tokens, o_idx, k, chunk_experts)
    return ref, ref_h


def oracle_outputs_act8(inp: LayerInputs, tokens: np.ndarray, o_idx=None, k: int = 1,
                        chunk_experts: int = 16):
    """The oracle's FP8-activation-mode outputs for `tokens` (its reading
    already holds every rounding the mode makes) and each token's hidden
    scale margin (oracle.forward(scale_margin=True))."""
    ref, _, margin = _oracle_eval(inp, tokens, o_idx, k, chunk_experts, act_fp8=True)
    return ref, margin


def _oracle_eval(inp, tokens, o_idx, k, chunk_experts, act_fp8=False):
    c = inp.cfg
    hidden = None if act_fp8 else HIDDEN[c.dtype]
    x = to_storage_numpy(inp.x)
    Wr = to_storage_numpy(inp.W_router)
    b = None if inp.bias is None else inp.bias.detach().cpu().numpy()
    Ws_gu, Ws_dn = w_storage(inp.Ws_gate_up, c.dtype), w_storage(inp.Ws_down, c.dtype)
    E = c.num_experts
    if o_idx is None or k > 1 or E == 0:
        groups = [(tokens, set(range(E)) if o_idx is None else
                   set(int(e) for e in np.asarray(o_idx)[tokens].ravel()))]
    else:
        te = np.asarray(o_idx)[tokens]
        experts = sorted(set(int(e) for e in te))
        groups = []
        for i in range(0, len(experts), chunk_experts):
            chunk = set(experts[i:i + chunk_experts])
            groups.append((tokens[np.isin(te, list(chunk))], chunk))
    ref = np.zeros((tokens.size, c.d_model))
    ref_h = np.zeros_like(ref) if hidden else None
    margin = np.full(tokens.size, np.inf) if act_fp8 else None
    pos = {int(t): i for i, t in enumerate(tokens)}
    for toks, need in groups:
        Wgu = [w_storage(inp.W_gate_up[e], c.dtype) if e in need else None for e in range(E)]
        Wdn = [w_storage(inp.W_down[e], c.dtype) if e in need else None for e in range(E)]
        kw = {}
        if c.dtype in CODED:
            kw = dict(s_gate_up=[inp.s_gate_up[e].cpu().numpy() if e in need else None for e in range(E)],
                      s_down=[inp.s_down[e].cpu().numpy() if e in need else None for e in range(E)],
                      ss_gate_up=inp.ss_gate_up.cpu().numpy(), ss_down=inp.ss_down.cpu().numpy())
        res = oracle.forward(x, Wr, Wgu, Wdn, Ws_gu, Ws_dn, bias=b, tokens=toks, k=k,
                             hidden_round=hidden, act_fp8=act_fp8, scale_margin=act_fp8, **kw)
        rows = np.array([pos[int(t)] for t in toks], dtype=np.int64)
        ref[rows] = res[0]
        if hidden:
            ref_h[rows] = res[3]
        if act_fp8:
            margin[rows] = res[-1]
        del Wgu, Wdn, kw, res
    return ref, ref_h, margin


def judge_outputs(got: np.ndarray, ref: np.ndarray, ref_h, dtype: str, tol: float | None = None,
                  slack: float | None = None) -> dict:
    """The two output assertions (module docstring) on aligned arrays."""
    assert np.all(np.isfinite(got)), "non-finite outputs"
    rms = float(np.sqrt(np.mean(ref ** 2)))
    err = np.abs(got - ref)
    tol = TOL[dtype] if tol is None else tol
    plain = float(np.max(err)) / rms if rms > 0 else float(np.max(err))
    rep = {"plain": plain, "n_tokens": int(got.shape[0])}
    if ref_h is None:
        rep.update(reading=None, floor=None, stated_bound_asserted=True)
        assert plain <= tol, f"max|err|/rms = {plain:.4g} exceeds tol {tol}"
        return rep
    slack = READING_SLACK[HIDDEN[dtype]] if slack is None else slack
    dev = np.abs(got - ref_h) - halfulp_bf16(got)
    reading = float(np.max(dev)) / rms
    floor = float(np.max(halfulp_bf16(ref_h) + np.abs(ref_h - ref))) / rms
    asserted = floor + slack <= tol
    rep.update(reading=reading, floor=floor, stated_bound_asserted=bool(asserted))
    assert reading <= slack, (
        f"output off the oracle's evaluation of the stated roundings by {reading:.3g} * rms beyond "
        f"its own rounding (allowed {slack}); max|err|/rms = {plain:.4g}")
    if asserted:
        assert plain <= tol, f"max|err|/rms = {plain:.4g} exceeds tol {tol} (floor {floor:.4g})"
    return rep


def check_outputs(inp: LayerInputs, out: torch.Tensor, tokens, same_mask=None, o_idx=None,
                  tol: float | None = None, k: int = 1) -> dict:
    """Oracle outputs for `tokens` (None = all) against the CUDA output rows.
    Tokens whose routing flipped on a near-tie are skipped.  Asserts the
    reading check and, where every exact implementation of the stated
    roundings meets it, the stated bound (see the module docstring).
    Returns {"plain": max|err| / rms, "reading": max over elements of
    (|out - ref_h| - halfulp(out)) / rms, "floor": the largest error an exact
    implementation could make / rms, "stated_bound_asserted": bool,
    "n_tokens": tokens compared}."""
    T = inp.cfg.T
    if tokens is None:
        tokens = np.arange(T, dtype=np.int32)
    tokens = np.asarray(tokens, dtype=np.int32)
    if same_mask is not None:
        tokens = tokens[same_mask[tokens]]
    ref, ref_h = oracle_outputs(inp, tokens, o_idx, k)
    got = out[torch.as_tensor(tokens, device=out.device, dtype=torch.long)].float().cpu().numpy().astype(np.float64)
    return judge_outputs(got, ref, ref_h, inp.cfg.dtype, tol)


def describe(rep: dict) -> str:
    """One line of a check_outputs report for the test log."""
    s = f"max|err|/rms = {rep['plain']:.3e} over {rep['n_tokens']} tokens"
    if rep.get("reading") is not None:
        s += (f", beyond own rounding {rep['reading']:.2e}, floor {rep['floor']:.3e}, stated bound "
              f"{'asserted' if rep['stated_bound_asserted'] else 'out of reach (floor + slack > tol)'}")
    return s


def sample_tokens(r: dict, rep: dict, T: int, seed: int = 0, n_min: int = 1024, tile: int = 256):
    """A stratified sample of at least `n_min` tokens (all of them when T is
    not larger): for every non-empty expert the first and last slot of its
    rows, the two slots on each side of every `tile`-row token-tile boundary
    inside them, and random slots in proportion to its rows; for the shared
    expert (token order) the same at every token-tile boundary; then evenly
    spaced tokens until `n_min` are reached.  Every GEMM token tile, every
    band of tiles and every expert is hit."""
    if T <= n_min:
        return np.arange(T, dtype=np.int32)
    rng = np.random.default_rng(seed)
    counts = np.asarray(rep["counts"])
    offs = np.concatenate([[0], np.cumsum(counts)])
    perm = r["perm"].cpu().numpy()
    toks = {0, T - 1}
    for j in range(tile, T, tile):            # shared expert's tile boundaries
        toks.update((j - 1, j))
    slots = set()
    for e in np.nonzero(counts)[0]:
        lo, hi = int(offs[e]), int(offs[e + 1])
        slots.update((lo, hi - 1))
        for j in range(lo + tile, hi, tile):
            slots.update((j - 1, j))
        n_rand = max(1, (n_min // 2) * (hi - lo) // max(1, int(counts.sum())))
        slots.update(int(v) for v in rng.integers(lo, hi, size=n_rand))
    toks.update(int(perm[s_]) for s_ in slots)
    if len(toks) < n_min:
        toks.update(int(v) for v in np.linspace(0, T - 1, n_min - len(toks) + 2).astype(np.int64))
    return np.array(sorted(toks), dtype=np.int32)


def check_outputs_act8(inp: LayerInputs, out: torch.Tensor, tokens, same_mask=None, o_idx=None,
                       k: int = 1) -> dict:
    """The FP8 activation mode's outputs against the oracle's reading of the
    mode (act_fp8): tokens whose routing flipped on a near-tie, or whose
    hidden-row scale may differ (margin below SCALE_MARGIN_EXCLUDE), are
    skipped and counted; the rest take the reading check with the "act8"
    slack and, where the output's own rounding leaves room, the E4M3 bound
    (6e-2 * rms)."""
    T = inp.cfg.T
    if tokens is None:
        tokens = np.arange(T, dtype=np.int32)
    tokens = np.asarray(tokens, dtype=np.int32)
    if same_mask is not None:
        tokens = tokens[same_mask[tokens]]
    ref, margin = oracle_outputs_act8(inp, tokens, o_idx, k)
    keep = margin >= SCALE_MARGIN_EXCLUDE
    got = out[torch.as_tensor(tokens, device=out.device, dtype=torch.long)].float().cpu().numpy().astype(np.float64)
    rep = judge_outputs(got[keep], ref[keep], ref[keep], "fp8", TOL["fp8"], READING_SLACK["act8"])
    rep["scale_excluded"] = int(np.count_nonzero(~keep))
    return rep
