"""Helpers shared by the GPU parity tests: run the CUDA path through the
C-ABI binding, run the oracle on the same seeded inputs, compare.

Acceptance (the layer's stated tolerances):
  * expert indices bit-exact on every token whose oracle top-2 fp32 logit
    margin is >= 1e-4 (closer tokens are excluded and counted);
  * per-expert counts equal the histogram of the indices, offsets/perm equal
    the oracle's stable permutation of the CUDA indices (exact);
  * outputs: per element |out - oracle| <= tol * rms(oracle) + u * |oracle|
    with tol = 2e-2 (f32 / bf16 weights) or 6e-2 (E4M3 weights) and u the
    unit roundoff of the output type (2^-8 for bf16, 2^-24 for f32).  The
    u * |oracle| term is the rounding of the exact result to the output type
    itself: a correctly rounded bf16 copy of the fp64 oracle already reaches
    1-2% of rms(oracle) at the tails of these layers, so a bound of
    tol * rms alone would fail even for exact arithmetic.  The plain
    max|err| / rms(oracle) is reported alongside.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from sparse_moe_transformer_router_b200.binding import L4MoE
from sparse_moe_transformer_router_b200.workloads import LayerInputs, to_storage_numpy

MARGIN_EXCLUDE = 1e-4
TOL = {"f32": 2e-2, "bf16": 2e-2, "fp8": 6e-2, "int8": 6e-2}
OUT_UNIT_ROUNDOFF = {"f32": 2.0 ** -24, "bf16": 2.0 ** -8, "fp8": 2.0 ** -8, "int8": 2.0 ** -8}


def make_layer(inp: LayerInputs) -> L4MoE:
    c = inp.cfg
    layer = L4MoE(c.d_model, c.expert_ffn, c.shared_ffn, c.num_experts, c.dtype)
    if inp.bias is not None:
        layer.set_router_bias(inp.bias)
    if c.dtype in ("fp8", "int8"):
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


def check_outputs(inp: LayerInputs, out: torch.Tensor, tokens, same_mask=None, o_idx=None,
                  tol: float | None = None, k: int = 1) -> float:
    """Oracle outputs for `tokens` (None = all) against the CUDA output rows.
    Tokens whose routing flipped on a near-tie are skipped.  Asserts the
    per-element bound (tol defaults to the dtype's); returns
    max|err| / rms(oracle)."""
    c = inp.cfg
    T = c.T
    if tokens is None:
        tokens = np.arange(T, dtype=np.int32)
    tokens = np.asarray(tokens, dtype=np.int32)
    if same_mask is not None:
        tokens = tokens[same_mask[tokens]]
    need = set(range(c.num_experts)) if o_idx is None else set(int(e) for e in np.asarray(o_idx)[tokens].ravel())
    x = to_storage_numpy(inp.x)
    Wr = to_storage_numpy(inp.W_router)
    b = None if inp.bias is None else inp.bias.detach().cpu().numpy()
    Wgu = [to_storage_numpy(inp.W_gate_up[e]) if e in need else None for e in range(c.num_experts)]
    Wdn = [to_storage_numpy(inp.W_down[e]) if e in need else None for e in range(c.num_experts)]
    kw = {}
    if c.dtype in ("fp8", "int8"):
        kw = dict(s_gate_up=[inp.s_gate_up[e].cpu().numpy() if e in need else None for e in range(c.num_experts)],
                  s_down=[inp.s_down[e].cpu().numpy() if e in need else None for e in range(c.num_experts)],
                  ss_gate_up=inp.ss_gate_up.cpu().numpy(), ss_down=inp.ss_down.cpu().numpy())
    ref, _, _ = oracle.forward(x, Wr, Wgu, Wdn, to_storage_numpy(inp.Ws_gate_up),
                               to_storage_numpy(inp.Ws_down), bias=b, tokens=tokens, k=k, **kw)
    got = out[torch.as_tensor(tokens, device=out.device, dtype=torch.long)].float().cpu().numpy().astype(np.float64)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    err = np.abs(got - ref)
    tol = TOL[c.dtype] if tol is None else tol
    bound = tol * rms + OUT_UNIT_ROUNDOFF[c.dtype] * np.abs(ref)
    worst = float(np.max(err / bound))
    ratio = float(np.max(err)) / rms if rms > 0 else float(np.max(err))
    assert worst <= 1.0, (f"|err| exceeds tol*rms + u*|ref| by {worst:.3f}x "
                          f"(max|err|/rms = {ratio:.4g}, tol {tol})")
    return ratio


def sample_tokens(r: dict, rep: dict, T: int, seed: int = 0, per_expert: int = 4, n_experts: int = 5):
    """Tokens to check at full size: from the most and least loaded non-empty
    experts plus random ones, the first and last slot of each (the ragged tail
    of its last token tile), a slot at a 256-token tile boundary and a random
    slot; plus tokens 0 and T-1."""
    rng = np.random.default_rng(seed)
    counts = rep["counts"]
    offs = np.concatenate([[0], np.cumsum(counts)])
    perm = r["perm"].cpu().numpy()
    nonempty = np.nonzero(counts)[0]
    order = nonempty[np.argsort(-counts[nonempty], kind="stable")]
    chosen = list(dict.fromkeys([int(order[0]), int(order[-1])] +
                                [int(e) for e in rng.choice(nonempty, size=min(len(nonempty), n_experts), replace=False)]))
    chosen = chosen[:n_experts]
    toks = {0, T - 1}
    for e in chosen:
        lo, hi = int(offs[e]), int(offs[e + 1])
        slots = {lo, hi - 1, int(rng.integers(lo, hi))}
        if hi - lo > 256:
            slots.add(lo + 256)
        for s in list(slots)[:per_expert]:
            toks.add(int(perm[s]))
    return np.array(sorted(toks), dtype=np.int32)
