"""The output tolerance, checked on the CPU with the oracle and library
roundings (no GPU).

The stated bound is max|out - oracle| <= 2e-2 * rms(oracle) for bf16 layers.
The layer's output is bf16, so even a correctly rounded copy of the exact
result carries the bf16 rounding of every element, up to half a bf16 spacing:
2^-8 of the value just above a power of two.  At the tails of a layer's
output (max|out| / rms reaches 5 to 7 on these workloads) that alone can
reach 2e-2 * rms.  These tests pin:
  * the half-spacing used by the parity check against torch's own bf16
    rounding (the bound is attained, so 2^-8, not 2^-9, is the unit);
  * that on the seeded inputs of the small parity layer `bf16_two_experts`
    a correctly rounded exact output exceeds 2e-2 * rms: there the stated
    bound is out of reach of exact arithmetic;
  * that the parity check accepts an exact implementation of the stated
    roundings (hidden rows rounded to bf16, output rounded once) and rejects
    an output one bf16 spacing off at a single element.
"""
import numpy as np
import pytest
import torch

import oracle
from parity_util import (HIDDEN, READING_SLACK, TOL, halfulp_bf16, judge_outputs, oracle_outputs,
                         round_out)
from sparse_moe_transformer_router_b200.workloads import LayerConfig, generate


def test_half_spacing_bounds_torch_bf16_rounding_and_is_attained():
    rng = np.random.default_rng(0)
    v = rng.standard_normal(200_000) * np.exp2(rng.integers(-20, 20, size=200_000))
    v = v.astype(np.float32).astype(np.float64)    # one rounding (fp32 -> bf16), as the GPU's output
    r = round_out(v, "bf16")
    ratio = np.abs(r - v) / halfulp_bf16(r)
    assert np.all(ratio <= 1.0)
    assert ratio.max() > 0.999                     # the bound is reached
    # relative to the value, just above a power of two: 2^-8, not 2^-9
    w = 1.0 + 2.0 ** -8 * (1 - 2.0 ** -20)         # just below the midpoint of 1 and 1 + 2^-7
    assert round_out(np.array([w]), "bf16")[0] == 1.0
    assert abs(1.0 - w) / w > 2.0 ** -8 * 0.99
    assert halfulp_bf16(np.array([1.0, 1.99, 2.0, 0.75, 0.0])).tolist() == \
        [2.0 ** -8, 2.0 ** -8, 2.0 ** -7, 2.0 ** -9, 0.0]


def _small(cfg, seed=0):
    inp = generate(cfg, seed=seed, device="cpu")
    toks = np.arange(cfg.T, dtype=np.int32)
    ref, ref_h = oracle_outputs(inp, toks)
    return inp, ref, ref_h


def test_correctly_rounded_output_already_exceeds_the_stated_bound_on_a_small_layer():
    """bf16_two_experts (T 1100, d 192, E 2, F 128, Fs 192; the GPU parity
    layer of that name), CPU-drawn inputs of the same recipe and seed."""
    cfg = LayerConfig("bf16_two_experts", 1100, 192, 2, 128, 192, "bf16", wr_std=0.1)
    _, ref, ref_h = _small(cfg)
    rms = np.sqrt(np.mean(ref ** 2))
    floor_out = np.max(np.abs(round_out(ref, "bf16") - ref)) / rms
    assert floor_out > TOL["bf16"]                  # exact arithmetic, one rounding: out of reach
    # the stated roundings (hidden rows in bf16) are further off still
    assert np.max(np.abs(round_out(ref_h, "bf16") - ref)) / rms > floor_out
    print(f"correctly rounded exact output: max|err|/rms = {floor_out:.4e}")


@pytest.mark.parametrize("dtype", ["bf16", "fp8", "int8"])
def test_parity_check_accepts_the_reading_and_rejects_one_spacing_off(dtype):
    cfg = LayerConfig(f"floor_{dtype}", 300, 256, 8, 384, 256, dtype, wr_std=0.1)
    _, ref, ref_h = _small(cfg)
    assert HIDDEN[dtype] is not None and ref_h is not None
    exact = round_out(ref_h, dtype)                 # the reading, evaluated exactly, rounded once
    rep = judge_outputs(exact, ref, ref_h, dtype)
    assert rep["reading"] <= 1e-6                   # the fp32 step before the bf16 rounding
    # one element moved by one bf16 spacing (at the largest output)
    bad = exact.copy()
    i = np.unravel_index(np.argmax(np.abs(bad)), bad.shape)
    bad[i] += 2 * halfulp_bf16(bad[i]) * np.sign(bad[i])
    with pytest.raises(AssertionError, match="stated roundings"):
        judge_outputs(bad, ref, ref_h, dtype)
    # a small extra error everywhere (an approximate contraction) is caught too
    rms = np.sqrt(np.mean(ref ** 2))
    noisy = round_out(ref_h + 3 * READING_SLACK[HIDDEN[dtype]] * rms * np.sign(ref_h), dtype)
    with pytest.raises(AssertionError):
        judge_outputs(noisy, ref, ref_h, dtype)


def test_oracle_hidden_rounding_matches_a_library_evaluation():
    """The oracle's second output (hidden values rounded through fp32 to bf16
    or f16 before the down projection) equals a torch fp64 evaluation with
    torch's own conversions, on a dense layer (E = 0) and on a one-expert
    layer with a saturated gate."""
    rng = np.random.default_rng(3)
    d, Fs, T = 64, 96, 20
    x = torch.from_numpy(rng.standard_normal((T, d)).astype(np.float32))
    Wgu = torch.from_numpy((rng.standard_normal((d, 2 * Fs)) * 0.1).astype(np.float32))
    Wd = torch.from_numpy((rng.standard_normal((Fs, d)) * 0.1).astype(np.float32))
    Wr = np.zeros((d, 0), np.float32)
    for kind, tdt in (("bf16", torch.bfloat16), ("f16", torch.float16)):
        out, _, _, out_h = oracle.forward(x.numpy(), Wr, [], [], Wgu.numpy(), Wd.numpy(), hidden_round=kind)
        a = x.double() @ Wgu.double()
        h = torch.nn.functional.silu(a[:, :Fs]) * a[:, Fs:]
        lib = h @ Wd.double()
        lib_h = h.float().to(tdt).double() @ Wd.double()
        np.testing.assert_allclose(out, lib.numpy(), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(out_h, lib_h.numpy(), rtol=1e-12, atol=1e-12)
        assert np.max(np.abs(out_h - out)) > 0      # the rounding does something
        # one routed expert (its own weights) next to the shared one; a router
        # bias of 100 makes the gate exactly 1 in fp64
        W2gu = torch.from_numpy((rng.standard_normal((d, 2 * Fs)) * 0.1).astype(np.float32))
        W2d = torch.from_numpy((rng.standard_normal((Fs, d)) * 0.1).astype(np.float32))
        _, _, gate, out_h1 = oracle.forward(x.numpy(), np.zeros((d, 1), np.float32), [W2gu.numpy()],
                                            [W2d.numpy()], Wgu.numpy(), Wd.numpy(),
                                            bias=np.array([100.0], np.float32), hidden_round=kind)
        assert np.all(gate == 1.0)
        a2 = x.double() @ W2gu.double()
        h2 = torch.nn.functional.silu(a2[:, :Fs]) * a2[:, Fs:]
        lib_h1 = lib_h + h2.float().to(tdt).double() @ W2d.double()
        np.testing.assert_allclose(out_h1, lib_h1.numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("hidden,tdt", [("bf16", torch.bfloat16), ("f16", torch.float16)])
def test_hidden_rounding_flips_stay_within_the_reading_slack(hidden, tdt):
    """The reading check's slack covers hidden values that fp32 arithmetic
    rounds to the other neighbour of the exact value's rounding.  Perturbing
    every hidden value of a layer by a relative 1e-6 (an fp32 accumulation
    error) flips a small fraction of them and moves outputs by up to a few
    thousandths of rms with bf16 rows -- more than any allowance for fp32
    noise alone, within READING_SLACK -- and by 8 times less with f16 rows."""
    cfg = LayerConfig("flips", 300, 256, 0, 0, 384, "bf16")
    inp = generate(cfg, seed=0, device="cpu")
    x, Wgu, Wd = inp.x.double(), inp.Ws_gate_up.double(), inp.Ws_down.double()
    a = x @ Wgu
    h = torch.nn.functional.silu(a[:, :384]) * a[:, 384:]
    rng = np.random.default_rng(1)
    hn = h * (1 + 1e-6 * torch.from_numpy(rng.standard_normal(tuple(h.shape))))
    hb, hnb = h.float().to(tdt).double(), hn.float().to(tdt).double()
    flipped = (hb != hnb).double().mean().item()
    y = hb @ Wd
    dy = ((hnb @ Wd) - y).abs().max().item() / y.pow(2).mean().sqrt().item()
    assert 0 < flipped < 1e-2
    assert dy <= READING_SLACK[hidden]
    if hidden == "bf16":
        assert dy > 1e-3      # far above fp32 noise: the flips themselves
    print(f"{hidden}: {flipped:.2e} of hidden values flipped, max output change {dy:.2e} * rms")


def _e4m3_rows_lib(v: torch.Tensor):
    """Per-row E4M3 quantisation with torch's casts (fp64 values out) and
    the row scales: s = fp32(max|v| / 448) (at least 2^-126, 1 for a zero
    row), codes from fp32(v * fp32(1 / s))."""
    m = v.float().abs().amax(dim=1, keepdim=True)
    s = torch.clamp_min(m / 448.0, 2.0 ** -126)
    s = torch.where(m == 0, torch.ones_like(s), s)
    q = (v.float() * (1.0 / s)).to(torch.float8_e4m3fn)
    return q.double() * s.double(), s


def _bf16_margin_lib(h: torch.Tensor) -> np.ndarray:
    """The hidden-scale margin of each row by torch's bf16 arithmetic: for
    every element within one bf16 spacing of the row's largest |fp32 value|,
    its distance to the midpoints between its bf16 neighbours (found with
    nextafter in bf16), relative to that largest value; the row minimum."""
    a = h.float().abs()
    m = a.amax(dim=1, keepdim=True)
    lo = torch.from_numpy((a.numpy().view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32))
    lo_b = lo.bfloat16()
    hi_b = torch.nextafter(lo_b, torch.full_like(lo_b, float("inf")))
    below_b = torch.nextafter(lo_b, torch.zeros_like(lo_b))
    a64, lo64 = a.double(), lo_b.double()
    d_up = (a64 - (lo64 + hi_b.double()) / 2).abs()
    d_dn = (a64 - (lo64 + below_b.double()) / 2).abs()
    dist = torch.minimum(d_up, d_dn) / m.double()
    near = (a64 >= m.double() * (1 - 2.0 ** -7)) & (a64 > 0)
    return torch.where(near, dist, torch.full_like(dist, float("inf"))).amin(dim=1).numpy()


def test_act8_scale_margin_matches_a_library_evaluation():
    """The oracle's hidden-scale margin (FP8 activation mode) equals a torch
    evaluation on the same hidden rows, on a dense layer (one hidden row per
    token); and rows whose margin is large keep their scale under a relative
    perturbation well below it, while perturbing a row's largest element
    across its nearest midpoint changes the scale."""
    cfg = LayerConfig("margin", 200, 128, 0, 0, 512, "bf16")
    inp = generate(cfg, seed=4, device="cpu")
    from parity_util import w_storage
    x = inp.x.double()
    xq, _ = _e4m3_rows_lib(x)
    a = xq @ inp.Ws_gate_up.double()
    h = torch.nn.functional.silu(a[:, :512]) * a[:, 512:]
    want = _bf16_margin_lib(h)
    res = oracle.forward(w_storage(inp.x, "bf16"), np.zeros((128, 0), np.uint16), [], [],
                         w_storage(inp.Ws_gate_up, "bf16"), w_storage(inp.Ws_down, "bf16"),
                         act_fp8=True, scale_margin=True)
    got = res[-1]
    np.testing.assert_allclose(got, want, rtol=1e-9, atol=1e-15)
    assert np.all(np.isfinite(got)) and got.min() < 1e-3 < got.max()
    _, s0 = _e4m3_rows_lib(h.float().bfloat16().double())
    wide = got > 1e-4
    hp = h * (1 + 3e-5 * torch.from_numpy(np.random.default_rng(5).standard_normal(tuple(h.shape))))
    _, s1 = _e4m3_rows_lib(hp.float().bfloat16().double())
    assert torch.equal(s0[wide], s1[wide])
    # the row with the smallest margin: push its largest element across the midpoint
    r = int(np.argmin(got))
    j = int(h[r].abs().argmax())
    hq = h.clone()
    step = 4 * got[r] * float(h[r].abs().max())
    for sgn in (1.0, -1.0):
        hq[r, j] = h[r, j] + sgn * step * np.sign(float(h[r, j]))
        _, s2 = _e4m3_rows_lib(hq.float().bfloat16().double())
        if not torch.equal(s2[r], s0[r]):
            break
    assert not torch.equal(s2[r], s0[r])


def test_act8_hidden_flips_stay_within_the_reading_slack():
    """The FP8 activation mode's reading slack: with every hidden value of a
    layer (hidden width 2048) perturbed by a relative 1e-6 (fp32 accumulation
    error) before its bf16 rounding and E4M3 quantisation, the tokens whose
    scale margin is at least SCALE_MARGIN_EXCLUDE keep their scales, and
    their outputs move by at most READING_SLACK["act8"] * rms -- by more than
    the bf16 slack: a flipped code moves its element by a whole E4M3 step."""
    from parity_util import SCALE_MARGIN_EXCLUDE
    F = 2048
    cfg = LayerConfig("act8_flips", 300, 512, 0, 0, F, "bf16")
    inp = generate(cfg, seed=0, device="cpu")
    xq, _ = _e4m3_rows_lib(inp.x.double())
    a = xq @ inp.Ws_gate_up.double()
    h = torch.nn.functional.silu(a[:, :F]) * a[:, F:]
    Wd = inp.Ws_down.double()
    margin = _bf16_margin_lib(h)
    keep = margin >= SCALE_MARGIN_EXCLUDE
    worst = 0.0
    for seed in (1, 2, 3):
        hn = h * (1 + 1e-6 * torch.from_numpy(np.random.default_rng(seed).standard_normal(tuple(h.shape))))
        q, s = _e4m3_rows_lib(h.float().bfloat16().double())
        qn, sn = _e4m3_rows_lib(hn.float().bfloat16().double())
        assert torch.equal(s[torch.from_numpy(keep)], sn[torch.from_numpy(keep)])
        y, yn = q @ Wd, qn @ Wd
        rms = y.pow(2).mean().sqrt().item()
        worst = max(worst, ((yn - y).abs().amax(dim=1).numpy()[keep]).max() / rms)
    assert 5e-3 < worst <= READING_SLACK["act8"]
    print(f"act8: {np.count_nonzero(~keep)} of {keep.size} tokens excluded, worst output change {worst:.3e} * rms")
