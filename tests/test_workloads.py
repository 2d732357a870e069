"""The seeded input generators (CPU): determinism, expert subsets, the Zipf
router bias and the loads it produces on the Maverick-shaped workload, and
the weight quantisers' ranges and rounding."""
import math

import numpy as np
import pytest
import torch

from sparse_moe_transformer_router_b200.workloads import (CONFIGS, LayerConfig, generate, int4_codes_columns,
                                                          pack_int4, quantize_e4m3_columns,
                                                          quantize_int8_columns, zipf_router_bias)


def test_generation_is_seeded_and_per_expert():
    cfg = LayerConfig("g", 16, 64, 4, 64, 64, "bf16")
    a, b, c = generate(cfg, seed=3), generate(cfg, seed=3), generate(cfg, seed=4)
    assert torch.equal(a.x, b.x) and torch.equal(a.W_router, b.W_router)
    assert all(torch.equal(u, v) for u, v in zip(a.W_gate_up, b.W_gate_up))
    assert not torch.equal(a.x, c.x)
    # an expert's weights do not depend on which other experts are drawn
    sub = generate(cfg, seed=3, experts=[2])
    assert sub.W_gate_up[0] is None and torch.equal(sub.W_gate_up[2], a.W_gate_up[2])
    assert torch.equal(sub.W_down[2], a.W_down[2])


def _zipf_target(n_live, s):
    p = np.arange(1, n_live + 1, dtype=np.float64) ** (-s)
    return p / p.sum()


def test_zipf_bias_gives_zipf_win_probabilities_under_its_logit_model():
    """Monte Carlo of the bias's own logit model (b_e + sigma * Z_e, Z iid
    normal): the win frequencies, sorted, follow Zipf(1.1) over the live
    experts, and the dead experts never win."""
    E, n_dead, s, sigma = 128, 10, 1.1, math.sqrt(5120) * 0.02
    b = zipf_router_bias(E, n_dead, s, sigma, seed=0).astype(np.float64)
    assert np.count_nonzero(b < -1e3) == n_dead
    rng = np.random.default_rng(1)
    n = 200_000
    wins = np.zeros(E, np.int64)
    for _ in range(10):
        z = b[None, :] + sigma * rng.standard_normal((n // 10, E))
        wins += np.bincount(z.argmax(axis=1), minlength=E)
    assert wins[b < -1e3].sum() == 0
    freq = np.sort(wins[b > -1e3])[::-1] / n
    p = _zipf_target(E - n_dead, s)
    se = np.sqrt(p * (1 - p) / n)
    assert np.all(np.abs(freq[:20] - p[:20]) <= 5 * se[:20] + 2e-3)
    assert abs(freq[0] - 0.228) < 0.01  # the largest expert's share


def test_maverick_prefill_loads_follow_the_zipf_recipe():
    """The realised routing of the Maverick-shaped prefill workload (T 8192,
    E 128, x ~ N(0, 1), W_router ~ N(0, 0.02), fitted bias): 118 experts
    receive tokens, the largest about 22.8 % of them."""
    cfg = CONFIGS["maverick_prefill_bf16"]
    inp = generate(cfg, seed=0, experts=[])
    logits = inp.x.float() @ inp.W_router.float() + inp.bias
    counts = np.bincount(logits.argmax(dim=1).numpy(), minlength=cfg.num_experts)
    assert np.count_nonzero(counts) == cfg.num_experts - cfg.n_dead
    assert abs(counts.max() / cfg.T - 0.228) < 0.03
    live = np.sort(counts[counts > 0])[::-1] / cfg.T
    p = _zipf_target(cfg.num_experts - cfg.n_dead, cfg.zipf_s)
    assert np.abs(live[:10] - p[:10]).max() < 0.03


@pytest.mark.parametrize("quant,qmax", [(quantize_int8_columns, 127), (int4_codes_columns, 7)])
def test_integer_quantisers_are_symmetric_per_column_and_round_to_nearest(quant, qmax):
    w = torch.randn(96, 40, generator=torch.Generator().manual_seed(5)) * 0.02
    w[:, 3] = 0.0  # an all-zero column keeps scale 1 and codes 0
    q, s = quant(w)
    assert q.dtype == torch.int8 and s.shape == (40,)
    qa = q.to(torch.int32).abs()
    assert int(qa.max()) == qmax and int(qa.min()) >= 0
    assert torch.all(qa[:, torch.arange(40) != 3].amax(dim=0) == qmax)   # each column reaches the range
    assert float(s[3]) == 1.0 and torch.all(q[:, 3] == 0)
    err = (w - q.double().float() * s[None, :]).abs()
    assert torch.all(err <= s[None, :] * 0.5 + 1e-7)


def test_e4m3_quantiser_fills_the_range_per_column():
    w = torch.randn(64, 24, generator=torch.Generator().manual_seed(6)) * 0.02
    q, s = quantize_e4m3_columns(w)
    deq = q.float() * s[None, :]
    assert torch.all(q.float().abs().amax(dim=0) == 448.0)
    assert torch.all((deq - w).abs() <= w.abs() * 2.0 ** -4 + s[None, :] * 2.0 ** -9)


def test_int4_packing_layout():
    q = torch.tensor([[-8, 7, 0, -1], [1, -2, 3, -4]], dtype=torch.int8)
    p = pack_int4(q)
    assert p.dtype == torch.uint8 and p.shape == (2, 2)
    # even column in the low nibble, two's complement
    assert p.tolist() == [[0x78, 0xF0], [0xE1, 0xC3]]
