"""CUDA path (through the C ABI) against the CPU oracle on the same seeded
inputs: small layers element by element (several tiles, ragged tails, empty
experts, degenerate routings), and the full-size workloads on sampled tokens
plus full routing."""
import numpy as np
import pytest
import torch

from parity_util import (check_outputs, check_outputs_act8, check_routing, check_routing_topk, describe,
                         make_layer, oracle_routing, run_gpu, sample_tokens)
from sparse_moe_transformer_router_b200.workloads import (CONFIGS, DECODE_TOKENS,
                                                          E4M3_FINITE_CODES, E4M3_SUBNORMAL_CODES,
                                                          INT4_CODES, INT8_CODES, LayerConfig, generate,
                                                          with_weight_codes)

pytestmark = pytest.mark.gpu

SMALL = {
    # tiny fp32 workload: T=64, d=128, E=4, F=Fs=256
    "tiny_f32": CONFIGS["tiny_f32"],
    # several feature tiles (F = 384 -> 3), ragged token tiles per expert
    "bf16_ragged": LayerConfig("bf16_ragged", 300, 256, 8, 384, 256, "bf16", wr_std=0.1),
    # d not a multiple of the 128-feature tile; 3 token tiles per expert
    "bf16_two_experts": LayerConfig("bf16_two_experts", 1100, 192, 2, 128, 192, "bf16", wr_std=0.1),
    "f32_ragged": LayerConfig("f32_ragged", 300, 256, 8, 384, 256, "f32", wr_std=0.1),
    # skewed loads with idle experts (router bias)
    "bf16_zipf": LayerConfig("bf16_zipf", 512, 128, 16, 128, 128, "bf16", router="zipf", n_dead=4,
                             wr_std=0.05),
    "bf16_T1": LayerConfig("bf16_T1", 1, 256, 8, 256, 256, "bf16", wr_std=0.1),
    "bf16_E1": LayerConfig("bf16_E1", 70, 128, 1, 128, 128, "bf16"),
    "bf16_E256": LayerConfig("bf16_E256", 600, 128, 256, 64, 64, "bf16", wr_std=0.1),
    # E4M3 weights with per-output-column scales, bf16 activations
    "fp8_ragged": LayerConfig("fp8_ragged", 300, 256, 8, 384, 256, "fp8", wr_std=0.1),
    "fp8_zipf": LayerConfig("fp8_zipf", 700, 192, 16, 128, 320, "fp8", router="zipf", n_dead=4,
                            wr_std=0.05),
    "fp8_T1": LayerConfig("fp8_T1", 1, 256, 8, 256, 256, "fp8", wr_std=0.1),
    # int8 weights with per-output-column scales, bf16 activations
    "int8_ragged": LayerConfig("int8_ragged", 300, 256, 8, 384, 256, "int8", wr_std=0.1),
    "int8_zipf": LayerConfig("int8_zipf", 700, 192, 16, 128, 320, "int8", router="zipf", n_dead=4,
                             wr_std=0.05),
    "int8_T1": LayerConfig("int8_T1", 1, 256, 8, 256, 256, "int8", wr_std=0.1),
    # int4 weights (two per byte) with per-output-column scales
    "int4_ragged": LayerConfig("int4_ragged", 300, 256, 8, 384, 256, "int4", wr_std=0.1),
    "int4_zipf": LayerConfig("int4_zipf", 700, 192, 16, 128, 320, "int4", router="zipf", n_dead=4,
                             wr_std=0.05),
    "int4_T1": LayerConfig("int4_T1", 1, 256, 8, 256, 256, "int4", wr_std=0.1),
    "int4_splitk": LayerConfig("int4_splitk", 2, 1024, 8, 1024, 1024, "int4", wr_std=0.03),
    # few tiles: split-K partials + finish kernels; T <= 128 with E % 16 == 0:
    # expert-split router with the arg-max in the permutation kernel
    "bf16_splitk": LayerConfig("bf16_splitk", 2, 1024, 8, 1024, 1024, "bf16", wr_std=0.03),
    "f32_splitk": LayerConfig("f32_splitk", 3, 1024, 8, 1024, 512, "f32", wr_std=0.03),
    "fp8_splitk": LayerConfig("fp8_splitk", 2, 1024, 8, 1024, 1024, "fp8", wr_std=0.03),
    "int8_splitk": LayerConfig("int8_splitk", 2, 1024, 8, 1024, 1024, "int8", wr_std=0.03),
    "bf16_router_split": LayerConfig("bf16_router_split", 1, 1024, 64, 512, 512, "bf16", wr_std=0.03),
    # the largest batch of the one-launch small-batch routing; fp32 with an
    # expert count that is not a multiple of 8
    "bf16_T16_E128": LayerConfig("bf16_T16_E128", 16, 512, 128, 256, 256, "bf16", wr_std=0.05),
    "f32_T16_E6": LayerConfig("f32_T16_E6", 16, 320, 6, 128, 192, "f32", wr_std=0.1),
    "fp8_T9_zipf": LayerConfig("fp8_T9_zipf", 9, 256, 16, 128, 128, "fp8", router="zipf", n_dead=4,
                               wr_std=0.05),
    "bf16_T40_E32": LayerConfig("bf16_T40_E32", 40, 512, 32, 512, 768, "bf16", wr_std=0.05),
    # few token tiles and E < 32: the router splits K into 4 slices per token
    # tile and reduces them inside a cluster (ragged last tile)
    "bf16_router_kslices": LayerConfig("bf16_router_kslices", 700, 1024, 16, 256, 256, "bf16",
                                       wr_std=0.03),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_small_layer_matches_oracle(name):
    cfg = SMALL[name]
    inp = generate(cfg, seed=0, device="cuda")
    layer = make_layer(inp)
    out, r = run_gpu(layer, inp)
    rep = check_routing(inp, r)
    res = check_outputs(inp, out, None, rep["same"])
    print(f"{name}: {describe(res)}, excluded {rep['excluded']}, flipped {rep['flipped']}")


@pytest.mark.parametrize("dtype,codes,scale", [("fp8", E4M3_FINITE_CODES, 4e-4),
                                               ("fp8", E4M3_SUBNORMAL_CODES, 20.0),
                                               ("int8", INT8_CODES, 1.5e-3),
                                               ("int4", INT4_CODES, 2.5e-2)],
                         ids=["e4m3_all_finite_codes", "e4m3_subnormal_codes", "int8_all_codes",
                              "int4_all_codes"])
def test_weight_widening_is_exact_for_every_code(dtype, codes, scale):
    """Weights drawn from every finite E4M3 code (or from the zero and
    subnormal codes alone), or from every int8 code, with one column scale:
    the widening to f16 is exact and the scale meets the fp32 accumulator, so
    the layer meets the bf16 tolerance, not just the 8-bit one (a flushed or
    mis-mapped code class would break it)."""
    cfg = LayerConfig(f"{dtype}_codes", 300, 256, 4, 256, 192, dtype, wr_std=0.1)
    inp = with_weight_codes(generate(cfg, seed=7, device="cuda"), codes, scale, seed=7)
    layer = make_layer(inp)
    out, r = run_gpu(layer, inp)
    rep = check_routing(inp, r)
    res = check_outputs(inp, out, None, rep["same"], tol=2e-2)
    print(describe(res))


TOPK = {
    # k experts per token: tensor-core router with the top-k epilogue
    "bf16_k2": (LayerConfig("bf16_k2", 300, 256, 8, 384, 256, "bf16", wr_std=0.1), 2),
    "bf16_k4_zipf": (LayerConfig("bf16_k4_zipf", 500, 128, 16, 128, 128, "bf16", router="zipf", n_dead=4,
                                 wr_std=0.05), 4),
    "fp8_k2": (LayerConfig("fp8_k2", 300, 256, 8, 384, 256, "fp8", wr_std=0.1), 2),
    "int8_k2": (LayerConfig("int8_k2", 300, 256, 8, 384, 256, "int8", wr_std=0.1), 2),
    "int4_k2": (LayerConfig("int4_k2", 300, 256, 8, 384, 256, "int4", wr_std=0.1), 2),
    # K slices reduced in a cluster before the top-k epilogue
    "bf16_k2_kslices": (LayerConfig("bf16_k2_kslices", 700, 1024, 16, 256, 256, "bf16", wr_std=0.03), 2),
    # one token tile with E >= 32: expert-split router, top-k in the permutation
    "bf16_k3_split_router": (LayerConfig("bf16_k3_sr", 40, 512, 32, 256, 384, "bf16", wr_std=0.05), 3),
    "bf16_k2_T1": (LayerConfig("bf16_k2_T1", 1, 1024, 64, 512, 512, "bf16", wr_std=0.03), 2),
    # the CUDA-core router's top-k: fp32 layers, and expert counts that are
    # not a multiple of 8 (one and several threads per token)
    "f32_k2": (LayerConfig("f32_k2", 300, 256, 8, 384, 256, "f32", wr_std=0.1), 2),
    "bf16_k3_E12": (LayerConfig("bf16_k3_E12", 300, 256, 12, 128, 256, "bf16", wr_std=0.1), 3),
    "f32_k4_E6_zipf": (LayerConfig("f32_k4_E6_zipf", 200, 128, 6, 128, 128, "f32", router="zipf", n_dead=1,
                                   wr_std=0.1), 4),
    "f32_k2_E40": (LayerConfig("f32_k2_E40", 100, 128, 40, 64, 64, "f32", wr_std=0.1), 2),
    # small-batch routing at its limits: 16 tokens x 4 experts of 256
    "bf16_k4_T16_E256": (LayerConfig("bf16_k4_T16_E256", 16, 512, 256, 64, 128, "bf16", wr_std=0.05), 4),
}


@pytest.mark.parametrize("name", list(TOPK))
def test_topk_layer_matches_oracle(name):
    cfg, k = TOPK[name]
    inp = generate(cfg, seed=0, device="cuda")
    layer = make_layer(inp)
    layer.set_top_k(k)
    out, r = run_gpu(layer, inp)
    rep = check_routing_topk(inp, r, k)
    res = check_outputs(inp, out, None, rep["same"], rep["o_idx"], k=k)
    print(f"{name}: k={k} {describe(res)}, excluded {rep['excluded']}, flipped {rep['flipped']}")


def test_launch_plan_of_small_and_large_batches():
    """Batches of up to 16 tokens route in one launch; with bf16 or fp32
    activations their gate/up starts with the shared expert's tiles while the
    routing runs and the two contractions go out as one fused launch (layers
    with coded weights read the routing's f16 copy of x and do not start
    early); larger batches take the separate launches."""
    for name, small, early in (("bf16_T1", 1, 1), ("bf16_T16_E128", 1, 1), ("f32_T16_E6", 1, 1),
                               ("fp8_T1", 1, 0), ("bf16_ragged", 0, 0)):
        inp = generate(SMALL[name], seed=0, device="cuda")
        layer = make_layer(inp)
        run_gpu(layer, inp)
        p = layer.plan()
        assert p["small_routing"] == small and p["early_shared"] == early, (name, p)
        assert p["fused"] == (early and p["split_gate_up"] == 1), (name, p)
        assert p["small_tiles"] == (SMALL[name].T <= 64), (name, p)


def test_top_k_bounds():
    from sparse_moe_transformer_router_b200.binding import ERR_ARG, L4MoEError
    inp = generate(TOPK["bf16_k2"][0], seed=0, device="cuda")
    layer = make_layer(inp)
    for bad in (0, 5, 9):
        with pytest.raises(L4MoEError) as ei:
            layer.set_top_k(bad)
        assert ei.value.status == ERR_ARG
    # back to one expert per token after a top-2 forward
    layer.set_top_k(2)
    run_gpu(layer, inp)
    layer.set_top_k(1)
    out, r = run_gpu(layer, inp)
    rep = check_routing(inp, r)
    check_outputs(inp, out, None, rep["same"])


DENSE = {
    # no experts: the layer is one SwiGLU feed-forward (ragged token and
    # feature tiles, fp32, E4M3 weights, a single token)
    "dense_bf16": LayerConfig("dense_bf16", 300, 256, 0, 0, 384, "bf16"),
    "dense_f32": LayerConfig("dense_f32", 130, 128, 0, 0, 192, "f32"),
    "dense_fp8": LayerConfig("dense_fp8", 300, 256, 0, 0, 320, "fp8"),
    "dense_int8": LayerConfig("dense_int8", 300, 256, 0, 0, 320, "int8"),
    "dense_int4": LayerConfig("dense_int4", 300, 256, 0, 0, 320, "int4"),
    "dense_T1": LayerConfig("dense_T1", 1, 1024, 0, 0, 1024, "bf16"),
}


def _dense_forward(inp):
    return _dense_forward_on(make_layer(inp), inp)


def _dense_forward_on(layer, inp):
    out = layer.forward(inp.x, None, [], [], inp.Ws_gate_up, inp.Ws_down)
    torch.cuda.synchronize()
    layer.check_device_status()
    return out


@pytest.mark.parametrize("name", list(DENSE))
def test_dense_layer_matches_oracle(name):
    inp = generate(DENSE[name], seed=0, device="cuda")
    res = check_outputs(inp, _dense_forward(inp), None)
    print(f"{name}: {describe(res)}")


ACT8 = {
    # FP8 activation mode: E4M3 x E4M3 tensor-core contractions with per-row
    # token scales (ragged token and feature tiles, idle experts)
    "act8_ragged": (LayerConfig("act8_ragged", 300, 256, 8, 384, 256, "fp8", wr_std=0.1), 1),
    # d = 192: the second 128-deep k-block is half past the rows (zero-filled)
    "act8_zipf_d192": (LayerConfig("act8_zipf_d192", 700, 192, 16, 128, 320, "fp8", router="zipf", n_dead=4,
                                   wr_std=0.05), 1),
    "act8_T1": (LayerConfig("act8_T1", 1, 256, 8, 256, 256, "fp8", wr_std=0.1), 1),
    # the one-launch small-batch routing writes the codes
    "act8_T9_zipf": (LayerConfig("act8_T9_zipf", 9, 256, 16, 128, 128, "fp8", router="zipf", n_dead=4,
                                 wr_std=0.05), 1),
    # split-K: gate/up partials finished in bf16 before the quantisation;
    # down partials take the hidden row scales
    "act8_splitk": (LayerConfig("act8_splitk", 2, 1024, 8, 1024, 1024, "fp8", wr_std=0.03), 1),
    "act8_k2": (LayerConfig("act8_k2", 300, 256, 8, 384, 256, "fp8", wr_std=0.1), 2),
    "act8_dense": (LayerConfig("act8_dense", 300, 256, 0, 0, 320, "fp8"), 1),
    "act8_T40_E32": (LayerConfig("act8_T40_E32", 40, 512, 32, 512, 768, "fp8", wr_std=0.05), 1),
}


def _act8_run(inp, k=1):
    layer = make_layer(inp)
    layer.set_act_fp8(True)
    if k > 1:
        layer.set_top_k(k)
    if inp.cfg.num_experts == 0:
        return layer, _dense_forward_on(layer, inp), None
    out, r = run_gpu(layer, inp)
    return layer, out, r


@pytest.mark.parametrize("name", list(ACT8))
def test_act8_layer_matches_oracle(name):
    cfg, k = ACT8[name]
    inp = generate(cfg, seed=0, device="cuda")
    _, out, r = _act8_run(inp, k)
    if r is None:
        res = check_outputs_act8(inp, out, None)
        print(f"{name}: {describe(res)}, scale-excluded {res['scale_excluded']}")
        return
    rep = check_routing(inp, r) if k == 1 else check_routing_topk(inp, r, k)
    res = check_outputs_act8(inp, out, None, rep["same"], rep["o_idx"], k=k)
    print(f"{name}: {describe(res)}, excluded {rep['excluded']}, flipped {rep['flipped']}, "
          f"scale-excluded {res['scale_excluded']}")


def test_act8_mode_is_opt_in_and_for_e4m3_weights_only():
    from sparse_moe_transformer_router_b200.binding import ERR_DTYPE, L4MoEError
    inp = generate(ACT8["act8_ragged"][0], seed=0, device="cuda")
    layer = make_layer(inp)
    plain, _ = run_gpu(layer, inp)
    layer.set_act_fp8(True)
    q, _ = run_gpu(layer, inp)
    layer.set_act_fp8(False)
    back, _ = run_gpu(layer, inp)
    assert torch.equal(plain, back) and not torch.equal(plain, q)
    bf = generate(SMALL["bf16_ragged"], seed=0, device="cuda")
    with pytest.raises(L4MoEError) as ei:
        make_layer(bf).set_act_fp8(True)
    assert ei.value.status == ERR_DTYPE


def test_full_size_maverick_fp8_act8():
    """Maverick-shaped E4M3 layer (T 16384, Zipf loads) in the FP8 activation
    mode: routing of every token, outputs of a stratified sample."""
    cfg = CONFIGS["maverick_fp8"]
    inp = generate(cfg, seed=0, device="cuda")
    layer, out, r = _act8_run(inp)
    ora = oracle_routing(inp)
    rep = check_routing(inp, r, ora)
    toks = sample_tokens(r, rep, cfg.T, seed=0)
    res = check_outputs_act8(inp, out, toks, rep["same"], rep["o_idx"])
    print(f"{cfg.name} act8: {describe(res)}, excluded {rep['excluded']}, flipped {rep['flipped']}, "
          f"scale-excluded {res['scale_excluded']}")
    del inp, layer
    torch.cuda.empty_cache()


def test_full_size_maverick_dense_layer():
    cfg = CONFIGS["maverick_dense_bf16"]
    inp = generate(cfg, seed=0, device="cuda")
    out = _dense_forward(inp)
    # every 256-token tile's first and last row, then evenly spaced rows
    toks = set()
    for j in range(0, cfg.T, 256):
        toks.update((j, min(cfg.T - 1, j + 255)))
    toks.update(np.linspace(0, cfg.T - 1, 1024 - len(toks) + 2).astype(np.int64).tolist())
    res = check_outputs(inp, out, np.array(sorted(toks), dtype=np.int32))
    print(f"{cfg.name}: {describe(res)}")


def test_zero_input_gives_zero_output_and_expert_zero():
    cfg = LayerConfig("zero", 200, 128, 6, 128, 128, "bf16")
    inp = generate(cfg, seed=1, device="cuda")
    inp.x.zero_()
    layer = make_layer(inp)
    out, r = run_gpu(layer, inp)
    assert torch.all(r["idx"] == 0)
    assert torch.all(r["gate"] == 0.5)
    assert torch.all(out == 0)


def test_all_tokens_to_one_expert_and_saturated_gate():
    cfg = LayerConfig("one_expert", 700, 128, 8, 128, 256, "bf16", wr_std=0.02)
    inp = generate(cfg, seed=2, device="cuda")
    bias = torch.full((8,), -50.0, device="cuda")
    bias[5] = 60.0
    inp.bias = bias
    layer = make_layer(inp)
    out, r = run_gpu(layer, inp)
    assert torch.all(r["idx"] == 5)
    assert torch.all(r["gate"] == 1.0)
    assert r["counts"].cpu().tolist() == [0, 0, 0, 0, 0, 700, 0, 0]
    rep = check_routing(inp, r)
    check_outputs(inp, out, None, rep["same"])


def test_repeatable_and_host_path_identical():
    cfg = SMALL["bf16_ragged"]
    inp = generate(cfg, seed=3, device="cuda")
    layer = make_layer(inp)
    out1, _ = run_gpu(layer, inp)
    out2, _ = run_gpu(layer, inp)
    assert torch.equal(out1, out2)
    x_host = inp.x.cpu().pin_memory()
    outs = [torch.empty_like(x_host).pin_memory() for _ in range(3)]
    for o in outs:  # pipelined calls: slots are reused while earlier copies may be in flight
        layer.forward_host(x_host, inp.W_router, inp.W_gate_up, inp.W_down, inp.Ws_gate_up,
                           inp.Ws_down, o)
    layer.join_host()
    torch.cuda.current_stream().synchronize()
    for o in outs:
        assert torch.equal(o, out1.cpu())
    layer.check_device_status()


def test_kernel_timing_records_only_the_selected_kernels():
    from sparse_moe_transformer_router_b200.binding import ERR_ARG, NUM_KERNELS, L4MoEError
    cfg = SMALL["bf16_ragged"]
    inp = generate(cfg, seed=3, device="cuda")
    layer = make_layer(inp)
    run_gpu(layer, inp)
    layer.read_timing()
    layer.set_timing(["gemm_gate_up"])
    run_gpu(layer, inp)
    layer.set_timing(False)
    t = layer.read_timing()
    assert t["gemm_gate_up"][1] == 1 and t["gemm_gate_up"][0] > 0
    assert all(n == 0 for k, (ms, n) in t.items() if k != "gemm_gate_up")
    with pytest.raises(L4MoEError) as ei:
        layer._check(layer._lib.l4moe_set_timing(layer._h, 1 << NUM_KERNELS))  # no such kernel slot
    assert ei.value.status == ERR_ARG


def test_weight_pointer_change_rebuilds_descriptors():
    cfg = LayerConfig("swap", 256, 128, 4, 128, 128, "bf16", wr_std=0.1)
    a = generate(cfg, seed=4, device="cuda")
    b = generate(cfg, seed=5, device="cuda")
    b.x, b.W_router = a.x, a.W_router  # same routing input, different experts
    layer = make_layer(a)
    out_a, _ = run_gpu(layer, a)
    out_b, r = run_gpu(layer, b)
    rep = check_routing(b, r)
    check_outputs(b, out_b, None, rep["same"])
    assert not torch.equal(out_a, out_b)


def _full_size(cfg, seed=0, all_tokens_up_to=4096):
    """Full-size workload: routing of every token against the oracle; outputs
    of every token when T <= 1024 (decode) or T = 4096 (Scout), else of a
    stratified sample of >= 1024 tokens covering every non-empty expert, every
    token-tile boundary and every band of tiles."""
    inp = generate(cfg, seed=seed, device="cuda")
    layer = make_layer(inp)
    out, r = run_gpu(layer, inp)
    ora = oracle_routing(inp)
    rep = check_routing(inp, r, ora)
    toks = np.arange(cfg.T, dtype=np.int32) if cfg.T <= all_tokens_up_to else sample_tokens(r, rep, cfg.T, seed=seed)
    res = check_outputs(inp, out, toks, rep["same"], rep["o_idx"])
    print(f"{cfg.name}: {describe(res)}, excluded {rep['excluded']}, flipped {rep['flipped']}, "
          f"experts with tokens {int(np.count_nonzero(rep['counts']))}")
    del inp, layer
    torch.cuda.empty_cache()


def test_full_size_scout_prefill():
    _full_size(CONFIGS["scout_prefill_bf16"])


def test_full_size_maverick_prefill_zipf():
    _full_size(CONFIGS["maverick_prefill_bf16"])


@pytest.mark.parametrize("T", DECODE_TOKENS)
def test_full_size_maverick_decode(T):
    _full_size(CONFIGS["maverick_decode_bf16"].with_tokens(T))


def test_full_size_maverick_fp8_zipf():
    _full_size(CONFIGS["maverick_fp8"])


def test_full_size_maverick_int8_zipf():
    _full_size(CONFIGS["maverick_int8"])


def test_full_size_scout_int4():
    _full_size(CONFIGS["scout_prefill_int4"], all_tokens_up_to=1024)


@pytest.mark.parametrize("dtype,T,E", [("fp8", 300, 8), ("int8", 5, 8), ("fp8", 3, 0), ("int8", 40, 0),
                                       ("int4", 64, 8)],
                         ids=["fp8_T300", "int8_T5_small_batch", "fp8_dense_T3", "int8_dense_T40", "int4_T64"])
def test_8bit_layers_take_inputs_beyond_f16_range(dtype, T, E):
    """E4M3 / int8 layers hold x in f16 for their contractions.  With bf16
    inputs around 1e5 (beyond f16's 65504) each token row is divided by a
    power of two on the way to f16 and the accumulators get it back: the
    outputs still match the oracle, which sees the inputs as they are.  The
    weights are small so that the hidden values stay in range."""
    cfg = LayerConfig(f"{dtype}_big_x", T, 256, E, 128 if E else 0, 192, dtype, x_std=1e5, w_std=1e-6,
                      wr_std=1e-6)
    inp = generate(cfg, seed=5, device="cuda")
    assert float(inp.x.float().abs().max()) > 65504.0
    layer = make_layer(inp)
    if E:
        out, r = run_gpu(layer, inp)
        rep = check_routing(inp, r)
        res = check_outputs(inp, out, None, rep["same"])
    else:
        res = check_outputs(inp, _dense_forward(inp), None)
    print(f"{cfg.name} T={T}: {describe(res)}")


def test_hidden_values_beyond_f16_range_are_reported():
    """A hidden value of an 8-bit-weight layer that f16 cannot hold is not
    stored silently as infinity: the device status says so."""
    from sparse_moe_transformer_router_b200.binding import ERR_RANGE, L4MoEError
    cfg = LayerConfig("fp8_big_hidden", 64, 256, 4, 128, 128, "fp8", x_std=1e3, wr_std=1e-4)
    inp = generate(cfg, seed=6, device="cuda")
    layer = make_layer(inp)
    layer.forward(inp.x, inp.W_router, inp.W_gate_up, inp.W_down, inp.Ws_gate_up, inp.Ws_down)
    with pytest.raises(L4MoEError) as ei:
        layer.check_device_status()
    assert ei.value.status == ERR_RANGE
    layer.check_device_status()  # the word was cleared


def test_a_bounded_wait_that_runs_out_is_reported_and_the_context_survives():
    """The failure path of every mbarrier wait in the kernels: a wait whose
    phase never completes gives up after its limit (here 5 ms), records a
    timeout in the device status and returns; the next forward still runs."""
    from sparse_moe_transformer_router_b200.binding import ERR_TIMEOUT, L4MoEError
    inp = generate(SMALL["bf16_ragged"], seed=3, device="cuda")
    layer = make_layer(inp)
    layer.selftest_wait(5.0)
    with pytest.raises(L4MoEError) as ei:
        layer.check_device_status()
    assert ei.value.status == ERR_TIMEOUT
    layer.check_device_status()  # cleared
    out, r = run_gpu(layer, inp)
    rep = check_routing(inp, r)
    check_outputs(inp, out, None, rep["same"])
