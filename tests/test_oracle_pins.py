"""Pins of the CPU oracle to things other than itself.

Each test reduces the layer to a case that the pages or the mathematics fix
(a library matmul, a closed form, an invariant, numpy's argmax / stable
argsort, torch's own dtype decoders), chosen so that a plausible slip in the
oracle (dropped shared expert, gate on the output instead of the input,
swapped gate/up halves, transposed down weight, wrong sigmoid sign, highest
index on ties, wrong subnormal decode, per-row instead of per-column FP8
scales) fails at least one of them.
"""
import numpy as np
import pytest
import torch
from scipy.special import expit

import oracle
from sparse_moe_transformer_router_b200.workloads import quantize_e4m3_columns


def _bf16_bits(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def _bf16_f64(bits: np.ndarray) -> np.ndarray:
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()


def _store(a: np.ndarray, dtype: str):
    """(storage array for the oracle, exact fp64 values it represents)."""
    if dtype == "f32":
        s = np.ascontiguousarray(a, np.float32)
        return s, s.astype(np.float64)
    s = _bf16_bits(a)
    return s, _bf16_f64(s)


def _dense_swiglu(u, Wgu, Wd):
    """Textbook SwiGLU FFN through library routines (torch fp64 matmul, F.silu)."""
    u = torch.from_numpy(u)
    Wgu = torch.from_numpy(Wgu)
    Wd = torch.from_numpy(Wd)
    F = Wd.shape[0]
    a = u @ Wgu
    h = torch.nn.functional.silu(a[:, :F]) * a[:, F:]
    return (h @ Wd).numpy()


def _layer(rng, T, d, E, F, Fs, dtype, wstd=0.2):
    x, x64 = _store(rng.standard_normal((T, d)), dtype)
    Wr, Wr64 = _store(rng.standard_normal((d, E)) * 0.3, dtype)
    Wgu, Wd, Wgu64, Wd64 = [], [], [], []
    for _ in range(E):
        a, a64 = _store(rng.standard_normal((d, 2 * F)) * wstd, dtype)
        b, b64 = _store(rng.standard_normal((F, d)) * wstd, dtype)
        Wgu.append(a), Wd.append(b), Wgu64.append(a64), Wd64.append(b64)
    Wsgu, Wsgu64 = _store(rng.standard_normal((d, 2 * Fs)) * wstd, dtype)
    Wsd, Wsd64 = _store(rng.standard_normal((Fs, d)) * wstd, dtype)
    return dict(x=x, x64=x64, Wr=Wr, Wr64=Wr64, Wgu=Wgu, Wd=Wd, Wgu64=Wgu64, Wd64=Wd64,
                Wsgu=Wsgu, Wsgu64=Wsgu64, Wsd=Wsd, Wsd64=Wsd64)


def test_bf16_decoder_matches_torch_for_every_code():
    codes = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = _bf16_f64(codes)
    got = np.array([oracle.bf16_to_f64(c) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])


def test_e4m3_decoder_matches_torch_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_to_f64(c) for c in codes])
    nan = np.isnan(ref)
    assert nan.sum() == 2  # S.1111.111 for both signs
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_single_expert_with_saturated_gate_is_two_dense_ffns(dtype):
    """E = 1 and router bias 100 force routing to expert 0 with
    sigmoid(>= 100 - small) == 1.0 exactly in fp64, so the layer must equal
    dense_swiglu(x; Wgu_0, Wd_0) + dense_swiglu(x; Ws_gu, Ws_d)."""
    rng = np.random.default_rng(1)
    T, d, F, Fs = 7, 48, 40, 24
    L = _layer(rng, T, d, 1, F, Fs, dtype)
    bias = np.array([100.0], np.float32)
    out, idx, gate = oracle.forward(L["x"], L["Wr"], L["Wgu"], L["Wd"], L["Wsgu"], L["Wsd"], bias=bias)
    assert np.all(idx == 0) and np.all(gate == 1.0)
    ref = _dense_swiglu(L["x64"], L["Wgu64"][0], L["Wd64"][0]) + \
        _dense_swiglu(L["x64"], L["Wsgu64"], L["Wsd64"])
    scale = np.sqrt(np.mean(ref ** 2))
    assert np.max(np.abs(out - ref)) <= 1e-12 * scale


@pytest.mark.parametrize("c", [0.7, -1.3])
def test_constant_logit_gives_sigmoid_gate_on_the_input(c):
    """A zero router weight and a bias with a unique maximum c make every
    logit constant: all tokens go to the arg-max expert with gate
    sigmoid(c), and the routed FFN sees gate * x (not gate * FFN(x))."""
    rng = np.random.default_rng(2)
    T, d, E, F, Fs = 5, 32, 3, 24, 16
    L = _layer(rng, T, d, E, F, Fs, "f32", wstd=0.5)
    Wr0 = np.zeros((d, E), np.float32)
    bias = np.array([c - 1.0, c, c - 0.5], np.float32)  # expert 1 wins
    Wgu = [None, L["Wgu"][1], None]
    Wd = [None, L["Wd"][1], None]
    out, idx, gate = oracle.forward(L["x"], Wr0, Wgu, Wd, L["Wsgu"], L["Wsd"], bias=bias)
    g = expit(np.float64(np.float32(c)))
    assert np.all(idx == 1)
    assert np.allclose(gate, g, rtol=0, atol=1e-15)
    shared = _dense_swiglu(L["x64"], L["Wsgu64"], L["Wsd64"])
    ref_in = shared + _dense_swiglu(g * L["x64"], L["Wgu64"][1], L["Wd64"][1])
    ref_out = shared + g * _dense_swiglu(L["x64"], L["Wgu64"][1], L["Wd64"][1])
    scale = np.sqrt(np.mean(ref_in ** 2))
    assert np.max(np.abs(out - ref_in)) <= 1e-12 * scale
    # the pin has power: gating the output instead would be far off
    assert np.max(np.abs(ref_out - ref_in)) > 1e-3 * scale


def test_argmax_takes_lowest_index_on_ties():
    """One-hot tokens make the logits exact copies of router rows; rows with
    duplicated maxima must resolve to the lowest index, as numpy.argmax does."""
    d, E = 6, 5
    Wr = np.array([[0.0, 2.0, 1.0, 2.0, 2.0],
                   [3.0, 3.0, 3.0, 3.0, 3.0],
                   [-1.0, -2.0, -1.0, -3.0, -1.0],
                   [0.5, 0.25, 0.75, 0.75, 0.1],
                   [0.0, 0.0, 0.0, 0.0, 1.0],
                   [-5.0, -4.0, -4.0, -6.0, -4.0]], np.float32)
    x = np.eye(d, dtype=np.float32)
    idx, lmax, margin = oracle.route(x, Wr)
    assert np.array_equal(idx, np.argmax(Wr, axis=1).astype(np.int32))
    assert list(idx) == [1, 0, 0, 2, 4, 1]
    assert np.array_equal(lmax, Wr.max(axis=1))
    assert list(margin[:3]) == [0.0, 0.0, 0.0] and margin[4] == 1.0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_router_equals_library_matmul_then_argmax(dtype):
    rng = np.random.default_rng(3)
    T, d, E = 257, 96, 16
    x, x64 = _store(rng.standard_normal((T, d)), dtype)
    Wr, Wr64 = _store(rng.standard_normal((d, E)) * 0.1, dtype)
    bias = (rng.standard_normal(E) * 0.05).astype(np.float32)
    idx, lmax, margin = oracle.route(x, Wr, bias)
    logits = (x64 @ Wr64 + bias.astype(np.float64)).astype(np.float32)
    assert np.array_equal(idx, np.argmax(logits, axis=1))
    assert np.array_equal(lmax, logits.max(axis=1))
    srt = np.sort(logits.astype(np.float64), axis=1)
    assert np.allclose(margin, (srt[:, -1] - srt[:, -2]).astype(np.float32), rtol=0, atol=0)


def test_permutation_is_the_stable_argsort():
    rng = np.random.default_rng(4)
    E, T = 12, 1000
    idx = rng.integers(0, E, T).astype(np.int32)
    idx[idx == 5] = 6          # expert 5 empty
    idx[:40] = 11              # heavy tail expert
    counts, offsets, perm = oracle.permutation(idx, E)
    assert counts.sum() == T
    assert np.array_equal(counts, np.bincount(idx, minlength=E))
    assert np.array_equal(offsets, np.concatenate([[0], np.cumsum(np.bincount(idx, minlength=E))]))
    assert np.array_equal(perm, np.argsort(idx, kind="stable"))
    inv = np.empty(T, np.int64)
    inv[perm] = np.arange(T)
    assert np.array_equal(np.sort(perm), np.arange(T))
    assert np.array_equal(perm[inv], np.arange(T))


def test_zero_input_gives_exact_zero_output():
    rng = np.random.default_rng(5)
    T, d, E, F, Fs = 9, 32, 4, 16, 16
    L = _layer(rng, T, d, E, F, Fs, "bf16")
    x = np.zeros_like(L["x"])
    out, idx, gate = oracle.forward(x, L["Wr"], L["Wgu"], L["Wd"], L["Wsgu"], L["Wsd"])
    assert np.all(idx == 0)            # all logits 0: tie -> lowest index
    assert np.all(gate == 0.5)
    assert np.all(out == 0.0)


def test_token_and_expert_relabelling_symmetries():
    """Per-token independence: permuting tokens permutes outputs exactly.
    Expert labels carry no meaning: relabelling experts (router columns and
    weight lists together) leaves every output bit-identical."""
    rng = np.random.default_rng(6)
    T, d, E, F, Fs = 23, 40, 6, 24, 16
    L = _layer(rng, T, d, E, F, Fs, "bf16")
    bias = (rng.standard_normal(E) * 0.3).astype(np.float32)
    out, idx, gate = oracle.forward(L["x"], L["Wr"], L["Wgu"], L["Wd"], L["Wsgu"], L["Wsd"], bias=bias)
    pt = rng.permutation(T)
    out_t, idx_t, _ = oracle.forward(L["x"][pt], L["Wr"], L["Wgu"], L["Wd"], L["Wsgu"], L["Wsd"], bias=bias)
    assert np.array_equal(out_t, out[pt]) and np.array_equal(idx_t, idx[pt])
    pe = rng.permutation(E)              # new expert j is old expert pe[j]
    out_e, idx_e, gate_e = oracle.forward(
        L["x"], np.ascontiguousarray(L["Wr"][:, pe]), [L["Wgu"][j] for j in pe],
        [L["Wd"][j] for j in pe], L["Wsgu"], L["Wsd"], bias=bias[pe])
    assert np.array_equal(out_e, out)
    assert np.array_equal(pe[idx_e], idx)
    assert np.array_equal(gate_e, gate)


def test_fp8_weights_dequantise_per_output_column():
    """E4M3 weights with per-output-column scales equal the dense layer on
    the dequantised weights (torch's float8 decoder times the column scale)."""
    rng = np.random.default_rng(7)
    T, d, F, Fs = 6, 64, 32, 48
    x, x64 = _store(rng.standard_normal((T, d)), "bf16")
    Wr, _ = _store(rng.standard_normal((d, 1)), "bf16")

    def q(shape):
        w = torch.from_numpy(rng.standard_normal(shape) * 0.02).float()
        w[:, 0] *= 50.0  # very different column ranges
        qq, s = quantize_e4m3_columns(w)
        deq = qq.to(torch.float64) * s.to(torch.float64)[None, :]
        return qq.view(torch.uint8).numpy(), s.numpy(), deq.numpy()

    gu, sgu, gu64 = q((d, 2 * F))
    dn, sdn, dn64 = q((F, d))
    sgu_s, ssgu, sgu64 = q((d, 2 * Fs))
    sdn_s, ssdn, sdn64 = q((Fs, d))
    out, idx, gate = oracle.forward(x, Wr, [gu], [dn], sgu_s, sdn_s, bias=np.array([100.0], np.float32),
                                    s_gate_up=[sgu], s_down=[sdn], ss_gate_up=ssgu, ss_down=ssdn)
    assert np.all(gate == 1.0)
    ref = _dense_swiglu(x64, gu64, dn64) + _dense_swiglu(x64, sgu64, sdn64)
    scale = np.sqrt(np.mean(ref ** 2))
    assert np.max(np.abs(out - ref)) <= 1e-12 * scale


def test_token_subset_equals_rows_of_full_run_and_missing_expert_raises():
    rng = np.random.default_rng(8)
    T, d, E, F, Fs = 17, 32, 4, 16, 24
    L = _layer(rng, T, d, E, F, Fs, "f32")
    full, idx, _ = oracle.forward(L["x"], L["Wr"], L["Wgu"], L["Wd"], L["Wsgu"], L["Wsd"])
    sel = np.array([16, 0, 5, 5, 9], np.int32)
    sub, sidx, _ = oracle.forward(L["x"], L["Wr"], L["Wgu"], L["Wd"], L["Wsgu"], L["Wsd"], tokens=sel)
    assert np.array_equal(sub, full[sel]) and np.array_equal(sidx, idx[sel])
    needed = set(idx[sel].tolist())
    Wgu = [w if e in needed else None for e, w in enumerate(L["Wgu"])]
    Wd = [w if e in needed else None for e, w in enumerate(L["Wd"])]
    sub2, _, _ = oracle.forward(L["x"], L["Wr"], Wgu, Wd, L["Wsgu"], L["Wsd"], tokens=sel)
    assert np.array_equal(sub2, sub)
    missing = next(e for e in range(E) if e not in needed) if len(needed) < E else None
    if missing is not None:
        t = int(np.nonzero(idx == missing)[0][0]) if np.any(idx == missing) else None
        if t is not None:
            with pytest.raises(ValueError):
                oracle.forward(L["x"], L["Wr"], Wgu, Wd, L["Wsgu"], L["Wsd"], tokens=np.array([t], np.int32))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_dense_layer_without_experts_is_one_swiglu_ffn(dtype):
    """E = 0 (the layers without experts): the output is the shared SwiGLU
    feed-forward alone, as a library matmul evaluates it."""
    rng = np.random.default_rng(11)
    L = _layer(rng, 9, 24, 0, 8, 40, dtype)
    out, idx, gate = oracle.forward(L["x"], L["Wr"], [], [], L["Wsgu"], L["Wsd"])
    ref = _dense_swiglu(L["x64"], L["Wsgu64"], L["Wsd64"])
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
    assert np.all(idx == -1)


def test_topk_takes_the_k_largest_lowest_index_first_on_ties():
    """One-hot tokens expose router rows as logits: the top-k list is the
    row sorted by (value descending, index ascending), as numpy's stable
    lexsort orders it; the margin is the k-th value minus the next one."""
    d, E = 6, 5
    Wr = np.array([[0.0, 2.0, 1.0, 2.0, 2.0],
                   [3.0, 3.0, 3.0, 3.0, 3.0],
                   [-1.0, -2.0, -1.0, -3.0, -1.0],
                   [0.5, 0.25, 0.75, 0.75, 0.1],
                   [0.0, 0.0, 0.0, 0.0, 1.0],
                   [-5.0, -4.0, -4.0, -6.0, -4.0]], np.float32)
    x = np.eye(d, dtype=np.float32)
    for k in (1, 2, 3, 5):
        idx, lsel, margin = oracle.route_topk(x, Wr, k)
        order = np.stack([np.lexsort((np.arange(E), -row)) for row in Wr])[:, :k]
        assert np.array_equal(idx, order.astype(np.int32))
        assert np.array_equal(lsel, np.take_along_axis(Wr, order, axis=1))
        if k < E:
            nxt = np.take_along_axis(Wr, np.stack([np.lexsort((np.arange(E), -r)) for r in Wr])[:, k:k + 1],
                                     axis=1)[:, 0]
            assert np.array_equal(margin, lsel[:, -1] - nxt)
        else:
            assert np.all(np.isinf(margin))
    idx1, lmax1, _ = oracle.route(x, Wr)
    assert np.array_equal(oracle.route_topk(x, Wr, 1)[0][:, 0], idx1)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_topk_with_every_expert_sums_each_gated_by_its_own_sigmoid(dtype):
    """k = E: every expert runs, each on sigmoid(its logit) * x, and their
    outputs add to the shared expert's -- library matmuls, expert by expert."""
    rng = np.random.default_rng(12)
    T, d, E, F, Fs = 5, 32, 3, 16, 24
    L = _layer(rng, T, d, E, F, Fs, dtype)
    out, idx, gate = oracle.forward(L["x"], L["Wr"], L["Wgu"], L["Wd"], L["Wsgu"], L["Wsd"], k=E)
    logits = (L["x64"] @ L["Wr64"]).astype(np.float32).astype(np.float64)
    ref = _dense_swiglu(L["x64"], L["Wsgu64"], L["Wsd64"])
    for e in range(E):
        g = expit(logits[:, e])[:, None]
        ref = ref + _dense_swiglu(g * L["x64"], L["Wgu64"][e], L["Wd64"][e])
    scale = np.sqrt(np.mean(ref ** 2))
    assert np.max(np.abs(out - ref)) <= 1e-12 * scale
    assert np.array_equal(np.sort(idx, axis=1), np.tile(np.arange(E), (T, 1)))


def test_topk_of_one_is_the_top1_layer():
    rng = np.random.default_rng(13)
    L = _layer(rng, 11, 32, 6, 16, 16, "bf16")
    a = oracle.forward(L["x"], L["Wr"], L["Wgu"], L["Wd"], L["Wsgu"], L["Wsd"])
    b = oracle.forward(L["x"], L["Wr"], L["Wgu"], L["Wd"], L["Wsgu"], L["Wsd"], k=1)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_int8_weights_dequantise_per_output_column():
    """int8 weights with per-output-column scales equal the dense layer on
    the dequantised weights (torch's int8 values times the column scale)."""
    from sparse_moe_transformer_router_b200.workloads import quantize_int8_columns
    rng = np.random.default_rng(17)
    T, d, F, Fs = 6, 64, 32, 48
    x, x64 = _store(rng.standard_normal((T, d)), "bf16")
    Wr, _ = _store(rng.standard_normal((d, 1)), "bf16")

    def q(shape):
        w = torch.from_numpy(rng.standard_normal(shape) * 0.02).float()
        w[:, 0] *= 50.0  # very different column ranges
        qq, s = quantize_int8_columns(w)
        deq = qq.to(torch.float64) * s.to(torch.float64)[None, :]
        return qq.numpy(), s.numpy(), deq.numpy()

    gu, sgu, gu64 = q((d, 2 * F))
    dn, sdn, dn64 = q((F, d))
    sgu_s, ssgu, sgu64 = q((d, 2 * Fs))
    sdn_s, ssdn, sdn64 = q((Fs, d))
    out, idx, gate = oracle.forward(x, Wr, [gu], [dn], sgu_s, sdn_s, bias=np.array([100.0], np.float32),
                                    s_gate_up=[sgu], s_down=[sdn], ss_gate_up=ssgu, ss_down=ssdn)
    assert np.all(gate == 1.0)
    ref = _dense_swiglu(x64, gu64, dn64) + _dense_swiglu(x64, sgu64, sdn64)
    scale = np.sqrt(np.mean(ref ** 2))
    assert np.max(np.abs(out - ref)) <= 1e-12 * scale


def test_int8_codes_with_unit_scales_equal_the_bf16_layer():
    """Every int8 code (-128 included) with unit column scales is the same
    layer as bf16 weights holding those integers (exact in bf16): a code read
    as unsigned, or with a sign slip, breaks the equality."""
    rng = np.random.default_rng(18)
    T, d, E, F, Fs = 9, 64, 3, 32, 48
    x, _ = _store(rng.standard_normal((T, d)), "bf16")
    Wr, _ = _store(rng.standard_normal((d, E)), "bf16")

    def codes(shape):
        q = rng.integers(-128, 128, size=shape).astype(np.int8)
        q.flat[:256] = np.arange(-128, 128, dtype=np.int8)
        return q, _bf16_bits(q.astype(np.float32) / 64.0)

    gu = [codes((d, 2 * F)) for _ in range(E)]
    dn = [codes((F, d)) for _ in range(E)]
    sgu, sdn = codes((d, 2 * Fs)), codes((Fs, d))
    ones = lambda n: np.ones(n, np.float32) / 64.0
    o8, i8, g8 = oracle.forward(x, Wr, [a for a, _ in gu], [a for a, _ in dn], sgu[0], sdn[0],
                                s_gate_up=[ones(2 * F)] * E, s_down=[ones(d)] * E,
                                ss_gate_up=ones(2 * Fs), ss_down=ones(d))
    ob, ib, gb = oracle.forward(x, Wr, [b for _, b in gu], [b for _, b in dn], sgu[1], sdn[1])
    assert np.array_equal(i8, ib) and np.array_equal(g8, gb)
    assert np.array_equal(o8, ob)


def test_int4_codes_equal_the_int8_layer_with_the_same_integers():
    """int4 weights (every code from -8 to 7, packed two per byte along the
    output columns) with per-column scales equal the int8 layer holding the
    same integers and scales: a swapped nibble order, a missing sign
    extension or a packing along the wrong axis breaks the equality."""
    from sparse_moe_transformer_router_b200.workloads import pack_int4
    rng = np.random.default_rng(19)
    T, d, E, F, Fs = 9, 64, 3, 32, 48
    x, _ = _store(rng.standard_normal((T, d)), "bf16")
    Wr, _ = _store(rng.standard_normal((d, E)), "bf16")

    def codes(shape):
        q = rng.integers(-8, 8, size=shape).astype(np.int8)
        q.flat[:16] = np.arange(-8, 8, dtype=np.int8)
        s = (rng.random(shape[1]) * 0.05 + 0.01).astype(np.float32)
        return q, oracle.as_int4x2(pack_int4(torch.from_numpy(q)).numpy()), s

    gu = [codes((d, 2 * F)) for _ in range(E)]
    dn = [codes((F, d)) for _ in range(E)]
    sgu, sdn = codes((d, 2 * Fs)), codes((Fs, d))
    scales = dict(s_gate_up=[g[2] for g in gu], s_down=[g[2] for g in dn], ss_gate_up=sgu[2], ss_down=sdn[2])
    o4, i4, g4 = oracle.forward(x, Wr, [g[1] for g in gu], [g[1] for g in dn], sgu[1], sdn[1], **scales)
    o8, i8, g8 = oracle.forward(x, Wr, [g[0] for g in gu], [g[0] for g in dn], sgu[0], sdn[0], **scales)
    assert np.array_equal(i4, i8) and np.array_equal(g4, g8)
    assert np.array_equal(o4, o8)
    assert np.any(o4 != 0)


def test_int4_quantised_weights_equal_their_codes_in_the_int8_layer():
    """The int4 workload's quantiser (per-column scale max|w| / 7, codes in
    [-7, 7]) fed packed to the oracle gives exactly the int8 layer on the
    unpacked codes; and at k = E with a saturated gate, the library
    evaluation of the dequantised weights."""
    from sparse_moe_transformer_router_b200.workloads import int4_codes_columns, pack_int4
    rng = np.random.default_rng(20)
    T, d, F, Fs = 5, 64, 32, 48
    x, x64 = _store(rng.standard_normal((T, d)), "bf16")
    Wr, _ = _store(rng.standard_normal((d, 1)), "bf16")

    def q(shape):
        w = torch.from_numpy(rng.standard_normal(shape) * 0.02).float()
        w[:, 1] *= 30.0
        qq, s = int4_codes_columns(w)
        assert int(qq.abs().max()) <= 7
        deq = qq.to(torch.float64) * s.to(torch.float64)[None, :]
        return qq.numpy(), oracle.as_int4x2(pack_int4(qq).numpy()), s.numpy(), deq.numpy()

    gu, dn, sgu, sdn = q((d, 2 * F)), q((F, d)), q((d, 2 * Fs)), q((Fs, d))
    kw = dict(bias=np.array([100.0], np.float32), s_gate_up=[gu[2]], s_down=[dn[2]], ss_gate_up=sgu[2],
              ss_down=sdn[2])
    o4, _, g4 = oracle.forward(x, Wr, [gu[1]], [dn[1]], sgu[1], sdn[1], **kw)
    o8, _, _ = oracle.forward(x, Wr, [gu[0]], [dn[0]], sgu[0], sdn[0], **kw)
    assert np.array_equal(o4, o8)
    assert np.all(g4 == 1.0)
    ref = _dense_swiglu(x64, gu[3], dn[3]) + _dense_swiglu(x64, sgu[3], sdn[3])
    assert np.max(np.abs(o4 - ref)) <= 1e-12 * np.sqrt(np.mean(ref ** 2))


def test_e4m3_encoder_round_trips_every_code_and_matches_torch():
    """The FP8 activation mode's encoder: every finite code decodes and
    re-encodes to itself (both zeros included); on random fp32 values across
    the whole range (subnormals, ties, the top binade) it agrees with torch's
    float8_e4m3fn cast (round to nearest even); beyond 448 it saturates."""
    for c in range(256):
        if c & 0x7F == 0x7F:
            continue
        assert oracle.e4m3_encode(oracle.e4m3_to_f64(c)) == c, hex(c)
    rng = np.random.default_rng(21)
    mag = np.exp2(rng.uniform(-12, np.log2(448.0), 20000)).astype(np.float32)
    v = mag * rng.choice([-1.0, 1.0], mag.size).astype(np.float32)
    ties = np.array([(a + b) / 2 for a, b in zip(range(0, 8), range(1, 9))], np.float32) * np.float32(2.0 ** -9)
    v = np.concatenate([v, ties, -ties, np.float32([1.0625, 1.1875, 416.0, 432.0, 440.0])])
    want = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(x) for x in v], np.uint8)
    assert np.array_equal(got, want)
    for big in (448.0, 449.0, 464.0, 1e6, float("inf")):
        assert oracle.e4m3_encode(big) == 0x7E and oracle.e4m3_encode(-big) == 0xFE


def _e4m3_scale_lib(v: torch.Tensor) -> torch.Tensor:
    """Row scales by torch's fp32 arithmetic: max|v| / 448, at least 2^-126,
    1 for a zero row."""
    m = v.abs().amax(dim=1, keepdim=True)
    s = torch.clamp_min(m / 448.0, 2.0 ** -126)
    return torch.where(m == 0, torch.ones_like(s), s)


def _e4m3_rows(v64: np.ndarray) -> np.ndarray:
    """Per-row E4M3 quantisation through torch: s as _e4m3_scale_lib, codes
    = float8 cast of fp32(v * fp32(1 / s)), values = codes * s (fp64)."""
    v = torch.from_numpy(np.ascontiguousarray(v64)).float()
    s = _e4m3_scale_lib(v)
    q = (v * (1.0 / s)).to(torch.float8_e4m3fn)
    return (q.double() * s.double()).numpy()


def _bf16_rows(v64: np.ndarray) -> np.ndarray:
    """Values rounded to fp32, then to bf16, by torch's casts (fp64)."""
    return torch.from_numpy(np.ascontiguousarray(v64)).float().bfloat16().double().numpy()


def test_fp8_activation_mode_is_the_layer_on_e4m3_rows():
    """FP8 activation mode: the layer equals a library evaluation where x and
    every hidden row (shared and routed) are quantised per row by torch's
    float8 cast with the same fp32 scale arithmetic, each hidden row first
    rounded to bf16 (the layer's activation type) by torch's casts, and the
    gate scales the routed expert's quantised input.  The hidden-rounding
    output has nothing more to round and equals the plain one."""
    rng = np.random.default_rng(22)
    T, d, E, F, Fs = 7, 64, 3, 32, 48
    L = _layer(rng, T, d, E, F, Fs, "bf16", wstd=0.2)
    out, idx, gate, out_h = oracle.forward(L["x"], L["Wr"], L["Wgu"], L["Wd"], L["Wsgu"], L["Wsd"],
                                           act_fp8=True, hidden_round="bf16")
    assert np.array_equal(out, out_h)
    xq = _e4m3_rows(L["x64"])

    def ffn(u, Wgu, Wd):
        a = u @ Wgu
        Fw = Wd.shape[0]
        h = torch.nn.functional.silu(torch.from_numpy(a[:, :Fw])).numpy() * a[:, Fw:]
        return _e4m3_rows(_bf16_rows(h)) @ Wd

    ref = ffn(xq, L["Wsgu64"], L["Wsd64"])
    for t in range(T):
        e = int(idx[t])
        ref[t] += ffn(gate[t] * xq[t:t + 1], L["Wgu64"][e], L["Wd64"][e])[0]
    scale = np.sqrt(np.mean(ref ** 2))
    assert np.max(np.abs(out - ref)) <= 1e-12 * scale
    # and it is a different layer from the bf16-activation one
    plain, _, _ = oracle.forward(L["x"], L["Wr"], L["Wgu"], L["Wd"], L["Wsgu"], L["Wsd"])
    rel = np.sqrt(np.mean((out - plain) ** 2)) / scale
    assert 1e-3 < rel < 0.2


def test_fp8_activation_mode_keeps_rows_already_in_e4m3():
    """Input rows that are E4M3 values times a power of two, with the row
    maximum at 448 times it, quantise to themselves: with one expert and a
    saturated gate the mode then equals the library evaluation that
    quantises only the hidden rows (a slip in the scale, say max / 447, or
    in the rounding would move some of the inputs)."""
    codes = np.array([oracle.e4m3_to_f64(c) for c in range(0x00, 0x7F)], np.float64)
    rng = np.random.default_rng(23)
    T, d, F, Fs = 4, 64, 32, 48
    x = rng.choice(np.concatenate([codes, -codes]), size=(T, d)) * 2.0 ** -6
    x[:, 0] = 448.0 * 2.0 ** -6
    xb = _bf16_bits(x)
    assert np.array_equal(_bf16_f64(xb), x)          # exact in bf16
    Wr, _ = _store(rng.standard_normal((d, 1)), "bf16")
    Wgu, Wgu64 = _store(rng.standard_normal((d, 2 * F)) * 0.2, "bf16")
    Wd, Wd64 = _store(rng.standard_normal((F, d)) * 0.2, "bf16")
    Wsgu, Wsgu64 = _store(rng.standard_normal((d, 2 * Fs)) * 0.2, "bf16")
    Wsd, Wsd64 = _store(rng.standard_normal((Fs, d)) * 0.2, "bf16")
    out, _, gate = oracle.forward(xb, Wr, [Wgu], [Wd], Wsgu, Wsd, bias=np.array([100.0], np.float32),
                                  act_fp8=True)
    assert np.all(gate == 1.0)

    def ffn(u, A, B):
        a = u @ A
        Fw = B.shape[0]
        h = torch.nn.functional.silu(torch.from_numpy(a[:, :Fw])).numpy() * a[:, Fw:]
        return _e4m3_rows(_bf16_rows(h)) @ B

    ref = ffn(x, Wsgu64, Wsd64) + ffn(x, Wgu64, Wd64)
    assert np.max(np.abs(out - ref)) <= 1e-12 * np.sqrt(np.mean(ref ** 2))


def test_expert_rows_equals_a_library_swiglu_on_gated_rows():
    """oracle.expert_rows (one expert on given rows, the routed part of each
    (token, expert) entry) against torch fp64: SwiGLU(g * x), bf16 and E4M3
    weights (the latter dequantised per output column)."""
    import torch
    rng = np.random.default_rng(11)
    n, d, F = 7, 64, 48
    x = torch.from_numpy(rng.standard_normal((n, d)).astype(np.float32)).bfloat16()
    g = rng.uniform(0.1, 1.0, size=n)
    Wgu = torch.from_numpy((rng.standard_normal((d, 2 * F)) * 0.1).astype(np.float32)).bfloat16()
    Wd = torch.from_numpy((rng.standard_normal((F, d)) * 0.1).astype(np.float32)).bfloat16()
    bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)  # noqa: E731
    y = oracle.expert_rows(bits(x), g, bits(Wgu), bits(Wd))
    a = (x.double() * torch.from_numpy(g)[:, None]) @ Wgu.double()
    lib = (torch.nn.functional.silu(a[:, :F]) * a[:, F:]) @ Wd.double()
    np.testing.assert_allclose(y, lib.numpy(), rtol=1e-12, atol=1e-13)
    # E4M3 weights with column scales
    q_gu = torch.from_numpy(rng.integers(0, 0x7F, size=(d, 2 * F), dtype=np.uint8)).view(torch.float8_e4m3fn)
    q_d = torch.from_numpy(rng.integers(0, 0x7F, size=(F, d), dtype=np.uint8)).view(torch.float8_e4m3fn)
    s_gu = rng.uniform(0.001, 0.01, size=2 * F).astype(np.float32)
    s_d = rng.uniform(0.001, 0.01, size=d).astype(np.float32)
    y8 = oracle.expert_rows(bits(x), g, q_gu.view(torch.uint8).numpy(), q_d.view(torch.uint8).numpy(),
                            s_gate_up=s_gu, s_down=s_d)
    a8 = (x.double() * torch.from_numpy(g)[:, None]) @ (q_gu.double() * torch.from_numpy(s_gu).double())
    lib8 = (torch.nn.functional.silu(a8[:, :F]) * a8[:, F:]) @ (q_d.double() * torch.from_numpy(s_d).double())
    np.testing.assert_allclose(y8, lib8.numpy(), rtol=1e-12, atol=1e-13)


def test_e4m3_row_quantisation_matches_torch_and_handles_ties_and_zero_rows():
    """oracle.e4m3_rows (the FP8 activation mode's per-row step): the scale
    is fp32(max|v| / 448) (at least 2^-126, 1 for a zero row) and the codes
    equal torch's float8_e4m3fn cast of fp32(v * fp32(1 / s)), including rows
    whose values scale to exact midpoints between two codes (ties to even),
    rows too small for 1 / s to be finite without the 2^-126 floor, and rows
    where dividing by s instead would give other codes."""
    rng = np.random.default_rng(31)
    v = (rng.standard_normal((50, 96)) * np.exp2(rng.uniform(-30, 30, size=(50, 1)))).astype(np.float32)
    vals = np.array([oracle.e4m3_to_f64(c) for c in range(0x00, 0x7F)])
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    tie = rng.choice(np.concatenate([mids, -mids]), size=96).astype(np.float32) * np.float32(2.0 ** -5)
    tie[0] = 448.0 * 2.0 ** -5
    tiny = (rng.standard_normal(96) * 1e-39).astype(np.float32)   # max / 448 below 2^-126
    # rows (bf16 values, as the layer's) where the reciprocal and the division disagree
    differ = []
    while len(differ) < 3:
        r = torch.from_numpy((rng.standard_normal(96) * np.exp2(rng.uniform(-10, 10))).astype(np.float32))
        r = r.bfloat16().float()
        sr = _e4m3_scale_lib(r[None])
        if not torch.equal((r * (1.0 / sr)).to(torch.float8_e4m3fn).view(torch.uint8),
                           (r / sr).to(torch.float8_e4m3fn).view(torch.uint8)):
            differ.append(r.numpy())
    v = np.vstack([v, np.array(differ), tiny[None], tie[None], np.zeros((1, 96), np.float32)])
    codes, scales = oracle.e4m3_rows(v)
    t = torch.from_numpy(v)
    s = _e4m3_scale_lib(t)
    want = (t * (1.0 / s)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(scales, s.numpy().ravel())
    assert np.array_equal(codes, want)
    assert scales[-1] == 1.0 and np.all(codes[-1] == 0)
    assert scales[-3] == np.float32(2.0 ** -126)
    # the tie row: every value is an exact midpoint times 2^-5 (but the
    # maximum), and half of the ties went up, half down (to the even code)
    q = t[-2] / s[-2]
    up = (torch.from_numpy(codes[-2]).view(torch.float8_e4m3fn).float().abs() > q.abs())[1:]
    assert 0 < int(up.sum()) < up.numel()
