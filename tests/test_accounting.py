"""The harness's FLOP accounting, pinned to the modelled costs printed on
llm-architectures-explained 'Llama 4 Maverick' (section 'Modelled costs'),
and to the Scout parameter counts of the superteams.ai glossary."""
import json
import os

from sparse_moe_transformer_router_b200.accounting import flops_per_token, layer_bytes, layer_flops

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "maverick_modelled_costs.json")))


def _model_totals():
    a = GOLD["architecture"]
    d, V, L = a["d_model"], a["vocab"], a["layers"]
    n_moe = L // a["moe_every"]
    n_dense = L - n_moe
    kv = a["kv_heads"] * a["head_dim"]
    attn_proj = d * (a["heads"] * a["head_dim"] + 2 * kv) + a["heads"] * a["head_dim"] * d
    moe_flops = flops_per_token(d, a["experts"], a["d_expert"], a["d_shared"])
    dense_flops = 6 * d * a["dense_d_ff"]
    head = 2 * d * V
    attn_ctx = 4 * a["heads"] * a["head_dim"] * a["context"]
    linear = n_moe * moe_flops + n_dense * dense_flops + L * 2 * attn_proj + head
    decode = linear + L * attn_ctx
    moe_active = moe_flops // 2
    moe_total = d * a["experts"] + a["experts"] * 3 * d * a["d_expert"] + 3 * d * a["d_shared"]
    body_active = n_moe * moe_active + n_dense * dense_flops // 2 + L * attn_proj
    body_total = n_moe * moe_total + n_dense * dense_flops // 2 + L * attn_proj
    emb = 2 * d * V
    return dict(decode_gflop_per_token_at_4k=decode / 1e9,
                prefill_tflop_4k_prompt=a["context"] * linear / 1e12,
                params_total_b=(body_total + emb) / 1e9,
                params_active_b=(body_active + emb) / 1e9,
                params_total_wo_embeddings_b=body_total / 1e9,
                params_active_wo_embeddings_b=body_active / 1e9)


def test_layer_flops_reproduce_the_printed_model_costs():
    got = _model_totals()
    for key, printed in GOLD["printed"].items():
        assert abs(got[key] - printed) <= GOLD["printed_rounding"][key], (key, got[key], printed)


def test_layer_counts():
    assert flops_per_token(5120, 16, 8192, 8192) == 503_480_320
    assert flops_per_token(5120, 128, 8192, 8192) == 504_627_200
    assert layer_flops(4096, 5120, 16, 8192, 8192) == 4096 * 503_480_320
    # Scout-shaped prefill: 16 experts touched, bf16
    b = layer_bytes(4096, 5120, 16, 8192, 8192, "bf16", 16)
    assert 4.6e9 < b < 4.8e9


def _scout_params(d_shared: int):
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "scout_glossary_params.json")))
    a = g["architecture"]
    d, V, L = a["d_model"], a["vocab"], a["layers"]
    assert a["moe_every"] == 1 and not a["tie_embeddings"]
    kv = a["kv_heads"] * a["head_dim"]
    attn_proj = d * (a["heads"] * a["head_dim"] + 2 * kv) + a["heads"] * a["head_dim"] * d
    moe_active = flops_per_token(d, a["experts"], a["d_expert"], d_shared) // 2
    moe_total = d * a["experts"] + a["experts"] * 3 * d * a["d_expert"] + 3 * d * d_shared
    emb = 2 * d * V  # untied embedding and output head
    return g, (L * (moe_total + attn_proj) + emb) / 1e9, (L * (moe_active + attn_proj) + emb) / 1e9


def test_scout_parameter_counts_select_the_8192_shared_width():
    """The glossary's Scout figures (about 109B stored, 17B active) follow from
    the KerasFormers Scout defaults with a shared expert of width 8192 (the
    Maverick table's d_shared), and not with KerasFormers' dense_mlp_dim of
    16384, which would make about 23B active per token."""
    g, total, active = _scout_params(8192)
    tol = g["printed_relative_tolerance"]
    assert abs(total - g["printed"]["params_total_b"]) <= tol["params_total_b"] * g["printed"]["params_total_b"]
    assert abs(active - g["printed"]["params_active_b"]) <= tol["params_active_b"] * g["printed"]["params_active_b"]
    _, total16, active16 = _scout_params(g["shared_width_readings"]["kerasformers_dense_mlp_dim"])
    assert abs(active16 - g["printed"]["params_active_b"]) > 0.3 * g["printed"]["params_active_b"]
    assert g["shared_width_readings"]["maverick_table_d_shared"] == 8192
