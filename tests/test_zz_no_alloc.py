"""The allocation-free entry point, l4moe_forward_static.

It exists for callers that may not allocate device memory while they run the
layer (work recorded under CUDA-graph stream capture, code inside another
framework's allocator callbacks, or a process whose device memory is fully
reserved up front).  It runs the same kernels as l4moe_forward but keeps its
workspace in the library's fixed device array.  This file runs last so that a
run stopping at the first failure has already run every other test.
"""
import pytest
import torch

from parity_util import make_layer
from sparse_moe_transformer_router_b200.binding import ERR_WORKSPACE, L4MoEError
from sparse_moe_transformer_router_b200.workloads import LayerConfig, generate

pytestmark = pytest.mark.gpu


def _assert_same(out: torch.Tensor, ref: torch.Tensor):
    """The two entry points run the same deterministic kernels on the same
    inputs (only the workspace's address differs), so the outputs are equal
    bit for bit."""
    assert torch.isfinite(out.float()).all()
    assert torch.equal(out, ref)


@pytest.mark.parametrize("dtype", ["bf16", "f32", "fp8", "int8", "int4"])
def test_static_forward_matches_allocating_forward_on_two_calls(dtype):
    cfg = LayerConfig(f"noalloc_{dtype}", 300, 256, 8, 384, 256, dtype, wr_std=0.1)
    inp = generate(cfg, seed=11, device="cuda")
    layer = make_layer(inp)
    args = (inp.x, inp.W_router, inp.W_gate_up, inp.W_down, inp.Ws_gate_up, inp.Ws_down)
    ref = layer.forward(*args)
    torch.cuda.synchronize()
    for _ in range(2):  # the shared scratch array keeps the previous call's contents
        out = torch.full_like(ref, float("nan"))
        layer.forward_static(*args, out)
        torch.cuda.synchronize()
        _assert_same(out, ref)


def test_static_forward_rejects_batches_beyond_its_array():
    cfg = LayerConfig("noalloc_big", 64, 256, 8, 384, 256, "bf16", wr_std=0.1)
    inp = generate(cfg, seed=12, device="cuda")
    layer = make_layer(inp)
    x_big = torch.zeros((20000, cfg.d_model), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(x_big)
    with pytest.raises(L4MoEError) as ei:
        layer.forward_static(x_big, inp.W_router, inp.W_gate_up, inp.W_down, inp.Ws_gate_up,
                             inp.Ws_down, out)
    assert ei.value.status == ERR_WORKSPACE
    assert "static" in str(ei.value)


@pytest.mark.parametrize("dtype", ["bf16", "fp8", "int8"])
def test_static_forward_replays_inside_a_cuda_graph(dtype):
    """The use it exists for: record the layer once under stream capture,
    replay it, including after the input values change in place.  The 8-bit
    layers' replays also re-read the handle's scale-pointer table."""
    cfg = LayerConfig(f"noalloc_graph_{dtype}", 200, 256, 8, 384, 256, dtype, wr_std=0.1)
    inp = generate(cfg, seed=13, device="cuda")
    layer = make_layer(inp)
    args = (inp.x, inp.W_router, inp.W_gate_up, inp.W_down, inp.Ws_gate_up, inp.Ws_down)
    out = torch.empty((cfg.T, cfg.d_model), dtype=inp.x.dtype, device="cuda")
    layer.forward_static(*args, out)  # first call outside capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        layer.forward_static(*args, out)
    for flip in (1.0, -0.5):
        inp.x.mul_(flip)
        ref = layer.forward(*args)
        out.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        _assert_same(out, ref)
    del graph
