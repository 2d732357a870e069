"""Argument checks of the Python binding (no GPU needed): the C ABI takes raw
pointers, so the binding compares every tensor's shape, dtype and device
with the layer before a call could make the kernels read past a buffer."""
import pytest
import torch

from sparse_moe_transformer_router_b200.binding import L4MoE


def _layer(d=64, F=32, Fs=48, E=3, dtype="bf16"):
    layer = object.__new__(L4MoE)  # no library call: only the host-side checks
    layer.d_model, layer.expert_ffn, layer.shared_ffn, layer.num_experts, layer.dtype = d, F, Fs, E, dtype
    return layer


def test_io_shapes_dtypes_and_devices_are_checked():
    layer = _layer()
    x = torch.zeros(5, 64, dtype=torch.bfloat16)
    Wr = torch.zeros(64, 3, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="shape"):
        layer._check_io(torch.zeros(5, 32, dtype=torch.bfloat16), Wr, None)
    with pytest.raises(ValueError, match="dtype"):
        layer._check_io(torch.zeros(5, 64, dtype=torch.float32), Wr, None)
    with pytest.raises(ValueError, match="shape"):
        layer._check_io(x, torch.zeros(64, 4, dtype=torch.bfloat16), None, host=True)
    with pytest.raises(ValueError, match="out has shape"):
        layer._check_io(x, Wr, torch.zeros(6, 64, dtype=torch.bfloat16), host=True)
    with pytest.raises(ValueError, match="x must be a CUDA tensor"):
        layer._check_io(x, Wr, None)  # right shape and dtype, but on the host
    # the host-buffer entry point takes host x / out (W_router stays on the device)
    with pytest.raises(ValueError, match="W_router must be a CUDA tensor"):
        layer._check_io(x, Wr, torch.zeros(5, 64, dtype=torch.bfloat16), host=True)
    with pytest.raises(ValueError, match="x must be"):
        layer._check_io(torch.zeros(64, dtype=torch.bfloat16), Wr, None)


def test_layers_without_experts_need_no_router():
    layer = _layer(E=0, F=0)
    x = torch.zeros(5, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        layer._check_io(x, None, None)   # reaches the device check: W_router is not asked for


@pytest.mark.parametrize("dtype,wdt", [("bf16", torch.bfloat16), ("fp8", torch.float8_e4m3fn),
                                       ("int8", torch.int8), ("f32", torch.float32)])
def test_weight_shapes_and_dtypes_are_checked(dtype, wdt):
    layer = _layer(dtype=dtype)
    d, F, Fs, E = 64, 32, 48, 3
    gu = [torch.zeros(d, 2 * F, dtype=wdt) for _ in range(E)]
    dn = [torch.zeros(F, d, dtype=wdt) for _ in range(E)]
    sgu, sdn = torch.zeros(d, 2 * Fs, dtype=wdt), torch.zeros(Fs, d, dtype=wdt)
    with pytest.raises(ValueError, match="expected 3 expert weights"):
        layer._weights(gu[:2], dn, sgu, sdn)
    with pytest.raises(ValueError, match=r"W_down\[1\] has shape"):
        layer._weights(gu, [dn[0], torch.zeros(d, F, dtype=wdt), dn[2]], sgu, sdn)
    other = torch.bfloat16 if wdt != torch.bfloat16 else torch.float32
    with pytest.raises(ValueError, match=r"W_gate_up\[0\] has dtype"):
        layer._weights([gu[0].to(other)] + gu[1:], dn, sgu, sdn)
    with pytest.raises(ValueError, match="Ws_down has shape"):
        layer._weights(gu, dn, sgu, torch.zeros(d, Fs, dtype=wdt))
    with pytest.raises(ValueError, match="CUDA tensor"):
        layer._weights(gu, dn, sgu, sdn)


def test_weight_arrays_are_cached_by_address_and_rechecked_on_change(monkeypatch):
    from sparse_moe_transformer_router_b200 import binding
    monkeypatch.setattr(binding, "_where", lambda t, name, host=False: None)  # host tensors stand in
    layer = _layer()
    d, F, Fs, E = 64, 32, 48, 3
    gu = [torch.zeros(d, 2 * F, dtype=torch.bfloat16) for _ in range(E)]
    dn = [torch.zeros(F, d, dtype=torch.bfloat16) for _ in range(E)]
    sgu, sdn = torch.zeros(d, 2 * Fs, dtype=torch.bfloat16), torch.zeros(Fs, d, dtype=torch.bfloat16)
    first = layer._weights(gu, dn, sgu, sdn)
    assert [first[0][i] for i in range(E)] == [w.data_ptr() for w in gu]
    assert layer._weights(list(gu), list(dn), sgu, sdn) is first      # same addresses: cached
    gu2 = gu[:2] + [torch.ones(d, 2 * F, dtype=torch.bfloat16)]
    second = layer._weights(gu2, dn, sgu, sdn)
    assert second is not first and second[0][2] == gu2[2].data_ptr()
    with pytest.raises(ValueError, match=r"W_down\[0\] is required"):
        layer._weights(gu, [None] + dn[1:], sgu, sdn)
    with pytest.raises(ValueError, match=r"W_gate_up\[1\] has shape"):
        layer._weights([gu[0], torch.zeros(d, F, dtype=torch.bfloat16), gu[2]], dn, sgu, sdn)
    with pytest.raises(ValueError, match="contiguous"):
        layer._weights([gu[0], torch.zeros(2 * F, d, dtype=torch.bfloat16).t(), gu[2]], dn, sgu, sdn)


def test_a_view_at_a_checked_address_is_checked_again(monkeypatch):
    """A transpose, a slice or a reinterpreting view of a checked weight
    shares its address but is another tensor: the cache must not let it
    through unchecked."""
    from sparse_moe_transformer_router_b200 import binding
    monkeypatch.setattr(binding, "_where", lambda t, name, host=False: None)  # host tensors stand in
    layer = _layer(d=64, F=48, Fs=32)
    d, F, Fs, E = 64, 48, 32, 3
    gu = [torch.zeros(d, 2 * F, dtype=torch.bfloat16) for _ in range(E)]
    dn = [torch.zeros(F, d, dtype=torch.bfloat16) for _ in range(E)]
    sgu, sdn = torch.zeros(d, 2 * Fs, dtype=torch.bfloat16), torch.zeros(Fs, d, dtype=torch.bfloat16)
    layer._weights(gu, dn, sgu, sdn)
    with pytest.raises(ValueError, match=r"W_gate_up\[0\] has shape"):
        layer._weights([gu[0].t()] + gu[1:], dn, sgu, sdn)          # same address, transposed
    with pytest.raises(ValueError, match=r"W_down\[0\] has shape"):
        layer._weights(gu, [dn[0][: F // 2]] + dn[1:], sgu, sdn)      # same address, fewer rows
    with pytest.raises(ValueError, match=r"W_gate_up\[1\] has dtype"):
        layer._weights([gu[0], gu[1].view(torch.float16)] + gu[2:], dn, sgu, sdn)
    with pytest.raises(ValueError, match="Ws_down has shape"):
        layer._weights(gu, dn, sgu, sdn.view(d, Fs))                  # same bytes, reshaped
    # the original tensors are accepted again (and held by the layer)
    layer._weights(gu, dn, sgu, sdn)
    assert layer._wkeep[0] is gu[0]


def test_int4_weights_are_packed_two_per_byte(monkeypatch):
    """int4 layers take uint8 weights packed along the output columns:
    W_gate_up [d, F] bytes (2F codes), W_down [F, d / 2]."""
    from sparse_moe_transformer_router_b200 import binding
    monkeypatch.setattr(binding, "_where", lambda t, name, host=False: None)
    layer = _layer(dtype="int4")
    d, F, Fs, E = 64, 32, 48, 3
    gu = [torch.zeros(d, F, dtype=torch.uint8) for _ in range(E)]
    dn = [torch.zeros(F, d // 2, dtype=torch.uint8) for _ in range(E)]
    sgu, sdn = torch.zeros(d, Fs, dtype=torch.uint8), torch.zeros(Fs, d // 2, dtype=torch.uint8)
    layer._weights(gu, dn, sgu, sdn)
    with pytest.raises(ValueError, match=r"W_gate_up\[0\] has shape"):
        layer._weights([torch.zeros(d, 2 * F, dtype=torch.uint8)] + gu[1:], dn, sgu, sdn)  # unpacked
    with pytest.raises(ValueError, match=r"W_down\[2\] has dtype"):
        layer._weights(gu, dn[:2] + [dn[2].view(torch.int8)], sgu, sdn)
