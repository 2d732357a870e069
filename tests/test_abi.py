"""The C-ABI library builds, loads without a GPU, exports every entry point
declared in include/l4moe.h, and rejects bad arguments on the host side
before touching a device."""
import ctypes
import os
import re

import pytest

from sparse_moe_transformer_router_b200 import build as build_mod
from sparse_moe_transformer_router_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "l4moe.h")).read()
    return re.findall(r"L4MOE_API[^;(]*?\b(l4moe_\w+)\s*\(", src)


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return binding.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 19
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(binding.EXPORTED)


def test_status_strings_and_version(lib):
    assert lib.l4moe_version() == 100
    assert lib.l4moe_status_string(0) == b"L4MOE_OK"
    assert lib.l4moe_status_string(6) == b"L4MOE_ERR_TIMEOUT"
    assert lib.l4moe_status_string(8) == b"L4MOE_ERR_RANGE"


def _create(lib, d, F, Fs, E, dtype):
    p = binding.Params(d, F, Fs, E, dtype)
    h = ctypes.c_void_p()
    st = lib.l4moe_create(ctypes.byref(p), ctypes.byref(h))
    return st, h


@pytest.mark.parametrize("args,status", [
    ((5120, 8192, 8192, 16, 7), binding.ERR_DTYPE),       # unknown dtype
    ((0, 8192, 8192, 16, 1), binding.ERR_ARG),            # d = 0
    ((5120, 8192, 8192, -1, 1), binding.ERR_ARG),         # E < 0
    ((5120, 0, 8192, 16, 1), binding.ERR_ARG),            # experts need F > 0
    ((5120, 8192, 0, 0, 1), binding.ERR_ARG),             # Fs = 0
    ((5120, 8192, 8192, 257, 1), binding.ERR_ARG),        # E > 256
    ((5100, 8192, 8192, 16, 1), binding.ERR_ALIGN),       # d not a multiple of 64
    ((5120, 8200, 8192, 16, 1), binding.ERR_ALIGN),       # F not a multiple of 64
])
def test_create_rejects_bad_params_without_a_device(lib, args, status):
    st, h = _create(lib, *args)
    assert st == status
    assert not h.value
    assert lib.l4moe_last_error(None)


def test_null_handle_calls_fail_cleanly(lib):
    assert lib.l4moe_forward(None, 1, None, None, None, None, None, None, None, None) == binding.ERR_ARG
    assert lib.l4moe_check_device_status(None, None) == binding.ERR_ARG
    assert lib.l4moe_workspace_size(None, 10) == 0
    assert lib.l4moe_launch_count(None) == 0
    lib.l4moe_destroy(None)


def test_valid_params_need_a_b200(lib):
    import torch
    st, h = _create(lib, 128, 256, 256, 4, 1)
    if torch.cuda.is_available():
        assert st in (binding.OK, binding.ERR_UNSUPPORTED)
        if st == binding.OK:
            lib.l4moe_destroy(h)
    else:
        assert st in (binding.ERR_CUDA, binding.ERR_UNSUPPORTED)


def test_binding_refuses_to_run_without_the_library(monkeypatch, tmp_path):
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(binding, "_lib", None)
    with pytest.raises(ImportError):
        binding.load_library()
