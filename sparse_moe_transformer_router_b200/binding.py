"""Thin ctypes binding over libl4moe.so (include/l4moe.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  torch is used for device memory and streams.  There is no fallback:
if the compiled library is missing or the call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libl4moe.so")

OK, ERR_ARG, ERR_DTYPE, ERR_ALIGN, ERR_CUDA, ERR_WORKSPACE, ERR_TIMEOUT, ERR_UNSUPPORTED, ERR_RANGE = range(9)
DTYPES = {"f32": 0, "bf16": 1, "fp8": 2, "int8": 3, "int4": 4}
EXPORTED = ("l4moe_create", "l4moe_destroy", "l4moe_workspace_size", "l4moe_set_workspace",
            "l4moe_set_router_bias", "l4moe_set_fp8_scales", "l4moe_forward",
            "l4moe_forward_host", "l4moe_get_routing", "l4moe_check_device_status",
            "l4moe_launch_count", "l4moe_last_error", "l4moe_status_string", "l4moe_version",
            "l4moe_set_timing", "l4moe_read_timing", "l4moe_kernel_name",
            "l4moe_forward_static", "l4moe_join_host", "l4moe_set_top_k",
            "l4moe_set_weight_scales", "l4moe_selftest_wait", "l4moe_set_act_fp8", "l4moe_get_plan")
STATIC_WORKSPACE_BYTES = 32 << 20
NUM_KERNELS = 6

_lib = None


class L4MoEError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{message} (status {status})")
        self.status = status


class Plan(ctypes.Structure):
    _fields_ = [("split_gate_up", ctypes.c_int), ("split_down", ctypes.c_int),
                ("small_routing", ctypes.c_int), ("early_shared", ctypes.c_int),
                ("fused", ctypes.c_int), ("small_tiles", ctypes.c_int)]


class Params(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int), ("expert_ffn", ctypes.c_int),
                ("shared_ffn", ctypes.c_int), ("num_experts", ctypes.c_int),
                ("dtype", ctypes.c_int)]


def load_library():
    """Load libl4moe.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m sparse_moe_transformer_router_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    pvp = ctypes.POINTER(ctypes.c_void_p)
    lib.l4moe_create.argtypes = [ctypes.POINTER(Params), ctypes.POINTER(vp)]
    lib.l4moe_destroy.argtypes = [vp]
    lib.l4moe_destroy.restype = None
    lib.l4moe_workspace_size.argtypes = [vp, i32]
    lib.l4moe_workspace_size.restype = sz
    lib.l4moe_set_workspace.argtypes = [vp, vp, sz, i32]
    lib.l4moe_set_router_bias.argtypes = [vp, vp]
    lib.l4moe_set_fp8_scales.argtypes = [vp, pvp, pvp, vp, vp]
    lib.l4moe_set_weight_scales.argtypes = [vp, pvp, pvp, vp, vp]
    fwd = [vp, i32, vp, vp, pvp, pvp, vp, vp, vp, vp]
    lib.l4moe_forward.argtypes = fwd
    lib.l4moe_forward_host.argtypes = fwd
    lib.l4moe_forward_static.argtypes = fwd
    lib.l4moe_join_host.argtypes = [vp, vp]
    lib.l4moe_get_routing.argtypes = [vp] + [pvp] * 7
    lib.l4moe_check_device_status.argtypes = [vp, vp]
    lib.l4moe_launch_count.argtypes = [vp]
    lib.l4moe_launch_count.restype = ctypes.c_uint64
    lib.l4moe_last_error.argtypes = [vp]
    lib.l4moe_last_error.restype = ctypes.c_char_p
    lib.l4moe_status_string.argtypes = [i32]
    lib.l4moe_status_string.restype = ctypes.c_char_p
    lib.l4moe_version.argtypes = []
    lib.l4moe_set_timing.argtypes = [vp, i32]
    lib.l4moe_set_top_k.argtypes = [vp, i32]
    lib.l4moe_set_act_fp8.argtypes = [vp, i32]
    lib.l4moe_get_plan.argtypes = [vp, ctypes.POINTER(Plan)]
    lib.l4moe_selftest_wait.argtypes = [vp, ctypes.c_double, vp]
    lib.l4moe_read_timing.argtypes = [vp, ctypes.POINTER(ctypes.c_double),
                                      ctypes.POINTER(ctypes.c_uint64)]
    lib.l4moe_kernel_name.argtypes = [i32]
    lib.l4moe_kernel_name.restype = ctypes.c_char_p
    for name in ("l4moe_create", "l4moe_set_workspace", "l4moe_set_router_bias",
                 "l4moe_set_fp8_scales", "l4moe_forward", "l4moe_forward_host",
                 "l4moe_get_routing", "l4moe_check_device_status", "l4moe_version",
                 "l4moe_set_timing", "l4moe_read_timing", "l4moe_forward_static",
                 "l4moe_join_host", "l4moe_set_top_k", "l4moe_set_weight_scales", "l4moe_selftest_wait",
                 "l4moe_set_act_fp8", "l4moe_get_plan"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("l4moe: tensors must be contiguous (row-major)")
    return t.data_ptr()


def _ptr_array(tensors):
    arr = (ctypes.c_void_p * len(tensors))()
    for i, t in enumerate(tensors):
        arr[i] = _ptr(t)
    return arr


def _stream_handle(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


_ACT_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16, "fp8": torch.bfloat16, "int8": torch.bfloat16,
              "int4": torch.bfloat16}
# int4 weights are packed two per byte along the output columns
_W_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16, "fp8": torch.float8_e4m3fn, "int8": torch.int8,
            "int4": torch.uint8}


def _expect(t, name, shape, dtype):
    """Shape / dtype check of one argument (the C ABI sees raw pointers, so a
    wrong shape would make the kernels read past a buffer)."""
    if t is None:
        raise ValueError(f"l4moe: {name} is required")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"l4moe: {name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise ValueError(f"l4moe: {name} has dtype {t.dtype}, expected {dtype}")


def _where(t, name, host=False):
    """Device check of one argument (after every shape and dtype check)."""
    if host == t.is_cuda:
        raise ValueError(f"l4moe: {name} must be a {'host' if host else 'CUDA'} tensor")


class _DevView:
    """Zero-copy torch view of a device buffer (CUDA array interface)."""

    def __init__(self, ptr, shape, typestr):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (int(ptr), False), "version": 3, "strides": None}


class L4MoE:
    """One MoE feed-forward layer (d_model, expert_ffn, shared_ffn, num_experts, dtype)."""

    def __init__(self, d_model: int, expert_ffn: int, shared_ffn: int, num_experts: int,
                 dtype: str = "bf16"):
        self._lib = load_library()
        self.params = Params(d_model, expert_ffn, shared_ffn, num_experts, DTYPES[dtype])
        self.d_model, self.expert_ffn, self.shared_ffn = d_model, expert_ffn, shared_ffn
        self.num_experts, self.dtype = num_experts, dtype
        h = ctypes.c_void_p()
        st = self._lib.l4moe_create(ctypes.byref(self.params), ctypes.byref(h))
        if st != OK:
            raise L4MoEError(st, self._lib.l4moe_last_error(None).decode())
        self._h = h
        self._keep = []
        self.last_T = 0
        # the handle belongs to the device current at creation (as in the C ABI)
        self.device = torch.device("cuda", torch.cuda.current_device()) if torch.cuda.is_available() else None

    def close(self):
        if getattr(self, "_h", None):
            self._lib.l4moe_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check(self, st: int):
        if st != OK:
            raise L4MoEError(st, self._lib.l4moe_last_error(self._h).decode())

    def workspace_size(self, max_tokens: int) -> int:
        return int(self._lib.l4moe_workspace_size(self._h, max_tokens))

    def set_workspace(self, buf: torch.Tensor, max_tokens: int):
        self._check(self._lib.l4moe_set_workspace(self._h, _ptr(buf), buf.numel() * buf.element_size(),
                                                  max_tokens))
        self._keep.append(buf)

    def set_router_bias(self, bias: torch.Tensor | None):
        self._check(self._lib.l4moe_set_router_bias(self._h, _ptr(bias)))
        self._bias = bias

    def set_weight_scales(self, s_gate_up, s_down, ss_gate_up, ss_down):
        """Per-output-column fp32 scales of E4M3, int8 or int4 weights (device tensors)."""
        a, b = _ptr_array(s_gate_up), _ptr_array(s_down)
        self._check(self._lib.l4moe_set_weight_scales(self._h, a, b, _ptr(ss_gate_up), _ptr(ss_down)))
        self._scales = (list(s_gate_up), list(s_down), ss_gate_up, ss_down)

    set_fp8_scales = set_weight_scales

    def _weights(self, W_gate_up, W_down, Ws_gate_up, Ws_down):
        """Pointer arrays of the expert weights; shapes, dtypes, devices and
        contiguity are checked whenever the weight tensors change.  The key is
        each tensor's identity and address: a view of a checked weight (a
        transpose, a slice, a reinterpreting .view) is another tensor object,
        so it is checked again even at the same address, and the checked
        tensors are held (self._wkeep) so that their identities cannot be
        reused by new tensors while the key stands.  (The per-call cost with
        128 experts is ~20 us of Python, against ~60 us when every call
        re-checked every tensor.)"""
        try:
            ws = list(W_gate_up) + list(W_down) + [Ws_gate_up, Ws_down]
            key = (tuple(id(w) for w in ws), tuple(w.data_ptr() for w in ws))
        except AttributeError:  # a missing weight: the checks below name it
            key = None
        if key is None or getattr(self, "_wkey", None) != key:
            d, F, Fs, E = self.d_model, self.expert_ffn, self.shared_ffn, self.num_experts
            wdt = _W_DTYPE[self.dtype]
            if len(W_gate_up) != E or len(W_down) != E:
                raise ValueError(f"l4moe: expected {E} expert weights, got {len(W_gate_up)} / {len(W_down)}")
            cols = (lambda n: n // 2) if self.dtype == "int4" else (lambda n: n)  # noqa: E731 (packed bytes)
            named = [(W_gate_up[e], f"W_gate_up[{e}]", (d, cols(2 * F))) for e in range(E)]
            named += [(W_down[e], f"W_down[{e}]", (F, cols(d))) for e in range(E)]
            named += [(Ws_gate_up, "Ws_gate_up", (d, cols(2 * Fs))), (Ws_down, "Ws_down", (Fs, cols(d)))]
            for t, name, shape in named:
                _expect(t, name, shape, wdt)
            for t, name, _ in named:
                _where(t, name)
            self._wkey = None
            self._warr = (_ptr_array(W_gate_up), _ptr_array(W_down))
            self._wkeep = ws
            self._wkey = key
        return self._warr

    def _check_io(self, x, W_router, out, host=False):
        if x.dim() != 2:
            raise ValueError(f"l4moe: x must be [T, d_model], got shape {tuple(x.shape)}")
        T = x.shape[0]
        act = _ACT_DTYPE[self.dtype]
        _expect(x, "x", (T, self.d_model), act)
        if self.num_experts > 0:
            _expect(W_router, "W_router", (self.d_model, self.num_experts), act)
        if out is not None:
            _expect(out, "out", (T, self.d_model), act)
        _where(x, "x", host)
        if self.num_experts > 0:
            _where(W_router, "W_router")
        if out is not None:
            _where(out, "out", host)
        return T

    def forward(self, x, W_router, W_gate_up, W_down, Ws_gate_up, Ws_down, out=None, stream=None):
        T = self._check_io(x, W_router, out)
        if out is None:
            out = torch.empty((T, self.d_model), dtype=x.dtype, device=x.device)
        gu, dn = self._weights(W_gate_up, W_down, Ws_gate_up, Ws_down)
        self._check(self._lib.l4moe_forward(self._h, T, _ptr(x), _ptr(W_router), gu, dn,
                                            _ptr(Ws_gate_up), _ptr(Ws_down), _ptr(out),
                                            _stream_handle(stream)))
        self.last_T = T
        return out

    def forward_static(self, x, W_router, W_gate_up, W_down, Ws_gate_up, Ws_down, out, stream=None):
        """l4moe_forward_static: the same layer with the library's fixed device
        scratch array instead of an allocated workspace (no device allocation
        in the call; `out` must be supplied)."""
        T = self._check_io(x, W_router, out)
        if out is None:
            raise ValueError("l4moe: forward_static needs `out`")
        gu, dn = self._weights(W_gate_up, W_down, Ws_gate_up, Ws_down)
        self._check(self._lib.l4moe_forward_static(self._h, T, _ptr(x), _ptr(W_router), gu, dn,
                                                   _ptr(Ws_gate_up), _ptr(Ws_down), _ptr(out),
                                                   _stream_handle(stream)))
        return out

    def forward_host(self, x_host, W_router, W_gate_up, W_down, Ws_gate_up, Ws_down, out_host,
                     stream=None):
        T = self._check_io(x_host, W_router, out_host, host=True)
        if out_host is None:
            raise ValueError("l4moe: forward_host needs `out_host`")
        gu, dn = self._weights(W_gate_up, W_down, Ws_gate_up, Ws_down)
        self._check(self._lib.l4moe_forward_host(self._h, T, _ptr(x_host), _ptr(W_router), gu, dn,
                                                 _ptr(Ws_gate_up), _ptr(Ws_down), _ptr(out_host),
                                                 _stream_handle(stream)))
        self.last_T = T
        return out_host

    def join_host(self, stream=None):
        """Make `stream` wait for the output copies of all forward_host calls."""
        self._check(self._lib.l4moe_join_host(self._h, _stream_handle(stream)))

    def set_top_k(self, k: int):
        """Experts per token (l4moe_set_top_k)."""
        self._check(self._lib.l4moe_set_top_k(self._h, int(k)))
        self.top_k = int(k)

    def plan(self) -> dict:
        """How the last forward was launched (l4moe_get_plan)."""
        p = Plan()
        self._check(self._lib.l4moe_get_plan(self._h, ctypes.byref(p)))
        return {name: int(getattr(p, name)) for name, _ in Plan._fields_}

    def set_act_fp8(self, on: bool = True):
        """FP8 activation mode (l4moe_set_act_fp8): E4M3 token and hidden rows."""
        self._check(self._lib.l4moe_set_act_fp8(self._h, 1 if on else 0))
        self.act_fp8 = bool(on)

    def routing(self):
        """Zero-copy device views of the last forward's routing (valid until
        the next forward on this handle); with top_k = k > 1, idx / gate /
        lmax / perm hold T * k entries (entry t * k + j: token t's j-th)."""
        ptrs = [ctypes.c_void_p() for _ in range(7)]
        self._check(self._lib.l4moe_get_routing(self._h, *[ctypes.byref(p) for p in ptrs]))
        T, E = self.last_T, self.num_experts
        Tv = T * getattr(self, "top_k", 1)
        spec = [("idx", (Tv,), "<i4"), ("gate", (Tv,), "<f4"), ("lmax", (Tv,), "<f4"),
                ("margin", (T,), "<f4"), ("counts", (E,), "<i4"), ("offsets", (E + 1,), "<i4"),
                ("perm", (Tv,), "<i4")]
        out = {}
        for (name, shape, ts), p in zip(spec, ptrs):
            out[name] = torch.as_tensor(_DevView(p.value, shape, ts), device=self.device)
        return out

    def selftest_wait(self, limit_ms: float = 5.0, stream=None):
        """l4moe_selftest_wait: a device wait that runs out after limit_ms; the
        next check_device_status raises with ERR_TIMEOUT."""
        self._check(self._lib.l4moe_selftest_wait(self._h, float(limit_ms), _stream_handle(stream)))

    def check_device_status(self, stream=None):
        self._check(self._lib.l4moe_check_device_status(self._h, _stream_handle(stream)))

    def set_timing(self, kernels=True):
        """Time every kernel (True), none (False), or the named kernels."""
        if kernels is True:
            mask = (1 << NUM_KERNELS) - 1
        elif kernels is False or kernels is None:
            mask = 0
        else:
            names = [self._lib.l4moe_kernel_name(i).decode() for i in range(NUM_KERNELS)]
            mask = sum(1 << names.index(k) for k in kernels)
        self._check(self._lib.l4moe_set_timing(self._h, mask))

    def read_timing(self) -> dict:
        """{kernel name: (total ms, launches)} recorded since the last read."""
        ms = (ctypes.c_double * NUM_KERNELS)()
        n = (ctypes.c_uint64 * NUM_KERNELS)()
        self._check(self._lib.l4moe_read_timing(self._h, ms, n))
        return {self._lib.l4moe_kernel_name(i).decode(): (ms[i], int(n[i]))
                for i in range(NUM_KERNELS)}

    @property
    def launch_count(self) -> int:
        return int(self._lib.l4moe_launch_count(self._h))
