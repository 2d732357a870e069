"""CPU oracle for the top-1 sigmoid-gated MoE feed-forward layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference legs of ``bench.py`` may import this package.  The
product path (the CUDA library and its Python binding) never imports, links or
calls anything here, and this package imports nothing from the product.

The arithmetic lives in ``oracle.c`` (plain C, fp64 accumulation, OpenMP over
tokens); this module only compiles it with gcc and marshals numpy arrays.
Inputs are numpy arrays in their storage dtype: float32, bf16 as uint16 bit
patterns, E4M3 as uint8 codes, int8 weights as int8, int4 weights as packed
bytes viewed with ``INT4X2``.

Every function is pinned by ``tests/test_oracle_pins.py`` and
``tests/test_tolerance_floor.py`` to something other than itself (library
matmuls on reductions of the layer, closed forms, invariants, numpy's argmax /
stable argsort, torch's bf16 and float8 decoders and conversions).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

F32, BF16, E4M3, INT8, INT4 = 0, 1, 2, 3, 4

# int4 weights: a [K, N] matrix stored as [K, N / 2] bytes (two's-complement
# nibbles, the even column in the low nibble), viewed with this one-byte
# record dtype so that it is told apart from E4M3 codes.
INT4X2 = np.dtype([("int4x2", np.uint8)])


def as_int4x2(packed: np.ndarray) -> np.ndarray:
    """View packed int4 bytes (uint8 [K, N / 2]) as the oracle's int4 storage."""
    return np.ascontiguousarray(packed, dtype=np.uint8).view(INT4X2)

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, OpenMP, no fast-math)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
           "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            vp, i32, f32p = ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p
            lib.oracle_bf16_to_double.restype = ctypes.c_double
            lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
            lib.oracle_e4m3_to_double.restype = ctypes.c_double
            lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
            lib.oracle_route.restype = None
            lib.oracle_route.argtypes = [i32, i32, i32, vp, i32, vp, i32, f32p,
                                         vp, vp, vp]
            lib.oracle_permutation.restype = None
            lib.oracle_permutation.argtypes = [i32, i32, vp, vp, vp, vp]
            lib.oracle_forward.restype = ctypes.c_int
            lib.oracle_route_topk.restype = None
            lib.oracle_route_topk.argtypes = [i32, i32, i32, i32, vp, i32, vp, i32, f32p,
                                              vp, vp, vp]
            lib.oracle_forward.argtypes = [i32, i32, i32, i32, i32, i32,
                                           vp, i32, vp, i32, f32p,
                                           vp, vp, vp, vp, i32,
                                           vp, vp, vp, vp, i32,
                                           i32, vp, vp, vp, vp, i32, vp, vp]
            lib.oracle_expert_rows.restype = None
            lib.oracle_expert_rows.argtypes = [i32, i32, i32, vp, i32, vp, vp, vp, i32, vp, vp, vp]
            lib.oracle_round_hidden.restype = ctypes.c_double
            lib.oracle_round_hidden.argtypes = [ctypes.c_double, i32]
            lib.oracle_e4m3_encode.restype = ctypes.c_uint8
            lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
            lib.oracle_e4m3_row.restype = ctypes.c_float
            lib.oracle_e4m3_row.argtypes = [i32, vp, vp]
            lib.oracle_num_threads.restype = ctypes.c_int
            lib.oracle_num_threads.argtypes = []
            _lib = lib
    return _lib


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    if a.dtype == np.uint8:
        return E4M3
    if a.dtype == np.int8:
        return INT8
    if a.dtype == INT4X2:
        return INT4
    raise TypeError(f"oracle: unsupported storage dtype {a.dtype}")


def _ptr(a):
    return None if a is None else a.ctypes.data


def num_threads() -> int:
    """OpenMP threads the oracle runs on (OMP_NUM_THREADS or all cores)."""
    return int(_load().oracle_num_threads())


def bf16_to_f64(bits: int) -> float:
    return float(_load().oracle_bf16_to_double(int(bits)))


def e4m3_to_f64(code: int) -> float:
    return float(_load().oracle_e4m3_to_double(int(code)))


def e4m3_encode(v: float) -> int:
    """E4M3 code of an fp32 value (round to nearest even, saturating)."""
    return int(_load().oracle_e4m3_encode(float(np.float32(v))))


def e4m3_rows(v: np.ndarray):
    """The FP8 activation mode's quantisation of each row of v (fp32 values):
    (codes uint8 [rows, n], scales float32 [rows])."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    rows, n = v.shape
    codes = np.empty((rows, n), np.uint8)
    scales = np.empty(rows, np.float32)
    lib = _load()
    for i in range(rows):
        scales[i] = lib.oracle_e4m3_row(n, v[i].ctypes.data, codes[i].ctypes.data)
    return codes, scales


def route(x: np.ndarray, Wr: np.ndarray, bias: np.ndarray | None = None):
    """Router for all tokens: (idx int32[T], lmax f32[T], margin f32[T]).

    x is [T, d], Wr is [d, E] (router weight, ``x @ Wr`` orientation); the
    fp32 logits are the fp64 sums rounded once; the top-1 index takes the
    lowest index on ties; margin is the winning logit minus the runner-up.
    """
    x = np.ascontiguousarray(x)
    Wr = np.ascontiguousarray(Wr)
    T, d = x.shape
    d2, E = Wr.shape
    assert d == d2
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    idx = np.empty(T, np.int32)
    lmax = np.empty(T, np.float32)
    margin = np.empty(T, np.float32)
    _load().oracle_route(T, d, E, _ptr(x), _dtype_code(x), _ptr(Wr),
                         _dtype_code(Wr), _ptr(b), _ptr(idx), _ptr(lmax),
                         _ptr(margin))
    return idx, lmax, margin


def route_topk(x: np.ndarray, Wr: np.ndarray, k: int, bias: np.ndarray | None = None):
    """Top-k router for all tokens: (idx int32[T, k], logits f32[T, k],
    margin f32[T]): the k largest fp32 logits in descending order, ties to
    the lower index; margin is the k-th selected logit minus the largest one
    left out (+inf when k == E)."""
    x = np.ascontiguousarray(x)
    Wr = np.ascontiguousarray(Wr)
    T, d = x.shape
    d2, E = Wr.shape
    assert d == d2 and 1 <= k <= E
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    idx = np.empty((T, k), np.int32)
    lsel = np.empty((T, k), np.float32)
    margin = np.empty(T, np.float32)
    _load().oracle_route_topk(T, d, E, k, _ptr(x), _dtype_code(x), _ptr(Wr), _dtype_code(Wr),
                              _ptr(b), _ptr(idx), _ptr(lsel), _ptr(margin))
    return idx, lsel, margin


def permutation(idx: np.ndarray, E: int):
    """(counts[E], offsets[E+1], perm[T]) with perm the stable expert order."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T = idx.shape[0]
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(T, np.int32)
    _load().oracle_permutation(T, E, _ptr(idx), _ptr(counts), _ptr(offsets),
                               _ptr(perm))
    return counts, offsets, perm


def expert_rows(x_rows, gates, W_gate_up, W_down, *, s_gate_up=None, s_down=None):
    """One expert's SwiGLU on given rows: out[i] = SwiGLU(g[i] * x[i]) in
    fp64 ([n, d]), the routed part of the layer for each (token, expert)
    entry that expert receives."""
    x_rows = np.ascontiguousarray(x_rows)
    n, d = x_rows.shape
    g = np.ascontiguousarray(gates, dtype=np.float64)
    assert g.shape == (n,)
    Wgu = np.ascontiguousarray(W_gate_up)
    Wdn = np.ascontiguousarray(W_down)
    F = Wdn.shape[0]
    w_code = _dtype_code(Wgu)
    sgu = sdn = None
    if w_code in (E4M3, INT8, INT4):
        sgu = np.ascontiguousarray(s_gate_up, dtype=np.float32)
        sdn = np.ascontiguousarray(s_down, dtype=np.float32)
    out = np.zeros((n, d), np.float64)
    if n:
        _load().oracle_expert_rows(n, d, F, _ptr(x_rows), _dtype_code(x_rows), _ptr(g), _ptr(Wgu), _ptr(Wdn),
                                   w_code, _ptr(sgu), _ptr(sdn), _ptr(out))
    return out


HIDDEN_ROUND = {None: 0, "bf16": 1, "f16": 2}


def round_hidden(v: float, kind: str) -> float:
    """The oracle's rounding of one hidden value (fp64 -> fp32 -> bf16 or
    f16, nearest even)."""
    return float(_load().oracle_round_hidden(float(v), HIDDEN_ROUND[kind]))


def forward(x, Wr, W_gate_up, W_down, Ws_gate_up, Ws_down, *, bias=None,
            s_gate_up=None, s_down=None, ss_gate_up=None, ss_down=None,
            tokens=None, k=1, act_fp8=False, hidden_round=None, scale_margin=False):
    """Layer output in fp64 for ``tokens`` (all tokens when None).

    W_gate_up / W_down are length-E lists of [d, 2F] / [F, d] arrays; entries
    may be None for experts no selected token reaches (int4 weights: packed
    [d, F] / [F, d / 2] byte arrays viewed as ``INT4X2``).  For E4M3, int8 and
    int4 weights the per-output-column fp32 scales are required.  k > 1: each token runs its
    k highest-scoring experts, each on the input gated by the sigmoid of its
    own logit, and their outputs add to the shared expert's.  Returns
    (out f64[n_sel, d], idx int32[n_sel], gate f64[n_sel]), or [n_sel, k]
    index and gate arrays for k > 1.  act_fp8: the FP8 activation mode (every
    contraction input row quantised to E4M3 with its own fp32 scale, the
    row multiplied by the scale's reciprocal; a hidden
    row is first held in the layer's activation type, bf16 for bf16 inputs;
    the hidden-rounding output then equals the plain one).
    hidden_round ("bf16" or "f16"): also return, as a fourth element, the
    same outputs with every hidden value rounded to that type (through fp32)
    before the down projection -- the roundings a GPU that keeps the hidden
    rows in that type makes, with everything else exact.
    scale_margin (FP8 activation mode, bf16 activations): also return, last,
    each token's smallest distance (relative to the row's largest value) of a
    near-largest hidden value to a bf16 rounding midpoint over its hidden
    rows -- where an fp32 evaluation may give the row another scale.
    """
    x = np.ascontiguousarray(x)
    Wr = np.ascontiguousarray(Wr)
    T, d = x.shape
    E = Wr.shape[1]
    assert len(W_gate_up) == E and len(W_down) == E
    Ws_gate_up = np.ascontiguousarray(Ws_gate_up)
    Ws_down = np.ascontiguousarray(Ws_down)
    Fs = Ws_down.shape[0]
    F = None
    keep = []
    gu_ptrs = (ctypes.c_void_p * E)()
    dn_ptrs = (ctypes.c_void_p * E)()
    w_code = _dtype_code(Ws_gate_up)
    for e in range(E):
        if W_gate_up[e] is not None:
            a = np.ascontiguousarray(W_gate_up[e])
            b = np.ascontiguousarray(W_down[e])
            assert _dtype_code(a) == w_code and _dtype_code(b) == w_code
            F = b.shape[0]
            keep += [a, b]
            gu_ptrs[e] = a.ctypes.data
            dn_ptrs[e] = b.ctypes.data
    if F is None:
        F = Fs
    sgu_ptrs = sdn_ptrs = None
    if w_code in (E4M3, INT8, INT4):
        sgu_ptrs = (ctypes.c_void_p * E)()
        sdn_ptrs = (ctypes.c_void_p * E)()
        for e in range(E):
            if s_gate_up is not None and s_gate_up[e] is not None:
                a = np.ascontiguousarray(s_gate_up[e], dtype=np.float32)
                b = np.ascontiguousarray(s_down[e], dtype=np.float32)
                keep += [a, b]
                sgu_ptrs[e] = a.ctypes.data
                sdn_ptrs[e] = b.ctypes.data
        ss_gate_up = np.ascontiguousarray(ss_gate_up, dtype=np.float32)
        ss_down = np.ascontiguousarray(ss_down, dtype=np.float32)
    else:
        ss_gate_up = ss_down = None
    bias = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    if tokens is None:
        sel = None
        n_sel = T
    else:
        sel = np.ascontiguousarray(tokens, dtype=np.int32)
        n_sel = sel.shape[0]
    assert 1 <= k <= max(E, 1) and k <= 8
    out = np.zeros((n_sel, d), np.float64)
    sel_idx = np.empty(n_sel * k, np.int32)
    sel_gate = np.empty(n_sel * k, np.float64)
    out_h = np.zeros((n_sel, d), np.float64) if hidden_round else None
    margin = np.full(n_sel, np.inf) if scale_margin else None
    rc = _load().oracle_forward(
        T, d, E, k, F, Fs, _ptr(x), _dtype_code(x), _ptr(Wr), _dtype_code(Wr),
        _ptr(bias), ctypes.cast(gu_ptrs, ctypes.c_void_p),
        ctypes.cast(dn_ptrs, ctypes.c_void_p), _ptr(Ws_gate_up), _ptr(Ws_down),
        w_code,
        None if sgu_ptrs is None else ctypes.cast(sgu_ptrs, ctypes.c_void_p),
        None if sdn_ptrs is None else ctypes.cast(sdn_ptrs, ctypes.c_void_p),
        _ptr(ss_gate_up), _ptr(ss_down), 1 if act_fp8 else 0, n_sel, _ptr(sel), _ptr(out),
        _ptr(sel_idx), _ptr(sel_gate), HIDDEN_ROUND[hidden_round], _ptr(out_h), _ptr(margin))
    del keep
    if rc != 0:
        raise ValueError("oracle.forward: a selected token routes to an expert "
                         "whose weights were not supplied")
    if k > 1:
        sel_idx = sel_idx.reshape(n_sel, k)
        sel_gate = sel_gate.reshape(n_sel, k)
    res = (out, sel_idx, sel_gate) + ((out_h,) if hidden_round else ()) + ((margin,) if scale_margin else ())
    return res
