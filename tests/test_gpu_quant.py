"""The FP8 activation mode's row quantisation on the GPU (the hidden-row
kernel of csrc/quant.cuh, built into tests/device/quant_rows.cu) against the
oracle's (oracle.e4m3_rows): codes and row scales bit-exact.  Both sides
take the same fp32 steps (max, scale = max / 448 floored at 2^-126, its
reciprocal, one product per value, round to nearest even), so the rows
cover what could still tell them apart: exact ties between two codes,
values in E4M3's subnormal range, rows whose scale takes the floor, a zero
row, rows wider than the kernel's registers hold, and millions of random
values over a wide range of magnitudes."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
NVCC = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"


def _bf16(v: np.ndarray) -> np.ndarray:
    """fp32 values (already bf16-representable) -> bf16 bit patterns."""
    u = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32)
    assert np.all(u & 0xFFFF == 0), "value not exact in bf16"
    return (u >> 16).astype(np.uint16)


def _round_bf16(v: np.ndarray) -> np.ndarray:
    """fp32 -> nearest bf16 value (ties to even), as fp32."""
    u = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def _midpoints() -> np.ndarray:
    """The midpoints between adjacent positive E4M3 values (0 .. 448)."""
    vals = np.array([oracle.e4m3_to_f64(c) for c in range(0x00, 0x7F)], np.float64)
    return ((vals[:-1] + vals[1:]) / 2).astype(np.float32)


def _cases(width: int, rng) -> np.ndarray:
    rows = []
    # random rows over a wide range of magnitudes
    for _ in range(400):
        rows.append(rng.standard_normal(width) * np.exp2(rng.uniform(-40, 40)))
    # exact ties: the row maximum is 448 * 2^k, so the scale is 2^k and every
    # midpoint times 2^k scales back to the midpoint exactly
    mids = _midpoints()
    for k in (-20, -3, 0, 5, 30):
        r = rng.choice(np.concatenate([mids, -mids]), size=width) * np.float32(2.0 ** k)
        r[0] = 448.0 * 2.0 ** k
        rows.append(r)
    # one large value, the rest in E4M3's subnormal range and below
    for _ in range(20):
        r = rng.standard_normal(width) * np.exp2(rng.uniform(-20, -8, size=width))
        r[rng.integers(width)] = 448.0
        rows.append(r)
    # scales at the 2^-126 floor (max below 448 * 2^-126)
    rows.append(rng.standard_normal(width) * 1e-37)
    rows.append(rng.standard_normal(width) * 1e-39)
    # zero row, one nonzero element
    rows.append(np.zeros(width))
    z = np.zeros(width)
    z[width // 2] = -3.0
    rows.append(z)
    v = _round_bf16(np.array(rows, dtype=np.float64).astype(np.float32))
    return v


@pytest.fixture(scope="module")
def quant_rows_exe(tmp_path_factory):
    exe = tmp_path_factory.mktemp("qr") / "quant_rows"
    subprocess.run([NVCC, "-std=c++17", "-O2", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-I", os.path.join(ROOT, "sparse_moe_transformer_router_b200", "csrc"),
                    os.path.join(ROOT, "tests", "device", "quant_rows.cu"), "-o", str(exe)],
                   check=True, capture_output=True, timeout=600)
    return exe


@pytest.mark.parametrize("width", [8192, 72, 16448])
def test_gpu_row_quantisation_matches_the_oracle_bit_for_bit(quant_rows_exe, tmp_path, width):
    rng = np.random.default_rng(width)
    v = _cases(width, rng)
    src, dst = tmp_path / "in.bin", tmp_path / "out.bin"
    with open(src, "wb") as f:
        np.array([v.shape[0], width], np.int32).tofile(f)
        _bf16(v).tofile(f)
    r = subprocess.run([str(quant_rows_exe), str(src), str(dst)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    raw = np.fromfile(dst, np.uint8)
    n = v.size
    codes = raw[:n].reshape(v.shape)
    scales = raw[n:].view(np.float32)
    want_codes, want_scales = oracle.e4m3_rows(v)
    assert np.array_equal(scales.view(np.uint32), want_scales.view(np.uint32))
    bad = np.argwhere(codes != want_codes)
    assert bad.size == 0, f"{len(bad)} codes differ, e.g. row/col {bad[:5].tolist()}"
    print(f"width {width}: {n} codes, {v.shape[0]} rows identical")
