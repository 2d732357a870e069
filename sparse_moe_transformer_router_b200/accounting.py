"""FLOP and byte accounting for one MoE feed-forward layer (host logic).

Active FLOPs per token count 2 FLOP per multiply-add over the work the layer
does for that token: the router (d x E), the selected expert's SwiGLU (three
matmuls of d x F) and the shared expert's SwiGLU (three of d x Fs):
    2*d*E + 6*d*F + 6*d*Fs.
With the Maverick shapes this reproduces the modelled per-token costs printed
on llm-architectures-explained "Llama 4 Maverick" ("Modelled costs"), which
the test suite checks.

Algorithmic bytes count each touched weight byte once (experts that receive no
token are not read), the input read, the output write, and one write plus one
read of the gated expert-ordered input and of the two hidden activations.
With E = 0 (a dense feed-forward layer) only the shared SwiGLU counts.
"""
from __future__ import annotations

import numpy as np

ACT_BYTES = {"f32": 4, "bf16": 2, "fp8": 2, "int8": 2, "int4": 2}
W_BYTES = {"f32": 4, "bf16": 2, "fp8": 1, "int8": 1, "int4": 0.5}


def flops_per_token(d: int, E: int, F: int, Fs: int) -> int:
    return 2 * d * E + 6 * d * F + 6 * d * Fs


def layer_flops(T: int, d: int, E: int, F: int, Fs: int) -> int:
    return T * flops_per_token(d, E, F, Fs)


def layer_bytes(T: int, d: int, E: int, F: int, Fs: int, dtype: str, experts_touched: int) -> int:
    a, w = ACT_BYTES[dtype], W_BYTES[dtype]
    weights = (experts_touched * 3 * d * F + 3 * d * Fs) * w
    if dtype in ("fp8", "int8", "int4"):  # per-output-column fp32 scales
        weights += (experts_touched * (2 * F + d) + (2 * Fs + d)) * 4
    router = d * E * a
    acts = T * d * a * 2                 # x read, out write
    if E > 0:
        acts += T * d * a * 2            # gated expert-ordered input: write + read
    acts += T * (F + Fs) * a * 2         # hidden activations: write + read
    return int(weights + router + acts)


def experts_touched(counts) -> int:
    return int(np.count_nonzero(np.asarray(counts)))
