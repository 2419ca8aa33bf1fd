"""Seeded synthetic inputs for the ternary GEMV path.

This module is shared by the CUDA path's tests and bench and by the oracle's
tests. It draws random numbers and nothing else: it holds no packing, no
quantisation and no accumulation. Every input either side sees comes from here.

Input recipe (the same for every workload):

* ternary weights ``w`` int8 ``[N, K]``, i.i.d. over {-1, 0, +1} with
  probabilities 0.3 / 0.4 / 0.3 (a uniform draw over 0..9 mapped through a
  fixed 10-entry table);
* the stored per-tensor weight scale ``w_scale`` = mean |w| as fp32, i.e. the
  absmean scale a BitNet b1.58 checkpoint stores next to its packed weights
  (lemon-mlx-engine issue "Feature request: BitNet 1.58-bit ternary inference
  on ROCm", section "What We Need", item 2: the ``.weight_scale`` keys);
* activations ``x`` bf16 ``[M, K]``: N(0, 1) fp32, then in every row
  ``round(0.01 * K)`` distinct positions chosen uniformly without replacement
  are multiplied by 20 (outliers), then rounded to bf16 (round to nearest
  even). They are returned as raw bf16 bit patterns (uint16).

Seeds: numpy ``Generator(PCG64)`` from ``SeedSequence``. A workload with P
projections spawns two children of ``SeedSequence(seed)``: the first spawns
one stream per projection for the weights, the second one stream per
projection for the activations, in projection order (layer-major for a layer
stack).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

# BitNet-b1.58-2B-4T projection shapes (N x K), from the lemon-mlx-engine issue
# "Feature request: BitNet 1.58-bit ternary inference on ROCm (gfx1151)",
# section "Weight mapping (bitnet-b1.58-2B-4T)": hidden 2560, intermediate 6912.
DECODER_LAYER = (
    ("q_proj", 2560, 2560),
    ("k_proj", 640, 2560),
    ("v_proj", 640, 2560),
    ("o_proj", 2560, 2560),
    ("gate_proj", 6912, 2560),
    ("up_proj", 6912, 2560),
    ("down_proj", 2560, 6912),
)

STACK_LAYERS = 30
SMALL_M_VALUES = (1, 2, 4, 8, 16, 24)
SMALL_M_SHAPES = (("gate_proj", 6912, 2560), ("up_proj", 6912, 2560), ("down_proj", 2560, 6912))
PREFILL_M = 512
PREFILL_SHAPES = (("ffn_6912x2560", 6912, 2560), ("ffn_2560x6912", 2560, 6912),
                  ("ffn27b_17408x5120", 17408, 5120))

_TERNARY_TABLE = np.array([-1, -1, -1, 0, 0, 0, 0, 1, 1, 1], dtype=np.int8)


@dataclass
class Projection:
    """One synthetic projection: unpacked ternary weights and M activation rows."""
    name: str
    N: int
    K: int
    M: int
    w: np.ndarray          # int8 [N, K] in {-1, 0, 1}
    w_scale: np.float32    # stored absmean scale
    x_bf16: np.ndarray     # uint16 [M, K] bf16 bit patterns


def ternary_weights(rng: np.random.Generator, N: int, K: int) -> np.ndarray:
    """int8 [N, K], i.i.d. P(-1, 0, +1) = 0.3 / 0.4 / 0.3."""
    u = rng.integers(0, 10, size=(N, K), dtype=np.uint8)
    return _TERNARY_TABLE[u]


def stored_weight_scale(w: np.ndarray) -> np.float32:
    """The checkpoint's stored per-tensor scale: mean |w|, exact ratio then fp32."""
    nnz = int(np.count_nonzero(w))
    return np.float32(nnz / float(w.size)) if w.size else np.float32(0.0)


def activations_bf16(rng: np.random.Generator, M: int, K: int,
                     outlier_frac: float = 0.01, outlier_gain: float = 20.0) -> np.ndarray:
    """uint16 [M, K] bf16 bits: N(0,1) with round(outlier_frac*K) x20 outliers per row."""
    import torch  # bf16 rounding (round to nearest even) via torch's CPU cast

    x = rng.standard_normal((M, K), dtype=np.float32)
    n_out = int(round(outlier_frac * K))
    if n_out:
        for m in range(M):
            pos = rng.choice(K, size=n_out, replace=False)
            x[m, pos] *= np.float32(outlier_gain)
    t = torch.from_numpy(x).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_float(xb: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (xb.astype(np.uint32) << 16).view(np.float32)


def make_projections(shapes, M: int, seed: int = 0, with_weights: bool = True):
    """Yield Projection objects for ``shapes`` (sequence of (name, N, K)).

    Weights and activations of projection j come from their own spawned streams,
    so a projection can be regenerated without drawing the ones before it.
    """
    shapes = list(shapes)
    root = np.random.SeedSequence(seed)
    w_root, x_root = root.spawn(2)
    w_seqs = w_root.spawn(len(shapes))
    x_seqs = x_root.spawn(len(shapes))
    for j, (name, N, K) in enumerate(shapes):
        w = None
        ws = np.float32(0.0)
        if with_weights:
            w = ternary_weights(np.random.Generator(np.random.PCG64(w_seqs[j])), N, K)
            ws = stored_weight_scale(w)
        x = activations_bf16(np.random.Generator(np.random.PCG64(x_seqs[j])), M, K)
        yield Projection(name, N, K, M, w, ws, x)


def stack_shapes(layers: int = STACK_LAYERS):
    """The decode layer stack: ``layers`` copies of the seven decoder projections."""
    return [(f"L{l}.{name}", N, K) for l in range(layers) for (name, N, K) in DECODER_LAYER]


# ------------------------------------------------------------ binary g128
# Binary weights (baguaai "BitNet" tag page, Bonsai 27B item: 1 bit per weight,
# one fp16 scale per 128 weights). The shapes are the 27B-scale FFN of the
# prefill configuration: gate/up [17408 x 5120], down [5120 x 17408].
BINARY_GROUP = 128
BINARY_FFN27B = (("gate_proj", 17408, 5120), ("up_proj", 17408, 5120),
                 ("down_proj", 5120, 17408))
BINARY_LAYERS = 8
# fp16 group scales are drawn uniformly from this range: the size of mean|W|
# over 128 latent weights of N(0, 0.02^2) (0.02 * sqrt(2 / pi) = 0.016); the
# page gives no distribution.
BINARY_SCALE_RANGE = (0.012, 0.020)


@dataclass
class BinaryProjection:
    """One synthetic binary g128 projection and M activation rows."""
    name: str
    N: int
    K: int
    M: int
    w: np.ndarray          # int8 [N, K] in {-1, +1}
    s_f16: np.ndarray      # uint16 [N, K/128] fp16 bit patterns (group scales)
    x_bf16: np.ndarray     # uint16 [M, K] bf16 bit patterns


def binary_weights(rng: np.random.Generator, N: int, K: int) -> np.ndarray:
    """int8 [N, K], i.i.d. -1 / +1 with probability 1/2 each."""
    return (rng.integers(0, 2, size=(N, K), dtype=np.int8) * 2 - 1).astype(np.int8)


def group_scales_f16(rng: np.random.Generator, N: int, K: int) -> np.ndarray:
    """uint16 [N, K/128] fp16 bit patterns, uniform on BINARY_SCALE_RANGE."""
    lo, hi = BINARY_SCALE_RANGE
    s = rng.uniform(lo, hi, size=(N, K // BINARY_GROUP)).astype(np.float16)
    return s.view(np.uint16)


def make_binary_projections(shapes, M: int, seed: int = 0):
    """Yield BinaryProjection objects for ``shapes`` (sequence of (name, N, K)).
    Spawned streams as in ``make_projections``: weights (and then scales) of
    projection j from the first child's stream j, activations from the
    second's."""
    shapes = list(shapes)
    root = np.random.SeedSequence(seed)
    w_root, x_root = root.spawn(2)
    w_seqs = w_root.spawn(len(shapes))
    x_seqs = x_root.spawn(len(shapes))
    for j, (name, N, K) in enumerate(shapes):
        rng = np.random.Generator(np.random.PCG64(w_seqs[j]))
        w = binary_weights(rng, N, K)
        s = group_scales_f16(rng, N, K)
        x = activations_bf16(np.random.Generator(np.random.PCG64(x_seqs[j])), M, K)
        yield BinaryProjection(name, N, K, M, w, s, x)


def binary_stack_shapes(layers: int = BINARY_LAYERS):
    """``layers`` copies of the 27B-scale FFN projections (binary weights)."""
    return [(f"L{l}.{name}", N, K) for l in range(layers) for (name, N, K) in BINARY_FFN27B]


def binary_bytes(N: int, K: int, M: int) -> int:
    """Bytes one binary GEMV must move: bits (N*K/8) + fp16 scales (N*K/128*2)
    + int8 activations + fp32 output + per-row scale (4 B)."""
    return N * K // 8 + N * (K // BINARY_GROUP) * 2 + M * K + M * N * 4 + M * 4


# Hadamard route: block size of the rotation. 256 is the largest power of two
# dividing every K of the prefill shapes (2560 = 10 x 256, 6912 = 27 x 256,
# 5120 = 20 x 256), and 1/sqrt(256) = 1/16 is exact.
HADAMARD_BLOCK = 256

# Named workloads. Each maps to (shapes, M).
WORKLOADS = {
    "single_640x2560_m1": ([("proj", 640, 2560)], 1),
    "layer_m1": (list(DECODER_LAYER), 1),
    "stack30_m1": (stack_shapes(STACK_LAYERS), 1),
    # a 10-layer stack (175 MB of weights, still larger than L2): the small case
    # for profiler captures of the stack kernel
    "stack10_m1": (stack_shapes(10), 1),
    # the same stack with several tokens per projection (small-batch decode)
    "stack30_m2": (stack_shapes(STACK_LAYERS), 2),
    "stack30_m4": (stack_shapes(STACK_LAYERS), 4),
    "stack30_m8": (stack_shapes(STACK_LAYERS), 8),
    "stack30_m16": (stack_shapes(STACK_LAYERS), 16),
    "stack30_m24": (stack_shapes(STACK_LAYERS), 24),
}
for _m in SMALL_M_VALUES:
    WORKLOADS[f"ffn_m{_m}"] = (list(SMALL_M_SHAPES), _m)
WORKLOADS["prefill_m512"] = (list(PREFILL_SHAPES), PREFILL_M)

# Workloads of the other two paths, (shapes, M): the prefill contraction with
# Hadamard-rotated 4-bit activations, and binary g128 weights (8 layers of the
# 27B-scale FFN, 302 MB of bits and scales per pass).
NEXT_WORKLOADS = {
    "prefill_had4_m512": (list(PREFILL_SHAPES), PREFILL_M),
    "binary_ffn27b_m1": (binary_stack_shapes(BINARY_LAYERS), 1),
}


def algorithmic_bytes(N: int, K: int, M: int) -> int:
    """Bytes one GEMV must move: packed weights + int8 activations + fp32 output
    + per-row scale and sum (8 B) + the weight scale (4 B)."""
    return N * K // 4 + M * K + M * N * 4 + M * 8 + 4
