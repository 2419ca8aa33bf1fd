"""GPU parity of the decode GEMV (tq_gemv) against the oracle.

Covers the single 640x2560 projection, one full decoder layer's seven
projections, the batched-decode FFN shapes at every M of that workload, and
edge cases: tiny and ragged shapes (packed row counts that leave partial
tiles), the K limit, all-zero / all-one weights, zero activation rows,
repeat-run byte identity. From 25 tokens the single-projection path is the
tensor-core kernel's cluster plan (through tq_gemm_prefill).
"""
import numpy as np
import pytest
import torch

import ternary_absmax_int8_b200 as tq
from tests._gpu import (assert_parity, gpu_forward, host_pack, oracle_forward)
from workloads import (DECODER_LAYER, SMALL_M_SHAPES, SMALL_M_VALUES, activations_bf16,
                       make_projections, stored_weight_scale, ternary_weights)

pytestmark = pytest.mark.gpu


def _run(p):
    P = host_pack(p.w)
    gpu = gpu_forward(P, p.N, p.w_scale, p.x_bf16)
    ref = oracle_forward(p.w, p.w_scale, p.x_bf16)
    assert_parity(gpu, ref, p.name)


def test_single_projection_640x2560(cuda_device):
    for p in make_projections([("proj", 640, 2560)], M=1, seed=0):
        _run(p)


def test_decoder_layer_m1(cuda_device):
    for p in make_projections(DECODER_LAYER, M=1, seed=0):
        _run(p)


@pytest.mark.parametrize("M", SMALL_M_VALUES)
def test_batched_decode(cuda_device, M):
    for p in make_projections(SMALL_M_SHAPES, M=M, seed=1000 + M):
        _run(p)


@pytest.mark.parametrize("N,K,M", [(4, 16, 1), (8, 32, 2), (12, 48, 3), (60, 112, 4),
                                   (6916, 2560, 1), (2564, 6928, 5), (100, 32768, 1),
                                   (36, 32768, 4), (1024, 16, 24), (400, 4096, 13),
                                   (520, 2560, 20), (2564, 6928, 28), (1024, 16, 32)])
def test_edge_shapes(cuda_device, N, K, M):
    rng = np.random.default_rng(N * 7 + K * 3 + M)
    w = ternary_weights(rng, N, K)
    xb = activations_bf16(rng, M, K)
    P = host_pack(w)
    ws = stored_weight_scale(w)
    assert_parity(gpu_forward(P, N, ws, xb), oracle_forward(w, ws, xb), f"{N}x{K} M={M}")


def test_degenerate_values(cuda_device):
    N, K, M = 256, 512, 3
    rng = np.random.default_rng(9)
    xb = activations_bf16(rng, M, K)
    xb[1, :] = 0  # an all-zero token row
    for w in (np.zeros((N, K), np.int8), np.ones((N, K), np.int8), -np.ones((N, K), np.int8)):
        assert_parity(gpu_forward(host_pack(w), N, 1.0, xb), oracle_forward(w, 1.0, xb))


def test_k_zero_and_empty(cuda_device):
    y = torch.full((2, 8), 7.0, device="cuda")
    acc = torch.full((2, 8), 7, dtype=torch.int32, device="cuda")
    xs = torch.zeros(2, device="cuda")
    xsum = torch.zeros(2, dtype=torch.int32, device="cuda")
    P = torch.zeros(16, dtype=torch.uint8, device="cuda")
    xq = torch.zeros(16, dtype=torch.int8, device="cuda")
    tq.tq_gemv(P, 1.0, xq, xs, xsum, y, acc, 2, 8, 0)
    torch.cuda.synchronize()
    assert (y == 0).all() and (acc == 0).all()
    tq.tq_gemv(P, 1.0, xq, xs, xsum, y, acc, 0, 8, 16)  # M = 0: untouched
    torch.cuda.synchronize()
    assert (y == 0).all()


def test_repeat_runs_identical(cuda_device):
    (p,) = make_projections([("gate", 6912, 2560)], M=4, seed=5)
    P = host_pack(p.w)
    a = gpu_forward(P, p.N, p.w_scale, p.x_bf16)
    b = gpu_forward(P, p.N, p.w_scale, p.x_bf16)
    for u, v in zip(a, b):
        assert u.tobytes() == v.tobytes()
    assert tq.tq_device_error(reset=True) == 0
