"""Pins for the oracle's int32 accumulation and fp64 epilogue (CPU only).

acc[m,n] = sum_k w[n,k] q[m,k], each weight an add, a subtract or a skip
(baguaai "BitNet" tag page, C99 engine item); y = acc * w_scale * x_scale[m]
with the per-tensor weight scale (lemon-mlx-engine issue, "What We Need" 2).
The dense products below start from the unpacked int8 weights the generator
drew, never from anything the oracle unpacked.
"""
import numpy as np
import pytest

import oracle
from workloads import (activations_bf16, bf16_bits_to_float, make_projections,
                       ternary_weights)


def _dense_acc(w, q):
    return (q.astype(np.int64) @ w.astype(np.int64).T)


@pytest.mark.parametrize("N,K,M", [(4, 16, 1), (8, 32, 3), (60, 112, 2), (128, 256, 5)])
def test_brute_force_tiny(N, K, M):
    rng = np.random.default_rng(N + 31 * K + M)
    w = ternary_weights(rng, N, K)
    q = rng.integers(-127, 128, size=(M, K), dtype=np.int8)
    acc = oracle.gemv(oracle.pack(w), N, q)
    assert acc.dtype == np.int32
    assert (acc == _dense_acc(w, q)).all()


def test_brute_force_single_projection_full():
    (p,) = make_projections([("proj", 640, 2560)], M=1, seed=0)
    q, xs, xsum = oracle.quant(p.x_bf16)
    acc = oracle.gemv(oracle.pack(p.w), p.N, q)
    assert (acc == _dense_acc(p.w, q)).all()


def test_invariants():
    rng = np.random.default_rng(1)
    N, K, M = 64, 320, 4
    w = ternary_weights(rng, N, K)
    q = rng.integers(-127, 128, size=(M, K), dtype=np.int8)
    P = oracle.pack(w)
    acc = oracle.gemv(P, N, q).astype(np.int64)
    # all-zero weights give zero
    assert (oracle.gemv(oracle.pack(np.zeros_like(w)), N, q) == 0).all()
    # negating every weight (code c -> 2 - c) negates the accumulator
    assert (oracle.gemv(oracle.pack(-w), N, q) == -acc).all()
    # all +1 gives the row sums of q
    ones = oracle.gemv(oracle.pack(np.ones_like(w)), N, q)
    assert (ones == q.astype(np.int64).sum(axis=1, keepdims=True)).all()
    # acc = (sum of q under +1 weights) - (sum of q under -1 weights)
    qq = q.astype(np.int64)
    plus = np.stack([(qq * (w[n] == 1)).sum(axis=1) for n in range(N)], axis=1)
    minus = np.stack([(qq * (w[n] == -1)).sum(axis=1) for n in range(N)], axis=1)
    assert (acc == plus - minus).all()
    # linear in q
    q1 = rng.integers(-63, 64, size=(M, K), dtype=np.int8)
    q2 = rng.integers(-63, 64, size=(M, K), dtype=np.int8)
    s = oracle.gemv(P, N, (q1 + q2).astype(np.int8)).astype(np.int64)
    assert (s == oracle.gemv(P, N, q1).astype(np.int64) + oracle.gemv(P, N, q2)).all()


def test_row_ranges_and_threads_agree():
    rng = np.random.default_rng(2)
    N, K = 96, 208
    w = ternary_weights(rng, N, K)
    q = rng.integers(-127, 128, size=(3, K), dtype=np.int8)
    P = oracle.pack(w)
    full = oracle.gemv(P, N, q)
    assert (oracle.gemv(P, N, q, 17, 61) == full[:, 17:61]).all()
    assert (oracle.gemv_threads(P, N, q, threads=5) == full).all()


def test_epilogue_matches_dense_float64():
    rng = np.random.default_rng(4)
    N, K, M = 32, 96, 3
    w = ternary_weights(rng, N, K)
    xb = activations_bf16(rng, M, K)
    w_scale = np.float32(0.6171875)
    q, xs, xsum, acc, y = oracle.forward(oracle.pack(w), N, w_scale, xb)
    ref = (q.astype(np.float64) * xs[:, None].astype(np.float64)) @ \
          (np.float64(w_scale) * w.astype(np.float64)).T
    assert np.allclose(y, ref, rtol=1e-12, atol=0)


def test_all_plus_one_reduces_to_row_sum():
    # w = +1 everywhere and w_scale = 1: y is the sum of the dequantised
    # activations, so it equals sum_k x within K half-steps of the quantiser.
    rng = np.random.default_rng(6)
    N, K, M = 8, 2560, 4
    xb = activations_bf16(rng, M, K)
    x = bf16_bits_to_float(xb).astype(np.float64)
    q, xs, xsum, acc, y = oracle.forward(oracle.pack(np.ones((N, K), np.int8)), N, 1.0, xb)
    bound = K * 0.5 * xs.astype(np.float64) * (1 + 1e-4)
    assert np.all(np.abs(y - x.sum(axis=1, keepdims=True)) <= bound[:, None])
    assert (acc == xsum[:, None]).all()
