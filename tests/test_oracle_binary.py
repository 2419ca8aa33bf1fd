"""Pins of the oracle's binary g128 path (baguaai "BitNet" tag page, Bonsai
27B item: 1-bit binary weights, 128 weights sharing one fp16 scale, about
1.125 bits per weight).

The fp16 decoder is pinned to numpy's float16 on every bit pattern; packing to
a hand-derived byte and exhaustive round trips; the accumulation to a dense
float64 product built from the unpacked weights and the broadcast scales, and
to invariants (all +1 weights give the token's sum, negation, linearity in a
group's scale, group independence).
"""
import numpy as np
import pytest

import oracle
from workloads import BINARY_GROUP, activations_bf16, binary_weights, group_scales_f16


def test_half_decoder_matches_numpy_on_every_pattern():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits])
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[np.isinf(ref)], ref[np.isinf(ref)])


def test_hand_packed_byte():
    # N = 8, K = 1: rows 0..7 are bits 0..7 of the single byte; +1 sets a bit.
    w = np.array([[1], [-1], [-1], [1], [1], [1], [-1], [-1]], np.int8)
    B = oracle.pack_binary(w)
    assert B.tolist() == [[0b00111001]]
    # N = 16: byte (i, k) holds rows i + 2p
    w16 = -np.ones((16, 1), np.int8)
    w16[3] = 1  # row 3 = i 1, bit 1
    assert oracle.pack_binary(w16).tolist() == [[0], [2]]


def test_exhaustive_round_trip_and_rejection():
    pats = np.arange(256, dtype=np.uint8)
    w = np.where((pats[None, :] >> np.arange(8)[:, None]) & 1, 1, -1).astype(np.int8)  # [8, 256]
    B = oracle.pack_binary(w)
    assert np.array_equal(B[0], pats)
    assert np.array_equal(oracle.unpack_binary(B, 8), w)
    rng = np.random.default_rng(1)
    w2 = binary_weights(rng, 64, 40)
    assert np.array_equal(oracle.unpack_binary(oracle.pack_binary(w2), 64), w2)
    with pytest.raises(oracle.OracleError):
        oracle.pack_binary(np.zeros((8, 4), np.int8))  # 0 is not a binary weight
    with pytest.raises(oracle.OracleError):
        oracle.pack_binary(np.ones((4, 4), np.int8))  # N % 8


def _dense_reference(w, s_f16, q, x_scale):
    """y = x_scale * (W o S) q in float64 with S the group scales broadcast over
    their 128 columns; acc = w q in int64."""
    S = np.repeat(s_f16.view(np.float16).astype(np.float64), BINARY_GROUP, axis=1)
    Wd = w.astype(np.float64) * S
    y = (q.astype(np.float64) @ Wd.T) * x_scale.astype(np.float64)[:, None]
    acc = q.astype(np.int64) @ w.astype(np.int64).T
    return acc, y


@pytest.mark.parametrize("N,K,M", [(8, 128, 1), (64, 512, 3), (640, 2560, 2)])
def test_gemv_binary_equals_dense_float64_product(N, K, M):
    rng = np.random.default_rng(N + K)
    w = binary_weights(rng, N, K)
    s = group_scales_f16(rng, N, K)
    q, xs, _ = oracle.quant(activations_bf16(rng, M, K))
    acc, y = oracle.gemv_binary(oracle.pack_binary(w), N, s, q, xs)
    racc, ry = _dense_reference(w, s, q, xs)
    assert np.array_equal(acc, racc)
    assert np.allclose(y, ry, rtol=1e-12, atol=1e-300)
    # row ranges and threads give the same values
    a2, y2 = oracle.gemv_binary(oracle.pack_binary(w), N, s, q, xs, 8, N)
    assert np.array_equal(a2, acc[:, 8:]) and np.array_equal(y2, y[:, 8:])
    a3, y3 = oracle.gemv_binary_threads(oracle.pack_binary(w), N, s, q, xs, threads=3)
    assert np.array_equal(a3, acc) and np.array_equal(y3, y)


def test_gemv_binary_invariants():
    rng = np.random.default_rng(9)
    N, K, M = 16, 384, 2
    q, xs, xsum = oracle.quant(activations_bf16(rng, M, K))
    ones = np.full((N, K // BINARY_GROUP), np.float16(1.0)).view(np.uint16)
    # all +1 with unit scales: acc = x_sum, y = x_sum * x_scale
    acc, y = oracle.gemv_binary(oracle.pack_binary(np.ones((N, K), np.int8)), N, ones, q, xs)
    assert (acc == xsum[:, None]).all()
    assert (y == xsum[:, None].astype(np.float64) * xs[:, None].astype(np.float64)).all()
    # negating every weight negates acc and y
    w = binary_weights(rng, N, K)
    s = group_scales_f16(rng, N, K)
    a1, y1 = oracle.gemv_binary(oracle.pack_binary(w), N, s, q, xs)
    a2, y2 = oracle.gemv_binary(oracle.pack_binary(-w), N, s, q, xs)
    assert np.array_equal(a2, -a1) and np.array_equal(y2, -y1)
    # doubling group 1's scale of row 5 adds exactly that group's term once more
    s2 = s.copy()
    s2[5, 1] = (s.view(np.float16)[5, 1] * np.float16(2)).view(np.uint16)
    _, y3 = oracle.gemv_binary(oracle.pack_binary(w), N, s2, q, xs)
    g1 = (q[:, 128:256].astype(np.int64) @ w[5, 128:256].astype(np.int64))
    term = g1 * np.float64(s.view(np.float16)[5, 1]) * xs.astype(np.float64)
    assert np.allclose(y3[:, 5] - y1[:, 5], term, rtol=1e-12, atol=1e-15)
    others = [n for n in range(N) if n != 5]
    assert np.array_equal(y3[:, others], y1[:, others])


def test_forward_binary_composes_quant_and_gemv():
    rng = np.random.default_rng(10)
    w = binary_weights(rng, 32, 256)
    s = group_scales_f16(rng, 32, 256)
    x = activations_bf16(rng, 2, 256)
    q, xs, xsum, acc, y = oracle.forward_binary(oracle.pack_binary(w), 32, s, x)
    q2, xs2, xsum2 = oracle.quant(x)
    assert np.array_equal(q, q2) and np.array_equal(xs, xs2) and np.array_equal(xsum, xsum2)
    racc, ry = _dense_reference(w, s, q, xs)
    assert np.array_equal(acc, racc) and np.allclose(y, ry, rtol=1e-12)
