"""Pins of the oracle's Hadamard-rotated 4-bit activation route (1bit engine
blog, "509 tokens a second of prompt: the Hadamard route ships": 4-bit
activations on the matrix units, kept accurate by a Hadamard rotation;
1bit.systems README, "Training-Runs -- BitNet v2 Hadamard").

The rotation is pinned to a hand-worked case, to a library construction of
the Sylvester-Hadamard matrix, to exact big-integer arithmetic on synthetic
rows (which also shows that the fp64 sums are exact, so any order of the
additions gives the same fp32 value), and to Parseval's identity. The 4-bit
quantiser is pinned to hand-worked ties and to its invariants.
"""
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from workloads import HADAMARD_BLOCK, activations_bf16, bf16_bits_to_float


def _bf16(x):
    t = torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def test_hand_worked_four_point_rotation():
    # H_4 = [[1,1,1,1],[1,-1,1,-1],[1,1,-1,-1],[1,-1,-1,1]];
    # H_4 [1,2,3,4] = [10, -2, -4, 0]; divided by sqrt(4) = 2.
    h = oracle.hadamard_rotate(_bf16([[1, 2, 3, 4]]), 4)
    assert h.tolist() == [[5.0, -1.0, -2.0, 0.0]]
    # two blocks of two: H_2 [a, b] = [a + b, a - b] / sqrt(2)
    h2 = oracle.hadamard_rotate(_bf16([[1, 2, 3, 4]]), 2)
    c = 1.0 / np.sqrt(2.0)
    assert h2.tolist() == [[np.float32(3 * c), np.float32(-1 * c),
                            np.float32(7 * c), np.float32(-1 * c)]]


@pytest.mark.parametrize("n", [2, 8, 16, 64, 256])
def test_rotation_matrix_is_the_sylvester_hadamard_matrix(n):
    # Rotating the unit vectors gives the columns of H_n / sqrt(n); scipy builds
    # H_n by the Sylvester construction.
    E = _bf16(np.eye(n, dtype=np.float32))
    R = oracle.hadamard_rotate(E, n).T  # column j = rotation of e_j
    expected = (scipy.linalg.hadamard(n).astype(np.float64) / np.sqrt(float(n))).astype(np.float32)
    assert np.array_equal(R, expected)
    # orthogonal: R R^T = I (exactly for a power of four)
    RR = R.astype(np.float64) @ R.astype(np.float64).T
    assert np.allclose(RR, np.eye(n), atol=1e-6)


def _exact_rotation(x_bits, n):
    """Rotation with exact rational arithmetic, then one rounding to fp32 via
    the fp64 product with fl64(1/sqrt(n)) (exact for powers of four)."""
    xf = bf16_bits_to_float(x_bits).astype(np.float64)
    M, K = xf.shape
    H = scipy.linalg.hadamard(n)
    c = 1.0 / np.sqrt(float(n))
    out = np.empty((M, K), np.float32)
    for m in range(M):
        for b in range(0, K, n):
            blk = [Fraction(float(v)) for v in xf[m, b:b + n]]
            for i in range(n):
                s = sum((blk[j] if H[i, j] > 0 else -blk[j]) for j in range(n))
                out[m, b + i] = np.float32(float(s) * c)  # float(s) exact here
    return out


def test_rotation_of_synthetic_rows_is_exact():
    rng = np.random.default_rng(3)
    x = activations_bf16(rng, 2, 2 * HADAMARD_BLOCK)
    h = oracle.hadamard_rotate(x, HADAMARD_BLOCK)
    assert np.array_equal(h, _exact_rotation(x, HADAMARD_BLOCK))


def test_parseval_and_block_independence():
    rng = np.random.default_rng(4)
    x = activations_bf16(rng, 3, 1024)
    xf = bf16_bits_to_float(x).astype(np.float64)
    h = oracle.hadamard_rotate(x, 256).astype(np.float64)
    for b in range(0, 1024, 256):
        e_x = (xf[:, b:b + 256] ** 2).sum(1)
        e_h = (h[:, b:b + 256] ** 2).sum(1)
        assert np.allclose(e_h, e_x, rtol=1e-6)
    # changing one block changes only that block's outputs
    x2 = x.copy()
    x2[:, 300] = _bf16([[5.0]])[0, 0]
    h2 = oracle.hadamard_rotate(x2, 256)
    assert np.array_equal(h2[:, :256], h[:, :256].astype(np.float32))
    assert np.array_equal(h2[:, 512:], h[:, 512:].astype(np.float32))
    assert not np.array_equal(h2[:, 256:512], h[:, 256:512].astype(np.float32))


def test_rotation_is_linear_in_sign_and_powers_of_two():
    rng = np.random.default_rng(5)
    x = activations_bf16(rng, 2, 512)
    h = oracle.hadamard_rotate(x, 256)
    assert np.array_equal(oracle.hadamard_rotate(x ^ np.uint16(0x8000), 256), -h)
    x4 = _bf16(bf16_bits_to_float(x) * 4)
    assert np.array_equal(oracle.hadamard_rotate(x4, 256), h * 4)


def test_rotation_rejects_bad_block_sizes():
    x = _bf16(np.ones((1, 96), np.float32))
    for n in (0, 3, 64, 128):  # not a power of two, or not dividing K
        with pytest.raises(oracle.OracleError):
            oracle.hadamard_rotate(x, n)


def test_quant4_hand_worked_ties_and_clamp():
    # amax = 7 gives s = 1: 2.5 -> 2 and -3.5 -> -4 (ties to even), 0.5 -> 0
    h = np.array([[7.0, 2.5, -3.5, 0.5, 1.5, -7.0]], np.float32)
    q, s, t = oracle.quant4(h)
    assert q.tolist() == [[7, 2, -4, 0, 2, -7]]
    assert s.tolist() == [1.0] and t.tolist() == [0]
    # amax = 3.5 gives s = 2: 1.75 -> 3.5 -> 4, 0.25 -> 0.5 -> 0
    q, s, t = oracle.quant4(np.array([[3.5, 1.75, 0.25, -1.25]], np.float32))
    assert q.tolist() == [[7, 4, 0, -2]] and s.tolist() == [0.5] and t.tolist() == [9]
    # a zero row
    q, s, t = oracle.quant4(np.zeros((1, 8), np.float32))
    assert not q.any() and s.tolist() == [0.0] and t.tolist() == [0]


def test_quant4_invariants():
    rng = np.random.default_rng(6)
    h = oracle.hadamard_rotate(activations_bf16(rng, 64, 512), 256)
    q, s, t = oracle.quant4(h)
    assert q.min() >= -7 and q.max() <= 7
    am = np.abs(h).argmax(1)
    assert (np.abs(q[np.arange(64), am]) == 7).all()
    assert (np.sign(q) * np.sign(h) >= 0).all()
    err = np.abs(q * s[:, None].astype(np.float64) - h)
    assert (err <= 0.5 * s[:, None] * (1 + 1e-5)).all()
    assert np.array_equal(t, q.astype(np.int64).sum(1))
    qn, sn, tn = oracle.quant4(-h)
    assert np.array_equal(qn, -q) and np.array_equal(sn, s) and np.array_equal(tn, -t)
    # s = amax / 7 within one rounding
    amax = np.abs(h).max(1).astype(np.float64)
    assert np.allclose(s, amax / 7, rtol=2 ** -23)


def test_forward_had4_is_rotation_quant_gemv_epilogue():
    rng = np.random.default_rng(7)
    from workloads import stored_weight_scale, ternary_weights
    w = ternary_weights(rng, 64, 512)
    x = activations_bf16(rng, 3, 512)
    ws = stored_weight_scale(w)
    q, xs, xsum, acc, y = oracle.forward_had4(oracle.pack(w), 64, ws, x, 256)
    q2, xs2, _ = oracle.quant4(oracle.hadamard_rotate(x, 256))
    assert np.array_equal(q, q2) and np.array_equal(xs, xs2)
    assert np.array_equal(acc, q.astype(np.int64) @ w.astype(np.int64).T)
    ref = acc.astype(np.float64) * np.float64(ws) * xs.astype(np.float64)[:, None]
    assert np.allclose(y, ref, rtol=1e-12, atol=0)
