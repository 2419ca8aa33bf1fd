"""Pins of the oracle's decoder-layer neighbours of the GEMV (RMSNorm,
relu_squared times up, absmax of fp32 rows) and of the absmean weight
quantiser, against hand-derived values, closed forms and exact invariants.

The pages (lemon-mlx-engine issue, section "Architecture"; 1bit.systems post
"the full arc ...", read-more item "Training-Runs") name these steps without
formulas; the readings pinned here are stated in oracle.c's header.
"""
import numpy as np
import pytest
import torch

import oracle


def bf16(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)


def f32_of_bf16(b):
    return (np.asarray(b, dtype=np.uint32) << 16).view(np.float32)


# ------------------------------------------------------------ relu^2 * up
def test_relu2_mul_hand_values():
    a = np.array([3.0, -1.0, 0.5, 0.0, -0.0, 2.0], np.float32)
    b = np.array([2.0, 5.0, 4.0, 7.0, 7.0, -0.25], np.float32)
    assert oracle.relu2_mul(a, b).tolist() == [18.0, 0.0, 1.0, 0.0, 0.0, -1.0]


def test_relu2_mul_one_rounding_per_product():
    rng = np.random.default_rng(0)
    a = rng.standard_normal(4096).astype(np.float32)
    b = rng.standard_normal(4096).astype(np.float32)
    r = np.maximum(a, 0).astype(np.float64)
    sq = (r * r).astype(np.float32)                      # fl32 of the exact square
    ref = (sq.astype(np.float64) * b).astype(np.float32)  # fl32 of the exact product
    assert np.array_equal(oracle.relu2_mul(a, b), ref)


# ---------------------------------------------------------------- RMSNorm
def test_rmsnorm_hand_example():
    h = oracle.rmsnorm(np.array([[3.0, 4.0]], np.float32), np.ones(2, np.float32), 0.0)
    # mean of squares 12.5; 1/sqrt(12.5) = 0.2828427...
    assert np.allclose(h[0], [3 / np.sqrt(12.5), 4 / np.sqrt(12.5)], rtol=2e-7, atol=0)


def test_rmsnorm_constant_row_gives_the_gain():
    g = np.array([1.0, -2.0, 0.5, 3.0, 0.0, 7.25, -1.0, 4.0], np.float32)
    h = oracle.rmsnorm(np.full((1, 8), 2.0, np.float32), g, 0.0)
    assert np.array_equal(h[0], g)          # r = 1/2 exactly, 2 * 1/2 = 1
    h = oracle.rmsnorm(np.full((1, 8), -2.0, np.float32), g, 0.0)
    assert np.array_equal(h[0], -g)


def test_rmsnorm_epsilon_enters_under_the_root():
    g = np.arange(1, 17, dtype=np.float32)
    # mean(x^2) = 1, eps = 3: r = 1 / sqrt(4) = 1/2 exactly
    h = oracle.rmsnorm(np.ones((1, 16), np.float32), g, 3.0)
    assert np.array_equal(h[0], g / 2)
    # zero row: r = 1/sqrt(eps), h = 0
    assert not oracle.rmsnorm(np.zeros((2, 16), np.float32), g, 1e-5).any()


def test_rmsnorm_scale_invariance_and_row_independence():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((3, 2560)).astype(np.float32)
    g = (1 + 0.1 * rng.standard_normal(2560)).astype(np.float32)
    h = oracle.rmsnorm(x, g, 0.0)
    # powers of two scale every square, the mean and the root exactly
    assert np.array_equal(oracle.rmsnorm(4 * x, g, 0.0), h)
    assert np.array_equal(oracle.rmsnorm(x[1:2], g, 0.0), h[1:2])


def test_rmsnorm_against_float64():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((4, 6912)) * 3).astype(np.float32)
    g = rng.uniform(0.5, 1.5, 6912).astype(np.float32)
    h = oracle.rmsnorm(x, g, 1e-5).astype(np.float64)
    x64 = x.astype(np.float64)
    ref = x64 / np.sqrt((x64 ** 2).mean(axis=1, keepdims=True) + 1e-5) * g
    # three fp32 roundings (r, x*r, *g): within 2e-7 relative each
    assert np.all(np.abs(h - ref) <= 4e-7 * np.abs(ref) + 1e-30)


# ------------------------------------------------------- absmax of fp32 rows
def test_quant_f32_hand_values():
    q, s, t = oracle.quant_f32(np.array([[1.0, -0.5, 0.25, 0.0, 0.7]], np.float32))
    # s = 127: -63.5 -> -64 (ties to even), 31.75 -> 32, 0.7 * 127 = 88.9 -> 89
    # (a scale of 128 would give 90)
    assert q[0].tolist() == [127, -64, 32, 0, 89]
    assert s[0] == np.float32(1.0) / np.float32(127.0) and t[0] == 127 - 64 + 32 + 89


def test_quant_f32_matches_bf16_entry_on_bf16_values():
    rng = np.random.default_rng(3)
    xb = bf16(rng.standard_normal((5, 512)) * 4)
    a = oracle.quant(xb)
    b = oracle.quant_f32(f32_of_bf16(xb))
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


# ----------------------------------------------------------------- absmean
def test_absmean_hand_example():
    w, g = oracle.absmean(bf16([[0.5, -1.5], [0.0, 3.0]]))
    # mean |W| = 5/4; W / g = 0.4, -1.2, 0, 2.4 -> 0, -1, 0, 1 (clamped)
    assert g == np.float32(1.25) and w.tolist() == [[0, -1], [0, 1]]


def test_absmean_rounding_ties_and_clamp():
    # mean |W| = 1: 0.5 -> 0 (tie to even), 0.75 -> 1 (a truncation gives 0),
    # 1.5 -> 2 -> 1 (clamp), -0.25 -> 0
    w, g = oracle.absmean(bf16([[0.5, 0.75, 1.5, -1.25]]))
    assert g == np.float32(1.0) and w.tolist() == [[0, 1, 1, -1]]


def test_absmean_recovers_dequantised_ternary_weights():
    # Pre-dequantised weights w * s (exact in bf16) quantise back to w, with
    # gamma = s * mean|w|.
    rng = np.random.default_rng(4)
    t = rng.choice(np.array([-1, 0, 1], np.int8), size=(64, 320), p=[0.3, 0.4, 0.3])
    for s in (0.75, 1.0, 3.5, 2.0 ** -7):
        w, g = oracle.absmean(bf16(t.astype(np.float32) * s))
        assert np.array_equal(w, t)
        assert g == np.float32(s * np.count_nonzero(t) / t.size)


def test_absmean_symmetries_and_zero():
    rng = np.random.default_rng(5)
    W = rng.standard_normal((32, 256)).astype(np.float32)
    w, g = oracle.absmean(bf16(W))
    wn, gn = oracle.absmean(bf16(-W))
    assert np.array_equal(wn, -w) and gn == g
    w2, g2 = oracle.absmean(bf16(2 * W))        # power of two: exact
    assert np.array_equal(w2, w) and g2 == 2 * g
    wz, gz = oracle.absmean(bf16(np.zeros((4, 16))))
    assert gz == 0 and not wz.any()


def test_absmean_against_float64():
    rng = np.random.default_rng(6)
    Wb = bf16(rng.standard_normal((128, 512)) * 0.02)
    w, g = oracle.absmean(Wb)
    W = f32_of_bf16(Wb).astype(np.float64)
    g64 = np.abs(W).mean()
    assert abs(float(g) - g64) <= 6e-8 * g64
    ref = np.clip(np.rint((W / float(g)).astype(np.float32)), -1, 1)
    assert np.array_equal(w, ref.astype(np.int8))


@pytest.mark.parametrize("shape", [(0, 16), (4, 0)])
def test_absmean_empty(shape):
    w, g = oracle.absmean(np.zeros(shape, np.uint16))
    assert g == 0 and w.shape == shape
