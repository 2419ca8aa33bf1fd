"""The GPU parity tests of the normalising quantisers and of the absmean
packer compare fp32 scales bit for bit although the GPU sums in a tree order
and the oracle left to right. That is sound only for inputs whose result is
the same for every order of the fp64 additions; tests/_exact.py checks this
per row with the exact sum and the (n - 1) u error bound of any order. These
CPU tests pin that check: it holds for the seeded inputs the GPU tests use,
and it does detect a constructed row whose factor sits on an fp32 rounding
boundary."""
import numpy as np
import torch

from tests._exact import U64, absmean_order_free, rms_factor, rms_interval_ok, rms_order_free
from workloads import activations_bf16


def test_seeded_rmsnorm_rows_are_order_free():
    for M, K in [(1, 2560), (4, 6912), (16, 2560), (3, 16), (2, 32768)]:
        rng = np.random.default_rng(M * 7 + K)
        xb = activations_bf16(rng, M, K)
        x = (xb.astype(np.uint32) << 16).view(np.float32)
        assert rms_order_free(x, 1e-5).all()
    for M, K in [(1, 2560), (5, 6912)]:
        rng = np.random.default_rng(100 + M + K)
        assert rms_order_free((rng.standard_normal((M, K)) * 3).astype(np.float32), 1e-5).all()


def test_seeded_absmean_inputs_are_order_free():
    for N, K in [(6912, 2560), (2560, 6912), (4, 16), (516, 272)]:
        rng = np.random.default_rng(N + K)
        W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
        Wb = torch.from_numpy(W).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert absmean_order_free(Wb)


def test_check_detects_a_factor_on_a_rounding_boundary():
    # Scan the sum of squares upward in steps far smaller than the error band
    # until the fp32 factor changes: a sum there is rejected, one halfway
    # between two boundaries is accepted.
    K, eps = 4096, 0.0
    S = 1000.0
    r0 = rms_factor(S, K, eps)
    step = S * K * U64 / 8
    while rms_factor(S, K, eps) == r0:
        S += step
    assert not rms_interval_ok(S, K, eps)
    assert not rms_interval_ok(S - 2 * step, K, eps)
    # fp32 factors near 1/sqrt(1000/4096) are about 2^-22 relative apart:
    # move half of that in S (twice in 1/sqrt), well away from both sides
    assert rms_interval_ok(S * (1 - 2.0 ** -23), K, eps)
    # and the row-level check uses the exact sum
    assert rms_order_free(np.ones((1, K), np.float32), 1e-5)[0]
