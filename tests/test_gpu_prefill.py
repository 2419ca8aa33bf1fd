"""GPU parity of tq_gemm_prefill (M = 512 prompt processing) against the oracle.

Full outputs at M = 128 and 256 for the FFN shapes and at M = 512 on the three
prefill shapes (including the 27B-scale 17408 x 5120). Ragged M and N exercise
partial tiles (128- and 256-token tiles); CTAs that take several tiles drain
and refill both tensor-memory accumulators.
"""
import numpy as np
import pytest

from tests._gpu import assert_parity, gpu_forward, host_pack, oracle_forward
from workloads import PREFILL_M, PREFILL_SHAPES, activations_bf16, make_projections, \
    stored_weight_scale, ternary_weights

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M", [128, 256])
def test_prefill_full_outputs(cuda_device, M):
    for p in make_projections(PREFILL_SHAPES[:2], M=M, seed=77 + M):
        P = host_pack(p.w)
        assert_parity(gpu_forward(P, p.N, p.w_scale, p.x_bf16),
                      oracle_forward(p.w, p.w_scale, p.x_bf16), f"{p.name} M={M}")


def test_prefill_m512_full_outputs(cuda_device):
    # The three prefill shapes at 512 tokens, every output: the oracle runs
    # over disjoint output-row ranges on all host threads (same function,
    # same result; 45.6 G multiply-adds on the largest shape).
    for p in make_projections(PREFILL_SHAPES, M=PREFILL_M, seed=0):
        P = host_pack(p.w)
        assert_parity(gpu_forward(P, p.N, p.w_scale, p.x_bf16),
                      oracle_forward(p.w, p.w_scale, p.x_bf16), f"{p.name} M={PREFILL_M}")


@pytest.mark.parametrize("N,K,M", [(516, 272, 130), (4, 16, 129), (2048, 1024, 384),
                                   (260, 2560, 200), (512, 128, 33), (2564, 6928, 64)])
def test_prefill_ragged(cuda_device, N, K, M):
    rng = np.random.default_rng(N + K + M)
    w = ternary_weights(rng, N, K)
    xb = activations_bf16(rng, M, K)
    ws = stored_weight_scale(w)
    assert_parity(gpu_forward(host_pack(w), N, ws, xb), oracle_forward(w, ws, xb),
                  f"{N}x{K} M={M}")


def test_prefill_second_tile_per_cta(cuda_device):
    # 136 x 4 = 544 tiles of 128 features x 256 tokens on 148 SMs: every CTA
    # takes three or four tiles, so both accumulators are drained and
    # refilled; sampled token rows from every token tile, all N outputs.
    N, K, M = 17408, 512, 1024
    rng = np.random.default_rng(5)
    w = ternary_weights(rng, N, K)
    xb = activations_bf16(rng, M, K)
    ws = stored_weight_scale(w)
    q, xs, xsum, acc, y = gpu_forward(host_pack(w), N, ws, xb)
    rows = np.array([0, 255, 256, 300, 511, 512, 700, 767, 768, 1000, 1023])
    sub = (q[rows], xs[rows], xsum[rows], acc[rows], y[rows])
    assert_parity(sub, oracle_forward(w, ws, xb[rows]), "17408x512 M=1024")


def test_prefill_repeated_and_after_error(cuda_device):
    # Repeated calls give identical bytes and match the oracle, also after a
    # device error has been reported in between.
    import torch

    import ternary_absmax_int8_b200 as tq
    from tests._gpu import dev, gpu_quant
    p = next(make_projections([("ffn_2560x6912", 2560, 6912)], M=PREFILL_M, seed=11))
    P = dev(host_pack(p.w))
    xq, xs, xsum = gpu_quant(p.x_bf16)
    ref = oracle_forward(p.w, p.w_scale, p.x_bf16)
    outs = []
    for i in range(3):
        if i == 2:
            tq.tq_selftest_wait_timeout(100)
            assert tq.tq_device_error(reset=True) != 0
        y = torch.full((p.M, p.N), float("nan"), device="cuda")
        acc = torch.full((p.M, p.N), -(2 ** 31), dtype=torch.int32, device="cuda")
        tq.tq_gemm_prefill(P, float(p.w_scale), xq, xs, xsum, y, acc, p.M, p.N, p.K)
        torch.cuda.synchronize()
        got = (xq.cpu().numpy(), xs.cpu().numpy(), xsum.cpu().numpy(), acc.cpu().numpy(),
               y.cpu().numpy())
        assert_parity(got, ref, f"call {i}")
        outs.append(got[4])
    assert all(np.array_equal(o.view(np.uint32), outs[0].view(np.uint32)) for o in outs)
    assert tq.tq_device_error(reset=True) == 0
