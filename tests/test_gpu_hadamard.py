"""GPU parity of the Hadamard route for prompt processing (1bit engine blog,
"509 tokens a second of prompt: the Hadamard route ships"): the fused
rotation + 4-bit quantiser (tq_hadamard_quantize_act) against the oracle's
plain matrix-vector rotation and quantiser, codes / scales / sums bit-exact;
then the ternary contraction of those codes (tq_gemm_prefill) at M = 512 on
the three prefill shapes, every int32 accumulator bit-exact and every fp32
output within the parity bar."""
import numpy as np
import pytest
import torch

import oracle
import ternary_absmax_int8_b200 as tq
from tests._gpu import THREADS, assert_parity, dev, host_pack
from workloads import HADAMARD_BLOCK, PREFILL_M, PREFILL_SHAPES, activations_bf16, \
    make_projections

pytestmark = pytest.mark.gpu


def gpu_had4(x_bf16, n):
    M, K = x_bf16.shape
    x = dev(x_bf16.view(np.int16))
    xq = torch.full((M, K), 99, dtype=torch.int8, device="cuda")
    xs = torch.full((M,), float("nan"), device="cuda")
    xsum = torch.full((M,), -(2 ** 31), dtype=torch.int32, device="cuda")
    tq.tq_hadamard_quantize_act(x, xq, xs, xsum, M, K, n)
    return xq, xs, xsum


def _check_quant(x_bf16, n):
    xq, xs, xsum = gpu_had4(x_bf16, n)
    torch.cuda.synchronize()
    rq, rxs, rxsum = oracle.hadamard_quant4(x_bf16, n)
    assert np.array_equal(xq.cpu().numpy(), rq)
    assert np.array_equal(xs.cpu().numpy().view(np.uint32), rxs.view(np.uint32))
    assert np.array_equal(xsum.cpu().numpy(), rxsum)


@pytest.mark.parametrize("n", [32, 64, 128, 256, 512, 1024])
def test_rotation_and_4bit_codes_match_oracle(cuda_device, n):
    rng = np.random.default_rng(100 + n)
    for M, K in ((3, n), (5, 5120), (2, 6144)):
        if K % n == 0:
            _check_quant(activations_bf16(rng, M, K), n)


def test_degenerate_rows(cuda_device):
    K = 1024
    x = np.zeros((4, K), np.float32)
    x[1] = 3.0                              # constant blocks: all energy in h[0] of each block
    x[2, ::2] = 1.0
    x[2, 1::2] = -1.0                       # alternating signs: one Walsh function
    x[3] = np.where(np.arange(K) % 3 == 0, 1e-3, -2.5)
    xb = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    _check_quant(xb, 256)


def test_prefill_m512_had4_every_output(cuda_device):
    # The three prefill shapes at 512 tokens through the Hadamard route, block
    # 256; the oracle over output-row ranges on all host threads.
    for p in make_projections(PREFILL_SHAPES, M=PREFILL_M, seed=3):
        xq, xs, xsum = gpu_had4(p.x_bf16, HADAMARD_BLOCK)
        Pd = dev(host_pack(p.w))
        y = torch.full((p.M, p.N), float("nan"), device="cuda")
        acc = torch.full((p.M, p.N), -(2 ** 31), dtype=torch.int32, device="cuda")
        tq.tq_gemm_prefill(Pd, float(p.w_scale), xq, xs, xsum, y, acc, p.M, p.N, p.K)
        torch.cuda.synchronize()
        got = (xq.cpu().numpy(), xs.cpu().numpy(), xsum.cpu().numpy(), acc.cpu().numpy(),
               y.cpu().numpy())
        ref = oracle.forward_had4(oracle.pack(p.w), p.N, p.w_scale, p.x_bf16, HADAMARD_BLOCK,
                                  threads=THREADS)
        assert_parity(got, ref, f"{p.name} had4 M={p.M}")
    assert tq.tq_device_error(reset=True) == 0


@pytest.mark.parametrize("M", [1, 8, 24, 40, 300])
def test_had4_codes_through_every_contraction_path(cuda_device, M):
    # streaming (1 token), warp MMA (8), tensor-core batched decode (24),
    # prefill GEMM on single CTAs (40) and on CTA pairs (300)
    for p in make_projections([("ffn", 2560, 6912)], M=M, seed=30 + M):
        xq, xs, xsum = gpu_had4(p.x_bf16, HADAMARD_BLOCK)
        Pd = dev(host_pack(p.w))
        y = torch.full((M, p.N), float("nan"), device="cuda")
        acc = torch.full((M, p.N), -(2 ** 31), dtype=torch.int32, device="cuda")
        tq.tq_gemm_prefill(Pd, float(p.w_scale), xq, xs, xsum, y, acc, M, p.N, p.K)
        torch.cuda.synchronize()
        got = (xq.cpu().numpy(), xs.cpu().numpy(), xsum.cpu().numpy(), acc.cpu().numpy(),
               y.cpu().numpy())
        ref = oracle.forward_had4(oracle.pack(p.w), p.N, p.w_scale, p.x_bf16, HADAMARD_BLOCK,
                                  threads=THREADS)
        assert_parity(got, ref, f"had4 M={M}")


@pytest.mark.parametrize("n", [256, 1024])
def test_stack_form_matches_the_oracle(cuda_device, n):
    # the grouped form over projections of different K (one launch): every
    # code, scale and sum against the oracle
    M = 7
    rng = np.random.default_rng(n)
    xs_in = [activations_bf16(rng, M, n * k) for k in (1, 3, 10, 27)]
    xd = [dev(x.view(np.int16)) for x in xs_in]
    xq = [torch.full((M, x.shape[1]), 99, dtype=torch.int8, device="cuda") for x in xs_in]
    xs = [torch.full((M,), float("nan"), device="cuda") for _ in xs_in]
    xsum = [torch.full((M,), -(2 ** 31), dtype=torch.int32, device="cuda") for _ in xs_in]
    table = [tq.make_proj(x=xd[j], xq=xq[j], x_scale=xs[j], x_sum=xsum[j], K=x.shape[1])
             for j, x in enumerate(xs_in)]
    tq.tq_hadamard_quantize_act_stack(table, M, n)
    torch.cuda.synchronize()
    for j, x in enumerate(xs_in):
        rq, rxs, rxsum = oracle.hadamard_quant4(x, n)
        assert np.array_equal(xq[j].cpu().numpy(), rq), j
        assert np.array_equal(xs[j].cpu().numpy().view(np.uint32), rxs.view(np.uint32)), j
        assert np.array_equal(xsum[j].cpu().numpy(), rxsum), j
