"""GPU parity of the binary g128 decode GEMV (baguaai "BitNet" tag page,
Bonsai 27B item: 1-bit weights, one fp16 scale per 128 weights) against the
oracle: the int32 total sum_k w q bit-exact and the group-scaled fp32 output
within 1e-5 relative (exactly 0 where the oracle gives 0), on the 27B-scale
FFN shapes at 1..4 tokens, ragged and minimal shapes, degenerate weights and
tokens, and the 8-layer stack the bench times (one launch)."""
import numpy as np
import pytest
import torch

import oracle
import ternary_absmax_int8_b200 as tq
from tests._gpu import THREADS, assert_y_close, dev, gpu_quant
from workloads import BINARY_FFN27B, binary_stack_shapes, make_binary_projections

pytestmark = pytest.mark.gpu


class BinDev:
    """Packed device copies of one binary projection and its outputs."""

    def __init__(self, p):
        self.p = p
        bits = np.empty((p.N // 8, p.K), np.uint8)
        sp = np.empty((p.N // 8, p.K // 128, 8), np.uint16)
        tq.tq_pack_binary_host(p.w, p.s_f16, bits, sp, p.N, p.K)
        self.bits, self.sp = dev(bits), dev(sp.view(np.int16))
        self.xq, self.xs, self.xsum = gpu_quant(p.x_bf16)
        self.y = torch.full((p.M, p.N), float("nan"), device="cuda")
        self.acc = torch.full((p.M, p.N), -(2 ** 31), dtype=torch.int32, device="cuda")

    def proj(self):
        return tq.make_binary_proj(bits=self.bits, scales_packed=self.sp, xq=self.xq,
                                   x_scale=self.xs, y=self.y, acc_out=self.acc, N=self.p.N,
                                   K=self.p.K)

    def check(self, threads=1):
        p = self.p
        _, _, _, racc, ry = oracle.forward_binary(oracle.pack_binary(p.w), p.N, p.s_f16,
                                                  p.x_bf16, threads=threads)
        acc = self.acc.cpu().numpy()
        bad = np.argwhere(acc != racc)
        assert bad.size == 0, (p.name, p.M, bad[:4].tolist())
        assert_y_close(self.y.cpu().numpy(), ry)


@pytest.mark.parametrize("M", [1, 2, 3, 4])
def test_27b_ffn_shapes(cuda_device, M):
    for p in make_binary_projections(BINARY_FFN27B, M=M, seed=60 + M):
        d = BinDev(p)
        tq.tq_gemv_binary(d.bits, d.sp, d.xq, d.xs, d.y, d.acc, M, p.N, p.K)
        torch.cuda.synchronize()
        d.check(threads=THREADS)
    assert tq.tq_device_error(reset=True) == 0


@pytest.mark.parametrize("N,K,M", [(8, 128, 1), (8, 256, 3), (4104, 384, 2), (640, 2560, 1),
                                   (2048, 32768, 1), (24, 1152, 4)])
def test_small_ragged_and_maximum_k(cuda_device, N, K, M):
    p = next(make_binary_projections([("r", N, K)], M=M, seed=N + K + M))
    d = BinDev(p)
    tq.tq_gemv_binary(d.bits, d.sp, d.xq, d.xs, d.y, d.acc, M, N, K)
    torch.cuda.synchronize()
    d.check(threads=THREADS)


def test_degenerate_weights_and_tokens(cuda_device):
    ps = list(make_binary_projections([("a", 640, 1280), ("b", 640, 1280)], M=3, seed=70))
    ps[0].w[:] = 1                      # all +1: acc = x_sum
    ps[0].x_bf16[1] = 0                 # a zero token
    ps[1].w[:, ::2] = -1
    ps[1].w[:, 1::2] = 1
    ps[1].x_bf16[2] = np.where(np.arange(1280) % 2 == 0, 0x4120, 0xC120).astype(np.uint16)
    for p in ps:
        d = BinDev(p)
        tq.tq_gemv_binary(d.bits, d.sp, d.xq, d.xs, d.y, d.acc, p.M, p.N, p.K)
        torch.cuda.synchronize()
        d.check()
        if p.name == "a":
            assert (d.acc.cpu().numpy() == d.xsum.cpu().numpy()[:, None]).all()


def test_stack_of_8_layers_one_launch(cuda_device):
    # bench.py's binary_ffn27b_m1: 24 projections, 2.14e9 weights, one launch
    projs = list(make_binary_projections(binary_stack_shapes(8), M=1, seed=0))
    ds = [BinDev(p) for p in projs]
    tq.tq_gemv_binary_stack([d.proj() for d in ds], 1)
    torch.cuda.synchronize()
    for d in ds:
        d.check(threads=THREADS)
    assert tq.tq_device_error(reset=True) == 0


def test_one_token_mixed_stack(cuda_device):
    # one token: a table of ragged projections (tiles of 16 packed rows that
    # end mid-tile, single-group rows, long rows) in one launch
    shapes = [("a", 8, 128), ("b", 24, 256), ("c", 4104, 384), ("d", 640, 2560),
              ("e", 136, 1152), ("f", 2048, 32768), ("g", 8, 30720)]
    projs = list(make_binary_projections(shapes, M=1, seed=91))
    ds = [BinDev(p) for p in projs]
    tq.tq_gemv_binary_stack([d.proj() for d in ds], 1)
    torch.cuda.synchronize()
    for d in ds:
        d.check(threads=THREADS)


def test_one_token_degenerate(cuda_device):
    ps = list(make_binary_projections([("a", 640, 1280), ("b", 264, 1280)], M=1, seed=92))
    ps[0].w[:] = 1                      # all +1: acc = x_sum
    ps[1].x_bf16[0] = 0                 # a zero token: x_scale 0, acc 0, y 0
    for p in ps:
        d = BinDev(p)
        tq.tq_gemv_binary(d.bits, d.sp, d.xq, d.xs, d.y, d.acc, 1, p.N, p.K)
        torch.cuda.synchronize()
        d.check()
        if p.name == "a":
            assert (d.acc.cpu().numpy() == d.xsum.cpu().numpy()[:, None]).all()
        else:
            assert not d.acc.cpu().numpy().any() and not d.y.cpu().numpy().any()
