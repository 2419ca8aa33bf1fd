"""GPU parity of tq_gemm_prefill_stack: several projections of a prompt in one
launch whose tiles are dealt to the CTAs longest first (1bit engine blog,
"Qwen3.8-27B at 45.7 tok/s ...": prefill is set by the matrix units). Each
projection's outputs must equal tq_gemm_prefill's bit for bit and the
oracle's (int32 accumulators bit-exact, fp32 outputs within 1e-5 relative):
the three prefill shapes at 512 tokens (the bench's launch), ragged shapes at
a token count that is not a multiple of the tile, more projections than one
launch takes, empty entries, and the small-batch route (M <= 32)."""
import numpy as np
import pytest
import torch

import ternary_absmax_int8_b200 as tq
from tests._gpu import assert_parity, dev, gpu_quant, host_pack, oracle_forward
from workloads import PREFILL_M, PREFILL_SHAPES, activations_bf16, make_projections, \
    stored_weight_scale, ternary_weights

pytestmark = pytest.mark.gpu


class Proj:
    """Device operands of one projection, its grouped-call entry and a
    separate tq_gemm_prefill call on the same inputs."""

    def __init__(self, w, ws, xb):
        self.w, self.ws, self.xb = w, float(ws), xb
        self.M, self.K = xb.shape
        self.N = w.shape[0]
        self.P = dev(host_pack(w)) if self.N and self.K else torch.zeros(16, dtype=torch.uint8,
                                                                          device="cuda")
        self.xq, self.xs, self.xsum = gpu_quant(xb)
        self.y = torch.full((self.M, self.N), float("nan"), device="cuda")
        self.acc = torch.full((self.M, self.N), -(2 ** 31), dtype=torch.int32, device="cuda")

    def entry(self):
        return tq.make_proj(packed=self.P, xq=self.xq, x_scale=self.xs, x_sum=self.xsum,
                            y=self.y, acc_out=self.acc, w_scale=self.ws, N=self.N, K=self.K)

    def got(self, rows=None):
        g = (self.xq.cpu().numpy(), self.xs.cpu().numpy(), self.xsum.cpu().numpy(),
             self.acc.cpu().numpy(), self.y.cpu().numpy())
        return g if rows is None else tuple(a[rows] for a in g)

    def single(self):
        y = torch.full_like(self.y, float("nan"))
        acc = torch.full_like(self.acc, -(2 ** 31))
        tq.tq_gemm_prefill(self.P, self.ws, self.xq, self.xs, self.xsum, y, acc, self.M, self.N,
                           self.K)
        torch.cuda.synchronize()
        return acc.cpu().numpy(), y.cpu().numpy()


def _same_as_single(p):
    acc, y = p.single()
    assert np.array_equal(acc, p.acc.cpu().numpy())
    assert np.array_equal(y.view(np.uint32), p.y.cpu().numpy().view(np.uint32))


def test_three_prefill_shapes_one_launch(cuda_device):
    # The bench's prefill_m512 launch: 6912x2560, 2560x6912 and 17408x5120 at
    # 512 tokens. Every output against tq_gemm_prefill (itself checked against
    # the oracle in full); all token rows of the two smaller shapes and 48
    # token rows of the largest against the oracle.
    ps = [Proj(p.w, p.w_scale, p.x_bf16)
          for p in make_projections(PREFILL_SHAPES, M=PREFILL_M, seed=3)]
    tq.tq_gemm_prefill_stack([p.entry() for p in ps], PREFILL_M)
    torch.cuda.synchronize()
    rows = np.r_[0:16, 240:272, 496:512][:48]
    for p in ps:
        _same_as_single(p)
        if p.N * p.K > 20_000_000:
            assert_parity(p.got(rows), oracle_forward(p.w, p.ws, p.xb[rows]), f"{p.N}x{p.K}")
        else:
            assert_parity(p.got(), oracle_forward(p.w, p.ws, p.xb), f"{p.N}x{p.K}")
    assert tq.tq_device_error(reset=True) == 0


@pytest.mark.parametrize("M", [300, 100])
def test_ragged_group(cuda_device, M):
    # shapes with partial feature tiles, K not a multiple of the 128-byte
    # stage, and M not a multiple of the token tile (256, or 128 at M <= 128)
    shapes = [(516, 272), (4, 16), (2564, 1168), (260, 2560), (1028, 128)]
    rng = np.random.default_rng(M)
    ps = []
    for N, K in shapes:
        w = ternary_weights(rng, N, K)
        ps.append(Proj(w, stored_weight_scale(w), activations_bf16(rng, M, K)))
    tq.tq_gemm_prefill_stack([p.entry() for p in ps], M)
    torch.cuda.synchronize()
    for p in ps:
        assert_parity(p.got(), oracle_forward(p.w, p.ws, p.xb), f"{p.N}x{p.K} M={M}")
        _same_as_single(p)


def test_more_projections_than_a_launch_and_empty_entries(cuda_device):
    # 19 projections (16 per launch), among them one with N = 0 and one with
    # K = 0 (outputs zero-filled)
    M = 64
    rng = np.random.default_rng(9)
    ps = []
    for j in range(19):
        N = 0 if j == 4 else 128 * (1 + j % 5)
        K = 256 * (1 + j % 3)
        w = ternary_weights(rng, N, K)
        p = Proj(w, stored_weight_scale(w) if N else 1.0, activations_bf16(rng, M, K))
        if j == 7:
            p.K = 0  # valid buffers, no columns: the call zero-fills y and acc
        ps.append(p)
    tq.tq_gemm_prefill_stack([p.entry() for p in ps], M)
    torch.cuda.synchronize()
    for j, p in enumerate(ps):
        if p.N == 0:
            continue
        if p.K == 0:
            assert not p.acc.cpu().numpy().any() and not p.y.cpu().numpy().any()
            continue
        assert_parity(p.got(), oracle_forward(p.w, p.ws, p.xb), f"entry {j}")


def test_small_batch_route(cuda_device):
    # M <= 32 runs the batched-decode kernels
    M = 20
    ps = [Proj(p.w, p.w_scale, p.x_bf16)
          for p in make_projections(PREFILL_SHAPES[:2], M=M, seed=21)]
    tq.tq_gemm_prefill_stack([p.entry() for p in ps], M)
    torch.cuda.synchronize()
    for p in ps:
        assert_parity(p.got(), oracle_forward(p.w, p.ws, p.xb), f"{p.N}x{p.K} M={M}")
