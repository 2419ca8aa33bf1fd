"""GPU parity of the small-batch grouped decode calls (tq_quantize_act_stack_batch
then tq_gemv_stack_batch, M = 2..32 tokens per projection: the streaming
kernel up to 2 tokens, the warp-MMA kernel for 3..24, the tensor-core group
plan from 25) against the oracle on every output: per-token codes, scales and
sums, int32 accumulators bit-exact and fp32 outputs within the parity bar.
Each projection's M rows are independent tokens (1bit engine blog, "One GPU,
many users")."""
import numpy as np
import pytest
import torch

import oracle
import ternary_absmax_int8_b200 as tq
from tests._gpu import assert_y_close, dev, host_pack, parallel_map
from workloads import SMALL_M_SHAPES, make_projections, stack_shapes

pytestmark = pytest.mark.gpu


class BatchStack:
    """Device buffers for a list of projections of M rows each."""

    def __init__(self, projs, M):
        self.projs, self.M = projs, M
        self.P = parallel_map(lambda p: dev(host_pack(p.w)), projs)
        self.x = [dev(p.x_bf16.view(np.int16)) for p in projs]
        self.xq = [torch.full((M, p.K), -128, dtype=torch.int8, device="cuda") for p in projs]
        self.xs = [torch.full((M,), float("nan"), device="cuda") for p in projs]
        self.xsum = [torch.full((M,), -(2 ** 31), dtype=torch.int32, device="cuda")
                     for p in projs]
        self.y = [torch.full((M, p.N), float("nan"), device="cuda") for p in projs]
        self.acc = [torch.full((M, p.N), -1, dtype=torch.int32, device="cuda") for p in projs]
        self.table = [
            tq.make_proj(packed=self.P[j], x=self.x[j], xq=self.xq[j], x_scale=self.xs[j],
                         x_sum=self.xsum[j], y=self.y[j], acc_out=self.acc[j],
                         w_scale=p.w_scale, N=p.N, K=p.K)
            for j, p in enumerate(projs)]

    def run(self, flags=0):
        tq.tq_quantize_act_stack_batch(self.table, self.M)
        tq.tq_gemv_stack_batch(self.table, self.M, flags=flags)
        torch.cuda.synchronize()


def _oracle(p):
    return oracle.forward(oracle.pack(p.w), p.N, p.w_scale, p.x_bf16)


def _check(st, refs):
    for j, (p, r) in enumerate(zip(st.projs, refs)):
        q, rxs, rxsum, racc, ry = r
        assert np.array_equal(st.xq[j].cpu().numpy(), q), p.name
        assert np.array_equal(st.xs[j].cpu().numpy().view(np.uint32), rxs.view(np.uint32)), p.name
        assert np.array_equal(st.xsum[j].cpu().numpy(), rxsum), p.name
        acc = st.acc[j].cpu().numpy()
        assert np.array_equal(acc, racc), (p.name, np.argwhere(acc != racc)[:4].tolist())
        assert_y_close(st.y[j].cpu().numpy(), ry)


@pytest.mark.parametrize("M", [2, 3, 4])
def test_ffn_projections_batched(cuda_device, M):
    # gate/up [6912 x 2560] and down [2560 x 6912] in one launch, M tokens each
    projs = list(make_projections(SMALL_M_SHAPES, M=M, seed=20 + M))
    st = BatchStack(projs, M)
    refs = parallel_map(_oracle, projs)
    st.run()
    _check(st, refs)
    st.run(tq.TQ_STACK_OVERLAP_PREV)
    _check(st, refs)
    assert tq.tq_device_error(reset=True) == 0


@pytest.mark.parametrize("M", [2, 4])
def test_layer_stack_batched(cuda_device, M):
    projs = list(make_projections(stack_shapes(2), M=M, seed=7))
    st = BatchStack(projs, M)
    refs = parallel_map(_oracle, projs)
    st.run()
    _check(st, refs)


def test_batch_of_one_is_the_stack(cuda_device):
    projs = list(make_projections(stack_shapes(1), M=1, seed=8))
    st = BatchStack(projs, 1)
    refs = parallel_map(_oracle, projs)
    st.run()
    _check(st, refs)
    y0 = [y.clone() for y in st.y]
    tq.tq_gemv_stack(st.table)
    torch.cuda.synchronize()
    for a, b in zip(y0, st.y):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))


def test_mixed_stack_batched_more_than_one_launch(cuda_device):
    # 300 projections of assorted shapes at M = 3: two GEMV launches; 900
    # token rows in one quantiser launch (a CTA per row).
    shapes = [(f"p{j}", 4 * (1 + (j * 37) % 97), 16 * (1 + (j * 11) % 40)) for j in range(300)]
    projs = list(make_projections(shapes, M=3, seed=12))
    st = BatchStack(projs, 3)
    refs = parallel_map(_oracle, projs)
    st.run()
    _check(st, refs)


def test_batched_degenerate_rows(cuda_device):
    # A zero token next to live ones, a token of +-max entries, all-(+1)
    # weights and an all-zero weight block.
    projs = list(make_projections([("a", 640, 2560), ("b", 2560, 6912), ("c", 64, 512)],
                                  M=4, seed=9))
    projs[0].x_bf16[1] = 0
    projs[1].x_bf16[2] = np.where(np.arange(6912) % 2 == 0, 0x4120, 0xC120).astype(np.uint16)
    projs[2].w[:] = 1
    projs[0].w[: 320] = 0
    st = BatchStack(projs, 4)
    refs = parallel_map(_oracle, projs)
    st.run()
    _check(st, refs)


# ------------------- 5 <= M <= 24: warp MMA; 25 <= M <= 32: the group plan
@pytest.mark.parametrize("M", [5, 8, 16, 17, 24, 25, 32])
def test_ffn_projections_warp_mma_and_group_plan(cuda_device, M):
    # gate/up and down in one launch; up to 24 tokens the warp-MMA kernel
    # (one, two or three token groups), from 25 the tensor-core group plan,
    # whose tiles of 10 and 27 K units share one stream-K partition, so some
    # tiles are split between CTAs.
    projs = list(make_projections(SMALL_M_SHAPES, M=M, seed=40 + M))
    st = BatchStack(projs, M)
    refs = parallel_map(_oracle, projs)
    st.run()
    _check(st, refs)
    # the scratch is left zeroed: a second call gives identical results
    y0 = [y.clone() for y in st.y]
    tq.tq_gemv_stack_batch(st.table, M, flags=tq.TQ_STACK_OVERLAP_PREV)
    torch.cuda.synchronize()
    for a, b in zip(y0, st.y):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    assert tq.tq_device_error(reset=True) == 0


def test_many_launches_mixed_shapes(cuda_device):
    # 40 projections, assorted N and K including K of one unit and ragged
    # tiles, at M = 8 and M = 20 (warp MMA) and then M = 28 (group plan).
    shapes = [(f"p{j}", 4 * (1 + (j * 53) % 700), 16 * (1 + (j * 29) % 300)) for j in range(40)]
    shapes[3] = ("k16", 512, 16)
    shapes[7] = ("n4", 4, 2560)
    for M, seed in ((8, 13), (20, 14), (28, 12)):
        projs = list(make_projections(shapes, M=M, seed=seed))
        st = BatchStack(projs, M)
        refs = parallel_map(_oracle, projs)
        st.run()
        _check(st, refs)


@pytest.mark.parametrize("M", [12, 20, 28])
def test_degenerate_rows(cuda_device, M):
    # a zero token, a token of alternating +-10, all-+1 and all-zero weight
    # blocks; warp MMA (12 and 20 tokens) and group plan (28)
    projs = list(make_projections([("a", 640, 2560), ("b", 2560, 6912), ("c", 64, 512)],
                                  M=M, seed=15 + M))
    projs[0].x_bf16[3] = 0
    projs[1].x_bf16[11] = np.where(np.arange(6912) % 2 == 0, 0x4120, 0xC120).astype(np.uint16)
    projs[2].w[:] = 1
    projs[0].w[: 320] = 0
    st = BatchStack(projs, M)
    refs = parallel_map(_oracle, projs)
    st.run()
    _check(st, refs)


def test_group_plan_after_a_reported_device_error(cuda_device):
    # A bounded wait that gives up sets the device error word; reading it
    # makes the next group call (28 tokens) zero-fill its scratch first.
    tq.tq_selftest_wait_timeout(200)
    assert tq.tq_device_error(reset=True) != 0
    projs = list(make_projections(SMALL_M_SHAPES, M=28, seed=16))
    st = BatchStack(projs, 28)
    refs = parallel_map(_oracle, projs)
    st.run()
    _check(st, refs)
    assert tq.tq_device_error(reset=True) == 0


@pytest.mark.parametrize("layers,M", [(1, 12), (2, 4), (3, 8), (4, 4), (2, 12), (2, 20)])
def test_layer_stacks_team_sizes(cuda_device, layers, M):
    # 1 to 4 decoder layers (356 to 1424 tiles, up to 3 to 12 per CTA) give
    # the warp-MMA kernel teams of 4 (of 12 warps), 5 and 3 (of 16: one warp
    # idle), 2 and 2 (three token groups); every output against the oracle.
    projs = list(make_projections(stack_shapes(layers), M=M, seed=60 + 7 * layers + M))
    st = BatchStack(projs, M)
    refs = parallel_map(_oracle, projs)
    st.run()
    _check(st, refs)
    assert tq.tq_device_error(reset=True) == 0


def test_full_stack_30_layers_m16_warp_mma(cuda_device):
    # The launch configuration bench.py times for stack30_m16: all 210
    # projections of the 30-layer stack at 16 tokens in one warp-MMA launch;
    # every output against the oracle.
    projs = list(make_projections(stack_shapes(30), M=16, seed=17))
    st = BatchStack(projs, 16)
    refs = parallel_map(_oracle, projs)
    st.run(tq.TQ_STACK_OVERLAP_PREV)
    _check(st, refs)
    assert tq.tq_device_error(reset=True) == 0


def test_full_stack_30_layers_m4_warp_mma(cuda_device):
    # bench.py's stack30_m4: all 210 projections at 4 tokens in one warp-MMA
    # launch; every output against the oracle.
    projs = list(make_projections(stack_shapes(30), M=4, seed=18))
    st = BatchStack(projs, 4)
    refs = parallel_map(_oracle, projs)
    st.run()
    _check(st, refs)
    assert tq.tq_device_error(reset=True) == 0


def test_full_stack_30_layers_m24_warp_mma(cuda_device):
    # bench.py's stack30_m24: all 210 projections at 24 tokens in one
    # warp-MMA launch (three token groups); every output against the oracle.
    projs = list(make_projections(stack_shapes(30), M=24, seed=19))
    st = BatchStack(projs, 24)
    refs = parallel_map(_oracle, projs)
    st.run(tq.TQ_STACK_OVERLAP_PREV)
    _check(st, refs)
    assert tq.tq_device_error(reset=True) == 0


def test_stack_10_layers_m32_group_plan(cuda_device):
    # 70 projections at 32 tokens: two tensor-core group launches (64 + 6
    # projections), each over one stream-K partition; every output.
    projs = list(make_projections(stack_shapes(10), M=32, seed=20))
    st = BatchStack(projs, 32)
    refs = parallel_map(_oracle, projs)
    st.run(tq.TQ_STACK_OVERLAP_PREV)
    _check(st, refs)
    assert tq.tq_device_error(reset=True) == 0


def test_stack_quantiser_warp_rows_and_two_launches(cuda_device):
    # 600 projections x 4 rows of assorted K: the first launch (512
    # projections, 2048 rows) takes a warp per row, the second (88
    # projections, 352 rows) a CTA per row; every code, scale and sum against
    # the oracle's quantiser.
    M = 4
    rng = np.random.default_rng(44)
    from workloads import activations_bf16
    xs_in = [activations_bf16(rng, M, 16 * (1 + (j * 13) % 64)) for j in range(600)]
    xd = [dev(x.view(np.int16)) for x in xs_in]
    xq = [torch.full((M, x.shape[1]), -128, dtype=torch.int8, device="cuda") for x in xs_in]
    xs = [torch.full((M,), float("nan"), device="cuda") for _ in xs_in]
    xsum = [torch.full((M,), -(2 ** 31), dtype=torch.int32, device="cuda") for _ in xs_in]
    table = [tq.make_proj(x=xd[j], xq=xq[j], x_scale=xs[j], x_sum=xsum[j], N=0, K=x.shape[1])
             for j, x in enumerate(xs_in)]
    tq.tq_quantize_act_stack_batch(table, M)
    torch.cuda.synchronize()
    for j, x in enumerate(xs_in):
        rq, rxs, rxsum = oracle.quant(x)
        assert np.array_equal(xq[j].cpu().numpy(), rq), j
        assert np.array_equal(xs[j].cpu().numpy().view(np.uint32), rxs.view(np.uint32)), j
        assert np.array_equal(xsum[j].cpu().numpy(), rxsum), j

