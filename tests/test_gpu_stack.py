"""GPU parity of the grouped decode calls on the full 30-layer stack (210
projections, M = 1) against the oracle on every output: the one-launch form
the bench times (tq_gemv_stack with TQ_STACK_QUANTIZE: quantise and multiply
in the same launch) and the two-launch form (tq_quantize_act_stack, then
tq_gemv_stack, allowed to overlap it)."""
import numpy as np
import pytest
import torch

import oracle
import ternary_absmax_int8_b200 as tq
from tests._gpu import assert_y_close, dev, host_pack, parallel_map
from workloads import DECODER_LAYER, make_projections, stack_shapes

pytestmark = pytest.mark.gpu


class Stack:
    """Device buffers for a list of projections at M = 1."""

    def __init__(self, projs):
        self.projs = projs
        self.P = parallel_map(lambda p: dev(host_pack(p.w)), projs)
        self.x = [dev(p.x_bf16.view(np.int16)) for p in projs]
        self.xq = [torch.empty(p.K, dtype=torch.int8, device="cuda") for p in projs]
        self.xs = torch.empty(len(projs), dtype=torch.float32, device="cuda")
        self.xsum = torch.empty(len(projs), dtype=torch.int32, device="cuda")
        self.y = [torch.full((p.N,), float("nan"), device="cuda") for p in projs]
        self.acc = [torch.full((p.N,), -1, dtype=torch.int32, device="cuda") for p in projs]
        es, ei = self.xs.element_size(), self.xsum.element_size()
        self.table = [
            tq.make_proj(packed=self.P[j], x=self.x[j], xq=self.xq[j],
                         x_scale=self.xs.data_ptr() + j * es, x_sum=self.xsum.data_ptr() + j * ei,
                         y=self.y[j], acc_out=self.acc[j], w_scale=p.w_scale, N=p.N, K=p.K)
            for j, p in enumerate(projs)]

    def run(self, flags):
        tq.tq_quantize_act_stack(self.table)
        tq.tq_gemv_stack(self.table, flags=flags)
        torch.cuda.synchronize()

    def run_fused(self):
        # Poison the quantiser's outputs first: the fused launch must write them.
        for q in self.xq:
            q.fill_(-128)
        self.xs.fill_(float("nan"))
        self.xsum.fill_(-(2 ** 31))
        tq.tq_gemv_stack(self.table, flags=tq.TQ_STACK_QUANTIZE)
        torch.cuda.synchronize()


def _oracle(p):
    P = oracle.pack(p.w)
    return oracle.forward(P, p.N, p.w_scale, p.x_bf16)


def _check(stack, refs):
    xs = stack.xs.cpu().numpy()
    xsum = stack.xsum.cpu().numpy()
    for j, (p, r) in enumerate(zip(stack.projs, refs)):
        q, rxs, rxsum, racc, ry = r
        assert (stack.xq[j].cpu().numpy() == q[0]).all(), p.name
        assert xs[j].view(np.uint32) == rxs[0].view(np.uint32), p.name
        assert xsum[j] == rxsum[0], p.name
        acc = stack.acc[j].cpu().numpy()
        assert (acc == racc[0]).all(), (p.name, np.argwhere(acc != racc[0])[:4].tolist())
        assert_y_close(stack.y[j].cpu().numpy(), ry[0])


def test_layer_stack_small(cuda_device):
    projs = list(make_projections(stack_shapes(2), M=1, seed=3))
    st = Stack(projs)
    refs = parallel_map(_oracle, projs)
    for flags in (0, tq.TQ_STACK_OVERLAP_PREV):
        st.run(flags)
        _check(st, refs)
    st.run_fused()
    _check(st, refs)


def test_full_stack_30_layers_fused(cuda_device):
    # The bench's launch: one tq_gemv_stack(TQ_STACK_QUANTIZE) for all 210.
    projs = list(make_projections(stack_shapes(30), M=1, seed=0))
    st = Stack(projs)
    refs = parallel_map(_oracle, projs)
    st.run_fused()
    _check(st, refs)
    # repeat: byte-identical outputs
    y0 = [y.clone() for y in st.y]
    st.run_fused()
    for a, b in zip(y0, st.y):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    assert tq.tq_device_error(reset=True) == 0


def test_full_stack_30_layers_two_launches(cuda_device):
    projs = list(make_projections(stack_shapes(30), M=1, seed=0))
    st = Stack(projs)
    refs = parallel_map(_oracle, projs)
    st.run(tq.TQ_STACK_OVERLAP_PREV)
    _check(st, refs)
    assert tq.tq_device_error(reset=True) == 0


def test_fused_stack_degenerate_rows(cuda_device):
    # An all-zero token (amax = 0), a token whose every entry is +-max, and
    # all-zero / all-(+1) weights, through the quantising launch.
    projs = list(make_projections([("a", 640, 2560), ("b", 2560, 6912), ("c", 64, 512)],
                                  M=1, seed=5))
    projs[0].x_bf16[:] = 0
    projs[1].x_bf16[:] = np.where(np.arange(6912) % 2 == 0, 0x4120, 0xC120).astype(np.uint16)
    projs[2].w[:] = 1
    projs[0].w[: 320] = 0
    st = Stack(projs)
    refs = parallel_map(_oracle, projs)
    st.run_fused()
    _check(st, refs)


def test_mixed_stack_more_than_one_launch(cuda_device):
    # 400 projections of assorted shapes: more than one launch's table.
    shapes = [(f"p{j}", 4 * (1 + (j * 37) % 97), 16 * (1 + (j * 11) % 40)) for j in range(400)]
    projs = list(make_projections(shapes, M=1, seed=11))
    st = Stack(projs)
    refs = parallel_map(_oracle, projs)
    st.run(0)
    _check(st, refs)
    st.run_fused()
    _check(st, refs)
