"""tq_gemv_noalloc, the entry point for callers that cannot allocate device
memory (their device memory belongs to another allocator, or an allocation's
implicit synchronisation is not acceptable on their path). It runs the
stream-K formulation of the batched-decode kernel on a fixed device array and
must give the same results as tq_gemv (the cluster formulation, no scratch) on
consecutive calls that share that array.

Collected last on purpose (file name), so that a run stopping at the first
failure has already run every other test; it also passes alone in a fresh
process.
"""
import numpy as np
import pytest
import torch

import ternary_absmax_int8_b200 as tq
from tests._gpu import assert_y_close, dev, gpu_quant, host_pack
from workloads import make_projections

pytestmark = pytest.mark.gpu


def _outputs(call, P, p, xq, xs, xsum):
    y = torch.full((p.M, p.N), float("nan"), dtype=torch.float32, device="cuda")
    acc = torch.full((p.M, p.N), -(2 ** 31), dtype=torch.int32, device="cuda")
    call(P, float(p.w_scale), xq, xs, xsum, y, acc, p.M, p.N, p.K)
    torch.cuda.synchronize()
    return y.cpu().numpy(), acc.cpu().numpy()


@pytest.mark.parametrize("M", [16, 24])
def test_noalloc_matches_tq_gemv_twice(cuda_device, M):
    # the FFN shapes of batched decode, one projection per K
    for p in make_projections([("gate_proj", 6912, 2560), ("down_proj", 2560, 6912)], M=M,
                              seed=900 + M):
        P = dev(host_pack(p.w))
        xq, xs, xsum = gpu_quant(p.x_bf16)
        y_ref, acc_ref = _outputs(tq.tq_gemv, P, p, xq, xs, xsum)
        for _ in range(2):  # the second call reuses the scratch the first one left
            y, acc = _outputs(tq.tq_gemv_noalloc, P, p, xq, xs, xsum)
            assert (acc == acc_ref).all()
            assert_y_close(y.astype(np.float64), y_ref.astype(np.float64))
    assert tq.tq_device_error(reset=True) == 0


def test_noalloc_rejects_what_its_scratch_cannot_hold(cuda_device):
    # M = 32 needs 16 KiB of scratch per 128 output features: N = 32,768 is
    # beyond the fixed 4 MiB (the limit is N <= 32,640 there).
    N, K, M = 32768, 64, 32
    P = torch.zeros((N // 4, K), dtype=torch.uint8, device="cuda")
    xq = torch.zeros((M, K), dtype=torch.int8, device="cuda")
    xs = torch.zeros(M, dtype=torch.float32, device="cuda")
    xsum = torch.zeros(M, dtype=torch.int32, device="cuda")
    y = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    with pytest.raises(tq.TQError) as e:
        tq.tq_gemv_noalloc(P, 1.0, xq, xs, xsum, y, None, M, N, K)
    assert e.value.name == "TQ_ERR_UNSUPPORTED" and "scratch" in str(e.value)
    with pytest.raises(tq.TQError):
        tq.tq_gemv_noalloc(P, 1.0, xq, xs, xsum, y, None, 4, N, K)  # M <= 4 is tq_gemv's
