"""tq_gemv_noalloc, the entry point for callers that cannot allocate device
memory: a process whose device memory is all owned by another allocator (a
framework's caching pool, a pre-reserved arena), or a latency-critical loop
that cannot take an allocation's implicit device synchronisation. It runs the
stream-K formulation of the batched-decode kernel, whose split-K partial sums
live in a fixed device array compiled into the library.

Each case checks two consecutive calls, which share that array, element by
element against the oracle (codes, scales and sums and int32 accumulators
bit-exact, fp32 outputs within the parity bar) and against the existing entry
point for the same M (tq_gemv up to 24 tokens, tq_gemm_prefill from 25: the
cluster formulation, no scratch).

Collected last on purpose (file name), so that a run stopping at the first
failure has already run every other test; it also passes alone in a fresh
process.
"""
import numpy as np
import pytest
import torch

import oracle
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


def _check_twice(p):
    P = dev(host_pack(p.w))
    xq, xs, xsum = gpu_quant(p.x_bf16)
    rq, rxs, rxsum, racc, ry = oracle.forward(oracle.pack(p.w), p.N, p.w_scale, p.x_bf16)
    assert np.array_equal(xq.cpu().numpy(), rq)
    assert np.array_equal(xs.cpu().numpy().view(np.uint32), rxs.view(np.uint32))
    assert np.array_equal(xsum.cpu().numpy(), rxsum)
    existing = tq.tq_gemv if p.M <= 24 else tq.tq_gemm_prefill
    y_ex, acc_ex = _outputs(existing, P, p, xq, xs, xsum)
    for call in range(2):  # the second call reuses the array the first one left
        y, acc = _outputs(tq.tq_gemv_noalloc, P, p, xq, xs, xsum)
        bad = np.argwhere(acc != racc)
        assert bad.size == 0, (p.name, p.M, call, bad[:4].tolist())
        assert_y_close(y, ry)
        assert np.array_equal(acc, acc_ex)
        assert_y_close(y.astype(np.float64), y_ex.astype(np.float64))


@pytest.mark.parametrize("M", [5, 13, 16, 24, 29, 32])
def test_noalloc_matches_oracle_and_existing_entry_twice(cuda_device, M):
    # The batched-decode FFN shapes. Spread over 148 SMs, their tiles of 10
    # and 27 K units are split between CTAs, several of them into a 1-unit
    # piece at the end or the start of a CTA's range.
    for p in make_projections([("gate_proj", 6912, 2560), ("down_proj", 2560, 6912)], M=M,
                              seed=900 + M):
        _check_twice(p)
    assert tq.tq_device_error(reset=True) == 0


def test_noalloc_small_and_ragged(cuda_device):
    # Five tiles over 50 CTAs (one unit each), and a ragged last tile.
    for p in make_projections([("k_proj", 640, 2560), ("ragged", 4 * 1001, 16 * 37)], M=9,
                              seed=950):
        _check_twice(p)
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
