"""Helpers for the GPU parity tests: run the product path through the C ABI and
the oracle on the same seeded inputs, then compare.

Bar (from the method's statement of correctness): int8 codes, int32
accumulators and the per-token sums bit-exact; x_scale exactly equal (a
correctly rounded fp32 divide on both sides); fp32 outputs within 1e-5
relative error of the oracle's fp64 product, and exactly 0 where it is 0.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle
import ternary_absmax_int8_b200 as tq

Y_RTOL = 1e-5
THREADS = os.cpu_count() or 1


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host_pack(w: np.ndarray) -> np.ndarray:
    N, K = w.shape
    P = np.empty((N // 4, K), dtype=np.uint8)
    tq.tq_pack_host(w, P, 1, N, K)
    return P


def gpu_quant(x_bf16: np.ndarray):
    M, K = x_bf16.shape
    x = dev(x_bf16.view(np.int16))
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    xs = torch.empty(M, dtype=torch.float32, device="cuda")
    xsum = torch.empty(M, dtype=torch.int32, device="cuda")
    tq.tq_quantize_act(x, xq, xs, xsum, M, 0, K)
    return xq, xs, xsum


def gpu_forward(P: np.ndarray, N: int, w_scale, x_bf16: np.ndarray, call=None):
    """Product path for one projection: quantise then GEMV. Returns numpy
    (q, x_scale, x_sum, acc, y)."""
    M, K = x_bf16.shape
    call = call or (tq.tq_gemv if M <= 24 else tq.tq_gemm_prefill)
    xq, xs, xsum = gpu_quant(x_bf16)
    Pd = dev(P)
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    acc = torch.full((M, N), -(2 ** 31), dtype=torch.int32, device="cuda")
    call(Pd, float(w_scale), xq, xs, xsum, y, acc, M, N, K)
    torch.cuda.synchronize()
    return (xq.cpu().numpy(), xs.cpu().numpy(), xsum.cpu().numpy(), acc.cpu().numpy(),
            y.cpu().numpy())


def oracle_forward(w: np.ndarray, w_scale, x_bf16: np.ndarray, threads: int = THREADS):
    N = w.shape[0]
    P = oracle.pack(w)
    return oracle.forward(P, N, w_scale, x_bf16, threads=threads)


def assert_y_close(y: np.ndarray, ref: np.ndarray, rtol: float = Y_RTOL):
    y64 = y.astype(np.float64)
    zero = ref == 0
    assert (y64[zero] == 0).all(), "nonzero output where the oracle gives 0"
    rel = np.abs(y64[~zero] - ref[~zero]) / np.abs(ref[~zero])
    assert rel.size == 0 or rel.max() <= rtol, f"max rel err {rel.max():.3e}"


def assert_parity(gpu, ref, what=""):
    q, xs, xsum, acc, y = gpu
    rq, rxs, rxsum, racc, ry = ref
    assert (q == rq).all(), f"{what}: int8 codes differ"
    assert (xs.view(np.uint32) == rxs.view(np.uint32)).all(), f"{what}: x_scale differs"
    assert (xsum == rxsum).all(), f"{what}: x_sum differs"
    bad = np.argwhere(acc != racc)
    assert bad.size == 0, f"{what}: {len(bad)} accumulators differ, first at {bad[:4].tolist()}"
    assert_y_close(y, ry)


def parallel_map(fn, items, threads: int = THREADS):
    with ThreadPoolExecutor(max(1, threads)) as ex:
        return list(ex.map(fn, items))
