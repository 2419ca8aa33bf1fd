"""ctypes wrapper over the CPU oracle (``oracle.c``).

TEST INFRASTRUCTURE: imported only by ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline / reference leg. The product package never
imports it.

``build()`` compiles ``oracle.c`` with gcc into ``liboracle.so`` next to it.
Every function takes and returns numpy arrays; shapes follow ``oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]

_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile the oracle if the library is missing or older than its source."""
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            i64 = ctypes.c_int64
            p = ctypes.c_void_p
            lib.oracle_pack.argtypes = [p, p, i64, i64]
            lib.oracle_unpack.argtypes = [p, p, i64, i64]
            lib.oracle_quant.argtypes = [p, i64, i64, p, p, p]
            lib.oracle_gemv.argtypes = [p, i64, i64, p, i64, i64, i64, p]
            lib.oracle_epilogue.argtypes = [p, i64, i64, ctypes.c_float, p, p]
            lib.oracle_quant_f32.argtypes = [p, i64, i64, p, p, p]
            lib.oracle_rmsnorm.argtypes = [p, i64, i64, p, ctypes.c_float, p]
            lib.oracle_relu2_mul.argtypes = [p, p, i64, p]
            lib.oracle_absmean.argtypes = [p, i64, i64, p, p]
            lib.oracle_hadamard_rotate.argtypes = [p, i64, i64, i64, p]
            lib.oracle_quant4.argtypes = [p, i64, i64, p, p, p]
            lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
            lib.oracle_half_to_double.restype = ctypes.c_double
            lib.oracle_pack_binary.argtypes = [p, p, i64, i64]
            lib.oracle_unpack_binary.argtypes = [p, p, i64, i64]
            lib.oracle_gemv_binary.argtypes = [p, i64, i64, p, p, i64, p, i64, i64, p, p]
            for f in (lib.oracle_pack, lib.oracle_unpack, lib.oracle_quant,
                      lib.oracle_gemv, lib.oracle_epilogue, lib.oracle_quant_f32,
                      lib.oracle_rmsnorm, lib.oracle_relu2_mul, lib.oracle_absmean,
                      lib.oracle_hadamard_rotate, lib.oracle_quant4, lib.oracle_pack_binary,
                      lib.oracle_unpack_binary, lib.oracle_gemv_binary):
                f.restype = ctypes.c_int
            _lib = lib
    return _lib


class OracleError(ValueError):
    pass


def _check(rc: int, what: str):
    if rc == 1:
        raise OracleError(f"{what}: value outside the domain")
    if rc == 2:
        raise OracleError(f"{what}: bad shape")
    if rc != 0:
        raise OracleError(f"{what}: status {rc}")


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def pack(w: np.ndarray) -> np.ndarray:
    """int8 [N,K] in {-1,0,1} -> uint8 [N/4,K]."""
    w = np.ascontiguousarray(w, dtype=np.int8)
    N, K = w.shape
    if N % 4:
        raise OracleError("pack: bad shape")
    P = np.empty((N // 4, K), dtype=np.uint8)
    _check(_load().oracle_pack(_ptr(w), _ptr(P), N, K), "pack")
    return P


def unpack(P: np.ndarray, N: int) -> np.ndarray:
    """uint8 [N/4,K] -> int8 [N,K]."""
    P = np.ascontiguousarray(P, dtype=np.uint8)
    K = P.shape[1]
    if P.shape[0] * 4 != N:
        raise OracleError("unpack: bad shape")
    w = np.empty((N, K), dtype=np.int8)
    _check(_load().oracle_unpack(_ptr(P), _ptr(w), N, K), "unpack")
    return w


def quant(x_bf16: np.ndarray):
    """uint16 bf16 bits [M,K] -> (q int8 [M,K], x_scale fp32 [M], x_sum int32 [M])."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    M, K = x.shape
    q = np.empty((M, K), dtype=np.int8)
    s = np.empty(M, dtype=np.float32)
    t = np.empty(M, dtype=np.int32)
    _check(_load().oracle_quant(_ptr(x), M, K, _ptr(q), _ptr(s), _ptr(t)), "quant")
    return q, s, t


def gemv(P: np.ndarray, N: int, q: np.ndarray, n0: int = 0, n1: int | None = None) -> np.ndarray:
    """int32 acc [M, n1-n0] for output rows n0..n1-1 of the packed projection P."""
    P = np.ascontiguousarray(P, dtype=np.uint8)
    q = np.ascontiguousarray(q, dtype=np.int8)
    if q.ndim == 1:
        q = q[None, :]
    K = P.shape[1]
    M = q.shape[0]
    if q.shape[1] != K or P.shape[0] * 4 != N:
        raise OracleError("gemv: bad shape")
    if n1 is None:
        n1 = N
    acc = np.empty((M, n1 - n0), dtype=np.int32)
    _check(_load().oracle_gemv(_ptr(P), N, K, _ptr(q), M, n0, n1, _ptr(acc)), "gemv")
    return acc


def gemv_threads(P: np.ndarray, N: int, q: np.ndarray, threads: int | None = None) -> np.ndarray:
    """``gemv`` over all rows, run as disjoint row ranges on several host threads
    (the C call releases the GIL). Same function, same result; for parity runs
    on large shapes only."""
    from concurrent.futures import ThreadPoolExecutor

    q = np.ascontiguousarray(q, dtype=np.int8)
    if q.ndim == 1:
        q = q[None, :]
    threads = threads or os.cpu_count() or 1
    bounds = np.linspace(0, N, min(threads, max(1, N)) + 1).astype(np.int64)
    out = np.empty((q.shape[0], N), dtype=np.int32)

    def run(i):
        a, b = int(bounds[i]), int(bounds[i + 1])
        if b > a:
            out[:, a:b] = gemv(P, N, q, a, b)

    with ThreadPoolExecutor(len(bounds) - 1) as ex:
        list(ex.map(run, range(len(bounds) - 1)))
    return out


def epilogue(acc: np.ndarray, w_scale: float, x_scale: np.ndarray) -> np.ndarray:
    """fp64 y [M,N] = acc * w_scale * x_scale[m]."""
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    if acc.ndim == 1:
        acc = acc[None, :]
    x_scale = np.ascontiguousarray(x_scale, dtype=np.float32).reshape(-1)
    M, N = acc.shape
    y = np.empty((M, N), dtype=np.float64)
    _check(_load().oracle_epilogue(_ptr(acc), M, N, np.float32(w_scale), _ptr(x_scale), _ptr(y)),
           "epilogue")
    return y


def forward(P: np.ndarray, N: int, w_scale: float, x_bf16: np.ndarray, threads: int = 1):
    """The whole path for one projection: quant, accumulate, scale.
    Returns (q, x_scale, x_sum, acc, y)."""
    q, xs, xsum = quant(x_bf16)
    acc = gemv(P, N, q) if threads == 1 else gemv_threads(P, N, q, threads)
    y = epilogue(acc, w_scale, xs)
    return q, xs, xsum, acc, y


def quant_f32(h: np.ndarray):
    """Absmax int8 quantisation of fp32 rows h [M, K] -> (q, x_scale, x_sum)."""
    h = np.ascontiguousarray(h, dtype=np.float32)
    M, K = h.shape
    q = np.empty((M, K), np.int8)
    s = np.empty(M, np.float32)
    t = np.empty(M, np.int32)
    _check(_load().oracle_quant_f32(_ptr(h), M, K, _ptr(q), _ptr(s), _ptr(t)), "quant_f32")
    return q, s, t


def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm of fp32 rows x [M, K] with gain g [K] -> fp32 [M, K]."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    g = np.ascontiguousarray(g, dtype=np.float32)
    M, K = x.shape
    h = np.empty((M, K), np.float32)
    _check(_load().oracle_rmsnorm(_ptr(x), M, K, _ptr(g), float(eps), _ptr(h)), "rmsnorm")
    return h


def relu2_mul(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """relu(a)^2 * b elementwise, fp32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    b = np.ascontiguousarray(b, dtype=np.float32)
    h = np.empty(a.shape, np.float32)
    _check(_load().oracle_relu2_mul(_ptr(a), _ptr(b), a.size, _ptr(h)), "relu2_mul")
    return h


def absmean(W_bf16: np.ndarray):
    """Absmean ternary quantisation of bf16 latent weights [N, K] ->
    (w int8 [N, K] in {-1, 0, 1}, gamma fp32)."""
    W = np.ascontiguousarray(W_bf16, dtype=np.uint16)
    N, K = W.shape
    w = np.empty((N, K), np.int8)
    g = np.empty(1, np.float32)
    _check(_load().oracle_absmean(_ptr(W), N, K, _ptr(w), _ptr(g)), "absmean")
    return w, g[0]


# ------------------------------------------------ Hadamard-rotated 4-bit route
def hadamard_rotate(x_bf16: np.ndarray, n: int) -> np.ndarray:
    """Blockwise normalised Sylvester-Hadamard rotation of bf16 rows [M, K]
    (blocks of n along K) -> fp32 [M, K]."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    M, K = x.shape
    h = np.empty((M, K), np.float32)
    _check(_load().oracle_hadamard_rotate(_ptr(x), M, K, int(n), _ptr(h)), "hadamard_rotate")
    return h


def quant4(h: np.ndarray):
    """4-bit absmax quantisation (codes -7..7, one per int8) of fp32 rows
    h [M, K] -> (q, x_scale, x_sum)."""
    h = np.ascontiguousarray(h, dtype=np.float32)
    M, K = h.shape
    q = np.empty((M, K), np.int8)
    s = np.empty(M, np.float32)
    t = np.empty(M, np.int32)
    _check(_load().oracle_quant4(_ptr(h), M, K, _ptr(q), _ptr(s), _ptr(t)), "quant4")
    return q, s, t


def hadamard_quant4(x_bf16: np.ndarray, n: int):
    """Rotation, then the 4-bit quantiser: (q, x_scale, x_sum)."""
    return quant4(hadamard_rotate(x_bf16, n))


def forward_had4(P: np.ndarray, N: int, w_scale: float, x_bf16: np.ndarray, n: int,
                 threads: int = 1):
    """The Hadamard route for one projection: rotate, quantise to 4 bits,
    accumulate against the ternary weights, scale. Returns (q, x_scale, x_sum,
    acc, y)."""
    q, xs, xsum = hadamard_quant4(x_bf16, n)
    acc = gemv(P, N, q) if threads == 1 else gemv_threads(P, N, q, threads)
    return q, xs, xsum, acc, epilogue(acc, w_scale, xs)


# ------------------------------------------------------------ binary g128
def half_to_double(h: int) -> float:
    """fp16 bit pattern -> float, by the IEEE binary16 definition."""
    return float(_load().oracle_half_to_double(int(h)))


def pack_binary(w: np.ndarray) -> np.ndarray:
    """int8 [N,K] in {-1,+1} -> uint8 [N/8,K]."""
    w = np.ascontiguousarray(w, dtype=np.int8)
    N, K = w.shape
    if N % 8:
        raise OracleError("pack_binary: bad shape")
    B = np.empty((N // 8, K), dtype=np.uint8)
    _check(_load().oracle_pack_binary(_ptr(w), _ptr(B), N, K), "pack_binary")
    return B


def unpack_binary(B: np.ndarray, N: int) -> np.ndarray:
    """uint8 [N/8,K] -> int8 [N,K] in {-1,+1}."""
    B = np.ascontiguousarray(B, dtype=np.uint8)
    K = B.shape[1]
    if B.shape[0] * 8 != N:
        raise OracleError("unpack_binary: bad shape")
    w = np.empty((N, K), dtype=np.int8)
    _check(_load().oracle_unpack_binary(_ptr(B), _ptr(w), N, K), "unpack_binary")
    return w


def gemv_binary(B: np.ndarray, N: int, s_f16: np.ndarray, q: np.ndarray, x_scale: np.ndarray,
                n0: int = 0, n1: int | None = None):
    """(acc int32 [M, n1-n0], y fp64 [M, n1-n0]) for output rows n0..n1-1 of
    the binary projection B with fp16 group scales s_f16 [N, K/128] (uint16
    bit patterns or float16)."""
    B = np.ascontiguousarray(B, dtype=np.uint8)
    s = np.ascontiguousarray(np.asarray(s_f16).view(np.uint16))
    q = np.ascontiguousarray(q, dtype=np.int8)
    if q.ndim == 1:
        q = q[None, :]
    x_scale = np.ascontiguousarray(x_scale, dtype=np.float32).reshape(-1)
    K = B.shape[1]
    M = q.shape[0]
    if q.shape[1] != K or B.shape[0] * 8 != N or s.shape != (N, K // 128) or x_scale.size != M:
        raise OracleError("gemv_binary: bad shape")
    if n1 is None:
        n1 = N
    acc = np.empty((M, n1 - n0), np.int32)
    y = np.empty((M, n1 - n0), np.float64)
    _check(_load().oracle_gemv_binary(_ptr(B), N, K, _ptr(s), _ptr(q), M, _ptr(x_scale), n0, n1,
                                      _ptr(acc), _ptr(y)), "gemv_binary")
    return acc, y


def gemv_binary_threads(B, N, s_f16, q, x_scale, threads: int | None = None):
    """``gemv_binary`` over all rows as disjoint row ranges on several host
    threads (same function, same result; for parity runs on large shapes)."""
    from concurrent.futures import ThreadPoolExecutor

    q = np.ascontiguousarray(q, dtype=np.int8)
    if q.ndim == 1:
        q = q[None, :]
    threads = threads or os.cpu_count() or 1
    bounds = (np.linspace(0, N // 8, min(threads, max(1, N // 8)) + 1).astype(np.int64)) * 8
    acc = np.empty((q.shape[0], N), np.int32)
    y = np.empty((q.shape[0], N), np.float64)

    def run(i):
        a, b = int(bounds[i]), int(bounds[i + 1])
        if b > a:
            acc[:, a:b], y[:, a:b] = gemv_binary(B, N, s_f16, q, x_scale, a, b)

    with ThreadPoolExecutor(len(bounds) - 1) as ex:
        list(ex.map(run, range(len(bounds) - 1)))
    return acc, y


def forward_binary(B: np.ndarray, N: int, s_f16: np.ndarray, x_bf16: np.ndarray,
                   threads: int = 1):
    """The binary g128 path for one projection: int8 absmax quantisation, then
    the group-scaled accumulation. Returns (q, x_scale, x_sum, acc, y)."""
    q, xs, xsum = quant(x_bf16)
    if threads == 1:
        acc, y = gemv_binary(B, N, s_f16, q, xs)
    else:
        acc, y = gemv_binary_threads(B, N, s_f16, q, xs, threads)
    return q, xs, xsum, acc, y
