"""Python binding of libtq (include/tq.h): the same names, argument marshalling only.

Every function forwards to the C ABI of the in-tree ``libtq.so``; all work runs
in its CUDA kernels. Tensors are passed as raw pointers (``data_ptr()``), an
``int`` is taken as a raw pointer, ``None`` as NULL. ``stream`` defaults to
PyTorch's current CUDA stream. A non-OK status raises :class:`TQError`.

There is no fallback: if ``libtq.so`` is missing, every call raises (the
package itself still imports, so that its ``build`` module can run). Build it
with ``python -m ternary_absmax_int8_b200.build``.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "TQError", "TQ_STACK_OVERLAP_PREV", "TQ_STACK_QUANTIZE", "TQ_STACK_RMSNORM",
    "TQ_STACK_RELU2_MUL", "TqProj", "lib_path",
    "tq_pack_host", "tq_quantize_act", "tq_gemv", "tq_gemm_prefill",
    "tq_quantize_act_stack", "tq_gemv_stack", "tq_quantize_act_stack_batch",
    "tq_gemv_stack_batch", "tq_gemm_prefill_stack", "tq_device_error", "tq_gemv_noalloc",
    "tq_status_string", "tq_last_error", "make_proj", "tq_rmsnorm_quantize",
    "tq_relu2_mul_rmsnorm_quantize", "tq_absmean_pack", "tq_selftest_wait_timeout",
    "tq_hadamard_quantize_act", "tq_hadamard_quantize_act_stack", "TqBinaryProj",
    "tq_pack_binary_host", "tq_gemv_binary",
    "tq_gemv_binary_stack", "make_binary_proj",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libtq.so")

TQ_STACK_OVERLAP_PREV = 1
TQ_STACK_QUANTIZE = 2
TQ_STACK_RMSNORM = 4
TQ_STACK_RELU2_MUL = 8
_STATUS = {0: "TQ_OK", 1: "TQ_ERR_NULL", 2: "TQ_ERR_SHAPE", 3: "TQ_ERR_ALIGN",
           4: "TQ_ERR_VALUE", 5: "TQ_ERR_CUDA", 6: "TQ_ERR_UNSUPPORTED"}


class TQError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        self.name = _STATUS.get(status, f"status {status}")
        super().__init__(f"{self.name}: {message}")


_vp, _i, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float


class TqProj(ctypes.Structure):
    """Mirror of ``struct tq_proj``."""
    _fields_ = [
        ("packed", ctypes.c_void_p),
        ("x", ctypes.c_void_p),
        ("xq", ctypes.c_void_p),
        ("x_scale", ctypes.c_void_p),
        ("x_sum", ctypes.c_void_p),
        ("y", ctypes.c_void_p),
        ("acc_out", ctypes.c_void_p),
        ("w_scale", ctypes.c_float),
        ("N", ctypes.c_int),
        ("K", ctypes.c_int),
        ("gain", ctypes.c_void_p),
        ("x_f32", ctypes.c_void_p),
        ("up", ctypes.c_void_p),
        ("eps", ctypes.c_float),
        ("reserved", ctypes.c_int),
    ]


class TqBinaryProj(ctypes.Structure):
    """Mirror of ``struct tq_binary_proj``."""
    _fields_ = [
        ("bits", ctypes.c_void_p),
        ("scales_packed", ctypes.c_void_p),
        ("xq", ctypes.c_void_p),
        ("x_scale", ctypes.c_void_p),
        ("y", ctypes.c_void_p),
        ("acc_out", ctypes.c_void_p),
        ("N", ctypes.c_int),
        ("K", ctypes.c_int),
    ]


_SIGS = {
    "tq_pack_host": [_vp, _vp, _i, _i, _i, _vp],
    "tq_quantize_act": [_vp, _vp, _vp, _vp, _i, _i, _i, _vp],
    "tq_gemv": [_vp, _f, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _vp],
    "tq_gemm_prefill": [_vp, _f, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _vp],
    "tq_gemv_noalloc": [_vp, _f, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _vp],
    "tq_quantize_act_stack": [ctypes.POINTER(TqProj), _i, _vp],
    "tq_gemv_stack": [ctypes.POINTER(TqProj), _i, ctypes.c_uint, _vp],
    "tq_quantize_act_stack_batch": [ctypes.POINTER(TqProj), _i, _i, _vp],
    "tq_gemv_stack_batch": [ctypes.POINTER(TqProj), _i, _i, ctypes.c_uint, _vp],
    "tq_gemm_prefill_stack": [ctypes.POINTER(TqProj), _i, _i, _vp],
    "tq_device_error": [ctypes.POINTER(ctypes.c_uint32), _i],
    "tq_rmsnorm_quantize": [_vp, _vp, _vp, _f, _vp, _vp, _vp, _i, _i, _vp],
    "tq_relu2_mul_rmsnorm_quantize": [_vp, _vp, _vp, _f, _vp, _vp, _vp, _i, _i, _vp],
    "tq_absmean_pack": [_vp, _vp, _vp, _i, _i, _vp],
    "tq_selftest_wait_timeout": [ctypes.c_uint, _vp],
    "tq_hadamard_quantize_act": [_vp, _vp, _vp, _vp, _i, _i, _i, _vp],
    "tq_hadamard_quantize_act_stack": [ctypes.POINTER(TqProj), _i, _i, _i, _vp],
    "tq_pack_binary_host": [_vp, _vp, _vp, _vp, _i, _i],
    "tq_gemv_binary": [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _vp],
    "tq_gemv_binary_stack": [ctypes.POINTER(TqBinaryProj), _i, _i, _vp],
}
_lib_handle = None


def _load():
    """Load libtq.so once; raise loudly if it has not been built."""
    global _lib_handle
    if _lib_handle is None:
        if not os.path.exists(lib_path):
            raise RuntimeError(
                f"{lib_path} is missing: build it with `python -m ternary_absmax_int8_b200.build`"
                " (there is no CPU fallback)")
        lib = ctypes.CDLL(lib_path)
        for name, args in _SIGS.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        lib.tq_status_string.argtypes = [ctypes.c_int]
        lib.tq_status_string.restype = ctypes.c_char_p
        lib.tq_last_error.argtypes = []
        lib.tq_last_error.restype = ctypes.c_char_p
        _lib_handle = lib
    return _lib_handle


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if hasattr(t, "data_ptr"):
        return t.data_ptr()
    if hasattr(t, "ctypes"):  # numpy array
        return t.ctypes.data
    raise TypeError(f"cannot pass {type(t).__name__} as a pointer")


def _stream(stream):
    if stream is None:
        import torch
        if not torch.cuda.is_available():
            return None
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int):
    if rc != 0:
        raise TQError(rc, _load().tq_last_error().decode())


def tq_status_string(status: int) -> str:
    return _load().tq_status_string(status).decode()


def tq_last_error() -> str:
    return _load().tq_last_error().decode()


def tq_pack_host(w, packed, M: int, N: int, K: int, stream=0) -> None:
    """Host packing: w int8 [N,K] (CPU tensor or numpy) -> packed uint8 [N/4,K]."""
    _check(_load().tq_pack_host(_ptr(w), _ptr(packed), M, N, K, None))


def tq_quantize_act(x, xq, x_scale, x_sum, M: int, N: int, K: int, stream=None) -> None:
    _check(_load().tq_quantize_act(_ptr(x), _ptr(xq), _ptr(x_scale), _ptr(x_sum), M, N, K,
                                _stream(stream)))


def tq_gemv(packed, w_scale: float, xq, x_scale, x_sum, y, acc_out, M: int, N: int, K: int,
            stream=None) -> None:
    _check(_load().tq_gemv(_ptr(packed), float(w_scale), _ptr(xq), _ptr(x_scale), _ptr(x_sum),
                        _ptr(y), _ptr(acc_out), M, N, K, _stream(stream)))


def tq_gemm_prefill(packed, w_scale: float, xq, x_scale, x_sum, y, acc_out, M: int, N: int,
                    K: int, stream=None) -> None:
    _check(_load().tq_gemm_prefill(_ptr(packed), float(w_scale), _ptr(xq), _ptr(x_scale),
                                _ptr(x_sum), _ptr(y), _ptr(acc_out), M, N, K, _stream(stream)))


def tq_gemv_noalloc(packed, w_scale: float, xq, x_scale, x_sum, y, acc_out, M: int, N: int,
                    K: int, stream=None) -> None:
    """tq_gemv for 5 <= M <= 32 on fixed library scratch (allocates nothing)."""
    _check(_load().tq_gemv_noalloc(_ptr(packed), float(w_scale), _ptr(xq), _ptr(x_scale),
                                _ptr(x_sum), _ptr(y), _ptr(acc_out), M, N, K, _stream(stream)))


def tq_rmsnorm_quantize(x_bf16, x_f32, gain, eps: float, xq, x_scale, x_sum, M: int, K: int,
                        stream=None) -> None:
    """RMSNorm (gain, eps) then the absmax quantiser; exactly one of x_bf16 / x_f32."""
    _check(_load().tq_rmsnorm_quantize(_ptr(x_bf16), _ptr(x_f32), _ptr(gain), float(eps),
                                    _ptr(xq), _ptr(x_scale), _ptr(x_sum), M, K,
                                    _stream(stream)))


def tq_relu2_mul_rmsnorm_quantize(gate, up, gain, eps: float, xq, x_scale, x_sum, M: int,
                                  K: int, stream=None) -> None:
    """relu(gate)^2 * up, RMSNorm (gain, eps), then the absmax quantiser."""
    _check(_load().tq_relu2_mul_rmsnorm_quantize(_ptr(gate), _ptr(up), _ptr(gain), float(eps),
                                              _ptr(xq), _ptr(x_scale), _ptr(x_sum), M, K,
                                              _stream(stream)))


def tq_absmean_pack(w_bf16, packed, w_scale, N: int, K: int, stream=None) -> None:
    """Absmean ternary quantisation of bf16 weights [N,K] -> packed [N/4,K], w_scale [1]."""
    _check(_load().tq_absmean_pack(_ptr(w_bf16), _ptr(packed), _ptr(w_scale), N, K,
                                _stream(stream)))


def tq_selftest_wait_timeout(limit_us: int, stream=None) -> None:
    """A bounded wait that nothing satisfies: sets the device error word."""
    _check(_load().tq_selftest_wait_timeout(int(limit_us), _stream(stream)))


def tq_hadamard_quantize_act(x, xq, x_scale, x_sum, M: int, K: int, n: int,
                             stream=None) -> None:
    """Blockwise Hadamard rotation (block n) then 4-bit absmax codes (-7..7 in int8)."""
    _check(_load().tq_hadamard_quantize_act(_ptr(x), _ptr(xq), _ptr(x_scale), _ptr(x_sum), M, K,
                                         int(n), _stream(stream)))


def tq_hadamard_quantize_act_stack(projs, M: int, n: int, stream=None) -> None:
    arr, cnt = _proj_array(projs)
    _check(_load().tq_hadamard_quantize_act_stack(arr, cnt, int(M), int(n), _stream(stream)))


def tq_pack_binary_host(w, scales, bits, scales_packed, N: int, K: int) -> None:
    """Host packing of binary g128 weights: w int8 [N,K] in {-1,+1}, fp16 scales
    [N,K/128] -> bits uint8 [N/8,K], scales_packed fp16 [N/8,K/128,8]."""
    _check(_load().tq_pack_binary_host(_ptr(w), _ptr(scales), _ptr(bits), _ptr(scales_packed),
                                    int(N), int(K)))


def tq_gemv_binary(bits, scales_packed, xq, x_scale, y, acc_out, M: int, N: int, K: int,
                   stream=None) -> None:
    _check(_load().tq_gemv_binary(_ptr(bits), _ptr(scales_packed), _ptr(xq), _ptr(x_scale),
                               _ptr(y), _ptr(acc_out), M, N, K, _stream(stream)))


def make_binary_proj(bits=None, scales_packed=None, xq=None, x_scale=None, y=None, acc_out=None,
                     N: int = 0, K: int = 0) -> TqBinaryProj:
    return TqBinaryProj(_ptr(bits), _ptr(scales_packed), _ptr(xq), _ptr(x_scale), _ptr(y),
                        _ptr(acc_out), int(N), int(K))


def tq_gemv_binary_stack(projs, M: int, stream=None) -> None:
    arr = (TqBinaryProj * len(projs))(*projs)
    _check(_load().tq_gemv_binary_stack(arr, len(projs), int(M), _stream(stream)))


def make_proj(packed=None, x=None, xq=None, x_scale=None, x_sum=None, y=None, acc_out=None,
              w_scale: float = 0.0, N: int = 0, K: int = 0, gain=None, x_f32=None, up=None,
              eps: float = 0.0) -> TqProj:
    return TqProj(_ptr(packed), _ptr(x), _ptr(xq), _ptr(x_scale), _ptr(x_sum), _ptr(y),
                  _ptr(acc_out), float(w_scale), int(N), int(K), _ptr(gain), _ptr(x_f32),
                  _ptr(up), float(eps), 0)


def _proj_array(projs):
    arr = (TqProj * len(projs))(*projs)
    return arr, len(projs)


def tq_quantize_act_stack(projs, stream=None) -> None:
    arr, n = _proj_array(projs)
    _check(_load().tq_quantize_act_stack(arr, n, _stream(stream)))


def tq_gemv_stack(projs, flags: int = 0, stream=None) -> None:
    arr, n = _proj_array(projs)
    _check(_load().tq_gemv_stack(arr, n, int(flags), _stream(stream)))


def tq_quantize_act_stack_batch(projs, M: int, stream=None) -> None:
    arr, n = _proj_array(projs)
    _check(_load().tq_quantize_act_stack_batch(arr, n, int(M), _stream(stream)))


def tq_gemv_stack_batch(projs, M: int, flags: int = 0, stream=None) -> None:
    arr, n = _proj_array(projs)
    _check(_load().tq_gemv_stack_batch(arr, n, int(M), int(flags), _stream(stream)))


def tq_gemm_prefill_stack(projs, M: int, stream=None) -> None:
    arr, n = _proj_array(projs)
    _check(_load().tq_gemm_prefill_stack(arr, n, int(M), _stream(stream)))


def tq_device_error(reset: bool = False) -> int:
    code = ctypes.c_uint32(0)
    _check(_load().tq_device_error(ctypes.byref(code), 1 if reset else 0))
    return int(code.value)
