"""The C ABI library loads, exports what include/tq.h declares, and its host-side
logic (argument checks, the host packer) behaves as documented. CPU only: no
call here reaches a kernel launch."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import ternary_absmax_int8_b200 as tq
from workloads import ternary_weights

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "tq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol():
    names = _declared_functions()
    assert {"tq_pack_host", "tq_quantize_act", "tq_gemv", "tq_gemm_prefill"} <= set(names)
    lib = ctypes.CDLL(tq.lib_path)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings():
    assert tq.tq_status_string(0) == "TQ_OK"
    assert tq.tq_status_string(2) == "TQ_ERR_SHAPE"
    assert tq.tq_status_string(6) == "TQ_ERR_UNSUPPORTED"


@pytest.mark.parametrize("N,K", [(4, 16), (8, 3), (640, 2560), (2560, 6912), (12, 0), (0, 16)])
def test_host_packer_matches_oracle(N, K):
    w = ternary_weights(np.random.default_rng(N * 13 + K), N, K)
    packed = np.zeros((N // 4, K), dtype=np.uint8)
    tq.tq_pack_host(w, packed, 1, N, K)
    if N and K:
        assert (packed == oracle.pack(w)).all()


def test_host_packer_rejects_bad_input():
    w = np.zeros((8, 16), dtype=np.int8)
    packed = np.zeros((2, 16), dtype=np.uint8)
    w[5, 3] = 2
    with pytest.raises(tq.TQError) as e:
        tq.tq_pack_host(w, packed, 1, 8, 16)
    assert e.value.name == "TQ_ERR_VALUE"
    w[5, 3] = -2
    with pytest.raises(tq.TQError):
        tq.tq_pack_host(w, packed, 1, 8, 16)
    with pytest.raises(tq.TQError) as e:
        tq.tq_pack_host(w, packed, 1, 6, 16)
    assert e.value.name == "TQ_ERR_SHAPE"
    with pytest.raises(tq.TQError) as e:
        tq.tq_pack_host(None, packed, 1, 8, 16)
    assert e.value.name == "TQ_ERR_NULL"


# Fake, aligned, never-dereferenced device addresses: every case below is
# rejected by the argument checks before anything is enqueued.
A = 1 << 20


def _gemv(fn, **kw):
    args = dict(packed=A, w_scale=1.0, xq=A, x_scale=A, x_sum=A, y=A, acc_out=None,
                M=1, N=640, K=2560)
    args.update(kw)
    fn(args["packed"], args["w_scale"], args["xq"], args["x_scale"], args["x_sum"], args["y"],
       args["acc_out"], args["M"], args["N"], args["K"], stream=0)


@pytest.mark.parametrize("fn", [tq.tq_gemv, tq.tq_gemm_prefill])
@pytest.mark.parametrize("kw,status", [
    (dict(N=6), "TQ_ERR_SHAPE"),
    (dict(K=24), "TQ_ERR_SHAPE"),
    (dict(M=-1), "TQ_ERR_SHAPE"),
    (dict(packed=None), "TQ_ERR_NULL"),
    (dict(x_sum=None), "TQ_ERR_NULL"),
    (dict(y=None), "TQ_ERR_NULL"),
    (dict(packed=A + 8), "TQ_ERR_ALIGN"),
    (dict(xq=A + 4), "TQ_ERR_ALIGN"),
    (dict(y=A + 2), "TQ_ERR_ALIGN"),
    (dict(K=32768 + 16), "TQ_ERR_UNSUPPORTED"),
])
def test_gemv_argument_checks(fn, kw, status):
    with pytest.raises(tq.TQError) as e:
        _gemv(fn, **kw)
    assert e.value.name == status, str(e.value)


def test_gemv_m_limit_and_noops():
    with pytest.raises(tq.TQError) as e:
        _gemv(tq.tq_gemv, M=25)
    assert e.value.name == "TQ_ERR_UNSUPPORTED"
    # M = 0 or N = 0 is a no-op even with NULL pointers
    _gemv(tq.tq_gemv, M=0, packed=None, y=None)
    _gemv(tq.tq_gemm_prefill, N=0, packed=None, y=None)


def test_quantize_argument_checks():
    with pytest.raises(tq.TQError) as e:
        tq.tq_quantize_act(A, A, A, A, 1, 0, 40, stream=0)
    assert e.value.name == "TQ_ERR_SHAPE"
    with pytest.raises(tq.TQError) as e:
        tq.tq_quantize_act(A + 2, A, A, A, 1, 0, 32, stream=0)
    assert e.value.name == "TQ_ERR_ALIGN"
    with pytest.raises(tq.TQError) as e:
        tq.tq_quantize_act(None, A, A, A, 1, 0, 32, stream=0)
    assert e.value.name == "TQ_ERR_NULL"
    tq.tq_quantize_act(None, None, None, None, 0, 0, 32, stream=0)  # M = 0: no-op


def test_stack_argument_checks():
    good = dict(packed=A, x=A, xq=A, x_scale=A, x_sum=A, y=A, w_scale=1.0, N=640, K=2560)
    bad = dict(good, N=642)
    with pytest.raises(tq.TQError) as e:
        tq.tq_gemv_stack([tq.make_proj(**good), tq.make_proj(**bad)], stream=0)
    assert e.value.name == "TQ_ERR_SHAPE" and "[1]" in str(e.value)
    with pytest.raises(tq.TQError) as e:
        tq.tq_gemv_stack([tq.make_proj(**good)], flags=16, stream=0)   # no such flag
    assert e.value.name == "TQ_ERR_VALUE"
    with pytest.raises(tq.TQError) as e:
        tq.tq_quantize_act_stack([tq.make_proj(**dict(good, K=20))], stream=0)
    assert e.value.name == "TQ_ERR_SHAPE"
    # the quantising launch needs the bf16 activations, 16-byte aligned
    with pytest.raises(tq.TQError) as e:
        tq.tq_gemv_stack([tq.make_proj(**dict(good, x=None))], flags=tq.TQ_STACK_QUANTIZE,
                         stream=0)
    assert e.value.name == "TQ_ERR_NULL" and "x is NULL" in str(e.value)
    with pytest.raises(tq.TQError) as e:
        tq.tq_gemv_stack([tq.make_proj(**dict(good, x=A + 8))], flags=tq.TQ_STACK_QUANTIZE,
                         stream=0)
    assert e.value.name == "TQ_ERR_ALIGN"
    # the normalising modes need the gain (and x_f32, up for relu^2); one mode
    with pytest.raises(tq.TQError) as e:
        tq.tq_gemv_stack([tq.make_proj(**good)], flags=tq.TQ_STACK_RMSNORM, stream=0)
    assert e.value.name == "TQ_ERR_NULL"
    with pytest.raises(tq.TQError) as e:
        tq.tq_gemv_stack([tq.make_proj(**dict(good, gain=A))], flags=tq.TQ_STACK_RELU2_MUL,
                         stream=0)
    assert e.value.name == "TQ_ERR_NULL"
    with pytest.raises(tq.TQError) as e:
        tq.tq_gemv_stack([tq.make_proj(**dict(good, gain=A, eps=-1.0))],
                         flags=tq.TQ_STACK_RMSNORM, stream=0)
    assert e.value.name == "TQ_ERR_VALUE"
    with pytest.raises(tq.TQError) as e:
        tq.tq_gemv_stack([tq.make_proj(**good)],
                         flags=tq.TQ_STACK_QUANTIZE | tq.TQ_STACK_RMSNORM, stream=0)
    assert e.value.name == "TQ_ERR_VALUE"
    tq.tq_gemv_stack([], stream=0)
    tq.tq_quantize_act_stack([], stream=0)


def test_stack_batch_argument_checks():
    good = dict(packed=A, x=A, xq=A, x_scale=A, x_sum=A, y=A, w_scale=1.0, N=640, K=2560)
    with pytest.raises(tq.TQError) as e:
        tq.tq_gemv_stack_batch([tq.make_proj(**good)], 33, stream=0)     # at most 32 tokens
    assert e.value.name == "TQ_ERR_UNSUPPORTED"
    with pytest.raises(tq.TQError) as e:
        tq.tq_gemv_stack_batch([tq.make_proj(**good)], 2, flags=tq.TQ_STACK_QUANTIZE, stream=0)
    assert e.value.name == "TQ_ERR_UNSUPPORTED"
    with pytest.raises(tq.TQError) as e:
        tq.tq_gemv_stack_batch([tq.make_proj(**good)], -1, stream=0)
    assert e.value.name == "TQ_ERR_SHAPE"
    with pytest.raises(tq.TQError) as e:
        tq.tq_gemv_stack_batch([tq.make_proj(**good)], 2, flags=16, stream=0)
    assert e.value.name == "TQ_ERR_VALUE"
    with pytest.raises(tq.TQError) as e:                            # checks run for every entry
        tq.tq_gemv_stack_batch([tq.make_proj(**good), tq.make_proj(**dict(good, xq=A + 4))], 3,
                               stream=0)
    assert e.value.name == "TQ_ERR_ALIGN" and "[1]" in str(e.value)
    with pytest.raises(tq.TQError) as e:
        tq.tq_quantize_act_stack_batch([tq.make_proj(**dict(good, x=None))], 2, stream=0)
    assert e.value.name == "TQ_ERR_NULL"
    with pytest.raises(tq.TQError) as e:
        tq.tq_quantize_act_stack_batch([tq.make_proj(**good)], -2, stream=0)
    assert e.value.name == "TQ_ERR_SHAPE"
    # M == 0 and empty tables are no-ops
    tq.tq_gemv_stack_batch([tq.make_proj(**good)], 0, stream=0)
    tq.tq_quantize_act_stack_batch([tq.make_proj(**good)], 0, stream=0)
    tq.tq_gemv_stack_batch([], 3, stream=0)


def test_tq_proj_layout_matches_header():
    # 7 pointers, a float and two ints (68, padded to 72), then 3 pointers, a
    # float and an int: 72 + 24 + 8 = 104
    assert ctypes.sizeof(tq.TqProj) == 104
    assert tq.TqProj.gain.offset == 72 and tq.TqProj.eps.offset == 96


def test_layer_op_argument_checks():
    rq = tq.tq_rmsnorm_quantize
    with pytest.raises(tq.TQError) as e:
        rq(A, None, A, 1e-5, A, A, A, 1, 20, stream=0)
    assert e.value.name == "TQ_ERR_SHAPE"
    with pytest.raises(tq.TQError) as e:
        rq(A, A, A, 1e-5, A, A, A, 1, 32, stream=0)          # both inputs
    assert e.value.name == "TQ_ERR_VALUE"
    with pytest.raises(tq.TQError) as e:
        rq(A, None, A, -1.0, A, A, A, 1, 32, stream=0)       # negative eps
    assert e.value.name == "TQ_ERR_VALUE"
    with pytest.raises(tq.TQError) as e:
        rq(A, None, None, 1e-5, A, A, A, 1, 32, stream=0)    # no gain
    assert e.value.name == "TQ_ERR_NULL"
    with pytest.raises(tq.TQError) as e:
        rq(A + 8, None, A, 1e-5, A, A, A, 1, 32, stream=0)
    assert e.value.name == "TQ_ERR_ALIGN"
    with pytest.raises(tq.TQError) as e:
        tq.tq_relu2_mul_rmsnorm_quantize(A, None, A, 1e-5, A, A, A, 2, 64, stream=0)
    assert e.value.name == "TQ_ERR_NULL"
    rq(None, None, None, 1e-5, None, None, None, 0, 32, stream=0)  # M = 0: no-op


def test_absmean_pack_argument_checks():
    with pytest.raises(tq.TQError) as e:
        tq.tq_absmean_pack(A, A, A, 6, 32, stream=0)
    assert e.value.name == "TQ_ERR_SHAPE"
    with pytest.raises(tq.TQError) as e:
        tq.tq_absmean_pack(A, None, A, 8, 32, stream=0)
    assert e.value.name == "TQ_ERR_NULL"
    with pytest.raises(tq.TQError) as e:
        tq.tq_absmean_pack(A + 4, A, A, 8, 32, stream=0)
    assert e.value.name == "TQ_ERR_ALIGN"


def test_header_is_c_and_struct_layout_matches_binding(tmp_path):
    # include/tq.h must compile as C (a C ABI), and the C compiler's layout of
    # tq_proj must be the one the ctypes binding marshals.
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "tq.h"\n'
        "int main(void) {\n"
        '  printf("%zu %zu %zu %zu %zu %zu\\n", sizeof(tq_proj), offsetof(tq_proj, w_scale),\n'
        "         offsetof(tq_proj, K), offsetof(tq_proj, gain), offsetof(tq_proj, eps),\n"
        "         offsetof(tq_proj, reserved));\n"
        "  return 0;\n}\n")
    exe = tmp_path / "layout"
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    subprocess.run([gcc, "-std=c11", "-Wall", "-Wextra", "-Werror",
                    "-I", os.path.join(root, "include"), "-isystem", cuda_inc,
                    str(src), "-o", str(exe)], check=True, capture_output=True)
    got = [int(v) for v in subprocess.run([str(exe)], check=True, capture_output=True,
                                          text=True).stdout.split()]
    T = tq.TqProj
    assert got == [ctypes.sizeof(T), T.w_scale.offset, T.K.offset, T.gain.offset,
                   T.eps.offset, T.reserved.offset]


# ------------------------------------------------------ binary g128, Hadamard
@pytest.mark.parametrize("N,K", [(8, 128), (64, 256), (5120, 384)])
def test_binary_host_packer_matches_oracle_and_scale_layout(N, K):
    from workloads import make_binary_projections
    p = next(make_binary_projections([("b", N, K)], M=1, seed=N + K))
    bits = np.zeros((N // 8, K), np.uint8)
    sp = np.zeros((N // 8, K // 128, 8), np.uint16)
    tq.tq_pack_binary_host(p.w, p.s_f16, bits, sp, N, K)
    assert (bits == oracle.pack_binary(p.w)).all()
    # entry (i, g, p) is the scale of row i + p N/8 on group g
    Q = N // 8
    for i in (0, Q // 2, Q - 1):
        for pl in range(8):
            assert (sp[i, :, pl] == p.s_f16[i + pl * Q]).all()


def test_binary_host_packer_rejects_bad_input():
    w = np.ones((8, 128), np.int8)
    s = np.zeros((8, 1), np.uint16)
    bits = np.zeros((1, 128), np.uint8)
    sp = np.zeros((1, 1, 8), np.uint16)
    w[3, 7] = 0
    with pytest.raises(tq.TQError) as e:
        tq.tq_pack_binary_host(w, s, bits, sp, 8, 128)
    assert e.value.name == "TQ_ERR_VALUE"
    with pytest.raises(tq.TQError) as e:
        tq.tq_pack_binary_host(w, s, bits, sp, 8, 64)  # K % 128
    assert e.value.name == "TQ_ERR_SHAPE"
    with pytest.raises(tq.TQError) as e:
        tq.tq_pack_binary_host(w, s, bits, sp, 4, 128)  # N % 8
    assert e.value.name == "TQ_ERR_SHAPE"
    with pytest.raises(tq.TQError) as e:
        tq.tq_pack_binary_host(w, None, bits, sp, 8, 128)
    assert e.value.name == "TQ_ERR_NULL"


@pytest.mark.parametrize("kw,status", [
    (dict(N=12), "TQ_ERR_SHAPE"),
    (dict(K=192), "TQ_ERR_SHAPE"),
    (dict(M=5), "TQ_ERR_UNSUPPORTED"),
    (dict(K=32768 + 128), "TQ_ERR_UNSUPPORTED"),
    (dict(bits=None), "TQ_ERR_NULL"),
    (dict(y=None), "TQ_ERR_NULL"),
    (dict(bits=A + 8), "TQ_ERR_ALIGN"),
    (dict(scales_packed=A + 4), "TQ_ERR_ALIGN"),
    (dict(y=A + 2), "TQ_ERR_ALIGN"),
])
def test_binary_gemv_argument_checks(kw, status):
    args = dict(bits=A, scales_packed=A, xq=A, x_scale=A, y=A, acc_out=None, M=1, N=640, K=2560)
    args.update(kw)
    with pytest.raises(tq.TQError) as e:
        tq.tq_gemv_binary(args["bits"], args["scales_packed"], args["xq"], args["x_scale"],
                          args["y"], args["acc_out"], args["M"], args["N"], args["K"], stream=0)
    assert e.value.name == status
    # the stack call checks every entry the same way
    with pytest.raises(tq.TQError) as e:
        tq.tq_gemv_binary_stack([tq.make_binary_proj(**{k: v for k, v in args.items()
                                                        if k != "M"})], args["M"], stream=0)
    assert e.value.name == status


def test_binary_noops():
    tq.tq_gemv_binary(None, None, None, None, None, None, 0, 640, 2560, stream=0)  # M = 0
    tq.tq_gemv_binary(None, None, None, None, None, None, 1, 0, 2560, stream=0)    # N = 0
    tq.tq_gemv_binary_stack([], 1, stream=0)


def test_binary_proj_layout_matches_header(tmp_path):
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "tq.h"\n'
        "int main(void) {\n"
        '  printf("%zu %zu %zu\\n", sizeof(tq_binary_proj), offsetof(tq_binary_proj, N),\n'
        "         offsetof(tq_binary_proj, K));\n"
        "  return 0;\n}\n")
    exe = tmp_path / "layout"
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    subprocess.run([gcc, "-std=c11", "-Wall", "-Wextra", "-Werror",
                    "-I", os.path.join(ROOT, "include"), "-isystem", cuda_inc,
                    str(src), "-o", str(exe)], check=True, capture_output=True)
    got = [int(v) for v in subprocess.run([str(exe)], check=True, capture_output=True,
                                          text=True).stdout.split()]
    T = tq.TqBinaryProj
    assert got == [ctypes.sizeof(T), T.N.offset, T.K.offset] == [56, 48, 52]


@pytest.mark.parametrize("kw,status", [
    (dict(n=48), "TQ_ERR_SHAPE"),
    (dict(n=16), "TQ_ERR_SHAPE"),
    (dict(n=2048), "TQ_ERR_SHAPE"),
    (dict(K=2560, n=1024), "TQ_ERR_SHAPE"),   # 1024 does not divide 2560
    (dict(K=65536, n=256), "TQ_ERR_UNSUPPORTED"),
    (dict(x=None), "TQ_ERR_NULL"),
    (dict(xq=A + 8), "TQ_ERR_ALIGN"),
    (dict(M=-1), "TQ_ERR_SHAPE"),
])
def test_hadamard_quantize_argument_checks(kw, status):
    args = dict(x=A, xq=A, x_scale=A, x_sum=A, M=4, K=2560, n=256)
    args.update(kw)
    with pytest.raises(tq.TQError) as e:
        tq.tq_hadamard_quantize_act(args["x"], args["xq"], args["x_scale"], args["x_sum"],
                                    args["M"], args["K"], args["n"], stream=0)
    assert e.value.name == status


def test_hadamard_quantize_noops():
    tq.tq_hadamard_quantize_act(None, None, None, None, 0, 2560, 256, stream=0)
    tq.tq_hadamard_quantize_act(None, None, None, None, 3, 0, 256, stream=0)


@pytest.mark.parametrize("kw,status", [
    (dict(n=48), "TQ_ERR_SHAPE"),
    (dict(K=2560, n=1024), "TQ_ERR_SHAPE"),
    (dict(K=65536, n=256), "TQ_ERR_UNSUPPORTED"),
    (dict(x=None), "TQ_ERR_NULL"),
    (dict(xq=A + 8), "TQ_ERR_ALIGN"),
    (dict(M=-1), "TQ_ERR_SHAPE"),
])
def test_hadamard_quantize_stack_argument_checks(kw, status):
    args = dict(x=A, xq=A, x_scale=A, x_sum=A, M=4, K=2560, n=256)
    args.update(kw)
    good = tq.make_proj(x=A, xq=A, x_scale=A, x_sum=A, K=2560)
    bad = tq.make_proj(x=args["x"], xq=args["xq"], x_scale=args["x_scale"], x_sum=args["x_sum"],
                       K=args["K"])
    with pytest.raises(tq.TQError) as e:
        # the faulty entry second: nothing may have been launched for the first
        tq.tq_hadamard_quantize_act_stack([good, bad], args["M"], args["n"], stream=0)
    assert e.value.name == status


def test_hadamard_quantize_stack_noops():
    good = tq.make_proj(x=A, xq=A, x_scale=A, x_sum=A, K=2560)
    tq.tq_hadamard_quantize_act_stack([], 4, 256, stream=0)
    tq.tq_hadamard_quantize_act_stack([good], 0, 256, stream=0)
