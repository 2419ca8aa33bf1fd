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
