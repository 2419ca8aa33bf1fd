"""GPU parity of tq_quantize_act against the oracle: int8 codes, x_scale and
x_sum bit-exact, on the activation shapes of every workload and edge cases."""
import numpy as np
import pytest

import oracle
from tests._gpu import gpu_quant
from workloads import activations_bf16

pytestmark = pytest.mark.gpu


def _check(xb):
    q, s, t = (a.cpu().numpy() for a in gpu_quant(xb))
    rq, rs, rt = oracle.quant(xb)
    assert (q == rq).all()
    assert (s.view(np.uint32) == rs.view(np.uint32)).all()
    assert (t == rt).all()


@pytest.mark.parametrize("M,K", [(1, 2560), (1, 6912), (3, 2560), (24, 6912), (512, 5120),
                                 (7, 16), (2, 32768)])
def test_quant_parity(cuda_device, M, K):
    _check(activations_bf16(np.random.default_rng(M * 100003 + K), M, K))


def test_quant_edge_rows(cuda_device):
    K = 256
    rows = np.zeros((6, K), dtype=np.uint16)
    rows[1, :] = 0x8000                     # negative zeros
    rows[2, :] = 0x3F80                     # all 1.0
    rows[3, ::2] = 0xBF00                   # -0.5 and 0
    rows[4, :] = 0x0001                     # the smallest subnormal bf16
    rows[5, 7] = 0x7F7F                     # the largest finite bf16, rest 0
    _check(rows)
    # ties: amax 2 -> s = 63.5; 1.0 -> 63.5 (even 64), -1.0 -> -64
    t = np.zeros((1, 16), dtype=np.uint16)
    t[0, :4] = [0x4000, 0x3F80, 0xBF80, 0x3F00]
    _check(t)
