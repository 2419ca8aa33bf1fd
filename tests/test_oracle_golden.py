"""The oracle still reproduces its stored seed-0 outputs (tests/golden/)."""
import hashlib
import os

import numpy as np

import oracle
from workloads import make_projections

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "oracle_single_640x2560.txt")


def _read():
    d = {}
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        k, v = line.split(" ", 1)
        d[k] = v.strip()
    return d


def _sha(a):
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def test_oracle_matches_stored_outputs():
    g = _read()
    (p,) = make_projections([("proj", 640, 2560)], M=1, seed=0)
    P = oracle.pack(p.w)
    q, xs, xsum, acc, y = oracle.forward(P, p.N, p.w_scale, p.x_bf16)
    assert f"{np.float32(p.w_scale).view(np.uint32):08x}" == g["w_scale_hex"]
    assert _sha(P) == g["packed_sha256"]
    assert _sha(q) == g["q_sha256"]
    assert f"{xs.view(np.uint32)[0]:08x}" == g["x_scale_hex"]
    assert int(xsum[0]) == int(g["x_sum"])
    assert _sha(acc) == g["acc_sha256"]
    assert [int(v) for v in acc[0, :8]] == [int(v) for v in g["acc_first8"].split()]
    assert [float(v) for v in y[0, :4]] == [float(v) for v in g["y_first4"].split()]
