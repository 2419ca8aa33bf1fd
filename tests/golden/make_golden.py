"""Write tests/golden/oracle_single_640x2560.txt.

Calls only the oracle and the seeded input generator. The pages print no worked
numeric example for the ternary GEMV, so the stored values here are the
oracle's own outputs on the seed-0 single-projection workload (N=640, K=2560,
M=1). They pin the oracle against later edits: a change to its arithmetic must
change this file, and the commit that does so names the passage or reading
behind it.

Run from the repository root:  python tests/golden/make_golden.py
"""
import hashlib
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from workloads import make_projections  # noqa: E402


def digest(a: np.ndarray) -> str:
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def main():
    (p,) = make_projections([("proj", 640, 2560)], M=1, seed=0)
    P = oracle.pack(p.w)
    q, xs, xsum, acc, y = oracle.forward(P, p.N, p.w_scale, p.x_bf16)
    lines = [
        "# oracle outputs, seed-0 single projection N=640 K=2560 M=1 (see make_golden.py)",
        f"w_scale_hex {np.float32(p.w_scale).view(np.uint32):08x}",
        f"packed_sha256 {digest(P)}",
        f"q_sha256 {digest(q)}",
        f"x_scale_hex {xs.view(np.uint32)[0]:08x}",
        f"x_sum {int(xsum[0])}",
        f"acc_sha256 {digest(acc)}",
        "acc_first8 " + " ".join(str(int(v)) for v in acc[0, :8]),
        "y_first4 " + " ".join(repr(float(v)) for v in y[0, :4]),
    ]
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_single_640x2560.txt")
    with open(out, "w") as f:
        f.write("\n".join(lines) + "\n")
    print(out)


if __name__ == "__main__":
    main()
