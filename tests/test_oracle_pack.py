"""Pins for the oracle's pack / unpack (CPU only).

Layout under test: the packed tensor of an [N, K] ternary projection is uint8
[N/4, K], four 2-bit values per byte (lemon-mlx-engine issue "Feature request:
BitNet 1.58-bit ternary inference on ROCm (gfx1151)", section "Weight mapping
(bitnet-b1.58-2B-4T)"). Code map and bit order are the reading taken where the
pages are silent: code = w + 1, byte (i, k) holds row i + p*N/4 in bits 2p..2p+1.
"""
import itertools

import numpy as np
import pytest

import oracle


def test_hand_byte():
    # Column of rows (0, N/4, N/2, 3N/4) with N = 4: w = (-1, 0, +1, +1)
    # codes (0, 1, 2, 2) at bits (0-1, 2-3, 4-5, 6-7) -> 0b10_10_01_00 = 0xA4.
    w = np.array([[-1], [0], [1], [1]], dtype=np.int8)
    assert oracle.pack(w).tolist() == [[0xA4]]


def test_all_zero_is_0x55():
    # w = 0 everywhere -> code 1 in every 2-bit field -> 0b01010101.
    w = np.zeros((16, 48), dtype=np.int8)
    P = oracle.pack(w)
    assert P.shape == (4, 48)
    assert (P == 0x55).all()


def test_single_nonzero_lands_in_its_plane():
    # A lone +1 at (n, k) of an N = 8 projection changes exactly one byte,
    # (n mod 2, k), and in it exactly the field of plane n div 2, to code 2.
    N, K = 8, 5
    for n in range(N):
        for k in range(K):
            for v in (-1, 1):
                w = np.zeros((N, K), dtype=np.int8)
                w[n, k] = v
                P = oracle.pack(w)
                changed = np.argwhere(P != 0x55)
                assert changed.tolist() == [[n % 2, k]]
                field = (int(P[n % 2, k]) >> (2 * (n // 2))) & 3
                assert field == v + 1
                # the other three fields still hold code 1
                others = [(int(P[n % 2, k]) >> (2 * p)) & 3 for p in range(4) if p != n // 2]
                assert others == [1, 1, 1]


def test_exhaustive_n4_k1():
    seen = set()
    for col in itertools.product((-1, 0, 1), repeat=4):
        w = np.array(col, dtype=np.int8).reshape(4, 1)
        P = oracle.pack(w)
        seen.add(int(P[0, 0]))
        assert (oracle.unpack(P, 4) == w).all()
    # 81 distinct columns give 81 distinct bytes, none holding code 3
    assert len(seen) == 81
    assert all(((b >> (2 * p)) & 3) != 3 for b in seen for p in range(4))


def test_exhaustive_n4_k2():
    cols = np.array(list(itertools.product((-1, 0, 1), repeat=8)), dtype=np.int8)
    for c in cols:
        w = c.reshape(4, 2)
        assert (oracle.unpack(oracle.pack(w), 4) == w).all()


@pytest.mark.parametrize("N,K", [(4, 16), (12, 32), (640, 48), (64, 2560)])
def test_random_roundtrip(N, K):
    rng = np.random.default_rng(N * 7919 + K)
    w = rng.integers(-1, 2, size=(N, K), dtype=np.int8)
    assert (oracle.unpack(oracle.pack(w), N) == w).all()


def test_rejects_non_ternary_and_code3():
    w = np.zeros((4, 4), dtype=np.int8)
    w[2, 3] = 2
    with pytest.raises(oracle.OracleError):
        oracle.pack(w)
    P = np.full((1, 4), 0x55, dtype=np.uint8)
    P[0, 1] = 0x55 | (3 << 4)  # plane 2 of column 1 holds code 3
    with pytest.raises(oracle.OracleError):
        oracle.unpack(P, 4)
    q = np.ones((1, 4), dtype=np.int8)
    with pytest.raises(oracle.OracleError):
        oracle.gemv(P, 4, q)


def test_rejects_bad_shape():
    with pytest.raises(oracle.OracleError):
        oracle.pack(np.zeros((6, 4), dtype=np.int8))
