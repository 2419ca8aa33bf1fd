// pack_host.cpp -- host-side packing of ternary weights, four 2-bit codes per
// byte: an [N, K] projection becomes uint8 [N/4, K] (lemon-mlx-engine issue
// "Feature request: BitNet 1.58-bit ternary inference on ROCm (gfx1151)",
// sections "Architecture" item 3 and "Weight mapping (bitnet-b1.58-2B-4T)").
// Code map and bit order (not given on the pages): code = w + 1, and byte
// (i, k) holds output row i + p*N/4 in bits 2p..2p+1. Plane p of the packed
// tensor is therefore the contiguous block of rows [p*N/4, (p+1)*N/4), so the
// kernels read one packed row and produce four output rows N/4 apart.
#include <cstddef>
#include <cstdint>

namespace tq {

// Returns false if some weight is outside {-1, 0, 1}.
bool pack_ternary_host(const int8_t *w, uint8_t *packed, int N, int K)
{
    const size_t Q = size_t(N) / 4;
    const size_t Ks = size_t(K);
    unsigned bad = 0;
    for (size_t i = 0; i < Q; ++i) {
        const int8_t *w0 = w + (i + 0 * Q) * Ks;
        const int8_t *w1 = w + (i + 1 * Q) * Ks;
        const int8_t *w2 = w + (i + 2 * Q) * Ks;
        const int8_t *w3 = w + (i + 3 * Q) * Ks;
        uint8_t *out = packed + i * Ks;
        for (size_t k = 0; k < Ks; ++k) {
            const unsigned c0 = unsigned(w0[k] + 1), c1 = unsigned(w1[k] + 1);
            const unsigned c2 = unsigned(w2[k] + 1), c3 = unsigned(w3[k] + 1);
            // a valid code is 0..2; anything else (incl. wrap-around) is >= 3
            bad |= unsigned(c0 > 2u) | unsigned(c1 > 2u) | unsigned(c2 > 2u) | unsigned(c3 > 2u);
            out[k] = uint8_t((c0 & 3u) | ((c1 & 3u) << 2) | ((c2 & 3u) << 4) | ((c3 & 3u) << 6));
        }
        if (bad)
            return false;
    }
    return true;
}

}  // namespace tq

namespace tq {

// Binary g128 packing (baguaai "BitNet" tag page, Bonsai 27B item: one bit
// per weight, 128 weights sharing one fp16 scale). Layout (not given on the
// page): bits [N/8, K], bit p of byte (i, k) = weight of row i + p*N/8 at
// column k, 1 for +1 and 0 for -1; the fp16 scales [N, K/128] are regrouped
// as [N/8, K/128, 8] so that a packed row's tile carries the eight scales of
// each of its groups in 16 contiguous bytes. Returns false if some weight is
// not -1 or +1.
bool pack_binary_host(const int8_t *w, const uint16_t *scales, uint8_t *bits,
                      uint16_t *scales_packed, int N, int K)
{
    const size_t Q = size_t(N) / 8;
    const size_t Ks = size_t(K);
    const size_t G = Ks / 128;
    unsigned bad = 0;
    for (size_t i = 0; i < Q; ++i) {
        uint8_t *out = bits + i * Ks;
        for (size_t k = 0; k < Ks; ++k)
            out[k] = 0;
        for (unsigned p = 0; p < 8; ++p) {
            const int8_t *wr = w + (i + p * Q) * Ks;
            for (size_t k = 0; k < Ks; ++k) {
                const int v = wr[k];
                bad |= unsigned(v != 1 && v != -1);
                out[k] = uint8_t(out[k] | (unsigned(v == 1) << p));
            }
            for (size_t g = 0; g < G; ++g)
                scales_packed[(i * G + g) * 8 + p] = scales[(i + p * Q) * G + g];
        }
        if (bad)
            return false;
    }
    return true;
}

}  // namespace tq
