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
