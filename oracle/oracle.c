/*
 * oracle.c -- plain, slow, single-threaded CPU statement of the ternary
 * absmax-int8 GEMV.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the bench's CPU
 * baseline leg load this file's library. The product library never calls it,
 * includes it or shares a line with it.
 *
 * What it computes, and the passages it follows:
 *
 *  - Ternary weights w in {-1, 0, +1}: BitNet b1.58 (the 1bit.systems post
 *    "the full arc ...", paper list item 1; the lemon-mlx-engine issue
 *    "Feature request: BitNet 1.58-bit ternary inference on ROCm (gfx1151)",
 *    section "Why This Matters").
 *  - Packing, four 2-bit values per byte, the packed tensor of an [N, K]
 *    projection being uint8 [N/4, K]: same issue, section "Architecture"
 *    item 3 and section "Weight mapping (bitnet-b1.58-2B-4T)". The pages do
 *    not print the code map or the bit order. Reading taken: code = w + 1, and
 *    byte (i, k) holds output row i + p*(N/4) in bits 2p..2p+1 (p = 0..3).
 *    Code 3 is not a weight.
 *  - Per-token absmax int8 activations. The pages name BitNet b1.58 but not
 *    the formula. Reading taken (one fp32 rounding per step):
 *        amax = max_k |x[m,k]|          (bf16 -> fp32 is exact)
 *        amax == 0  ->  q = 0, x_scale = 0, x_sum = 0
 *        s = 127 / amax                 (fp32 divide, round to nearest)
 *        q = clamp(rint(x * s), -127, 127)  (fp32 product, ties to even)
 *        x_scale = amax / 127           (fp32 divide)
 *        x_sum = sum_k q
 *  - int32 accumulation of weight x activation, which for ternary weights is
 *    an add, a subtract or a skip (baguaai "BitNet" tag page, the C99 engine
 *    item): acc[m,n] = sum_k w[n,k] * q[m,k], each w[n,k] unpacked from its
 *    byte one element at a time.
 *  - Scale epilogue y[m,n] = acc[m,n] * w_scale * x_scale[m] with the
 *    per-tensor weight scale (issue above, "What We Need" item 2, the
 *    .weight_scale keys). Computed in fp64 here.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fPIC -shared.
 * Status codes: 0 ok; 1 a value outside the domain (a weight not in
 * {-1,0,1}, or a packed code 3); 2 a bad shape.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static float bf16_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Pack w [N,K] (int8, row-major) into P [N/4,K]. */
int oracle_pack(const int8_t *w, uint8_t *P, int64_t N, int64_t K)
{
    if (N < 0 || K < 0 || N % 4 != 0)
        return 2;
    const int64_t Q = N / 4; /* packed rows; plane p holds rows p*Q .. p*Q+Q-1 */
    for (int64_t i = 0; i < Q; ++i) {
        for (int64_t k = 0; k < K; ++k) {
            unsigned byte = 0;
            for (int p = 0; p < 4; ++p) {
                int v = w[(i + p * Q) * K + k];
                if (v < -1 || v > 1)
                    return 1;
                unsigned code = (unsigned)(v + 1);
                byte |= code << (2 * p);
            }
            P[i * K + k] = (uint8_t)byte;
        }
    }
    return 0;
}

/* The weight of output row n at column k, read out of P by definition.
 * Returns 2 for the invalid code 3 (the caller turns that into status 1). */
static int weight_at(const uint8_t *P, int64_t Q, int64_t K, int64_t n, int64_t k)
{
    int64_t i = n % Q;      /* packed row */
    int p = (int)(n / Q);   /* plane, 0..3 */
    int code = (P[i * K + k] >> (2 * p)) & 3;
    return code - 1;
}

/* Unpack P [N/4,K] into w [N,K]. */
int oracle_unpack(const uint8_t *P, int8_t *w, int64_t N, int64_t K)
{
    if (N < 0 || K < 0 || N % 4 != 0)
        return 2;
    const int64_t Q = N / 4;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            int v = weight_at(P, Q, K, n, k);
            if (v == 2)
                return 1;
            w[n * K + k] = (int8_t)v;
        }
    return 0;
}

/* Per-token absmax int8 quantisation of x [M,K] (bf16 bit patterns). */
int oracle_quant(const uint16_t *x, int64_t M, int64_t K,
                 int8_t *q, float *x_scale, int32_t *x_sum)
{
    if (M < 0 || K < 0)
        return 2;
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t *row = x + m * K;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(bf16_to_float(row[k]));
            if (a > amax)
                amax = a;
        }
        int32_t sum = 0;
        if (amax == 0.0f) {
            for (int64_t k = 0; k < K; ++k)
                q[m * K + k] = 0;
            x_scale[m] = 0.0f;
        } else {
            volatile float s = 127.0f / amax; /* one fp32 rounding */
            for (int64_t k = 0; k < K; ++k) {
                volatile float t = bf16_to_float(row[k]) * s; /* one fp32 rounding */
                float r = rintf(t); /* default mode: nearest, ties to even */
                if (r > 127.0f) r = 127.0f;
                if (r < -127.0f) r = -127.0f;
                q[m * K + k] = (int8_t)r;
                sum += (int32_t)r;
            }
            x_scale[m] = amax / 127.0f;
        }
        x_sum[m] = sum;
    }
    return 0;
}

/* acc[m, n - n0] = sum_k w[n,k] * q[m,k] for output rows n0 <= n < n1 and all
 * M rows of q [M,K]. acc is [M, n1-n0] row-major. */
int oracle_gemv(const uint8_t *P, int64_t N, int64_t K, const int8_t *q, int64_t M,
                int64_t n0, int64_t n1, int32_t *acc)
{
    if (N < 0 || K < 0 || M < 0 || N % 4 != 0 || n0 < 0 || n1 > N || n0 > n1)
        return 2;
    const int64_t Q = N / 4;
    const int64_t W = n1 - n0;
    int bad = 0;
    for (int64_t m = 0; m < M; ++m) {
        const int8_t *qm = q + m * K;
        for (int64_t n = n0; n < n1; ++n) {
            int32_t s = 0;
            for (int64_t k = 0; k < K; ++k) {
                int v = weight_at(P, Q, K, n, k);
                bad |= (v == 2);
                s += v * (int32_t)qm[k];
            }
            acc[m * W + (n - n0)] = s;
        }
    }
    return bad ? 1 : 0;
}

/* y[m,n] = acc[m,n] * w_scale * x_scale[m], in fp64. acc and y are [M,N]. */
int oracle_epilogue(const int32_t *acc, int64_t M, int64_t N, float w_scale,
                    const float *x_scale, double *y)
{
    if (M < 0 || N < 0)
        return 2;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            y[m * N + n] = (double)acc[m * N + n] * (double)w_scale * (double)x_scale[m];
    return 0;
}
