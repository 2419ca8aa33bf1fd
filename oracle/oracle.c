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
 *
 * The steps on either side of the GEMV in a BitNet decoder layer (the
 * lemon-mlx-engine issue, section "Architecture": a Llama variant with
 * relu_squared instead of silu and sub-layer norms, attn_sub_norm before
 * o_proj and ffn_sub_norm before down_proj; RMSNorm is named among the ops
 * that pass) and the absmean weight quantiser (1bit.systems post "the full
 * arc ...", read-more item "Training-Runs -- absmean QAT"; the stored scale is
 * the .weight_scale of "What We Need" item 2). The pages print none of their
 * formulas. Readings taken:
 *  - RMSNorm of a row x [K] with gain g [K] and epsilon e: the mean of x^2
 *    is accumulated in fp64 (each square exact), r = 1 / sqrt(mean + e) in
 *    fp64 rounded once to fp32, h[k] = fl32(fl32(x[k] * r) * g[k]).
 *  - relu_squared(a) * b = fl32(fl32(max(a,0) * max(a,0)) * b), fp32.
 *  - absmean: gamma = fl32(sum |W| / (N K)) with the sum in fp64;
 *    w = clamp(rint(fl32(W / gamma)), -1, 1) (ties to even); gamma == 0
 *    gives w = 0. The packed weights then follow oracle_pack, and gamma is
 *    the stored per-tensor scale.
 *
 * Two further paths, with their readings next to their code below: the
 * Hadamard-rotated 4-bit activations of prompt processing and the binary
 * g128 weight format.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fPIC -shared.
 * Status codes: 0 ok; 1 a value outside the domain (a weight not in
 * {-1,0,1} -- {-1,+1} for the binary format --, or a packed code 3); 2 a bad
 * shape.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
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

/* Absmax quantisation of one fp32 row to the symmetric levels -qb..qb (the
 * reading above, with qb = 127 for int8 and qb = 7 for the 4-bit codes of
 * the Hadamard route). */
static void quant_row_levels(const float *row, int64_t K, float qb, int8_t *q, float *x_scale,
                             int32_t *x_sum)
{
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        float a = fabsf(row[k]);
        if (a > amax)
            amax = a;
    }
    int32_t sum = 0;
    if (amax == 0.0f) {
        for (int64_t k = 0; k < K; ++k)
            q[k] = 0;
        *x_scale = 0.0f;
    } else {
        volatile float s = qb / amax; /* one fp32 rounding */
        for (int64_t k = 0; k < K; ++k) {
            volatile float t = row[k] * s; /* one fp32 rounding */
            float r = rintf(t); /* default mode: nearest, ties to even */
            if (r > qb) r = qb;
            if (r < -qb) r = -qb;
            q[k] = (int8_t)r;
            sum += (int32_t)r;
        }
        *x_scale = amax / qb;
    }
    *x_sum = sum;
}

/* Absmax int8 quantisation of one fp32 row (the reading above). */
static void quant_row(const float *row, int64_t K, int8_t *q, float *x_scale, int32_t *x_sum)
{
    quant_row_levels(row, K, 127.0f, q, x_scale, x_sum);
}

/* Per-token absmax int8 quantisation of x [M,K] (bf16 bit patterns). */
int oracle_quant(const uint16_t *x, int64_t M, int64_t K,
                 int8_t *q, float *x_scale, int32_t *x_sum)
{
    if (M < 0 || K < 0)
        return 2;
    float *row = malloc((size_t)(K > 0 ? K : 1) * sizeof(float));
    if (!row)
        return 2;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t k = 0; k < K; ++k)
            row[k] = bf16_to_float(x[m * K + k]); /* exact */
        quant_row(row, K, q + m * K, &x_scale[m], &x_sum[m]);
    }
    free(row);
    return 0;
}

/* The same quantisation of fp32 rows h [M,K]. */
int oracle_quant_f32(const float *h, int64_t M, int64_t K,
                     int8_t *q, float *x_scale, int32_t *x_sum)
{
    if (M < 0 || K < 0)
        return 2;
    for (int64_t m = 0; m < M; ++m)
        quant_row(h + m * K, K, q + m * K, &x_scale[m], &x_sum[m]);
    return 0;
}

/* RMSNorm of each row of x [M,K] with gain g [K] (the reading above). */
int oracle_rmsnorm(const float *x, int64_t M, int64_t K, const float *g, float eps, float *h)
{
    if (M < 0 || K <= 0)
        return 2;
    for (int64_t m = 0; m < M; ++m) {
        const float *row = x + m * K;
        double ss = 0.0;
        for (int64_t k = 0; k < K; ++k)
            ss += (double)row[k] * (double)row[k]; /* each square exact in fp64 */
        const float r = (float)(1.0 / sqrt(ss / (double)K + (double)eps));
        for (int64_t k = 0; k < K; ++k) {
            volatile float t = row[k] * r; /* one fp32 rounding */
            h[m * K + k] = t * g[k];
        }
    }
    return 0;
}

/* h[i] = relu(a[i])^2 * b[i] for n elements (the reading above). */
int oracle_relu2_mul(const float *a, const float *b, int64_t n, float *h)
{
    if (n < 0)
        return 2;
    for (int64_t i = 0; i < n; ++i) {
        const float r = a[i] > 0.0f ? a[i] : 0.0f;
        volatile float sq = r * r; /* one fp32 rounding */
        h[i] = sq * b[i];
    }
    return 0;
}

/* Absmean ternary quantisation of latent weights W [N,K] (bf16 bit
 * patterns): w [N,K] in {-1,0,1} and the per-tensor scale gamma. */
int oracle_absmean(const uint16_t *W, int64_t N, int64_t K, int8_t *w, float *gamma)
{
    if (N < 0 || K < 0)
        return 2;
    const int64_t n = N * K;
    double s = 0.0;
    for (int64_t i = 0; i < n; ++i)
        s += fabs((double)bf16_to_float(W[i]));
    const float g = n > 0 ? (float)(s / (double)n) : 0.0f;
    *gamma = g;
    for (int64_t i = 0; i < n; ++i) {
        if (g == 0.0f) {
            w[i] = 0;
            continue;
        }
        volatile float t = bf16_to_float(W[i]) / g; /* one fp32 rounding */
        float r = rintf(t);
        if (r > 1.0f) r = 1.0f;
        if (r < -1.0f) r = -1.0f;
        w[i] = (int8_t)r;
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

/* ------------------------------------------------------------------------
 * Hadamard-rotated 4-bit activations for prompt processing (1bit engine blog,
 * "509 tokens a second of prompt: the Hadamard route ships" and "Qwen3.8-27B
 * at 45.7 tok/s ...": 4-bit activations on the matrix units, kept accurate by
 * a Hadamard rotation; 1bit.systems README, read-more item "Training-Runs --
 * BitNet v2 Hadamard"). The pages print no formula. Readings taken:
 *  - The rotation acts on each block of n consecutive entries of a token row
 *    (n a power of two dividing K): h = H_n x / sqrt(n), with H_n the
 *    Sylvester-Hadamard matrix, H_n[i][j] = (-1)^popcount(i & j).
 *  - Each sum over j is accumulated in fp64. For bf16 inputs every partial
 *    sum is then exact (the inputs are multiples of the block's smallest
 *    unit in the last place, and n * 2^8 times the largest over that unit
 *    stays below 2^53 unless the block's magnitudes span more than ~2^35),
 *    so the result does not depend on the order of the additions. The sum
 *    times fl64(1/sqrt(n)) is rounded once to fp32 (for n a power of four,
 *    1/sqrt(n) is a power of two and that product is exact).
 *  - 4-bit codes: the absmax quantiser above with 7 levels each side
 *    (q in -7..7, s = 7 / amax, x_scale = amax / 7), one code per int8.
 * ---------------------------------------------------------------------- */

/* (-1)^popcount(i & j), written out bit by bit. */
static int hadamard_sign(int64_t i, int64_t j)
{
    int64_t b = i & j;
    int odd = 0;
    while (b) {
        odd ^= (int)(b & 1);
        b >>= 1;
    }
    return odd ? -1 : 1;
}

/* h [M,K] = the blockwise normalised Hadamard rotation of x [M,K] (bf16 bit
 * patterns), n the block size. */
int oracle_hadamard_rotate(const uint16_t *x, int64_t M, int64_t K, int64_t n, float *h)
{
    if (M < 0 || K < 0 || n < 1 || (n & (n - 1)) != 0 || K % n != 0)
        return 2;
    const double c = 1.0 / sqrt((double)n);
    for (int64_t m = 0; m < M; ++m)
        for (int64_t b = 0; b < K; b += n)
            for (int64_t i = 0; i < n; ++i) {
                double s = 0.0;
                for (int64_t j = 0; j < n; ++j)
                    s += (double)hadamard_sign(i, j) * (double)bf16_to_float(x[m * K + b + j]);
                h[m * K + b + i] = (float)(s * c);
            }
    return 0;
}

/* Per-token 4-bit absmax quantisation of fp32 rows h [M,K]. */
int oracle_quant4(const float *h, int64_t M, int64_t K, int8_t *q, float *x_scale, int32_t *x_sum)
{
    if (M < 0 || K < 0)
        return 2;
    for (int64_t m = 0; m < M; ++m)
        quant_row_levels(h + m * K, K, 7.0f, q + m * K, &x_scale[m], &x_sum[m]);
    return 0;
}

/* ------------------------------------------------------------------------
 * Binary g128 weights (baguaai "BitNet" tag page, the Bonsai 27B item: a
 * true 1-bit binary scheme in which 128 weights share one fp16 scale, about
 * 1.125 bits per weight). The page gives no bit order, no group direction
 * and no activation format. Readings taken:
 *  - A weight is +1 or -1: bit 1 is +1, bit 0 is -1.
 *  - Eight weights per byte in the plane layout of the ternary format: the
 *    packed tensor of an [N, K] projection is uint8 [N/8, K], bit p of byte
 *    (i, k) holding output row i + p*(N/8).
 *  - Groups are 128 consecutive k of one output row (K a multiple of 128);
 *    scale s[n, g] (fp16) belongs to row n, columns 128 g .. 128 g + 127.
 *  - Activations: the per-token absmax int8 quantiser above.
 *  - acc[m, n, g] = sum over the group of w * q (int32, exact);
 *    y[m, n] = x_scale[m] * sum_g s[n, g] * acc[m, n, g], in fp64 here.
 *    The group-free total sum_g acc[m, n, g] is also returned (int32).
 * ---------------------------------------------------------------------- */

/* fp16 bit pattern to double, by the IEEE binary16 definition. */
double oracle_half_to_double(uint16_t h)
{
    const int sign = (h >> 15) & 1;
    const int e = (h >> 10) & 0x1F;
    const int f = h & 0x3FF;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24); /* subnormal: f * 2^-14 * 2^-10 */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25); /* (1 + f/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* Pack w [N,K] in {-1,+1} into B [N/8,K]. */
int oracle_pack_binary(const int8_t *w, uint8_t *B, int64_t N, int64_t K)
{
    if (N < 0 || K < 0 || N % 8 != 0)
        return 2;
    const int64_t Q = N / 8;
    for (int64_t i = 0; i < Q; ++i)
        for (int64_t k = 0; k < K; ++k) {
            unsigned byte = 0;
            for (int p = 0; p < 8; ++p) {
                int v = w[(i + p * Q) * K + k];
                if (v != 1 && v != -1)
                    return 1;
                if (v == 1)
                    byte |= 1u << p;
            }
            B[i * K + k] = (uint8_t)byte;
        }
    return 0;
}

/* The weight of output row n at column k, read out of B by definition. */
static int binary_weight_at(const uint8_t *B, int64_t Q, int64_t K, int64_t n, int64_t k)
{
    int64_t i = n % Q;    /* packed row */
    int p = (int)(n / Q); /* bit, 0..7 */
    return ((B[i * K + k] >> p) & 1) ? 1 : -1;
}

/* Unpack B [N/8,K] into w [N,K]. */
int oracle_unpack_binary(const uint8_t *B, int8_t *w, int64_t N, int64_t K)
{
    if (N < 0 || K < 0 || N % 8 != 0)
        return 2;
    const int64_t Q = N / 8;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            w[n * K + k] = (int8_t)binary_weight_at(B, Q, K, n, k);
    return 0;
}

/* For output rows n0 <= n < n1 and all M rows of q [M,K]: acc [M, n1-n0]
 * (int32, sum over all K of w * q) and y [M, n1-n0] (fp64, the group-scaled
 * sum times x_scale). s holds the fp16 scales [N, K/128] as bit patterns. */
int oracle_gemv_binary(const uint8_t *B, int64_t N, int64_t K, const uint16_t *s,
                       const int8_t *q, int64_t M, const float *x_scale, int64_t n0, int64_t n1,
                       int32_t *acc, double *y)
{
    if (N < 0 || K < 0 || M < 0 || N % 8 != 0 || K % 128 != 0 || n0 < 0 || n1 > N || n0 > n1)
        return 2;
    const int64_t Q = N / 8, G = K / 128, W = n1 - n0;
    for (int64_t m = 0; m < M; ++m) {
        const int8_t *qm = q + m * K;
        for (int64_t n = n0; n < n1; ++n) {
            int32_t total = 0;
            double sum = 0.0;
            for (int64_t g = 0; g < G; ++g) {
                int32_t a = 0;
                for (int64_t k = 128 * g; k < 128 * g + 128; ++k)
                    a += binary_weight_at(B, Q, K, n, k) * (int32_t)qm[k];
                total += a;
                sum += (double)a * oracle_half_to_double(s[n * G + g]);
            }
            acc[m * W + (n - n0)] = total;
            y[m * W + (n - n0)] = sum * (double)x_scale[m];
        }
    }
    return 0;
}
