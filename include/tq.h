/*
 * tq.h -- C ABI of libtq, the B200 (sm_100a) ternary absmax-int8 GEMV library.
 *
 * The method: BitNet b1.58 style projections. Weights are ternary {-1, 0, +1}
 * (1bit.systems post "the full arc ...", paper list item 1), stored four 2-bit
 * codes per byte so that an [N, K] projection becomes uint8 [N/4, K]
 * (lemon-mlx-engine issue "Feature request: BitNet 1.58-bit ternary inference
 * on ROCm (gfx1151)", section "Weight mapping (bitnet-b1.58-2B-4T)"), with one
 * fp32 scale per tensor (same issue, "What We Need" item 2, the .weight_scale
 * keys). Activations are quantised per token to int8 by absmax, products are
 * accumulated in int32 (adds and subtracts only: baguaai "BitNet" tag page,
 * the C99 engine item) and a scale epilogue produces fp32. Decode is bound by
 * the bytes of weights read per token (1bit engine blog, "Qwen3.8-27B at 45.7
 * tok/s ..." and "Smaller files ..."); prompt processing by the matrix units
 * (same blog, first of those two posts).
 *
 * Layout and value conventions (the pages leave these open; readings taken):
 *   - packed[i, k] (row-major, K contiguous) holds, in bits 2p..2p+1
 *     (p = 0..3), the code of weight w[i + p*N/4, k]; code = w + 1 in {0,1,2};
 *     code 3 is not a weight and the output for a byte holding it is undefined
 *     (the kernels neither fault nor detect it).
 *   - per token m: amax = max_k |x[m,k]|; s = fl32(127 / amax);
 *     xq = clamp(round_half_even(fl32(x * s)), -127, 127);
 *     x_scale = fl32(amax / 127); x_sum = sum_k xq. An all-zero row gives
 *     xq = 0, x_scale = 0, x_sum = 0. NaN or Inf input is outside the contract.
 *   - acc[m, n] = sum_k w[n, k] * xq[m, k] (int32, exact);
 *     y[m, n] = fl32(float(acc) * fl32(w_scale * x_scale[m])).
 *
 * Conventions for every call:
 *   - The caller owns every buffer. "device" pointers are CUDA device memory
 *     (any allocator); "host" pointers are ordinary host memory.
 *   - Device work is enqueued on `stream` and returns without synchronising;
 *     argument checks happen before anything is enqueued, and a failed check
 *     enqueues nothing.
 *   - Shapes: N % 4 == 0 and K % 16 == 0; M, N, K >= 0. M = 0 or N = 0 is a
 *     no-op. Device pointers to byte tensors (packed, xq) and to x must be
 *     16-byte aligned; fp32/int32 vectors 4-byte aligned.
 *   - Errors are returned as tq_status; tq_last_error() gives a message for
 *     the last failure on the calling thread. A kernel-launch failure is
 *     TQ_ERR_CUDA. Kernel execution errors surface on the stream as usual.
 *   - The library keeps no state between calls apart from per-device launch
 *     settings and one device-side error word (tq_device_error).
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum tq_status {
    TQ_OK = 0,
    TQ_ERR_NULL = 1,        /* a required pointer is NULL */
    TQ_ERR_SHAPE = 2,       /* M, N or K outside the contract */
    TQ_ERR_ALIGN = 3,       /* a pointer is not aligned as required */
    TQ_ERR_VALUE = 4,       /* a value outside its domain (e.g. a weight not in {-1,0,1}) */
    TQ_ERR_CUDA = 5,        /* a CUDA runtime call or a kernel launch failed */
    TQ_ERR_UNSUPPORTED = 6  /* valid input this build does not handle (see each call) */
} tq_status;

/* Name of a status code (static string). */
const char *tq_status_string(tq_status s);

/* Message for the last failed call on this thread (static per thread; "" if none). */
const char *tq_last_error(void);

/*
 * tq_pack_host -- pack ternary weights on the host.
 *   w      host, int8 [N, K] row-major, every value in {-1, 0, 1}.
 *   packed host, uint8 [N/4, K] row-major, written.
 *   M, stream: unused (kept so that every call takes M, N, K and a stream).
 * Synchronous. TQ_ERR_VALUE if any w is outside {-1, 0, 1} (packed is then
 * partly written). Packing: lemon-mlx-engine issue, "Architecture" item 3 and
 * "Weight mapping".
 */
tq_status tq_pack_host(const int8_t *w, uint8_t *packed, int M, int N, int K,
                       cudaStream_t stream);

/*
 * tq_quantize_act -- per-token absmax int8 quantisation (BitNet b1.58
 * activations; formula as in the header comment).
 *   x       device, bf16 [M, K] row-major (raw bf16 bit patterns).
 *   xq      device, int8 [M, K], written.
 *   x_scale device, fp32 [M], written (amax / 127).
 *   x_sum   device, int32 [M], written (sum of xq over k); may be NULL when the
 *           caller will not pass it to a GEMV call.
 *   N: unused. Any M >= 0; K % 16 == 0.
 */
tq_status tq_quantize_act(const uint16_t *x, int8_t *xq, float *x_scale, int32_t *x_sum,
                          int M, int N, int K, cudaStream_t stream);

/*
 * tq_gemv -- decode-shaped ternary GEMV, 1 <= M <= 24 tokens.
 *   packed  device, uint8 [N/4, K] (layout above).
 *   w_scale the projection's fp32 scale.
 *   xq, x_scale, x_sum  device, as written by tq_quantize_act for [M, K].
 *   y       device, fp32 [M, N], written.
 *   acc_out device, int32 [M, N], written when not NULL (the exact
 *           accumulator; for checking), else untouched.
 * TQ_ERR_UNSUPPORTED for M > 24 (use tq_gemm_prefill) or K > 32768.
 * Kernels (chosen by M from B200 measurements; many concurrent users make
 * decode a small batch: 1bit engine blog, "One GPU, many users"): M <= 2 the
 * streaming dp4a kernel; 3 <= M <= 24 the warp-MMA kernel (mma.sync int8 on
 * the masked packed bytes). The tensor-core (tcgen05) batched-decode kernel
 * runs the grouped calls from 25 tokens and tq_gemv_noalloc. The environment
 * variable TQ_BATCH_KERNEL=stream|mma|tc forces one where it applies (for
 * measurement).
 */
tq_status tq_gemv(const uint8_t *packed, float w_scale, const int8_t *xq,
                  const float *x_scale, const int32_t *x_sum, float *y, int32_t *acc_out,
                  int M, int N, int K, cudaStream_t stream);

/*
 * tq_gemm_prefill -- the same contract as tq_gemv for any M >= 1 (prompt
 * processing; prefill is set by the matrix units: 1bit engine blog, "Qwen3.8-27B
 * at 45.7 tok/s ..."). M >= 33 runs on the tensor cores (tcgen05, int8 in,
 * int32 accumulators in tensor memory, the 2-bit codes expanded in shared
 * memory, 128-feature x 256-token tiles, 128-token tiles for M <= 128);
 * smaller M runs tq_gemv's kernels. TQ_ERR_UNSUPPORTED for K > 32768,
 * N > 2^21 or M > 2^22.
 */
tq_status tq_gemm_prefill(const uint8_t *packed, float w_scale, const int8_t *xq,
                          const float *x_scale, const int32_t *x_sum, float *y,
                          int32_t *acc_out, int M, int N, int K, cudaStream_t stream);

/*
 * One projection of a decode layer stack, for the grouped calls below. All
 * pointers are device pointers with the meanings they have in
 * tq_quantize_act / tq_gemv; the shapes below are for M = 1 and become
 * [M, K], [M] and [M, N] in the _batch calls. tq_quantize_act_stack reads x
 * and writes xq, x_scale, x_sum (packed, y, acc_out unused, may be NULL);
 * tq_gemv_stack reads packed, xq, x_scale, x_sum and writes y and, when not
 * NULL, acc_out (x unused, may be NULL).
 */
typedef struct tq_proj {
    const uint8_t *packed;  /* [N/4, K] */
    const uint16_t *x;      /* bf16 [K]   (read by tq_quantize_act_stack) */
    int8_t *xq;             /* int8 [K]   (written by quantize, read by gemv) */
    float *x_scale;         /* fp32 [1] */
    int32_t *x_sum;         /* int32 [1] */
    float *y;               /* fp32 [N]   (written by gemv) */
    int32_t *acc_out;       /* int32 [N] or NULL */
    float w_scale;
    int N;
    int K;
    /* TQ_STACK_RMSNORM / TQ_STACK_RELU2_MUL only (else ignored): */
    const float *gain;      /* fp32 [K] RMSNorm gain */
    const float *x_f32;     /* fp32 [K] TQ_STACK_RELU2_MUL: the gate projection's output */
    const float *up;        /* fp32 [K] TQ_STACK_RELU2_MUL: the up projection's output */
    float eps;              /* RMSNorm epsilon, finite, >= 0 */
    int reserved;           /* set to 0 */
} tq_proj;

/* Flags for tq_gemv_stack. */
#define TQ_STACK_OVERLAP_PREV 1u /* weights are not written by work still in flight on
                                    the stream: the kernel may start streaming them
                                    before the previous kernel on the stream ends
                                    (programmatic dependent launch); activations,
                                    scales and sums are read only after it ends. */
#define TQ_STACK_QUANTIZE 2u     /* the same launch also quantises: x (bf16, 16-byte
                                    aligned) is the input, and xq, x_scale and x_sum
                                    are written with exactly the values
                                    tq_quantize_act_stack would write, instead of
                                    being read. One launch per call replaces the
                                    quantiser launch and the GEMV launch. */
#define TQ_STACK_RMSNORM 4u      /* as TQ_STACK_QUANTIZE, with RMSNorm (gain, eps)
                                    applied to x first: the values
                                    tq_rmsnorm_quantize would write. */
#define TQ_STACK_RELU2_MUL 8u    /* as TQ_STACK_RMSNORM on v = relu(x_f32)^2 * up
                                    (fp32 rows, 16-byte aligned): the values
                                    tq_relu2_mul_rmsnorm_quantize would write.
                                    With TQ_STACK_OVERLAP_PREV the launch streams
                                    weights while the kernel producing x_f32 and up
                                    finishes. At most one of the three quantising
                                    flags; the launch quantises its own inputs, so
                                    entries sharing one input each write identical
                                    xq, x_scale and x_sum. */

/*
 * tq_quantize_act_stack -- tq_quantize_act for each projection's single
 * token, all in one launch. projs is a HOST array of n_proj entries (read
 * during the call only). K % 16 == 0 for every entry.
 */
tq_status tq_quantize_act_stack(const tq_proj *projs, int n_proj, cudaStream_t stream);

/*
 * tq_gemv_stack -- tq_gemv (M = 1) for every projection, in one persistent
 * launch per 256 projections that streams all their weights back to back, in
 * projection order, with no drain between projections. projs is a HOST array
 * (read during the call only; the table travels in the launch parameters).
 * flags: TQ_STACK_OVERLAP_PREV, and at most one of TQ_STACK_QUANTIZE,
 * TQ_STACK_RMSNORM, TQ_STACK_RELU2_MUL. Without those, xq, x_scale and x_sum
 * are inputs (from tq_quantize_act_stack); with one, the launch computes
 * them from x (or x_f32 and up) and writes them.
 * Projections are independent: y of one must not be another's input within
 * the same call, and no buffer may be shared between two entries.
 */
tq_status tq_gemv_stack(const tq_proj *projs, int n_proj, unsigned flags, cudaStream_t stream);

/*
 * The same two calls for M tokens per projection (small-batch decode: each
 * projection's weights streamed once for all M rows): x bf16 [M, K], xq int8
 * [M, K], x_scale fp32 [M], x_sum int32 [M], y fp32 [M, N], acc_out int32
 * [M, N] or NULL, row-major. tq_quantize_act_stack_batch quantises every row
 * exactly as tq_quantize_act does (any M >= 0). tq_gemv_stack_batch takes
 * 0 <= M <= 32 (TQ_ERR_UNSUPPORTED above); M == 0 is a no-op and M == 1 is
 * tq_gemv_stack. The quantising flags need M == 1 (TQ_ERR_UNSUPPORTED
 * otherwise); TQ_STACK_OVERLAP_PREV is accepted at every M.
 *   M <= 2: the streaming kernel, one launch per 256 projections.
 *   3 <= M <= 24: the warp-MMA kernel, one launch per 256 projections (16-row
 *   tiles of all projections balanced over the SMs); no scratch memory.
 *   25 <= M <= 32: the tensor-core batched-decode kernel, one launch per 64
 *   projections, its K work split evenly over the SMs across projection
 *   boundaries. Tiles split between CTAs finish through a fixed device array
 *   compiled into the library (one slot per CTA), which every launch leaves
 *   zeroed, also one whose bounded wait gave up; the first call on a device
 *   (make it before any stream capture) and the first call after
 *   tq_device_error reported a nonzero code zero-fill it on `stream` first.
 *   Calls whose work overlaps on the GPU (two streams) race on that array and
 *   must be serialised by the caller.
 * TQ_STACK_OVERLAP_PREV lets the first launch start while the previous
 * kernel on the stream drains (programmatic dependent launch: weights may be
 * streamed early, activations, scales and outputs are touched only after
 * the previous kernel completes); later launches of the call always may.
 * TQ_BATCH_KERNEL (see tq_gemv) applies here too.
 */
tq_status tq_quantize_act_stack_batch(const tq_proj *projs, int n_proj, int M,
                                      cudaStream_t stream);

/*
 * tq_gemm_prefill_stack -- tq_gemm_prefill for several independent
 * projections at the same M (the rows of a prompt through, say, the gate
 * and up projections of a layer, or through several layers' projections
 * whose inputs are ready), each with the [M, K] / [M] / [M, N] shapes of the
 * _batch calls above. projs is a HOST array read during the call only; x,
 * flags-only fields and `reserved` are ignored. For M >= 33 one launch takes
 * up to 16 projections: the 128-feature tiles of all of them are dealt to
 * persistent CTAs longest first (by K), so that projections too small to
 * fill the GPU alone fill it together, and each CTA's accumulator is
 * double-buffered in tensor memory so that its output stores overlap the
 * next tile's MMAs. M <= 32 runs tq_gemv_stack_batch. Results are those of
 * tq_gemm_prefill on each projection, bit for bit. Projections are
 * independent: no output may be another's input and no buffer may be shared.
 * Errors: those of tq_gemm_prefill for any entry (nothing is launched).
 */
tq_status tq_gemm_prefill_stack(const tq_proj *projs, int n_proj, int M, cudaStream_t stream);
tq_status tq_gemv_stack_batch(const tq_proj *projs, int n_proj, int M, unsigned flags,
                              cudaStream_t stream);

/*
 * tq_gemv_noalloc -- tq_gemv for 5 <= M <= 32 tokens computed by the
 * stream-K formulation of the batched-decode kernel, which allocates no device
 * memory at all. No passage of the method corresponds to this call; it exists
 * for callers that cannot call cudaMalloc: a host process whose device memory
 * is all owned by another allocator (a framework's caching pool, a
 * pre-reserved arena) or a latency-critical loop that cannot afford the
 * implicit device synchronisation of an allocation. tq_gemv splits K inside
 * thread-block clusters and needs no scratch; the stream-K formulation spreads
 * every projection over all SMs and keeps its split-K partial sums in a fixed
 * 4 MiB device array compiled into the library, so it works for N up to the
 * size that fits there (TQ_ERR_UNSUPPORTED beyond it; at M <= 16 that is
 * N <= 65,408, at 17 <= M <= 32 N <= 32,640).
 *   Same arguments, results and alignment rules as tq_gemv.
 *   The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress); make that first call before any stream capture.
 *   Every call shares the one array: the part a call uses is zero-filled on
 *   `stream` before its kernel, but calls whose work overlaps on the GPU
 *   (e.g. on two streams) race on it and must be serialised by the caller.
 */
tq_status tq_gemv_noalloc(const uint8_t *packed, float w_scale, const int8_t *xq,
                          const float *x_scale, const int32_t *x_sum, float *y, int32_t *acc_out,
                          int M, int N, int K, cudaStream_t stream);

/*
 * The steps either side of the GEMV in a BitNet decoder layer, each fused
 * with the activation quantiser so that only int8 codes leave the kernel
 * (lemon-mlx-engine issue, section "Architecture": relu_squared in place of
 * silu, sub-layer norms attn_sub_norm before o_proj and ffn_sub_norm before
 * down_proj, RMSNorm). The pages give no formulas; the reading:
 *   r = fl32(1 / sqrt(sum_k v^2 / K + eps))   (the sum and root in fp64)
 *   h[k] = fl32(fl32(v[k] * r) * gain[k]),  then the absmax quantiser of
 *   tq_quantize_act on h (xq, x_scale, x_sum as there).
 * One CTA per token row, launched with programmatic stream serialisation:
 * the kernel waits for the previous kernel on the stream to complete before
 * it touches memory, and lets the next one start early (a tq_gemv_stack with
 * TQ_STACK_OVERLAP_PREV streams weights meanwhile).
 * Host checks: 0 <= M, 0 < K <= 32768, K % 16 == 0,
 * eps >= 0 and finite; byte tensors and fp32 rows 16-byte aligned, vectors
 * 4-byte aligned. M == 0 is a no-op.
 *
 * tq_rmsnorm_quantize -- v = x: exactly one of x_bf16 [M, K] (bf16 bits) and
 * x_f32 [M, K] is non-NULL (TQ_ERR_VALUE otherwise). gain fp32 [K].
 */
tq_status tq_rmsnorm_quantize(const uint16_t *x_bf16, const float *x_f32, const float *gain,
                              float eps, int8_t *xq, float *x_scale, int32_t *x_sum, int M,
                              int K, cudaStream_t stream);

/*
 * tq_relu2_mul_rmsnorm_quantize -- the FFN's down_proj input: v =
 * fl32(fl32(relu(gate)^2) * up) from the gate and up projections' fp32
 * outputs gate, up [M, K], then RMSNorm (ffn_sub_norm, gain [K]) and the
 * quantiser, in one pass over the rows.
 */
tq_status tq_relu2_mul_rmsnorm_quantize(const float *gate, const float *up, const float *gain,
                                        float eps, int8_t *xq, float *x_scale, int32_t *x_sum,
                                        int M, int K, cudaStream_t stream);

/*
 * tq_absmean_pack -- quantise latent (or pre-dequantised) weights to ternary
 * by absmean and pack them (1bit.systems post "the full arc ...", read-more
 * item "Training-Runs": absmean; the result is the packed tensor and its
 * .weight_scale). Reading: gamma = fl32(sum |W| / (N K)) with the sum in
 * fp64, w = clamp(rne(fl32(W / gamma)), -1, 1) (gamma == 0: w = 0), codes
 * w + 1 packed as tq_pack_host does.
 *   w_bf16  device, bf16 bits [N, K], 16-byte aligned
 *   packed  device, uint8 [N/4, K], 16-byte aligned (written)
 *   w_scale device, fp32 [1] (written: gamma)
 * N % 4 == 0, K % 16 == 0. Two launches (reduction, then quantise-and-pack);
 * the reduction's partial sums live in a fixed device array, so calls that
 * overlap on the GPU (on several streams) race on it.
 */
tq_status tq_absmean_pack(const uint16_t *w_bf16, uint8_t *packed, float *w_scale, int N, int K,
                          cudaStream_t stream);

/*
 * tq_hadamard_quantize_act -- 4-bit activation codes for prompt processing by
 * the Hadamard route (1bit engine blog, "509 tokens a second of prompt: the
 * Hadamard route ships" and "Qwen3.8-27B at 45.7 tok/s ...": 4-bit
 * activations on the matrix units, kept accurate by a Hadamard rotation;
 * 1bit.systems README, read-more item "Training-Runs -- BitNet v2 Hadamard").
 * The pages print no formula. Reading: per token row, each block of n
 * consecutive entries is rotated, h = H_n x / sqrt(n), H_n the
 * Sylvester-Hadamard matrix (H_n[i][j] = (-1)^popcount(i & j)); the sums are
 * exact in fp64 (bf16 inputs) and fl64(sum * fl64(1/sqrt(n))) is rounded once
 * to fp32. Then amax = max |h|, s = fl32(7 / amax),
 * xq = clamp(round_half_even(fl32(h * s)), -7, 7), x_scale = fl32(amax / 7),
 * x_sum = sum xq (an all-zero row gives zeros).
 * The codes, one per int8, feed tq_gemm_prefill (or tq_gemv) exactly like
 * 8-bit codes; the weights are those of the rotated basis (the rotation's
 * transpose is folded into them when they are trained or converted).
 *   x       device, bf16 bit patterns [M, K], 16-byte aligned
 *   xq      device, int8 [M, K], 16-byte aligned (written; values -7..7)
 *   x_scale device, fp32 [M] (written); x_sum device, int32 [M] (written;
 *           may be NULL)
 *   n       block size: 32, 64, 128, 256, 512 or 1024, dividing K
 * 0 <= K <= 32768 (M == 0 or K == 0: no-op); TQ_ERR_SHAPE if n is not one
 * of those or does not divide K. One CTA per token row; asynchronous.
 */
tq_status tq_hadamard_quantize_act(const uint16_t *x, int8_t *xq, float *x_scale, int32_t *x_sum,
                                   int M, int K, int n, cudaStream_t stream);

/*
 * tq_hadamard_quantize_act_stack -- tq_hadamard_quantize_act for M token rows
 * of each of n_proj projections (tq_proj's x, xq, x_scale, x_sum and K, with
 * the [M, K] / [M] shapes of the _batch calls; other fields ignored) in one
 * launch per 512 projections, every K a multiple of n. Results are those of
 * tq_hadamard_quantize_act on each projection, byte for byte. projs is a HOST
 * array read during the call only. Errors as tq_hadamard_quantize_act's, for
 * any entry (nothing is launched).
 */
tq_status tq_hadamard_quantize_act_stack(const tq_proj *projs, int n_proj, int M, int n,
                                         cudaStream_t stream);

/*
 * Binary g128 weights (baguaai "BitNet" tag page, Bonsai 27B item: a true
 * 1-bit binary scheme in which 128 weights share one fp16 scale, about 1.125
 * bits per weight). The page gives no bit order, group direction or
 * activation format. Readings:
 *   - a weight is +1 or -1; bit 1 is +1, bit 0 is -1;
 *   - bits uint8 [N/8, K]: bit p of byte (i, k) is the weight of output row
 *     i + p*N/8 at column k (the plane layout of the ternary format);
 *   - a group is 128 consecutive k of one output row (K % 128 == 0), with one
 *     fp16 scale; the device keeps the scales as [N/8, K/128, 8], entry
 *     (i, g, p) scaling row i + p*N/8 on group g;
 *   - activations: the per-token int8 absmax codes of tq_quantize_act;
 *   - acc[m, n] = sum_k w[n, k] xq[m, k] (int32, exact);
 *     y[m, n] = fl32(x_scale[m] * sum_g scale[n, g] * sum_{k in g} w xq),
 *     each product exact in fp64 and the sum in fp64.
 *
 * tq_pack_binary_host -- host packing, synchronous.
 *   w             host, int8 [N, K], every value -1 or +1
 *   scales        host, fp16 bit patterns [N, K/128] (scales[n, g] for
 *                 columns 128 g .. 128 g + 127)
 *   bits          host, uint8 [N/8, K] (written)
 *   scales_packed host, fp16 bit patterns [N/8, K/128, 8] (written)
 * N % 8 == 0, K % 128 == 0, N, K >= 0 (TQ_ERR_SHAPE). TQ_ERR_VALUE if a
 * weight is not -1 or +1 (outputs then partly written).
 */
tq_status tq_pack_binary_host(const int8_t *w, const uint16_t *scales, uint8_t *bits,
                              uint16_t *scales_packed, int N, int K);

/*
 * tq_gemv_binary -- decode GEMV over binary g128 weights, 1 <= M <= 4 tokens.
 *   bits          device, uint8 [N/8, K], 16-byte aligned
 *   scales_packed device, fp16 bits [N/8, K/128, 8], 16-byte aligned
 *   xq            device, int8 [M, K], 16-byte aligned
 *   x_scale       device, fp32 [M]
 *   y             device, fp32 [M, N] (written)
 *   acc_out       device, int32 [M, N] (written: sum_k w xq) or NULL
 * N % 8 == 0, K % 128 == 0, K <= 32768; M > 4 is TQ_ERR_UNSUPPORTED; M == 0,
 * N == 0 or K == 0 (all outputs 0) handled. One persistent launch streaming
 * the bits and scales; asynchronous on `stream`.
 *
 * tq_gemv_binary_stack -- the same for a table of projections (one launch per
 * 128 of them), each with its own shapes and buffers, M tokens each.
 */
tq_status tq_gemv_binary(const uint8_t *bits, const uint16_t *scales_packed, const int8_t *xq,
                         const float *x_scale, float *y, int32_t *acc_out, int M, int N, int K,
                         cudaStream_t stream);

typedef struct tq_binary_proj {
    const uint8_t *bits;            /* device, [N/8, K] */
    const uint16_t *scales_packed;  /* device, [N/8, K/128, 8] fp16 */
    const int8_t *xq;               /* device, [M, K] */
    const float *x_scale;           /* device, [M] */
    float *y;                       /* device, [M, N] */
    int32_t *acc_out;               /* device, [M, N] or NULL */
    int N, K;
} tq_binary_proj;

tq_status tq_gemv_binary_stack(const tq_binary_proj *projs, int n_proj, int M,
                               cudaStream_t stream);

/*
 * tq_selftest_wait_timeout -- exercise the failure path of the kernels'
 * bounded waits without a fault: one thread waits, with the same bounded
 * wait the kernels use, on an mbarrier that nothing ever arrives on. After
 * limit_us (1 .. 2,000,000) microseconds the wait gives up, sets bit 1 of the
 * device error word and the kernel returns; the context stays usable. Read
 * the result with tq_device_error. Asynchronous on `stream`.
 */
tq_status tq_selftest_wait_timeout(unsigned limit_us, cudaStream_t stream);

/*
 * tq_device_error -- read (and if reset != 0, clear) the library's device
 * error word on the current device. Synchronises the device. 0 means no
 * kernel has reported an error. A nonzero value means a kernel gave up a
 * bounded wait (its outputs are then invalid); bits: 1 = pipeline wait timed
 * out.
 */
tq_status tq_device_error(uint32_t *code, int reset);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
