// layer_ops.cu -- the steps either side of the ternary GEMV in a BitNet
// decoder layer, fused with the activation quantiser, and the absmean weight
// quantiser-packer.
//
// The pages describe the model as a Llama variant with relu_squared in place
// of silu and sub-layer norms (attn_sub_norm before o_proj, ffn_sub_norm
// before down_proj), RMSNorm among its ops (lemon-mlx-engine issue, section
// "Architecture"), and absmean quantisation-aware training (1bit.systems post
// "the full arc ...", read-more item "Training-Runs"); the packed weights
// carry one .weight_scale per tensor (same issue, "What We Need" item 2).
// No formula is printed; the arithmetic here (shared with no other code but
// quant_core.cuh's quantiser):
//   RMSNorm:  r = fl32(1 / sqrt(sum_k v^2 / K + eps)) with the sum and the
//             root in fp64, h = fl32(fl32(v * r) * gain)
//   relu^2:   v = fl32(fl32(max(a,0)^2) * b) for the FFN's gate a and up b
//   absmean:  gamma = fl32(sum |W| / (N K)) (fp64 sum), w = clamp(rne(fl32(W
//             / gamma)), -1, 1), code w + 1 packed four rows to a byte
//
// The normalise-and-quantise kernels take one CTA of 1024 threads per token:
// pass 1 reads the row into shared memory and reduces the sum of squares
// (fp64), pass 2 the largest |h| (exact), pass 3 writes the codes and
// reduces their sum; passes 2 and 3 recompute h from shared memory, so the
// row is read once and nothing but the codes is written. They are launched
// with programmatic stream serialisation and wait for the previous grid
// before any memory access, so a following stack GEMV launched with
// TQ_STACK_OVERLAP_PREV streams its weights while they run.
#include <atomic>
#include <algorithm>
#include <cfloat>

#include "quant_core.cuh"
#include "tq_internal.h"

namespace tq {

namespace {

constexpr int kRowThreads = 1024;

enum RowInput : int { kInBf16 = 0, kInF32 = 1, kInRelu2Mul = 2 };

struct RowParams {
    const uint16_t *x_bf16;  // kInBf16: [M, K]
    const float *x_f32;      // kInF32: [M, K]; kInRelu2Mul: the gate [M, K]
    const float *up;         // kInRelu2Mul: [M, K]
    const float *gain;       // [K]
    float eps;
    int8_t *xq;              // [M, K]
    float *x_scale;          // [M]
    int32_t *x_sum;          // [M]
    int K;
};

// Four consecutive inputs v[k .. k+3] of row m (k a multiple of 4).
template <int In>
__device__ __forceinline__ float4 load4(const RowParams &p, size_t base, int k)
{
    if constexpr (In == kInBf16) {
        const uint2 u = __ldg(reinterpret_cast<const uint2 *>(p.x_bf16 + base + k));
        return make_float4(bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y));
    } else if constexpr (In == kInF32) {
        return __ldg(reinterpret_cast<const float4 *>(p.x_f32 + base + k));
    } else {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(p.x_f32 + base + k));
        const float4 b = __ldg(reinterpret_cast<const float4 *>(p.up + base + k));
        auto r2 = [](float g, float u) {
            const float r = fmaxf(g, 0.0f);
            return __fmul_rn(__fmul_rn(r, r), u);
        };
        return make_float4(r2(a.x, b.x), r2(a.y, b.y), r2(a.z, b.z), r2(a.w, b.w));
    }
}

// Reduce over the CTA; every thread gets the result. `red` has one slot per
// warp. The operations are exact in any order except the fp64 sum, whose
// order is fixed (lanes in a butterfly, then warps in index order).
template <typename T, typename Op>
__device__ __forceinline__ T cta_reduce(T v, Op op, T *red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
    if ((threadIdx.x & 31) == 0)
        red[threadIdx.x >> 5] = v;
    __syncthreads();
    T r = red[0];
#pragma unroll
    for (int w = 1; w < kRowThreads / 32; ++w)
        r = op(r, red[w]);
    __syncthreads();
    return r;
}

template <int In>
__global__ void __launch_bounds__(kRowThreads)
rms_quant_kernel(const RowParams p)
{
    __shared__ double red_d[kRowThreads / 32];
    __shared__ float red_f[kRowThreads / 32];
    __shared__ int red_i[kRowThreads / 32];
    extern __shared__ float4 row[];  // the row's inputs v, K / 4 vectors
    const int K = p.K;
    const size_t base = size_t(blockIdx.x) * K;
    // Launched with programmatic stream serialisation: let the next grid (a
    // GEMV that streams weights first) start, and wait for the previous grid
    // (which may produce this row) before touching memory.
    pdl_launch_dependents();
    pdl_wait();

    // Pass 1 reads the row once from global memory into shared memory.
    double ss = 0.0;
    for (int k = 4 * threadIdx.x; k < K; k += 4 * kRowThreads) {
        const float4 v = load4<In>(p, base, k);
        row[k >> 2] = v;
        ss += double(v.x) * v.x;  // each square exact in fp64
        ss += double(v.y) * v.y;
        ss += double(v.z) * v.z;
        ss += double(v.w) * v.w;
    }
    ss = cta_reduce(ss, [](double a, double b) { return a + b; }, red_d);
    const float r = __double2float_rn(1.0 / sqrt(ss / double(K) + double(p.eps)));

    auto h_of = [&](float v, int k) { return __fmul_rn(__fmul_rn(v, r), __ldg(p.gain + k)); };
    float amax = 0.0f;
    for (int k = 4 * threadIdx.x; k < K; k += 4 * kRowThreads) {
        const float4 v = row[k >> 2];
        amax = fmaxf(amax, fabsf(h_of(v.x, k)));
        amax = fmaxf(amax, fabsf(h_of(v.y, k + 1)));
        amax = fmaxf(amax, fabsf(h_of(v.z, k + 2)));
        amax = fmaxf(amax, fabsf(h_of(v.w, k + 3)));
    }
    amax = cta_reduce(amax, [](float a, float b) { return fmaxf(a, b); }, red_f);
    const float s = quant_inv_scale(amax);

    int sum = 0;
    for (int k = 4 * threadIdx.x; k < K; k += 4 * kRowThreads) {
        const float4 v = row[k >> 2];
        const int a = code_of(h_of(v.x, k), s), b = code_of(h_of(v.y, k + 1), s);
        const int c = code_of(h_of(v.z, k + 2), s), d = code_of(h_of(v.w, k + 3), s);
        sum += a + b + c + d;
        *reinterpret_cast<uint32_t *>(p.xq + base + k) =
            (uint32_t(a) & 0xFFu) | ((uint32_t(b) & 0xFFu) << 8) | ((uint32_t(c) & 0xFFu) << 16) |
            ((uint32_t(d) & 0xFFu) << 24);
    }
    sum = cta_reduce(sum, [](int a, int b) { return a + b; }, red_i);
    if (threadIdx.x == 0) {
        p.x_scale[blockIdx.x] = quant_scale(amax);
        p.x_sum[blockIdx.x] = sum;
    }
}

// ----------------------------------------------------------- absmean pack
constexpr int kAbsThreads = 256;
constexpr int kAbsMaxBlocks = 1024;

// Fixed device scratch of the absmean reduction: one fp64 partial per block
// and a counter that the last block resets (calls on one stream are ordered;
// calls overlapping on several streams race on it).
__device__ double g_abs_partial[kAbsMaxBlocks];
__device__ unsigned g_abs_count;

// Pass 1: sum |W| (fp64) per block; the last block to finish adds the
// partials in block order and writes gamma = fl32(sum / n).
__global__ void __launch_bounds__(kAbsThreads)
absmean_sum_kernel(const uint16_t *__restrict__ w, size_t n, float *w_scale)
{
    __shared__ double red[kAbsThreads / 32];
    __shared__ bool last;
    const size_t n8 = n / 8;  // 16-byte vectors of 8 bf16 (n is a multiple of 16)
    double s = 0.0;
    for (size_t i = size_t(blockIdx.x) * kAbsThreads + threadIdx.x; i < n8;
         i += size_t(gridDim.x) * kAbsThreads) {
        const uint4 u = __ldg(reinterpret_cast<const uint4 *>(w) + i);
        s += double(fabsf(bf16_lo(u.x))) + double(fabsf(bf16_hi(u.x))) +
             double(fabsf(bf16_lo(u.y))) + double(fabsf(bf16_hi(u.y))) +
             double(fabsf(bf16_lo(u.z))) + double(fabsf(bf16_hi(u.z))) +
             double(fabsf(bf16_lo(u.w))) + double(fabsf(bf16_hi(u.w)));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        s += __shfl_xor_sync(0xffffffffu, s, o);
    if ((threadIdx.x & 31) == 0)
        red[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        double b = 0.0;
        for (int i = 0; i < kAbsThreads / 32; ++i)
            b += red[i];
        g_abs_partial[blockIdx.x] = b;
        __threadfence();
        last = atomicAdd(&g_abs_count, 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (last && threadIdx.x == 0) {
        __threadfence();
        double t = 0.0;
        for (unsigned b = 0; b < gridDim.x; ++b)
            t += __ldcg(&g_abs_partial[b]);
        *w_scale = n > 0 ? __double2float_rn(t / double(n)) : 0.0f;
        g_abs_count = 0;
    }
}

// Pass 2: each thread writes four packed bytes (packed row i, columns k..k+3):
// byte (i, k) holds the codes of rows i + p N/4, p = 0..3, in bits 2p..2p+1.
__global__ void __launch_bounds__(kAbsThreads)
absmean_pack_kernel(const uint16_t *__restrict__ w, uint8_t *__restrict__ packed,
                    const float *__restrict__ w_scale, int N4, int K)
{
    const float g = *w_scale;
    const int K4 = K / 4;
    const size_t total = size_t(N4) * K4;
    for (size_t t = size_t(blockIdx.x) * kAbsThreads + threadIdx.x; t < total;
         t += size_t(gridDim.x) * kAbsThreads) {
        const int i = int(t / K4), k = int(t - size_t(i) * K4) * 4;
        uint32_t word = 0;
#pragma unroll
        for (int p4 = 0; p4 < 4; ++p4) {
            const uint2 u = __ldg(reinterpret_cast<const uint2 *>(
                w + (size_t(i) + size_t(p4) * N4) * K + k));
            const float v[4] = {bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y)};
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                int c = 1;  // gamma == 0: every weight quantises to 0
                if (g != 0.0f)
                    c = min(max(__float2int_rn(__fdiv_rn(v[b], g)), -1), 1) + 1;
                word |= uint32_t(c) << (8 * b + 2 * p4);
            }
        }
        *reinterpret_cast<uint32_t *>(packed + size_t(i) * K + k) = word;
    }
}

}  // namespace

cudaError_t launch_rms_quant(int input, const uint16_t *x_bf16, const float *x_f32,
                             const float *up, const float *gain, float eps, int8_t *xq,
                             float *x_scale, int32_t *x_sum, int M, int K, cudaStream_t stream)
{
    RowParams p{x_bf16, x_f32, up, gain, eps, xq, x_scale, x_sum, K};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(M);
    cfg.blockDim = dim3(kRowThreads);
    cfg.dynamicSmemBytes = size_t(K) * sizeof(float);
    cfg.stream = stream;
    static std::atomic<int> configured_dev{-1};  // the row may need more than 48 KB
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        const int most = int(kStreamMaxK * sizeof(float));
        cudaError_t e = cudaFuncSetAttribute(rms_quant_kernel<kInBf16>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, most);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(rms_quant_kernel<kInF32>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, most);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(rms_quant_kernel<kInRelu2Mul>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, most);
        if (e != cudaSuccess)
            return e;
        configured_dev = dev;
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (input == kInBf16)
        e = cudaLaunchKernelEx(&cfg, rms_quant_kernel<kInBf16>, p);
    else if (input == kInF32)
        e = cudaLaunchKernelEx(&cfg, rms_quant_kernel<kInF32>, p);
    else
        e = cudaLaunchKernelEx(&cfg, rms_quant_kernel<kInRelu2Mul>, p);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_absmean_pack(const uint16_t *w, uint8_t *packed, float *w_scale, int N, int K,
                                cudaStream_t stream)
{
    const size_t n = size_t(N) * K;
    const int sms = device_sm_count();
    const size_t want = (n / 8 + kAbsThreads - 1) / kAbsThreads;
    const int blocks = int(std::min<size_t>(std::max<size_t>(want, 1), size_t(std::min(
                                                                   kAbsMaxBlocks, 4 * sms))));
    absmean_sum_kernel<<<blocks, kAbsThreads, 0, stream>>>(w, n, w_scale);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || n == 0)
        return e;
    const size_t words = n / 16;  // four packed bytes per thread
    const int blocks2 = int(std::min<size_t>((words + kAbsThreads - 1) / kAbsThreads,
                                             size_t(8 * sms)));
    absmean_pack_kernel<<<blocks2, kAbsThreads, 0, stream>>>(w, packed, w_scale, N / 4, K);
    return cudaGetLastError();
}

}  // namespace tq
