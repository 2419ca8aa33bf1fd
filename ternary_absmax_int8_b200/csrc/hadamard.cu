// hadamard.cu -- Hadamard-rotated 4-bit activation codes for prompt
// processing.
//
// The pages' engine reads prompts faster with 4-bit activations on the
// matrix units, a Hadamard rotation keeping them accurate (1bit engine blog,
// "509 tokens a second of prompt: the Hadamard route ships"; 1bit.systems
// README, "Training-Runs -- BitNet v2 Hadamard"). Per token row:
//
//   h = H_n x / sqrt(n) on each block of n consecutive entries (n a power of
//       two, 32..1024), H_n the Sylvester-Hadamard matrix
//       (H_n[i][j] = (-1)^popcount(i & j));
//   amax = max |h|, s = fl32(7 / amax), q = clamp(rne(fl32(h * s)), -7, 7),
//   x_scale = fl32(amax / 7), x_sum = sum q (amax == 0 gives zeros).
//
// The codes, one per int8, then enter the same int8 tensor-core contraction
// as 8-bit codes (sm_100 has no integer 4-bit MMA kind). The rotation is the
// fast Walsh-Hadamard butterfly in fp64: for bf16 inputs every partial sum
// is exact, so the butterfly's order gives the same value as the plain
// matrix-vector sum; fl64(sum * fl64(1/sqrt(n))) is then rounded once to fp32.
//
// One CTA of 256 threads per token row (one launch per call, or per table of
// projections in the stack form). Warp w rotates blocks w, w + 8, ...:
// lane l holds entries l*E .. l*E + E - 1 of a block (E = n / 32) in fp64
// registers; butterfly stages with a stride below E stay in the lane, the
// others pair lane l with lane l ^ (stride / E) through shuffles. The fp32
// results wait in shared memory for the row's amax, then become codes.
#include <atomic>
#include <cmath>

#include "tq_internal.h"

namespace tq {

namespace {

constexpr int kHadThreads = 256;
constexpr int kHadWarps = kHadThreads / 32;

template <typename T, typename Op>
__device__ __forceinline__ T block_reduce_had(T v, Op op, T *red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0)
        red[warp] = v;
    __syncthreads();
    T r = red[0];
#pragma unroll
    for (int w = 1; w < kHadWarps; ++w)
        r = op(r, red[w]);
    __syncthreads();  // red is reused by the next reduction
    return r;
}

struct HMax {
    __device__ float operator()(float a, float b) const { return fmaxf(a, b); }
};
struct HAdd {
    __device__ int operator()(int a, int b) const { return a + b; }
};

__device__ __forceinline__ int code4(float h, float s)
{
    const int r = __float2int_rn(__fmul_rn(h, s));  // one fp32 rounding, ties to even
    return min(max(r, -7), 7);
}

// One token row (the whole CTA): E entries per lane (block size n = 32 E).
template <int E>
__device__ __forceinline__ void hadamard_row(const uint16_t *__restrict__ row,
                                             int8_t *__restrict__ qrow, float *__restrict__ x_scale,
                                             int32_t *__restrict__ x_sum, int K, double c)
{
    extern __shared__ __align__(16) float hs[];  // [K] rotated row, fp32
    __shared__ float red_f[kHadWarps];
    __shared__ int red_i[kHadWarps];
    constexpr int n = 32 * E;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    float amax = 0.0f;
    for (int b = warp; b < K / n; b += kHadWarps) {
        const uint16_t *src = row + size_t(b) * n + lane * E;
        double v[E];
        if constexpr (E >= 8) {
#pragma unroll
            for (int i = 0; i < E; i += 8) {
                const uint4 u = __ldg(reinterpret_cast<const uint4 *>(src + i));
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    v[i + 2 * j] = double(__uint_as_float(w[j] << 16));
                    v[i + 2 * j + 1] = double(__uint_as_float(w[j] & 0xFFFF0000u));
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < E; ++i)
                v[i] = double(__uint_as_float(uint32_t(__ldg(src + i)) << 16));
        }
        // in-lane stages: stride h < E
#pragma unroll
        for (int h = 1; h < E; h <<= 1) {
#pragma unroll
            for (int i = 0; i < E; ++i) {
                if ((i & h) == 0) {
                    const double a = v[i], d = v[i + h];
                    v[i] = __dadd_rn(a, d);
                    v[i + h] = __dsub_rn(a, d);
                }
            }
        }
        // cross-lane stages: stride E t pairs lane l with lane l ^ t; the
        // lower lane keeps a + b, the upper b' = a - b
#pragma unroll
        for (int t = 1; t < 32; t <<= 1) {
            const bool upper = lane & t;
#pragma unroll
            for (int i = 0; i < E; ++i) {
                const double o = __shfl_xor_sync(0xffffffffu, v[i], t);
                v[i] = upper ? __dsub_rn(o, v[i]) : __dadd_rn(v[i], o);
            }
        }
        float *dst = hs + b * n + lane * E;
#pragma unroll
        for (int i = 0; i < E; ++i) {
            const float h = __double2float_rn(__dmul_rn(v[i], c));
            dst[i] = h;
            amax = fmaxf(amax, fabsf(h));
        }
    }
    amax = block_reduce_had(amax, HMax(), red_f);  // also orders the hs stores

    const float s = amax > 0.0f ? __fdiv_rn(7.0f, amax) : 0.0f;
    int sum = 0;
    uint32_t *qw = reinterpret_cast<uint32_t *>(qrow);
    for (int k4 = threadIdx.x; k4 < K / 4; k4 += kHadThreads) {
        const float4 h = reinterpret_cast<const float4 *>(hs)[k4];
        const int a = code4(h.x, s), b = code4(h.y, s), cc = code4(h.z, s), d = code4(h.w, s);
        sum += a + b + cc + d;
        qw[k4] = (uint32_t(a) & 0xFFu) | ((uint32_t(b) & 0xFFu) << 8) |
                 ((uint32_t(cc) & 0xFFu) << 16) | ((uint32_t(d) & 0xFFu) << 24);
    }
    sum = block_reduce_had(sum, HAdd(), red_i);
    if (threadIdx.x == 0) {
        *x_scale = amax > 0.0f ? __fdiv_rn(amax, 7.0f) : 0.0f;
        if (x_sum)
            *x_sum = sum;
    }
}

template <int E>
__global__ void __launch_bounds__(kHadThreads)
hadamard_quant4_kernel(const uint16_t *__restrict__ x, int8_t *__restrict__ xq,
                       float *__restrict__ x_scale, int32_t *__restrict__ x_sum, int K, double c)
{
    const size_t m = blockIdx.x;
    hadamard_row<E>(x + m * size_t(K), xq + m * size_t(K), x_scale + m, x_sum ? x_sum + m : nullptr,
                    K, c);
}

// The rows of a table of projections, one CTA per row (row r belongs to the
// entry with the largest row0 <= r).
template <int E>
__global__ void __launch_bounds__(kHadThreads)
hadamard_quant4_stack_kernel(const __grid_constant__ QuantStackParams p, double c)
{
    const int r = blockIdx.x;
    int lo = 0, hi = p.n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.e[mid].row0 <= r)
            lo = mid;
        else
            hi = mid - 1;
    }
    const QuantStackEntry &e = p.e[lo];
    const size_t m = size_t(r - e.row0);
    hadamard_row<E>(e.x + m * e.K, e.xq + m * e.K, e.x_scale + m, e.x_sum ? e.x_sum + m : nullptr,
                    e.K, c);
}

template <int E>
cudaError_t launch_e(const uint16_t *x, int8_t *xq, float *x_scale, int32_t *x_sum, int M, int K,
                     cudaStream_t stream)
{
    const size_t smem = size_t(K) * sizeof(float);
    static std::atomic<int> configured_dev{-1};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (configured_dev != dev) {
        // the rotated row of the longest K (32768 fp32), next to 64 bytes of
        // static reduction slots
        e = cudaFuncSetAttribute(hadamard_quant4_kernel<E>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(kStreamMaxK * sizeof(float)));
        if (e != cudaSuccess)
            return e;
        configured_dev = dev;
    }
    const int n = 32 * E;
    const double c = 1.0 / sqrt(double(n));  // IEEE sqrt and divide: the oracle's constant
    hadamard_quant4_kernel<E><<<M, kHadThreads, smem, stream>>>(x, xq, x_scale, x_sum, K, c);
    return cudaGetLastError();
}

template <int E>
cudaError_t launch_stack_e(const QuantStackParams &p, int max_k, cudaStream_t stream)
{
    static std::atomic<int> configured_dev{-1};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (configured_dev != dev) {
        e = cudaFuncSetAttribute(hadamard_quant4_stack_kernel<E>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(kStreamMaxK * sizeof(float)));
        if (e != cudaSuccess)
            return e;
        configured_dev = dev;
    }
    const double c = 1.0 / sqrt(double(32 * E));  // IEEE sqrt and divide: the oracle's constant
    hadamard_quant4_stack_kernel<E><<<p.rows, kHadThreads, size_t(max_k) * sizeof(float), stream>>>(p, c);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_hadamard_quant4_stack(const QuantStackParams &p, int max_k, int n,
                                         cudaStream_t stream)
{
    if (p.rows <= 0)
        return cudaSuccess;
    switch (n) {
    case 32: return launch_stack_e<1>(p, max_k, stream);
    case 64: return launch_stack_e<2>(p, max_k, stream);
    case 128: return launch_stack_e<4>(p, max_k, stream);
    case 256: return launch_stack_e<8>(p, max_k, stream);
    case 512: return launch_stack_e<16>(p, max_k, stream);
    case 1024: return launch_stack_e<32>(p, max_k, stream);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_hadamard_quant4(const uint16_t *x, int8_t *xq, float *x_scale, int32_t *x_sum,
                                   int M, int K, int n, cudaStream_t stream)
{
    if (M == 0)
        return cudaSuccess;
    switch (n) {
    case 32: return launch_e<1>(x, xq, x_scale, x_sum, M, K, stream);
    case 64: return launch_e<2>(x, xq, x_scale, x_sum, M, K, stream);
    case 128: return launch_e<4>(x, xq, x_scale, x_sum, M, K, stream);
    case 256: return launch_e<8>(x, xq, x_scale, x_sum, M, K, stream);
    case 512: return launch_e<16>(x, xq, x_scale, x_sum, M, K, stream);
    case 1024: return launch_e<32>(x, xq, x_scale, x_sum, M, K, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace tq
