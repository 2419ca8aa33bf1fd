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
// One CTA of 128 threads per token row (one launch per call, or per table of
// projections in the stack form). A block of n entries is held by E = n / 32
// lanes, 32 consecutive entries each in fp64 registers, so a warp rotates
// 32 / E blocks at a time: the five butterfly stages with a stride below 32
// stay in the lane, the log2(E) others pair lane l with lane l ^ (stride /
// 32) through shuffles. The fp32 results wait in shared memory for the
// row's amax, then become codes.
#include <atomic>
#include <cmath>

#include "tq_internal.h"

namespace tq {

namespace {

constexpr int kHadThreads = 128;
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

// The rotated row waits in shared memory as fp32, each lane's run of 32
// values followed by 4 floats of padding, so that the lanes' 16-byte stores
// fall in distinct banks: value k sits at k + 4 (k / 32).
__host__ __device__ constexpr size_t had_smem_floats(int K) { return size_t(K) + size_t(K / 32) * 4; }

// One token row (the whole CTA), block size n = 32 E: a block is held by E
// lanes of 32 consecutive entries each, so a warp takes 32 / E blocks at a
// time; the five butterfly stages with a stride below 32 stay in the lane,
// the log2(E) others pair lanes through shuffles.
template <int E>
__device__ __forceinline__ void hadamard_row(const uint16_t *__restrict__ row,
                                             int8_t *__restrict__ qrow, float *__restrict__ x_scale,
                                             int32_t *__restrict__ x_sum, int K, double c)
{
    extern __shared__ __align__(16) float hs[];  // rotated row, fp32, padded
    __shared__ float red_f[kHadWarps];
    __shared__ int red_i[kHadWarps];
    constexpr int n = 32 * E;
    constexpr int kEL = 32;       // entries per lane
    constexpr int kBPW = 32 / E;  // blocks per warp pass
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slot = lane / E, sl = lane % E;  // block slot of the pass, lane within the block
    const int nblk = K / n;

    float amax = 0.0f;
    for (int b0 = warp * kBPW; b0 < nblk; b0 += kHadWarps * kBPW) {
        const int b = b0 + slot;
        const bool ok = b < nblk;  // lanes past the last block run on zeros
        const uint16_t *src = row + size_t(ok ? b : 0) * n + sl * kEL;
        double v[kEL];
#pragma unroll
        for (int i = 0; i < kEL; i += 8) {
            const uint4 u = ok ? __ldg(reinterpret_cast<const uint4 *>(src + i)) : make_uint4(0, 0, 0, 0);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                v[i + 2 * j] = double(__uint_as_float(w[j] << 16));
                v[i + 2 * j + 1] = double(__uint_as_float(w[j] & 0xFFFF0000u));
            }
        }
        // in-lane stages: stride h < 32
#pragma unroll
        for (int h = 1; h < kEL; h <<= 1) {
#pragma unroll
            for (int i = 0; i < kEL; ++i) {
                if ((i & h) == 0) {
                    const double a = v[i], d = v[i + h];
                    v[i] = __dadd_rn(a, d);
                    v[i + h] = __dsub_rn(a, d);
                }
            }
        }
        // cross-lane stages: stride 32 t pairs lane sl with lane sl ^ t of
        // the same block; the lower lane keeps a + b, the upper a - b, as
        // (+-own) + other (a negation is exact, the add commutes)
#pragma unroll
        for (int t = 1; t < E; t <<= 1) {
            const uint32_t flip = (sl & t) ? 0x80000000u : 0u;
#pragma unroll
            for (int i = 0; i < kEL; ++i) {
                const double o = __shfl_xor_sync(0xffffffffu, v[i], t);
                const double own = __hiloint2double(int(uint32_t(__double2hiint(v[i])) ^ flip),
                                                    __double2loint(v[i]));
                v[i] = __dadd_rn(own, o);
            }
        }
        if (ok) {
            float4 *dst = reinterpret_cast<float4 *>(hs + had_smem_floats(b * n + sl * kEL));
#pragma unroll
            for (int i = 0; i < kEL; i += 4) {
                float4 f;
                f.x = __double2float_rn(__dmul_rn(v[i], c));
                f.y = __double2float_rn(__dmul_rn(v[i + 1], c));
                f.z = __double2float_rn(__dmul_rn(v[i + 2], c));
                f.w = __double2float_rn(__dmul_rn(v[i + 3], c));
                dst[i / 4] = f;
                amax = fmaxf(amax, fmaxf(fmaxf(fabsf(f.x), fabsf(f.y)), fmaxf(fabsf(f.z), fabsf(f.w))));
            }
        }
    }
    amax = block_reduce_had(amax, HMax(), red_f);  // also orders the hs stores

    const float s = amax > 0.0f ? __fdiv_rn(7.0f, amax) : 0.0f;
    int sum = 0;
    uint32_t *qw = reinterpret_cast<uint32_t *>(qrow);
    for (int k4 = threadIdx.x; k4 < K / 4; k4 += kHadThreads) {
        const float4 h = *reinterpret_cast<const float4 *>(hs + had_smem_floats(4 * k4));
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
    const size_t smem = had_smem_floats(K) * sizeof(float);
    static std::atomic<int> configured_dev{-1};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (configured_dev != dev) {
        // the rotated row of the longest K (32768 fp32 and its padding), next
        // to 64 bytes of static reduction slots
        e = cudaFuncSetAttribute(hadamard_quant4_kernel<E>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(had_smem_floats(kStreamMaxK) * sizeof(float)));
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
                                 int(had_smem_floats(kStreamMaxK) * sizeof(float)));
        if (e != cudaSuccess)
            return e;
        configured_dev = dev;
    }
    const double c = 1.0 / sqrt(double(32 * E));  // IEEE sqrt and divide: the oracle's constant
    hadamard_quant4_stack_kernel<E>
        <<<p.rows, kHadThreads, had_smem_floats(max_k) * sizeof(float), stream>>>(p, c);
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
