// quant.cu -- per-token absmax int8 quantisation of bf16 activations.
//
// BitNet b1.58 quantises activations to 8 bits per token by their largest
// magnitude (1bit.systems post "the full arc ...", paper list item 1). The
// per-element arithmetic (quant_core.cuh, shared with the stack GEMV's fused
// quantiser):
//   amax = max_k |x|, s = fl32(127/amax), q = clamp(rne(fl32(x*s)), -127, 127),
//   x_scale = fl32(amax/127), x_sum = sum q; amax == 0 gives zeros.
//
// A row is read twice as 16-byte vectors: pass 1 reduces |x| to amax, pass
// 2 (an L1/L2 hit) converts and writes 8 codes per vector and reduces the code
// sum. HBM traffic: 2K bytes in, K + 8 out. One CTA per row (block-wide
// reductions) while rows are few; once there are enough rows to give every
// SM eight, one warp per row (shuffle reductions only), its row copied whole
// into shared memory with every 16-byte copy in flight at once (one memory
// latency per row instead of one per batch of loads and pass), or, for rows
// too long for that, read twice from global memory.
#include <algorithm>
#include <atomic>

#include "mma_common.cuh"
#include "quant_core.cuh"
#include "tq_internal.h"

namespace tq {

namespace {

constexpr int kQuantThreads = 256;

// Reduce v over the block with op; `identity` is op's neutral element (it
// fills the lanes of the final warp that have no partial to contribute).
template <typename T, typename Op>
__device__ __forceinline__ T block_reduce(T v, Op op, T identity, T *red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0)
        red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < int(blockDim.x >> 5) ? red[lane] : identity;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0)
            red[0] = v;
    }
    __syncthreads();
    T r = red[0];
    __syncthreads();  // red may be reused by the caller's next reduction
    return r;
}

struct MaxOp {
    __device__ float operator()(float a, float b) const { return fmaxf(a, b); }
};
struct AddOp {
    __device__ int operator()(int a, int b) const { return a + b; }
};

__device__ void quant_row(const uint16_t *__restrict__ x, int8_t *__restrict__ xq,
                          float *__restrict__ x_scale, int32_t *__restrict__ x_sum, int K)
{
    __shared__ float red_f[32];
    __shared__ int red_i[32];
    const int nvec = K >> 3;  // 8 bf16 per 16-byte vector
    const uint4 *xv = reinterpret_cast<const uint4 *>(x);

    float amax = 0.0f;
    for (int v = threadIdx.x; v < nvec; v += blockDim.x)
        amax = fmaxf(amax, absmax8(__ldg(xv + v)));
    amax = block_reduce(amax, MaxOp(), 0.0f, red_f);

    const float s = quant_inv_scale(amax);
    int sum = 0;
    uint2 *qv = reinterpret_cast<uint2 *>(xq);
    for (int v = threadIdx.x; v < nvec; v += blockDim.x)
        qv[v] = quant8(__ldg(xv + v), s, &sum);
    sum = block_reduce(sum, AddOp(), 0, red_i);
    if (threadIdx.x == 0) {
        *x_scale = quant_scale(amax);
        if (x_sum)
            *x_sum = sum;
    }
}

__global__ void __launch_bounds__(kQuantThreads)
quant_rows_kernel(const uint16_t *__restrict__ x, int8_t *__restrict__ xq,
                  float *__restrict__ x_scale, int32_t *__restrict__ x_sum, int K)
{
    const size_t m = blockIdx.x;
    quant_row(x + m * K, xq + m * K, x_scale + m, x_sum ? x_sum + m : nullptr, K);
}

// The entry holding launch row r (entries' rows are consecutive).
__device__ __forceinline__ int entry_of_row(const QuantStackParams &p, int r)
{
    int lo = 0, hi = p.n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.e[mid].row0 <= r)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

__global__ void __launch_bounds__(kQuantThreads)
quant_stack_kernel(const __grid_constant__ QuantStackParams p)
{
    // Let a dependent grid (the stack GEMV) launch now: it streams weights,
    // which do not depend on this grid, and waits for it before reading xq.
    pdl_launch_dependents();
    const int r = blockIdx.x;
    const QuantStackEntry &e = p.e[entry_of_row(p, r)];
    const size_t m = size_t(r - e.row0);
    quant_row(e.x + m * e.K, e.xq + m * e.K, e.x_scale + m, e.x_sum ? e.x_sum + m : nullptr, e.K);
}

// One warp per row, rows strided over all warps of the grid.
__global__ void __launch_bounds__(kQuantThreads)
quant_stack_warp_kernel(const __grid_constant__ QuantStackParams p)
{
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int nwarps = int(gridDim.x) * (kQuantThreads / 32);
    for (int r = int(blockIdx.x) * (kQuantThreads / 32) + int(threadIdx.x >> 5); r < p.rows;
         r += nwarps) {
        const QuantStackEntry &e = p.e[entry_of_row(p, r)];
        const size_t m = size_t(r - e.row0);
        const uint4 *xv = reinterpret_cast<const uint4 *>(e.x + m * e.K);
        const int nvec = e.K >> 3;
        // eight 16-byte loads per lane in flight before any is used (a warp
        // has few rows' worth of neighbours on its SM to hide latency with)
        constexpr int kB = 8;
        float amax = 0.0f;
        for (int v0 = lane; v0 < nvec; v0 += 32 * kB) {
            uint4 u[kB];
#pragma unroll
            for (int b = 0; b < kB; ++b)
                u[b] = v0 + 32 * b < nvec ? __ldg(xv + v0 + 32 * b) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int b = 0; b < kB; ++b)
                amax = fmaxf(amax, absmax8(u[b]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float s = quant_inv_scale(amax);
        int sum = 0;
        uint2 *qv = reinterpret_cast<uint2 *>(e.xq + m * e.K);
        for (int v0 = lane; v0 < nvec; v0 += 32 * kB) {
            uint4 u[kB];
#pragma unroll
            for (int b = 0; b < kB; ++b)
                u[b] = v0 + 32 * b < nvec ? __ldg(xv + v0 + 32 * b) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int b = 0; b < kB; ++b)
                if (v0 + 32 * b < nvec)
                    qv[v0 + 32 * b] = quant8(u[b], s, &sum);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0) {
            e.x_scale[m] = quant_scale(amax);
            if (e.x_sum)
                e.x_sum[m] = sum;
        }
    }
}

// One warp per row, the row staged in shared memory: [warps][row_bytes].
constexpr int kQsWarps = 4;
constexpr int kQsMaxRowBytes = 48 * 1024;  // K <= 24576 on this path

__global__ void __launch_bounds__(kQsWarps * 32)
quant_stack_smem_kernel(const __grid_constant__ QuantStackParams p, int row_bytes)
{
    extern __shared__ __align__(16) uint8_t qs_buf[];
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint4 *sv = reinterpret_cast<const uint4 *>(qs_buf + size_t(warp) * row_bytes);
    const uint32_t sv_s = smem_u32(sv);
    const int nwarps = int(gridDim.x) * kQsWarps;
    for (int r = int(blockIdx.x) * kQsWarps + warp; r < p.rows; r += nwarps) {
        const QuantStackEntry &e = p.e[entry_of_row(p, r)];
        const size_t m = size_t(r - e.row0);
        const uint4 *xv = reinterpret_cast<const uint4 *>(e.x + m * e.K);
        const int nvec = e.K >> 3;
        __syncwarp();  // every lane is done reading the previous row
        for (int v = lane; v < nvec; v += 32)
            cp_async16(sv_s + uint32_t(v) * 16u, xv + v, true);
        cp_async_commit();
        cp_async_wait<0>();
        __syncwarp();
        float amax = 0.0f;
        for (int v = lane; v < nvec; v += 32)
            amax = fmaxf(amax, absmax8(sv[v]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float s = quant_inv_scale(amax);
        int sum = 0;
        uint2 *qv = reinterpret_cast<uint2 *>(e.xq + m * e.K);
        for (int v = lane; v < nvec; v += 32)
            qv[v] = quant8(sv[v], s, &sum);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0) {
            e.x_scale[m] = quant_scale(amax);
            if (e.x_sum)
                e.x_sum[m] = sum;
        }
    }
}

}  // namespace

cudaError_t launch_quant_rows(const uint16_t *x, int8_t *xq, float *x_scale, int32_t *x_sum,
                              int M, int K, cudaStream_t stream)
{
    quant_rows_kernel<<<M, kQuantThreads, 0, stream>>>(x, xq, x_scale, x_sum, K);
    return cudaGetLastError();
}

cudaError_t launch_quant_stack(const QuantStackParams &p, cudaStream_t stream)
{
    if (p.rows <= 0)
        return cudaSuccess;
    constexpr int kWarps = kQuantThreads / 32;
    const int sms = device_sm_count();
    if (p.rows < sms * kWarps) {
        quant_stack_kernel<<<p.rows, kQuantThreads, 0, stream>>>(p);
        return cudaGetLastError();
    }
    int max_k = 0;
    for (int j = 0; j < p.n; ++j)
        max_k = std::max(max_k, p.e[j].K);
    const int row_bytes = 2 * max_k;
    if (row_bytes == 0 || row_bytes > kQsMaxRowBytes) {
        const int grid = std::min((p.rows + kWarps - 1) / kWarps, sms * 8);  // 8 CTAs of 8 warps per SM
        quant_stack_warp_kernel<<<grid, kQuantThreads, 0, stream>>>(p);
        return cudaGetLastError();
    }
    static std::atomic<int> configured_dev{-1};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess)
        return err;
    if (configured_dev != dev) {
        err = cudaFuncSetAttribute(quant_stack_smem_kernel,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   kQsWarps * kQsMaxRowBytes);
        if (err != cudaSuccess)
            return err;
        configured_dev = dev;
    }
    const size_t smem = size_t(kQsWarps) * row_bytes;
    // CTAs per SM that the row buffers allow (227 KB per SM, 1 KB of it
    // reserved per CTA; up to 8 CTAs of 4 warps)
    const int per_sm = std::max(1, std::min(8, int((227 * 1024) / (smem + 1024))));
    const int grid = std::min((p.rows + kQsWarps - 1) / kQsWarps, sms * per_sm);
    quant_stack_smem_kernel<<<grid, kQsWarps * 32, smem, stream>>>(p, row_bytes);
    return cudaGetLastError();
}

}  // namespace tq
