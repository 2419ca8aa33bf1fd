// quant.cu -- per-token absmax int8 quantisation of bf16 activations.
//
// BitNet b1.58 quantises activations to 8 bits per token by their largest
// magnitude (1bit.systems post "the full arc ...", paper list item 1). The
// pages give no formula; the one used (shared with the header tq.h):
//   amax = max_k |x|, s = fl32(127/amax), q = clamp(rne(fl32(x*s)), -127, 127),
//   x_scale = fl32(amax/127), x_sum = sum q; amax == 0 gives zeros.
// Each rounding is an explicit _rn intrinsic, so the result does not depend
// on compiler contraction or fast-math settings.
//
// One CTA per token row. Pass 1 reads the row as 16-byte vectors and reduces
// |x| to amax; pass 2 re-reads it (an L1/L2 hit), converts and writes 8 codes
// per vector, and reduces the code sum. HBM traffic: 2K bytes in, K + 8 out.
#include "tq_internal.h"

namespace tq {

namespace {

constexpr int kQuantThreads = 256;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float absmax8(uint4 u)
{
    float a = fmaxf(fabsf(bf16_lo(u.x)), fabsf(bf16_hi(u.x)));
    a = fmaxf(a, fmaxf(fabsf(bf16_lo(u.y)), fabsf(bf16_hi(u.y))));
    a = fmaxf(a, fmaxf(fabsf(bf16_lo(u.z)), fabsf(bf16_hi(u.z))));
    a = fmaxf(a, fmaxf(fabsf(bf16_lo(u.w)), fabsf(bf16_hi(u.w))));
    return a;
}

__device__ __forceinline__ int code_of(float v, float s)
{
    int r = __float2int_rn(__fmul_rn(v, s));  // one fp32 rounding, then ties-to-even
    return min(max(r, -127), 127);
}

// Quantise two bf16 values held in one 32-bit word; returns two int8 codes in
// the low 16 bits and adds them to *sum.
__device__ __forceinline__ uint32_t quant2(uint32_t w, float s, int *sum)
{
    int a = code_of(bf16_lo(w), s);
    int b = code_of(bf16_hi(w), s);
    *sum += a + b;
    return (uint32_t(a) & 0xFFu) | ((uint32_t(b) & 0xFFu) << 8);
}

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

    const float s = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
    int sum = 0;
    uint2 *qv = reinterpret_cast<uint2 *>(xq);
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
        const uint4 u = __ldg(xv + v);
        uint2 o;
        o.x = quant2(u.x, s, &sum) | (quant2(u.y, s, &sum) << 16);
        o.y = quant2(u.z, s, &sum) | (quant2(u.w, s, &sum) << 16);
        qv[v] = o;
    }
    sum = block_reduce(sum, AddOp(), 0, red_i);
    if (threadIdx.x == 0) {
        *x_scale = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
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

__global__ void __launch_bounds__(kQuantThreads)
quant_stack_kernel(const __grid_constant__ QuantStackParams p)
{
    // Let a dependent grid (the stack GEMV) launch now: it streams weights,
    // which do not depend on this grid, and waits for it before reading xq.
    pdl_launch_dependents();
    const QuantStackEntry &e = p.e[blockIdx.x];
    quant_row(e.x, e.xq, e.x_scale, e.x_sum, e.K);
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
    quant_stack_kernel<<<p.n, kQuantThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace tq
