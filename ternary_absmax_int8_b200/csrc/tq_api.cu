// tq_api.cu -- the C ABI of libtq (declared in include/tq.h): argument
// checks, then kernel launches. Nothing here allocates device memory.
#include <atomic>
#include <cfloat>
#include <cstdarg>
#include <cstdio>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <vector>

#include "tq.h"
#include "tq_internal.h"

namespace tq {

__device__ unsigned int g_device_error = 0;

bool pack_ternary_host(const int8_t *w, uint8_t *packed, int N, int K);
bool pack_binary_host(const int8_t *w, const uint16_t *scales, uint8_t *bits,
                      uint16_t *scales_packed, int N, int K);
unsigned *device_error_word()
{
    static std::atomic<unsigned *> cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return nullptr;
    if (!cache[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess)
            return nullptr;
        cache[dev] = static_cast<unsigned *>(p);
    }
    return cache[dev];
}

int device_sm_count()
{
    static std::atomic<int> cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return 1;
    if (dev < 0 || dev >= 64)
        dev = 0;
    if (cache[dev] == 0) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cache[dev] = n > 0 ? n : 1;
    }
    return cache[dev];
}

}  // namespace tq

namespace {

thread_local char g_msg[512] = "";

tq_status fail(tq_status s, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof g_msg, fmt, ap);
    va_end(ap);
    return s;
}

tq_status ok()
{
    g_msg[0] = '\0';
    return TQ_OK;
}

tq_status cuda_fail(cudaError_t e, const char *where)
{
    if (e == cudaErrorInvalidValue)
        return fail(TQ_ERR_UNSUPPORTED, "%s: launch plan rejected (shape beyond this build's limits)",
                    where);
    return fail(TQ_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned(const void *p, size_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; }

constexpr int kGemvMaxM = 24;
constexpr int kStackMaxM = 32;  // tq_gemv_stack_batch

// Shared checks of the GEMV-shaped calls.
tq_status check_gemv_args(const char *fn, const uint8_t *packed, const int8_t *xq,
                          const float *x_scale, const int32_t *x_sum, const float *y,
                          const int32_t *acc_out, int M, int N, int K)
{
    if (M < 0 || N < 0 || K < 0)
        return fail(TQ_ERR_SHAPE, "%s: negative size (M=%d N=%d K=%d)", fn, M, N, K);
    if (N % 4 != 0)
        return fail(TQ_ERR_SHAPE, "%s: N=%d is not a multiple of 4", fn, N);
    if (K % 16 != 0)
        return fail(TQ_ERR_SHAPE, "%s: K=%d is not a multiple of 16", fn, K);
    if (M == 0 || N == 0)
        return TQ_OK;
    if (!packed || !xq || !x_scale || !x_sum || !y)
        return fail(TQ_ERR_NULL, "%s: a required pointer is NULL", fn);
    if (!aligned(packed, 16) || !aligned(xq, 16))
        return fail(TQ_ERR_ALIGN, "%s: packed and xq must be 16-byte aligned", fn);
    if (!aligned(x_scale, 4) || !aligned(x_sum, 4) || !aligned(y, 4) ||
        (acc_out && !aligned(acc_out, 4)))
        return fail(TQ_ERR_ALIGN, "%s: x_scale, x_sum, y, acc_out must be 4-byte aligned", fn);
    if (K > tq::kStreamMaxK)
        return fail(TQ_ERR_UNSUPPORTED, "%s: K=%d exceeds %d", fn, K, tq::kStreamMaxK);
    return TQ_OK;
}

// Host staging of the stack quantiser's launch parameters (too large for
// the stack), one per calling thread.
tq::QuantStackParams *quant_params()
{
    static thread_local tq::QuantStackParams params;
    return &params;
}

// K == 0: every accumulator is 0 and so is every output.
tq_status zero_outputs(float *y, int32_t *acc_out, size_t count, cudaStream_t s)
{
    cudaError_t e = cudaMemsetAsync(y, 0, count * sizeof(float), s);
    if (e == cudaSuccess && acc_out)
        e = cudaMemsetAsync(acc_out, 0, count * sizeof(int32_t), s);
    return e == cudaSuccess ? ok() : cuda_fail(e, "zero outputs");
}

// Which kernel runs a group of M-token projections: the streaming dp4a kernel
// (M <= 4 per launch), the warp-MMA kernel (2 <= M <= 32) or the tensor-core
// group plan (5 <= M <= 32). The choice by M follows B200 measurements of the
// 30-layer stack and the FFN projections (streaming up to 2 tokens, warp MMA
// for 3..24, the group plan for 25..32); TQ_BATCH_KERNEL=stream|mma|tc forces
// one where it applies (for measurement).
enum class BatchKernel { kStream, kWarpMma, kTensor };

BatchKernel batch_kernel(int M)
{
    static const int forced = [] {
        const char *v = getenv("TQ_BATCH_KERNEL");
        if (!v)
            return -1;
        if (!strcmp(v, "stream"))
            return 0;
        if (!strcmp(v, "mma"))
            return 1;
        if (!strcmp(v, "tc"))
            return 2;
        return -1;
    }();
    if (M <= 1)
        return BatchKernel::kStream;
    if (forced == 0 && M <= tq::kStreamMaxTokens)
        return BatchKernel::kStream;
    if (forced == 1)
        return BatchKernel::kWarpMma;
    if (forced == 2 && M >= 5)
        return BatchKernel::kTensor;
    if (M <= 2)
        return BatchKernel::kStream;
    return M <= 24 ? BatchKernel::kWarpMma : BatchKernel::kTensor;
}

// Tokens in groups of up to four, one streaming launch per group.
tq_status stream_groups(const uint8_t *packed, float w_scale, const int8_t *xq,
                        const float *x_scale, const int32_t *x_sum, float *y, int32_t *acc_out,
                        int M, int N, int K, cudaStream_t stream, const char *fn)
{
    for (int m0 = 0; m0 < M; m0 += tq::kStreamMaxTokens) {
        const int mg = M - m0 < tq::kStreamMaxTokens ? M - m0 : tq::kStreamMaxTokens;
        tq::StreamEntry e = {};
        e.packed = packed;
        // Inputs only: a launch that does not quantise never writes them.
        e.xq = const_cast<int8_t *>(xq) + size_t(m0) * K;
        e.x_scale = const_cast<float *>(x_scale) + m0;
        e.x_sum = const_cast<int32_t *>(x_sum) + m0;
        e.y = y + size_t(m0) * N;
        e.acc_out = acc_out ? acc_out + size_t(m0) * N : nullptr;
        e.w_scale = w_scale;
        e.N4 = N / 4;
        e.K = K;
        cudaError_t err = tq::launch_stream_gemv(&e, 1, mg, false, true, 0, stream);
        if (err != cudaSuccess)
            return cuda_fail(err, fn);
    }
    return ok();
}

// One projection at 1 <= M <= 32 tokens, by the kernel batch_kernel(M)
// picks: streaming (tokens in groups of four), warp MMA, or the tensor-core
// batched-decode kernel (thread-block clusters split K when tiles are few).
tq_status small_batch(const uint8_t *packed, float w_scale, const int8_t *xq, const float *x_scale,
                      const int32_t *x_sum, float *y, int32_t *acc_out, int M, int N, int K,
                      cudaStream_t stream, const char *fn)
{
    cudaError_t err;
    switch (batch_kernel(M)) {
    case BatchKernel::kStream:
        return stream_groups(packed, w_scale, xq, x_scale, x_sum, y, acc_out, M, N, K, stream, fn);
    case BatchKernel::kWarpMma: {
        const tq::MmaEntry e{packed, xq, x_scale, x_sum, y, acc_out, w_scale, N / 4, K, 0};
        err = tq::launch_mma_gemv(&e, 1, M, false, stream);
        break;
    }
    default:
        err = tq::launch_smallm_tc(packed, w_scale, xq, x_scale, x_sum, y, acc_out, M, N, K,
                                   stream);
    }
    return err == cudaSuccess ? ok() : cuda_fail(err, fn);
}

// One thread waits, with the library's bounded wait, on an mbarrier that
// nothing ever arrives on: the wait gives up after limit_ns, records
// kErrWaitTimeout in the error word and the kernel returns normally.
__global__ void wait_selftest_kernel(unsigned *err, unsigned long long limit_ns)
{
    __shared__ uint64_t bar;
    if (threadIdx.x != 0)
        return;
    tq::mbar_init(&bar, 1);
    tq::fence_mbar_init();
    tq::mbar_wait(&bar, 0u, err, limit_ns);
}

// The quantiser over M token rows of each projection: one entry of the stack
// quantiser per projection, one launch per kMaxQuantStack projections.
tq_status quantize_stack_impl(const char *fname, const tq_proj *projs, int n_proj, int M,
                              cudaStream_t stream)
{
    if (n_proj < 0 || M < 0)
        return fail(TQ_ERR_SHAPE, "%s: n_proj=%d M=%d", fname, n_proj, M);
    if (n_proj == 0 || M == 0)
        return ok();
    if (!projs)
        return fail(TQ_ERR_NULL, "%s: projs is NULL", fname);
    std::vector<tq::QuantStackEntry> list;
    list.reserve(size_t(n_proj));
    for (int j = 0; j < n_proj; ++j) {
        const tq_proj &p = projs[j];
        if (p.K < 0 || p.K % 16 != 0)
            return fail(TQ_ERR_SHAPE, "%s: entry %d: K=%d", fname, j, p.K);
        if (!p.x_scale || (p.K > 0 && (!p.x || !p.xq)))
            return fail(TQ_ERR_NULL, "%s: entry %d: NULL pointer", fname, j);
        if ((p.K > 0 && (!aligned(p.x, 16) || !aligned(p.xq, 16))) || !aligned(p.x_scale, 4) ||
            (p.x_sum && !aligned(p.x_sum, 4)))
            return fail(TQ_ERR_ALIGN, "%s: entry %d: misaligned pointer", fname, j);
    }
    for (int j = 0; j < n_proj; ++j) {
        const tq_proj &p = projs[j];
        if (p.K == 0) {
            cudaError_t e = cudaMemsetAsync(p.x_scale, 0, size_t(M) * sizeof(float), stream);
            if (e == cudaSuccess && p.x_sum)
                e = cudaMemsetAsync(p.x_sum, 0, size_t(M) * sizeof(int32_t), stream);
            if (e != cudaSuccess)
                return cuda_fail(e, fname);
            continue;
        }
        list.push_back(tq::QuantStackEntry{p.x, p.xq, p.x_scale, p.x_sum, p.K, M, 0, 0});
    }
    tq::QuantStackParams &params = *quant_params();
    for (size_t base = 0; base < list.size(); base += tq::kMaxQuantStack) {
        const size_t n = std::min(list.size() - base, size_t(tq::kMaxQuantStack));
        params.n = int(n);
        long long rows = 0;
        for (size_t i = 0; i < n; ++i) {
            params.e[i] = list[base + i];
            params.e[i].row0 = int(rows);
            rows += M;
        }
        if (rows > INT32_MAX)
            return fail(TQ_ERR_UNSUPPORTED, "%s: %lld rows in one call", fname, rows);
        params.rows = int(rows);
        cudaError_t e = tq::launch_quant_stack(params, stream);
        if (e != cudaSuccess)
            return cuda_fail(e, fname);
    }
    return ok();
}

tq_status gemv_stack_impl(const char *fname, const tq_proj *projs, int n_proj, int M,
                          unsigned flags, cudaStream_t stream)
{
    if (n_proj < 0 || M < 0)
        return fail(TQ_ERR_SHAPE, "%s: n_proj=%d M=%d", fname, n_proj, M);
    const unsigned qflags = flags & (TQ_STACK_QUANTIZE | TQ_STACK_RMSNORM | TQ_STACK_RELU2_MUL);
    if ((flags & ~(unsigned(TQ_STACK_OVERLAP_PREV) | qflags)) || (qflags & (qflags - 1)))
        return fail(TQ_ERR_VALUE, "%s: bad flags 0x%x", fname, flags);
    if (M > kStackMaxM)
        return fail(TQ_ERR_UNSUPPORTED, "%s: M=%d > %d", fname, M, kStackMaxM);
    if (qflags && M > 1)
        return fail(TQ_ERR_UNSUPPORTED, "%s: quantising flags need M == 1 (M=%d)", fname, M);
    if (n_proj == 0 || M == 0)
        return ok();
    if (!projs)
        return fail(TQ_ERR_NULL, "%s: projs is NULL", fname);
    // the launch's quantising mode: 1 absmax of bf16 x, 2 RMSNorm then absmax,
    // 3 relu(x_f32)^2 * up, RMSNorm, absmax
    const int mode = qflags == TQ_STACK_QUANTIZE ? 1
                     : qflags == TQ_STACK_RMSNORM ? 2
                     : qflags == TQ_STACK_RELU2_MUL ? 3 : 0;
    std::vector<tq::StreamEntry> list;
    list.reserve(size_t(n_proj));
    for (int j = 0; j < n_proj; ++j) {
        const tq_proj &p = projs[j];
        char fn[64];
        snprintf(fn, sizeof fn, "%s[%d]", fname, j);
        tq_status st =
            check_gemv_args(fn, p.packed, p.xq, p.x_scale, p.x_sum, p.y, p.acc_out, M, p.N, p.K);
        if (st != TQ_OK)
            return st;
        const void *xin = mode == 3 ? static_cast<const void *>(p.x_f32)
                                    : static_cast<const void *>(p.x);
        if (mode && p.K > 0) {
            if (!xin || (mode == 3 && !p.up) || (mode >= 2 && !p.gain))
                return fail(TQ_ERR_NULL, "%s: x is NULL (or x_f32, up or gain for its mode)", fn);
            if (!aligned(xin, 16) || (mode == 3 && !aligned(p.up, 16)) ||
                (mode >= 2 && !aligned(p.gain, 4)))
                return fail(TQ_ERR_ALIGN, "%s: x must be 16-byte aligned (x_f32, up too)", fn);
            if (mode >= 2 && (!(p.eps >= 0.0f) || p.eps > FLT_MAX))
                return fail(TQ_ERR_VALUE, "%s: eps must be finite and >= 0", fn);
        }
        if (p.N == 0 && !mode)
            continue;
        if (p.K == 0) {
            // Every accumulator is 0; a quantising call also reports the
            // empty token's scale and sum as 0.
            cudaError_t e = cudaSuccess;
            if (mode)
                e = cudaMemsetAsync(p.x_scale, 0, sizeof(float), stream);
            if (e == cudaSuccess && mode)
                e = cudaMemsetAsync(p.x_sum, 0, sizeof(int32_t), stream);
            if (e != cudaSuccess)
                return cuda_fail(e, fn);
            st = zero_outputs(p.y, p.acc_out, size_t(M) * size_t(p.N), stream);
            if (st != TQ_OK)
                return st;
            continue;
        }
        if (p.N == 0) {
            // Nothing to multiply, but the quantiser's outputs are owed.
            cudaError_t e;
            if (mode == 1) {
                tq::QuantStackParams *qp = quant_params();
                qp->n = 1;
                qp->rows = 1;
                qp->e[0] = tq::QuantStackEntry{p.x, p.xq, p.x_scale, p.x_sum, p.K, 1, 0, 0};
                e = tq::launch_quant_stack(*qp, stream);
            } else {
                e = tq::launch_rms_quant(mode == 2 ? 0 : 2, p.x, p.x_f32, p.up, p.gain, p.eps,
                                         p.xq, p.x_scale, p.x_sum, 1, p.K, stream);
            }
            if (e != cudaSuccess)
                return cuda_fail(e, fn);
            continue;
        }
        tq::StreamEntry e = {};
        e.packed = p.packed;
        e.xin = xin;
        e.gain = p.gain;
        e.up = p.up;
        e.eps = p.eps;
        e.xq = p.xq;
        e.x_scale = p.x_scale;
        e.x_sum = p.x_sum;
        e.y = p.y;
        e.acc_out = p.acc_out;
        e.w_scale = p.w_scale;
        e.N4 = p.N / 4;
        e.K = p.K;
        list.push_back(e);
    }
    const BatchKernel bk = batch_kernel(M);
    if (bk == BatchKernel::kTensor) {
        // the tensor-core batched-decode kernel's group plan, up to 64
        // projections per launch (TQ_STACK_OVERLAP_PREV: its first launch
        // may start while the previous kernel drains)
        std::vector<tq::GroupEntry> group;
        group.reserve(list.size());
        for (const tq::StreamEntry &e : list)
            group.push_back(tq::GroupEntry{e.packed, e.w_scale, e.xq, e.x_scale, e.x_sum, e.y,
                                           e.acc_out, 4 * e.N4, e.K});
        cudaError_t e = tq::launch_smallm_group(group.data(), int(group.size()), M,
                                                (flags & TQ_STACK_OVERLAP_PREV) != 0, stream);
        return e == cudaSuccess ? ok() : cuda_fail(e, fname);
    }
    if (bk == BatchKernel::kWarpMma) {
        // the warp-MMA small-batch kernel, one launch per 256 projections
        // (TQ_STACK_OVERLAP_PREV: the first launch may start while the
        // previous kernel drains)
        std::vector<tq::MmaEntry> mma;
        mma.reserve(list.size());
        for (const tq::StreamEntry &e : list)
            mma.push_back(tq::MmaEntry{e.packed, e.xq, e.x_scale, e.x_sum, e.y, e.acc_out,
                                       e.w_scale, e.N4, e.K, 0});
        cudaError_t e = tq::launch_mma_gemv(mma.data(), int(mma.size()), M,
                                            (flags & TQ_STACK_OVERLAP_PREV) != 0, stream);
        return e == cudaSuccess ? ok() : cuda_fail(e, fname);
    }
    const bool overlap = (flags & TQ_STACK_OVERLAP_PREV) != 0;
    for (size_t base = 0; base < list.size(); base += tq::kStreamStackMax) {
        const int n = int(std::min(list.size() - base, size_t(tq::kStreamStackMax)));
        cudaError_t e = tq::launch_stream_gemv(list.data() + base, n, M, overlap && base == 0,
                                               false, mode, stream);
        if (e != cudaSuccess)
            return cuda_fail(e, fname);
    }
    return ok();
}

}  // namespace

extern "C" {

const char *tq_status_string(tq_status s)
{
    switch (s) {
    case TQ_OK: return "TQ_OK";
    case TQ_ERR_NULL: return "TQ_ERR_NULL";
    case TQ_ERR_SHAPE: return "TQ_ERR_SHAPE";
    case TQ_ERR_ALIGN: return "TQ_ERR_ALIGN";
    case TQ_ERR_VALUE: return "TQ_ERR_VALUE";
    case TQ_ERR_CUDA: return "TQ_ERR_CUDA";
    case TQ_ERR_UNSUPPORTED: return "TQ_ERR_UNSUPPORTED";
    }
    return "TQ_ERR_UNKNOWN";
}

const char *tq_last_error(void) { return g_msg; }

tq_status tq_pack_host(const int8_t *w, uint8_t *packed, int M, int N, int K, cudaStream_t stream)
{
    (void)M;
    (void)stream;
    if (N < 0 || K < 0)
        return fail(TQ_ERR_SHAPE, "tq_pack_host: negative size (N=%d K=%d)", N, K);
    if (N % 4 != 0)
        return fail(TQ_ERR_SHAPE, "tq_pack_host: N=%d is not a multiple of 4", N);
    if (N == 0 || K == 0)
        return ok();
    if (!w || !packed)
        return fail(TQ_ERR_NULL, "tq_pack_host: a required pointer is NULL");
    if (!tq::pack_ternary_host(w, packed, N, K))
        return fail(TQ_ERR_VALUE, "tq_pack_host: a weight is outside {-1, 0, 1}");
    return ok();
}

tq_status tq_quantize_act(const uint16_t *x, int8_t *xq, float *x_scale, int32_t *x_sum, int M,
                          int N, int K, cudaStream_t stream)
{
    (void)N;
    if (M < 0 || K < 0)
        return fail(TQ_ERR_SHAPE, "tq_quantize_act: negative size (M=%d K=%d)", M, K);
    if (K % 16 != 0)
        return fail(TQ_ERR_SHAPE, "tq_quantize_act: K=%d is not a multiple of 16", K);
    if (M == 0)
        return ok();
    if (!x_scale || (K > 0 && (!x || !xq)))
        return fail(TQ_ERR_NULL, "tq_quantize_act: a required pointer is NULL");
    if ((K > 0 && (!aligned(x, 16) || !aligned(xq, 16))) || !aligned(x_scale, 4) ||
        (x_sum && !aligned(x_sum, 4)))
        return fail(TQ_ERR_ALIGN, "tq_quantize_act: x, xq need 16-byte, x_scale, x_sum 4-byte alignment");
    if (K == 0) {
        cudaError_t e = cudaMemsetAsync(x_scale, 0, size_t(M) * sizeof(float), stream);
        if (e == cudaSuccess && x_sum)
            e = cudaMemsetAsync(x_sum, 0, size_t(M) * sizeof(int32_t), stream);
        return e == cudaSuccess ? ok() : cuda_fail(e, "tq_quantize_act");
    }
    cudaError_t e = tq::launch_quant_rows(x, xq, x_scale, x_sum, M, K, stream);
    return e == cudaSuccess ? ok() : cuda_fail(e, "tq_quantize_act");
}

tq_status tq_gemv(const uint8_t *packed, float w_scale, const int8_t *xq, const float *x_scale,
                  const int32_t *x_sum, float *y, int32_t *acc_out, int M, int N, int K,
                  cudaStream_t stream)
{
    tq_status st = check_gemv_args("tq_gemv", packed, xq, x_scale, x_sum, y, acc_out, M, N, K);
    if (st != TQ_OK)
        return st;
    if (M > kGemvMaxM)
        return fail(TQ_ERR_UNSUPPORTED, "tq_gemv: M=%d > %d (use tq_gemm_prefill)", M, kGemvMaxM);
    if (M == 0 || N == 0)
        return ok();
    if (K == 0)
        return zero_outputs(y, acc_out, size_t(M) * N, stream);
    return small_batch(packed, w_scale, xq, x_scale, x_sum, y, acc_out, M, N, K, stream,
                       "tq_gemv");
}

tq_status tq_gemm_prefill(const uint8_t *packed, float w_scale, const int8_t *xq,
                          const float *x_scale, const int32_t *x_sum, float *y, int32_t *acc_out,
                          int M, int N, int K, cudaStream_t stream)
{
    tq_status st =
        check_gemv_args("tq_gemm_prefill", packed, xq, x_scale, x_sum, y, acc_out, M, N, K);
    if (st != TQ_OK)
        return st;
    if (M == 0 || N == 0)
        return ok();
    if (K == 0)
        return zero_outputs(y, acc_out, size_t(M) * N, stream);
    if (M <= 32)
        return small_batch(packed, w_scale, xq, x_scale, x_sum, y, acc_out, M, N, K, stream,
                           "tq_gemm_prefill");
    bool handled = false;
    cudaError_t e = tq::launch_prefill_tc(packed, w_scale, xq, x_scale, x_sum, y, acc_out, M, N, K,
                                          stream, &handled);
    if (e == cudaErrorInvalidValue && !handled)
        return fail(TQ_ERR_UNSUPPORTED, "tq_gemm_prefill: N=%d or M=%d exceeds the tile fields",
                    N, M);
    if (e != cudaSuccess)
        return cuda_fail(e, "tq_gemm_prefill");
    if (handled)
        return ok();
    return stream_groups(packed, w_scale, xq, x_scale, x_sum, y, acc_out, M, N, K, stream,
                         "tq_gemm_prefill");
}

tq_status tq_gemm_prefill_stack(const tq_proj *projs, int n_proj, int M, cudaStream_t stream)
{
    const char *fn = "tq_gemm_prefill_stack";
    if (n_proj < 0 || (n_proj > 0 && !projs))
        return fail(TQ_ERR_NULL, "%s: projs is NULL", fn);
    if (M < 0)
        return fail(TQ_ERR_SHAPE, "%s: negative M=%d", fn, M);
    for (int j = 0; j < n_proj; ++j) {
        const tq_proj &p = projs[j];
        const tq_status st =
            check_gemv_args(fn, p.packed, p.xq, p.x_scale, p.x_sum, p.y, p.acc_out, M, p.N, p.K);
        if (st != TQ_OK)
            return st;
    }
    if (M == 0 || n_proj == 0)
        return ok();
    if (M <= 32)  // small batches: the decode kernels
        return gemv_stack_impl(fn, projs, n_proj, M, 0, stream);
    std::vector<tq::PrefillEntry> list;
    list.reserve(size_t(n_proj));
    for (int j = 0; j < n_proj; ++j) {
        const tq_proj &p = projs[j];
        if (p.N == 0)
            continue;
        if (p.K == 0) {
            const tq_status st = zero_outputs(p.y, p.acc_out, size_t(M) * p.N, stream);
            if (st != TQ_OK)
                return st;
            continue;
        }
        list.push_back(tq::PrefillEntry{p.packed, p.w_scale, p.xq, p.x_scale, p.x_sum, p.y,
                                        p.acc_out, p.N, p.K});
    }
    for (size_t base = 0; base < list.size(); base += tq::kPrefillMaxGroup) {
        const int n = int(std::min(list.size() - base, size_t(tq::kPrefillMaxGroup)));
        bool handled = false;
        const cudaError_t e = tq::launch_prefill_group(list.data() + base, n, M, stream, &handled);
        if (e == cudaErrorInvalidValue && !handled)
            return fail(TQ_ERR_UNSUPPORTED, "%s: a shape exceeds the prefill tile fields", fn);
        if (e != cudaSuccess)
            return cuda_fail(e, fn);
    }
    return ok();
}

tq_status tq_quantize_act_stack(const tq_proj *projs, int n_proj, cudaStream_t stream)
{
    return quantize_stack_impl("tq_quantize_act_stack", projs, n_proj, 1, stream);
}

tq_status tq_quantize_act_stack_batch(const tq_proj *projs, int n_proj, int M,
                                      cudaStream_t stream)
{
    return quantize_stack_impl("tq_quantize_act_stack_batch", projs, n_proj, M, stream);
}

tq_status tq_gemv_stack(const tq_proj *projs, int n_proj, unsigned flags, cudaStream_t stream)
{
    return gemv_stack_impl("tq_gemv_stack", projs, n_proj, 1, flags, stream);
}

tq_status tq_gemv_stack_batch(const tq_proj *projs, int n_proj, int M, unsigned flags,
                              cudaStream_t stream)
{
    return gemv_stack_impl("tq_gemv_stack_batch", projs, n_proj, M, flags, stream);
}

tq_status tq_gemv_noalloc(const uint8_t *packed, float w_scale, const int8_t *xq,
                          const float *x_scale, const int32_t *x_sum, float *y, int32_t *acc_out,
                          int M, int N, int K, cudaStream_t stream)
{
    tq_status st =
        check_gemv_args("tq_gemv_noalloc", packed, xq, x_scale, x_sum, y, acc_out, M, N, K);
    if (st != TQ_OK)
        return st;
    if (M == 0 || N == 0)
        return ok();
    if (M < 5 || M > 32)
        return fail(TQ_ERR_UNSUPPORTED,
                    "tq_gemv_noalloc: M=%d outside 5..32 (tq_gemv needs no scratch for M <= 4)", M);
    if (K == 0)
        return fail(TQ_ERR_UNSUPPORTED, "tq_gemv_noalloc: K=0 (use tq_gemv)");
    const size_t need = tq::smallm_workspace_bytes(N, M);
    if (need > tq::noalloc_scratch_capacity())
        return fail(TQ_ERR_UNSUPPORTED,
                    "tq_gemv_noalloc: N=%d at M=%d needs %zu bytes of scratch, more than the fixed "
                    "%zu",
                    N, M, need, tq::noalloc_scratch_capacity());
    cudaError_t e = tq::launch_smallm_tc_noalloc(packed, w_scale, xq, x_scale, x_sum, y, acc_out, M,
                                                 N, K, stream);
    return e == cudaSuccess ? ok() : cuda_fail(e, "tq_gemv_noalloc");
}

static tq_status rms_quant_call(const char *fn, int input, const uint16_t *x_bf16,
                                const float *x_f32, const float *up, const float *gain, float eps,
                                int8_t *xq, float *x_scale, int32_t *x_sum, int M, int K,
                                cudaStream_t stream)
{
    if (M < 0 || K <= 0 || K % 16 != 0)
        return fail(TQ_ERR_SHAPE, "%s: M=%d K=%d (need M >= 0, K > 0, K %% 16 == 0)", fn, M, K);
    if (K > tq::kStreamMaxK)
        return fail(TQ_ERR_UNSUPPORTED, "%s: K=%d exceeds %d", fn, K, tq::kStreamMaxK);
    if (!(eps >= 0.0f) || eps > FLT_MAX)
        return fail(TQ_ERR_VALUE, "%s: eps must be finite and >= 0", fn);
    if (M == 0)
        return ok();
    const void *x = input == 0 ? static_cast<const void *>(x_bf16) : static_cast<const void *>(x_f32);
    if (!x || !gain || !xq || !x_scale || !x_sum || (input == 2 && !up))
        return fail(TQ_ERR_NULL, "%s: a required pointer is NULL", fn);
    if (!aligned(x, 16) || !aligned(xq, 16) || (up && !aligned(up, 16)) || !aligned(gain, 4) ||
        !aligned(x_scale, 4) || !aligned(x_sum, 4))
        return fail(TQ_ERR_ALIGN, "%s: rows and codes must be 16-byte aligned, vectors 4-byte",
                    fn);
    cudaError_t e = tq::launch_rms_quant(input, x_bf16, x_f32, up, gain, eps, xq, x_scale, x_sum,
                                         M, K, stream);
    return e == cudaSuccess ? ok() : cuda_fail(e, fn);
}

tq_status tq_rmsnorm_quantize(const uint16_t *x_bf16, const float *x_f32, const float *gain,
                              float eps, int8_t *xq, float *x_scale, int32_t *x_sum, int M, int K,
                              cudaStream_t stream)
{
    if ((x_bf16 != nullptr) == (x_f32 != nullptr) && M > 0)
        return fail(TQ_ERR_VALUE, "tq_rmsnorm_quantize: give exactly one of x_bf16 and x_f32");
    return rms_quant_call("tq_rmsnorm_quantize", x_bf16 ? 0 : 1, x_bf16, x_f32, nullptr, gain,
                          eps, xq, x_scale, x_sum, M, K, stream);
}

tq_status tq_relu2_mul_rmsnorm_quantize(const float *gate, const float *up, const float *gain,
                                        float eps, int8_t *xq, float *x_scale, int32_t *x_sum,
                                        int M, int K, cudaStream_t stream)
{
    return rms_quant_call("tq_relu2_mul_rmsnorm_quantize", 2, nullptr, gate, up, gain, eps, xq,
                          x_scale, x_sum, M, K, stream);
}

tq_status tq_absmean_pack(const uint16_t *w_bf16, uint8_t *packed, float *w_scale, int N, int K,
                          cudaStream_t stream)
{
    if (N < 0 || K < 0 || N % 4 != 0 || K % 16 != 0)
        return fail(TQ_ERR_SHAPE, "tq_absmean_pack: N=%d K=%d (need N %% 4 == 0, K %% 16 == 0)",
                    N, K);
    if (!w_scale || (N > 0 && K > 0 && (!w_bf16 || !packed)))
        return fail(TQ_ERR_NULL, "tq_absmean_pack: a required pointer is NULL");
    if ((w_bf16 && !aligned(w_bf16, 16)) || (packed && !aligned(packed, 16)) ||
        !aligned(w_scale, 4))
        return fail(TQ_ERR_ALIGN, "tq_absmean_pack: weights and packed bytes 16-byte aligned");
    cudaError_t e = tq::launch_absmean_pack(w_bf16, packed, w_scale, N, K, stream);
    return e == cudaSuccess ? ok() : cuda_fail(e, "tq_absmean_pack");
}

tq_status tq_hadamard_quantize_act(const uint16_t *x, int8_t *xq, float *x_scale, int32_t *x_sum,
                                   int M, int K, int n, cudaStream_t stream)
{
    const char *fn = "tq_hadamard_quantize_act";
    if (M < 0 || K < 0)
        return fail(TQ_ERR_SHAPE, "%s: negative size (M=%d K=%d)", fn, M, K);
    if (n < 32 || n > 1024 || (n & (n - 1)) != 0 || K % n != 0)
        return fail(TQ_ERR_SHAPE, "%s: block size n=%d must be a power of two in 32..1024 dividing K=%d",
                    fn, n, K);
    if (M == 0 || K == 0)
        return ok();
    if (K > tq::kStreamMaxK)
        return fail(TQ_ERR_UNSUPPORTED, "%s: K=%d exceeds %d", fn, K, tq::kStreamMaxK);
    if (!x || !xq || !x_scale)
        return fail(TQ_ERR_NULL, "%s: a required pointer is NULL", fn);
    if (!aligned(x, 16) || !aligned(xq, 16) || !aligned(x_scale, 4) || (x_sum && !aligned(x_sum, 4)))
        return fail(TQ_ERR_ALIGN, "%s: x and xq 16-byte aligned, vectors 4-byte aligned", fn);
    cudaError_t e = tq::launch_hadamard_quant4(x, xq, x_scale, x_sum, M, K, n, stream);
    return e == cudaSuccess ? ok() : cuda_fail(e, fn);
}

tq_status tq_hadamard_quantize_act_stack(const tq_proj *projs, int n_proj, int M, int n,
                                         cudaStream_t stream)
{
    const char *fn = "tq_hadamard_quantize_act_stack";
    if (n_proj < 0 || M < 0)
        return fail(TQ_ERR_SHAPE, "%s: n_proj=%d M=%d", fn, n_proj, M);
    if (n < 32 || n > 1024 || (n & (n - 1)) != 0)
        return fail(TQ_ERR_SHAPE, "%s: block size n=%d must be a power of two in 32..1024", fn, n);
    if (n_proj == 0 || M == 0)
        return ok();
    if (!projs)
        return fail(TQ_ERR_NULL, "%s: projs is NULL", fn);
    for (int j = 0; j < n_proj; ++j) {
        const tq_proj &p = projs[j];
        if (p.K < 0 || p.K % n != 0)
            return fail(TQ_ERR_SHAPE, "%s: entry %d: K=%d is not a multiple of n=%d", fn, j, p.K, n);
        if (p.K > tq::kStreamMaxK)
            return fail(TQ_ERR_UNSUPPORTED, "%s: entry %d: K=%d exceeds %d", fn, j, p.K,
                        tq::kStreamMaxK);
        if (!p.x_scale || (p.K > 0 && (!p.x || !p.xq)))
            return fail(TQ_ERR_NULL, "%s: entry %d: NULL pointer", fn, j);
        if ((p.K > 0 && (!aligned(p.x, 16) || !aligned(p.xq, 16))) || !aligned(p.x_scale, 4) ||
            (p.x_sum && !aligned(p.x_sum, 4)))
            return fail(TQ_ERR_ALIGN, "%s: entry %d: misaligned pointer", fn, j);
    }
    std::vector<tq::QuantStackEntry> list;
    int max_k = 0;
    for (int j = 0; j < n_proj; ++j) {
        const tq_proj &p = projs[j];
        if (p.K == 0) {  // no entries: zero scale and sum, as tq_quantize_act_stack
            cudaError_t e = cudaMemsetAsync(p.x_scale, 0, size_t(M) * sizeof(float), stream);
            if (e == cudaSuccess && p.x_sum)
                e = cudaMemsetAsync(p.x_sum, 0, size_t(M) * sizeof(int32_t), stream);
            if (e != cudaSuccess)
                return cuda_fail(e, fn);
            continue;
        }
        list.push_back(tq::QuantStackEntry{p.x, p.xq, p.x_scale, p.x_sum, p.K, M, 0, 0});
        max_k = std::max(max_k, p.K);
    }
    tq::QuantStackParams &params = *quant_params();
    for (size_t base = 0; base < list.size(); base += tq::kMaxQuantStack) {
        const size_t cnt = std::min(list.size() - base, size_t(tq::kMaxQuantStack));
        params.n = int(cnt);
        long long rows = 0;
        for (size_t i = 0; i < cnt; ++i) {
            params.e[i] = list[base + i];
            params.e[i].row0 = int(rows);
            rows += M;
        }
        if (rows > INT32_MAX)
            return fail(TQ_ERR_UNSUPPORTED, "%s: %lld rows in one call", fn, rows);
        params.rows = int(rows);
        const cudaError_t e = tq::launch_hadamard_quant4_stack(params, max_k, n, stream);
        if (e != cudaSuccess)
            return cuda_fail(e, fn);
    }
    return ok();
}

tq_status tq_pack_binary_host(const int8_t *w, const uint16_t *scales, uint8_t *bits,
                              uint16_t *scales_packed, int N, int K)
{
    if (N < 0 || K < 0 || N % 8 != 0 || K % 128 != 0)
        return fail(TQ_ERR_SHAPE, "tq_pack_binary_host: N=%d K=%d (need N %% 8 == 0, K %% 128 == 0)",
                    N, K);
    if (N == 0 || K == 0)
        return ok();
    if (!w || !scales || !bits || !scales_packed)
        return fail(TQ_ERR_NULL, "tq_pack_binary_host: a required pointer is NULL");
    if (!tq::pack_binary_host(w, scales, bits, scales_packed, N, K))
        return fail(TQ_ERR_VALUE, "tq_pack_binary_host: a weight is not -1 or +1");
    return ok();
}

namespace {

tq_status check_binary_args(const char *fn, const tq_binary_proj &p, int M)
{
    if (M < 0 || p.N < 0 || p.K < 0)
        return fail(TQ_ERR_SHAPE, "%s: negative size (M=%d N=%d K=%d)", fn, M, p.N, p.K);
    if (p.N % 8 != 0 || p.K % 128 != 0)
        return fail(TQ_ERR_SHAPE, "%s: N=%d K=%d (need N %% 8 == 0, K %% 128 == 0)", fn, p.N, p.K);
    if (M > tq::kBinMaxTokens)
        return fail(TQ_ERR_UNSUPPORTED, "%s: M=%d (1..%d tokens)", fn, M, tq::kBinMaxTokens);
    if (M == 0 || p.N == 0)
        return TQ_OK;
    if (!p.y || (p.K > 0 && (!p.bits || !p.scales_packed || !p.xq || !p.x_scale)))
        return fail(TQ_ERR_NULL, "%s: a required pointer is NULL", fn);
    if ((p.bits && !aligned(p.bits, 16)) || (p.scales_packed && !aligned(p.scales_packed, 16)) ||
        (p.xq && !aligned(p.xq, 16)))
        return fail(TQ_ERR_ALIGN, "%s: bits, scales and xq must be 16-byte aligned", fn);
    if ((p.x_scale && !aligned(p.x_scale, 4)) || !aligned(p.y, 4) ||
        (p.acc_out && !aligned(p.acc_out, 4)))
        return fail(TQ_ERR_ALIGN, "%s: x_scale, y, acc_out must be 4-byte aligned", fn);
    if (p.K > tq::kStreamMaxK)
        return fail(TQ_ERR_UNSUPPORTED, "%s: K=%d exceeds %d", fn, p.K, tq::kStreamMaxK);
    return TQ_OK;
}

tq::BinEntry bin_entry(const tq_binary_proj &p)
{
    tq::BinEntry e = {};
    e.bits = p.bits;
    e.scales = p.scales_packed;
    e.xq = p.xq;
    e.x_scale = p.x_scale;
    e.y = p.y;
    e.acc_out = p.acc_out;
    e.N8 = p.N / 8;
    e.K = p.K;
    return e;
}

}  // namespace

tq_status tq_gemv_binary_stack(const tq_binary_proj *projs, int n_proj, int M, cudaStream_t stream)
{
    const char *fn = "tq_gemv_binary_stack";
    if (n_proj < 0 || (n_proj > 0 && !projs))
        return fail(TQ_ERR_NULL, "%s: projs is NULL", fn);
    std::vector<tq::BinEntry> list;
    list.reserve(size_t(n_proj));
    for (int j = 0; j < n_proj; ++j) {
        const tq_status st = check_binary_args(fn, projs[j], M);
        if (st != TQ_OK)
            return st;
    }
    if (M == 0)
        return ok();
    for (int j = 0; j < n_proj; ++j) {
        const tq_binary_proj &p = projs[j];
        if (p.N == 0)
            continue;
        if (p.K == 0) {
            const tq_status st = zero_outputs(p.y, p.acc_out, size_t(M) * p.N, stream);
            if (st != TQ_OK)
                return st;
            continue;
        }
        list.push_back(bin_entry(p));
    }
    for (size_t base = 0; base < list.size(); base += tq::kBinStackMax) {
        const int n = int(std::min(list.size() - base, size_t(tq::kBinStackMax)));
        cudaError_t e = tq::launch_binary_gemv(list.data() + base, n, M, stream);
        if (e != cudaSuccess)
            return cuda_fail(e, fn);
    }
    return ok();
}

tq_status tq_gemv_binary(const uint8_t *bits, const uint16_t *scales_packed, const int8_t *xq,
                         const float *x_scale, float *y, int32_t *acc_out, int M, int N, int K,
                         cudaStream_t stream)
{
    const tq_binary_proj p = {bits, scales_packed, xq, x_scale, y, acc_out, N, K};
    const tq_status st = check_binary_args("tq_gemv_binary", p, M);
    if (st != TQ_OK)
        return st;
    return tq_gemv_binary_stack(&p, 1, M, stream);
}

tq_status tq_selftest_wait_timeout(unsigned limit_us, cudaStream_t stream)
{
    if (limit_us == 0 || limit_us > 2000000u)
        return fail(TQ_ERR_VALUE, "tq_selftest_wait_timeout: limit_us=%u (1..2000000)", limit_us);
    unsigned *err = tq::device_error_word();
    if (!err)
        return fail(TQ_ERR_CUDA, "tq_selftest_wait_timeout: no device error word");
    wait_selftest_kernel<<<1, 32, 0, stream>>>(err, 1000ull * limit_us);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ok() : cuda_fail(e, "tq_selftest_wait_timeout");
}

tq_status tq_device_error(uint32_t *code, int reset)
{
    if (!code)
        return fail(TQ_ERR_NULL, "tq_device_error: code is NULL");
    cudaError_t e = cudaDeviceSynchronize();
    unsigned v = 0;
    if (e == cudaSuccess)
        e = cudaMemcpyFromSymbol(&v, tq::g_device_error, sizeof v);
    if (e == cudaSuccess && reset) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(tq::g_device_error, &zero, sizeof zero);
    }
    if (e != cudaSuccess)
        return cuda_fail(e, "tq_device_error");
    if (v != 0)
        tq::group_scratch_mark_dirty();  // a kernel that gave up may have left partial sums
    *code = v;
    return ok();
}

}  // extern "C"
