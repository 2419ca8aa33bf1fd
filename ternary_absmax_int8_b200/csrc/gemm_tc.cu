// gemm_tc.cu -- prompt-processing (M >= 128 tokens) ternary GEMM on the
// 5th-generation tensor cores (tcgen05, int8, accumulators in tensor memory).
//
// Prompt processing is bound by the GPU's matrix units rather than by bytes
// (1bit engine blog, "Qwen3.8-27B at 45.7 tok/s ..."): at M = 512 every
// weight is reused 512 times, so this path expands the 2-bit codes to bytes
// on chip and runs an int8 contraction on the tensor cores.
//
//   D[n, m] = sum_k c[n, k] * xq[m, k]    (u8 codes c = w + 1 in {0,1,2},
//                                          s8 activations, s32 in TMEM)
//   acc[m, n] = D[n, m] - x_sum[m]          (since w = c - 1)
//   y[m, n] = float(acc) * (w_scale * x_scale[m])
//
// Tile: 128 output features x BN = 256 tokens, K in stages of 128 bytes.
// The 128 features of a tile are 32 packed rows i0 .. i0+31 times the four
// planes: MMA row r = 32 p + j is feature i0 + j + p N/4. So one 4 KB tile of
// packed bytes (TMA, 128B-swizzled) expands into the 16 KB A operand.
//
// Warp roles (10 warps, one CTA per SM, persistent over tiles):
//   warp 0      TMA producer: packed tile + activation tile per K stage
//   warp 1      TMEM allocator; lane 0 issues the MMAs and commits
//   warps 2..5  expand the codes into the A stage (canonical K-major,
//               128B swizzle), fence to the async proxy, signal the MMA
//   warps 6..9  epilogue: tcgen05.ld the accumulator (warp w reads TMEM lanes
//               32 (w % 4) ..), subtract x_sum, scale, store y
// Accumulators are double-buffered in TMEM (2 x 256 columns) so the epilogue
// of tile t overlaps the MMAs of tile t + 1. Every mbarrier wait is bounded.
#include <algorithm>
#include <cstring>

#include "tc_common.cuh"

namespace tq {

namespace {

constexpr int kBM = 128;         // features per tile (MMA M)
constexpr int kBN = 256;         // tokens per tile (MMA N)
constexpr int kBK = 128;         // bytes of K per stage
constexpr int kStages = 4;
constexpr int kPackedRows = kBM / 4;
constexpr int kABytes = kBM * kBK;           // 16 KB
constexpr int kBBytes = kBN * kBK;           // 32 KB
constexpr int kPBytes = kPackedRows * kBK;   // 4 KB
constexpr int kThreads = 320;
constexpr int kTmemCols = 2 * kBN;           // two accumulator buffers
constexpr uint32_t kIdesc = idesc_i8_u8s8(kBM, kBN);

struct PrefillParams {
    int N4, K, M;
    int feat_tiles, tok_tiles, k_stages;
    float w_scale;
    const float *x_scale;
    const int32_t *x_sum;
    float *y;
    int32_t *acc_out;
    unsigned *err;
};

struct PrefillSmem {
    // 1024-byte aligned operand stages (the 128B swizzle atom is 1 KB)
    static constexpr size_t a_off = 0;
    static constexpr size_t b_off = a_off + size_t(kStages) * kABytes;
    static constexpr size_t p_off = b_off + size_t(kStages) * kBBytes;
    static constexpr size_t bar_off = p_off + size_t(kStages) * kPBytes;
    // barriers: tma_full, a_full, mma_done, p_free per stage; acc_full, acc_empty x2
    static constexpr int kBarCount = 4 * kStages + 4;
    static constexpr size_t tmem_slot_off = bar_off + kBarCount * 8;
    static constexpr size_t bytes = tmem_slot_off + 16;
};

__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap map_p, const __grid_constant__ CUtensorMap map_x,
                  const __grid_constant__ PrefillParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // the dynamic base is only guaranteed 16-byte aligned: round up to 1 KB
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem + PrefillSmem::a_off;
    uint8_t *sB = smem + PrefillSmem::b_off;
    uint8_t *sP = smem + PrefillSmem::p_off;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + PrefillSmem::bar_off);
    uint64_t *tma_full = bars;
    uint64_t *a_full = bars + kStages;
    uint64_t *mma_done = bars + 2 * kStages;
    uint64_t *p_free = bars + 3 * kStages;
    uint64_t *acc_full = bars + 4 * kStages;
    uint64_t *acc_empty = acc_full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + PrefillSmem::tmem_slot_off);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tiles = p.feat_tiles * p.tok_tiles;
    const int KS = p.k_stages;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&tma_full[s], 1);
            mbar_init(&a_full[s], 4);
            mbar_init(&mma_done[s], 1);
            mbar_init(&p_free[s], 4);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        fence_mbar_init();
    }
    if (warp == 1)
        tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
                const int ft = t / p.tok_tiles, tt = t - ft * p.tok_tiles;
                for (int ks = 0; ks < KS; ++ks) {
                    if (issued >= kStages) {
                        if (!mbar_wait(&mma_done[stage], phase ^ 1u, p.err) ||
                            !mbar_wait(&p_free[stage], phase ^ 1u, p.err)) {
                            ok = false;
                            break;
                        }
                    }
                    mbar_arrive_expect_tx(&tma_full[stage], kPBytes + kBBytes);
                    tma_load_2d(sP + stage * kPBytes, &map_p, ks * kBK, ft * kPackedRows,
                                &tma_full[stage]);
                    tma_load_2d(sB + stage * kBBytes, &map_x, ks * kBK, tt * kBN, &tma_full[stage]);
                    ++issued;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // wait for the copies still in flight before the CTA may retire
            for (int s = 0; s < kStages && s < issued; ++s) {
                const int last = issued - 1 - ((issued - 1 - s) % kStages);  // last use of stage s
                mbar_wait(&tma_full[s], uint32_t((last / kStages) & 1), p.err);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int local = 0;
            bool ok = true;
            int issued = 0;
            for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++local) {
                const int buf = local & 1;
                if (local >= 2 && !mbar_wait(&acc_empty[buf], uint32_t(((local >> 1) - 1) & 1), p.err))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + uint32_t(buf * kBN);
                for (int ks = 0; ks < KS; ++ks) {
                    if (!mbar_wait(&tma_full[stage], phase, p.err) ||
                        !mbar_wait(&a_full[stage], phase, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sA + stage * kABytes);
                    const uint32_t b0 = smem_u32(sB + stage * kBBytes);
#pragma unroll
                    for (int kk = 0; kk < kBK / 32; ++kk)
                        umma_i8(d_tmem, umma_desc_sw128(a0 + kk * 32), umma_desc_sw128(b0 + kk * 32), kIdesc,
                                (ks > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&mma_done[stage]);
                    ++issued;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok)
                    umma_commit(&acc_full[buf]);
            }
            // the last commit tracks every MMA this thread issued
            if (issued > 0) {
                const int s = (issued - 1) % kStages;
                mbar_wait(&mma_done[s], uint32_t(((issued - 1) / kStages) & 1), p.err);
            }
        }
    } else if (warp < 6) {
        // ------------------------------------------------ code expansion
        const int et = threadIdx.x - 64;  // 0..127
        int stage = 0;
        uint32_t phase = 0;
        int seen = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
            for (int ks = 0; ks < KS; ++ks) {
                bool w1 = mbar_wait_warp(&tma_full[stage], phase, p.err);
                bool w2 = w1 && (seen < kStages || mbar_wait_warp(&mma_done[stage], phase ^ 1u, p.err));
                if (!w2) {
                    ok = false;
                    break;
                }
                const uint8_t *P = sP + stage * kPBytes;
                uint8_t *A = sA + stage * kABytes;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int idx = et + h * 128;  // (packed row j, chunk c)
                    const int j = idx >> 3, c = idx & 7;
                    const uint4 v = *reinterpret_cast<const uint4 *>(P + sw128_off(j, c));
#pragma unroll
                    for (int pl = 0; pl < 4; ++pl) {
                        uint4 o;
                        o.x = (v.x >> (2 * pl)) & 0x03030303u;
                        o.y = (v.y >> (2 * pl)) & 0x03030303u;
                        o.z = (v.z >> (2 * pl)) & 0x03030303u;
                        o.w = (v.w >> (2 * pl)) & 0x03030303u;
                        *reinterpret_cast<uint4 *>(A + sw128_off(j + 32 * pl, c)) = o;
                    }
                }
                fence_proxy_async_smem();  // make the codes visible to the tensor cores
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&p_free[stage]);
                    mbar_arrive(&a_full[stage]);
                }
                ++seen;
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else {
        // ------------------------------------------------ epilogue
        const int q = warp & 3;  // TMEM lane quarter this warp may access = plane
        int local = 0;
        for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++local) {
            const int ft = t / p.tok_tiles, tt = t - ft * p.tok_tiles;
            const int buf = local & 1;
            if (!mbar_wait_warp(&acc_full[buf], uint32_t((local >> 1) & 1), p.err))
                break;
            tc_fence_after();
            const int prow = ft * kPackedRows + lane;  // packed row of this lane
            const bool row_ok = prow < p.N4;
            const int n = prow + q * p.N4;
            const int N = 4 * p.N4;
            const uint32_t tbase = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(buf * kBN);
            for (int c0 = 0; c0 < kBN; c0 += 32) {
                const int mbase = tt * kBN + c0;
                if (mbase >= p.M)
                    break;
                uint32_t v[32];
                tmem_ld32(tbase + uint32_t(c0), v);
                const int my_m = mbase + lane;
                const float my_t = my_m < p.M ? __fmul_rn(p.w_scale, __ldg(p.x_scale + my_m)) : 0.0f;
                const int32_t my_s = my_m < p.M ? __ldg(p.x_sum + my_m) : 0;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float ts = __shfl_sync(0xffffffffu, my_t, i);
                    const int32_t xs = __shfl_sync(0xffffffffu, my_s, i);
                    const int m = mbase + i;
                    if (row_ok && m < p.M) {
                        const int32_t acc = int32_t(v[i]) - xs;
                        const size_t o = size_t(m) * N + n;
                        p.y[o] = __fmul_rn(__int2float_rn(acc), ts);
                        if (p.acc_out)
                            p.acc_out[o] = acc;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&acc_empty[buf]);
        }
    }

    __syncwarp();  // single-lane roles rejoin their warps before the CTA barrier
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        tmem_dealloc(tmem_base, kTmemCols);
}

}  // namespace

constexpr int kPrefillMinM = 33;

cudaError_t launch_prefill_tc(const uint8_t *packed, float w_scale, const int8_t *xq,
                              const float *x_scale, const int32_t *x_sum, float *y,
                              int32_t *acc_out, int M, int N, int K, cudaStream_t stream,
                              bool *handled)
{
    *handled = false;
    if (M < kPrefillMinM)
        return cudaSuccess;
    CUtensorMap map_p, map_x;
    if (!make_map(&map_p, packed, K, N / 4, kPackedRows) || !make_map(&map_x, xq, K, M, kBN))
        return cudaErrorInvalidValue;
    PrefillParams prm;
    prm.N4 = N / 4;
    prm.K = K;
    prm.M = M;
    prm.feat_tiles = (prm.N4 + kPackedRows - 1) / kPackedRows;
    prm.tok_tiles = (M + kBN - 1) / kBN;
    prm.k_stages = (K + kBK - 1) / kBK;
    prm.w_scale = w_scale;
    prm.x_scale = x_scale;
    prm.x_sum = x_sum;
    prm.y = y;
    prm.acc_out = acc_out;
    prm.err = device_error_word();
    if (!prm.err)
        return cudaErrorUnknown;
    const size_t smem = PrefillSmem::bytes + 1024;  // + alignment slack
    static int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess)
            return e;
        configured_dev = dev;
    }
    const int tiles = prm.feat_tiles * prm.tok_tiles;
    const int grid = std::min(tiles, device_sm_count());
    prefill_tc_kernel<<<grid, kThreads, smem, stream>>>(map_p, map_x, prm);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess)
        *handled = true;
    return e;
}

}  // namespace tq
