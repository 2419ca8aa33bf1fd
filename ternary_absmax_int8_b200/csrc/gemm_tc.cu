// gemm_tc.cu -- prompt-processing (M >= 33 tokens) ternary GEMM on the
// 5th-generation tensor cores (tcgen05, int8, accumulators in tensor memory).
//
// Prompt processing is bound by the GPU's matrix units rather than by bytes
// (1bit engine blog, "Qwen3.8-27B at 45.7 tok/s ..."): at M = 512 every
// weight is reused 512 times, so this path expands the 2-bit codes to bytes
// on chip and runs an int8 contraction on the tensor cores.
//
//   D[n, m] = sum_k c[n, k] * xq[m, k]    (u8 codes c = w + 1 in {0,1,2},
//                                          s8 activations, s32 in TMEM;
//                                          plane p's codes enter as c * 4^p,
//                                          its sums leave shifted by 2p)
//   acc[m, n] = D[n, m] - x_sum[m]          (since w = c - 1)
//   y[m, n] = float(acc) * (w_scale * x_scale[m])
//
// Tile: G x 128 output features x BN tokens, K in stages of 128 bytes; G (1
// or 2) MMA groups of 128 rows share each activation stage, so the
// activation operand is read from L2 once per G x 128 features. In group g,
// MMA row r = 32 p + j is feature i0 + 32 g + j + p N/4: one TMA tile of
// G x 32 packed rows (128B-swizzled) expands into the G A operands of 16 KB.
// The host picks (G, BN) in {(2,256), (1,256), (1,128)} for the least
// estimated time (waves of tiles over the SMs x cycles per K stage;
// larger tiles on ties), since a 512-token prompt through a 2560-feature
// projection makes only 20 tiles of the largest shape.
//
// Warp roles (14 warps, one CTA per SM, persistent over tiles):
//   warp 0       TMA producer: packed tile + activation tile per K stage
//   warp 1       TMEM allocator; lane 0 issues the MMAs and commits
//   warps 2..13  expand the codes into the A stage (canonical K-major, 128B
//                swizzle), fence to the async proxy, signal the MMA
//   warps 6..13  then run the tile's epilogue: warp w reads TMEM lane
//                quarter w % 4 of its group (G = 2) or of its half of the
//                columns (G = 1), subtracts x_sum, scales, stores y
// The accumulator (G x BN columns) is single-buffered: a CTA's next tile
// starts its MMAs once the epilogue has drained it, so the epilogue warps
// are free to expand codes during the main loop (expansion, 16 bytes of
// shared-memory stores per 4 bytes of weights, is what bounds a stage
// otherwise). Every mbarrier wait is
// bounded; loads never use cluster multicast.
#include <atomic>
#include <algorithm>
#include <cstring>

#include "tc_common.cuh"

namespace tq {

namespace {

constexpr int kGM = 128;                // MMA M: rows of one group
constexpr int kBK = 128;                // bytes of K per stage
constexpr int kAGroupBytes = kGM * kBK; // 16 KB
constexpr int kThreads = 448;
constexpr int kExpWarp0 = 2;             // warps 2..13 expand codes
constexpr int kExpWarps = 12;
constexpr int kEpiWarp0 = 6;             // warps 6..13 also run the epilogue
constexpr int kEpiWarps = 8;
constexpr size_t kSmemLimit = 227 * 1024;

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

template <int G, int BN>
struct PrefillShape {
    static constexpr int kPackedRows = 32 * G;          // packed rows per tile
    static constexpr int kABytes = G * kAGroupBytes;
    static constexpr int kBBytes = BN * kBK;
    static constexpr int kPBytes = kPackedRows * kBK;
    static constexpr int kStageBytes = kABytes + kBBytes + kPBytes;
    static constexpr int kBarCount_(int s) { return 4 * s + 2; }
    // as many stages as fit next to the barriers and the 1 KB alignment slack
    static constexpr int kStages =
        int((kSmemLimit - 1024 - 256) / size_t(kStageBytes)) > 6
            ? 6
            : int((kSmemLimit - 1024 - 256) / size_t(kStageBytes));
    static constexpr int kAccCols = G * BN;
    static constexpr int kTmemCols = kAccCols < 32 ? 32 : kAccCols;  // a power of two here
    // 1024-byte aligned operand stages (the 128B swizzle atom is 1 KB)
    static constexpr size_t a_off = 0;
    static constexpr size_t b_off = a_off + size_t(kStages) * kABytes;
    static constexpr size_t p_off = b_off + size_t(kStages) * kBBytes;
    static constexpr size_t bar_off = p_off + size_t(kStages) * kPBytes;
    // barriers: tma_full, a_full, mma_done, p_free per stage; acc_full, acc_empty
    static constexpr size_t tmem_slot_off = bar_off + size_t(kBarCount_(kStages)) * 8;
    static constexpr size_t bytes = tmem_slot_off + 16;
    static_assert(kStages >= 2, "two stages at least");
    static_assert(bytes + 1024 <= kSmemLimit, "shared memory");
    static_assert((kTmemCols & (kTmemCols - 1)) == 0 && kTmemCols <= 512, "tensor memory");
};

// One output element: y (and the exact accumulator when asked).
__device__ __forceinline__ void store_out(const PrefillParams &p, int m, int n, int32_t d,
                                          float t, int32_t xs)
{
    const int32_t acc = d - xs;
    const size_t o = size_t(m) * (4 * size_t(p.N4)) + n;
    p.y[o] = __fmul_rn(__int2float_rn(acc), t);
    if (p.acc_out)
        p.acc_out[o] = acc;
}

template <int G, int BN>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap map_p, const __grid_constant__ CUtensorMap map_x,
                  const __grid_constant__ PrefillParams p)
{
    using S = PrefillShape<G, BN>;
    constexpr int kStages = S::kStages;
    constexpr uint32_t kIdesc = idesc_i8_u8s8(kGM, BN);
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // the dynamic base is only guaranteed 16-byte aligned: round up to 1 KB
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem + S::a_off;
    uint8_t *sB = smem + S::b_off;
    uint8_t *sP = smem + S::p_off;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S::bar_off);
    uint64_t *tma_full = bars;
    uint64_t *a_full = bars + kStages;
    uint64_t *mma_done = bars + 2 * kStages;
    uint64_t *p_free = bars + 3 * kStages;
    uint64_t *acc_full = bars + 4 * kStages;
    uint64_t *acc_empty = acc_full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + S::tmem_slot_off);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tiles = p.feat_tiles * p.tok_tiles;
    const int KS = p.k_stages;

    if (threadIdx.x == 0) {
        prefetch_tensormap(&map_p);
        prefetch_tensormap(&map_x);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&tma_full[s], 1);
            mbar_init(&a_full[s], kExpWarps);
            mbar_init(&mma_done[s], 1);
            mbar_init(&p_free[s], kExpWarps);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, kEpiWarps);
        fence_mbar_init();
    }
    if (warp == 1)
        tmem_alloc(tmem_slot, S::kTmemCols);
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
                    mbar_arrive_expect_tx(&tma_full[stage], S::kPBytes + S::kBBytes);
                    tma_load_2d(sP + stage * S::kPBytes, &map_p, ks * kBK, ft * S::kPackedRows,
                                &tma_full[stage]);
                    tma_load_2d(sB + stage * S::kBBytes, &map_x, ks * kBK, tt * BN, &tma_full[stage]);
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
                if (local >= 1 && !mbar_wait(acc_empty, uint32_t((local - 1) & 1), p.err))
                    break;
                tc_fence_after();
                for (int ks = 0; ks < KS; ++ks) {
                    if (!mbar_wait(&tma_full[stage], phase, p.err) ||
                        !mbar_wait(&a_full[stage], phase, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    // one descriptor per operand and stage, advanced by adds
                    const uint64_t da = umma_desc_sw128(smem_u32(sA + stage * S::kABytes));
                    const uint64_t db = umma_desc_sw128(smem_u32(sB + stage * S::kBBytes));
#pragma unroll
                    for (int g = 0; g < G; ++g)
#pragma unroll
                        for (int kk = 0; kk < kBK / 32; ++kk)
                            umma_i8(tmem_base + uint32_t(g * BN),
                                    umma_desc_advance(da, uint32_t(g * kAGroupBytes + kk * 32)),
                                    umma_desc_advance(db, uint32_t(kk * 32)), kIdesc,
                                    (ks > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&mma_done[stage]);
                    ++issued;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok)
                    umma_commit(acc_full);
            }
            // the last commit tracks every MMA this thread issued
            if (issued > 0) {
                const int s = (issued - 1) % kStages;
                mbar_wait(&mma_done[s], uint32_t(((issued - 1) / kStages) & 1), p.err);
            }
        }
    } else {
        // -------------------------- code expansion, then (warps 6..13) epilogue
        const int et = threadIdx.x - kExpWarp0 * 32;  // 0..383
        const bool epi = warp >= kEpiWarp0;
        const int q = warp & 3;                  // TMEM lane quarter = plane
        const int sub = (warp - kEpiWarp0) >> 2;
        const int eg = G == 2 ? sub : 0;         // MMA group of this epilogue warp
        const int cb = G == 2 ? 0 : sub * (BN / 2);  // its columns: [cb, cb + ncol)
        constexpr int ncol = G == 2 ? BN : BN / 2;
        constexpr int kUnits = S::kPackedRows * 8;   // 16-byte chunks of packed bytes per stage
        int stage = 0;
        uint32_t phase = 0;
        int seen = 0;
        int local = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++local) {
            for (int ks = 0; ks < KS; ++ks) {
                bool w1 = mbar_wait_warp(&tma_full[stage], phase, p.err);
                bool w2 = w1 && (seen < kStages || mbar_wait_warp(&mma_done[stage], phase ^ 1u, p.err));
                if (!w2) {
                    ok = false;
                    break;
                }
                const uint8_t *P = sP + stage * S::kPBytes;
                uint8_t *A = sA + stage * S::kABytes;
#pragma unroll
                for (int h = 0; h < (kUnits + kExpWarps * 32 - 1) / (kExpWarps * 32); ++h) {
                    const int idx = et + h * kExpWarps * 32;  // (packed row j of the tile, chunk c)
                    if (idx < kUnits) {
                        const int j = idx >> 3, c = idx & 7;
                        const int g = j >> 5, jj = j & 31;
                        const uint4 v = *reinterpret_cast<const uint4 *>(P + sw128_off(j, c));
                        uint8_t *Ag = A + g * kAGroupBytes;
// plane bits left in place: code c held as c * 4^pl (<= 128, a u8),
                        // one AND per word; the epilogue shifts the sums back
#pragma unroll
                        for (int pl = 0; pl < 4; ++pl) {
                            const uint32_t m = 0x03030303u << (2 * pl);
                            const uint4 o = make_uint4(v.x & m, v.y & m, v.z & m, v.w & m);
                            *reinterpret_cast<uint4 *>(Ag + sw128_off(jj + 32 * pl, c)) = o;
                        }
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
            if (!epi || !ok)
                continue;
            // ---- epilogue of tile t
            const int ft = t / p.tok_tiles, tt = t - ft * p.tok_tiles;
            if (!mbar_wait_warp(acc_full, uint32_t(local & 1), p.err))
                break;
            tc_fence_after();
            const int prow = ft * S::kPackedRows + eg * 32 + lane;  // packed row of this lane
            const bool row_ok = prow < p.N4;
            const int n = prow + q * p.N4;
            const uint32_t tbase = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(eg * BN + cb);
            for (int c0 = 0; c0 < ncol; c0 += 32) {
                const int mbase = tt * BN + cb + c0;
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
                    if (row_ok && mbase + i < p.M)
                        store_out(p, mbase + i, n, int32_t(v[i]) >> (2 * q), ts, xs);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(acc_empty);
        }
    }

    __syncwarp();  // single-lane roles rejoin their warps before the CTA barrier
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        tmem_dealloc(tmem_base, S::kTmemCols);
}

template <int G, int BN>
cudaError_t launch_shape(const uint8_t *packed, const int8_t *xq, PrefillParams prm,
                         cudaStream_t stream)
{
    using S = PrefillShape<G, BN>;
    CUtensorMap map_p, map_x;
    if (!make_map(&map_p, packed, prm.K, prm.N4, S::kPackedRows) ||
        !make_map(&map_x, xq, prm.K, prm.M, BN))
        return cudaErrorInvalidValue;
    prm.feat_tiles = (prm.N4 + S::kPackedRows - 1) / S::kPackedRows;
    prm.tok_tiles = (prm.M + BN - 1) / BN;
    const size_t smem = S::bytes + 1024;  // + alignment slack
    static std::atomic<int> configured_dev{-1};  // set by any host thread
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel<G, BN>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess)
            return e;
        configured_dev = dev;
    }
    const int tiles = prm.feat_tiles * prm.tok_tiles;
    const int grid = std::min(tiles, device_sm_count());
    prefill_tc_kernel<G, BN><<<grid, kThreads, smem, stream>>>(map_p, map_x, prm);
    return cudaGetLastError();
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
    PrefillParams prm = {};
    prm.N4 = N / 4;
    prm.K = K;
    prm.M = M;
    prm.k_stages = (K + kBK - 1) / kBK;
    prm.w_scale = w_scale;
    prm.x_scale = x_scale;
    prm.x_sum = x_sum;
    prm.y = y;
    prm.acc_out = acc_out;
    prm.err = device_error_word();
    if (!prm.err)
        return cudaErrorUnknown;
    // Tile shape: the least estimated time = waves of tiles over the SMs x
    // cycles per K stage of one tile. A stage is 4 G MMAs of K = 32, each
    // costing its execution (BN / 2 cycles at the int8 rate) or its issue by
    // the single MMA thread (~100 cycles, measured), whichever is longer,
    // plus ~100 cycles of pipeline overhead. The larger tile wins ties (fewer
    // operand re-reads from L2).
    const int sms = device_sm_count();
    const int shapes[3][2] = {{2, 256}, {1, 256}, {1, 128}};
    int best = 0;
    long long best_cost = -1;
    for (int i = 0; i < 3; ++i) {
        const int G = shapes[i][0], BN = shapes[i][1];
        const long long tiles =
            (long long)((prm.N4 + 32 * G - 1) / (32 * G)) * ((M + BN - 1) / BN);
        const long long stage = 4LL * G * std::max(BN / 2, 100) + 100;
        const long long cost = (tiles + sms - 1) / sms * stage;
        if (best_cost < 0 || cost < best_cost) {
            best = i;
            best_cost = cost;
        }
    }
    cudaError_t e;
    switch (best) {
    case 0: e = launch_shape<2, 256>(packed, xq, prm, stream); break;
    case 1: e = launch_shape<1, 256>(packed, xq, prm, stream); break;
    default: e = launch_shape<1, 128>(packed, xq, prm, stream); break;
    }
    if (e == cudaSuccess)
        *handled = true;
    return e;
}

}  // namespace tq
