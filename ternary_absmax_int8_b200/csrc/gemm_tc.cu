// gemm_tc.cu -- prompt-processing (M >= 33 tokens) ternary GEMM on the
// 5th-generation tensor cores (tcgen05, int8, accumulators in tensor memory),
// one projection or a group of projections per launch.
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
// Tile: 128 output features x BN tokens (BN = 256, or 128 for M <= 128), K in
// stages of 128 bytes. MMA row r = 32 p + j is feature i0 + j + p N/4: one
// TMA tile of 32 packed rows (128B-swizzled) expands into the 16 KB A
// operand of the stage. A launch takes the tiles of all its projections
// (shapes and K may differ) and deals them to persistent CTAs by a static
// longest-first schedule computed on the host, so that projections too
// small to fill the GPU alone fill it together.
//
// Warp roles (18 warps, one CTA per SM):
//   warp 0       TMA producer: packed tile + activation tile per K stage
//   warp 1       TMEM allocator; lane 0 issues the MMAs and commits
//   warps 2..9   expand the codes into the A stage (canonical K-major, 128B
//                swizzle), fence to the async proxy, signal the MMA
//   warps 10..17 epilogue: warp w reads TMEM lane quarter w % 4 (the plane)
//                over half of the tile's columns, subtracts x_sum, scales and
//                stores y; of a CTA's last tile the expansion warps, idle by
//                then, drain half of the columns
// Launched with programmatic serialisation: the set-up (barriers, tensor
// memory, tensor-map prefetch) overlaps the previous grid's tail, and every
// access to global memory waits for that grid (griddepcontrol.wait).
// The accumulator is double-buffered in tensor memory (2 x BN columns): the
// MMAs of a CTA's next tile run while the epilogue warps drain the previous
// one, so the output stores (4 bytes per element, as many bytes as the
// weights many times over at M = 512) overlap the contraction. Every mbarrier
// wait is bounded; loads never use cluster multicast.
#include <atomic>
#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <vector>

#include "tc_common.cuh"

namespace tq {

namespace {

constexpr int kGM = 128;                 // MMA M: rows of a tile
constexpr int kBK = 128;                 // bytes of K per stage
constexpr int kABytes = kGM * kBK;       // 16 KB
constexpr int kPackedRows = 32;          // packed rows per tile
constexpr int kPBytes = kPackedRows * kBK;
constexpr int kExpWarp0 = 2, kExpWarps = 8;
constexpr int kEpiWarp0 = kExpWarp0 + kExpWarps, kEpiWarps = 8;
constexpr int kThreads = (kEpiWarp0 + kEpiWarps) * 32;  // 576
constexpr size_t kSmemLimit = 227 * 1024;

// A tile of a group launch: projection (4 bits), token tile (14 bits),
// feature tile (14 bits).
__host__ __device__ constexpr uint32_t tile_code(int e, int tt, int ft)
{
    return (uint32_t(e) << 28) | (uint32_t(tt) << 14) | uint32_t(ft);
}
constexpr int kTileField = 1 << 14;

struct PrefillProj {
    int N4, KS;  // packed rows, K stages
    int vec;     // outputs written four features per 16-byte store (N4 % 4 == 0, aligned)
    float w_scale;
    const float *x_scale;
    const int32_t *x_sum;
    float *y;
    int32_t *acc_out;
};

// The launch's table (a kernel parameter; tensor maps 64-byte aligned).
struct PrefillTable {
    CUtensorMap map_p[kPrefillMaxGroup];
    CUtensorMap map_x[kPrefillMaxGroup];
    PrefillProj e[kPrefillMaxGroup];
    int n, M;
    unsigned *err;
    int cta0[kPrefillMaxGrid + 1];  // CTA b works through tile[cta0[b] .. cta0[b + 1] - 1]
    uint32_t tile[kPrefillMaxTiles];
};
static_assert(sizeof(PrefillTable) <= 32000, "kernel parameters");

template <int BN>
struct PrefillShape {
    static constexpr int kBBytes = BN * kBK;
    static constexpr int kStageBytes = kABytes + kBBytes + kPBytes;
    static constexpr int kBarCount_(int s) { return 4 * s + 4; }
    // as many stages as fit next to the barriers and the 1 KB alignment slack
    static constexpr int kStages =
        int((kSmemLimit - 1024 - 512) / size_t(kStageBytes)) > 6
            ? 6
            : int((kSmemLimit - 1024 - 512) / size_t(kStageBytes));
    static constexpr int kTmemCols = 2 * BN;  // two accumulators
    // 1024-byte aligned operand stages (the 128B swizzle atom is 1 KB)
    static constexpr size_t a_off = 0;
    static constexpr size_t b_off = a_off + size_t(kStages) * kABytes;
    static constexpr size_t p_off = b_off + size_t(kStages) * kBBytes;
    static constexpr size_t bar_off = p_off + size_t(kStages) * kPBytes;
    // barriers: tma_full, a_full, mma_done, p_free per stage; acc_full[2], acc_empty[2]
    static constexpr size_t tmem_slot_off = bar_off + size_t(kBarCount_(kStages)) * 8;
    static constexpr size_t bytes = tmem_slot_off + 16;
    static_assert(kStages >= 3, "three stages at least");
    static_assert(bytes + 1024 <= kSmemLimit, "shared memory");
    static_assert((kTmemCols & (kTmemCols - 1)) == 0 && kTmemCols <= 512, "tensor memory");
};

// One output element: y (and the exact accumulator when asked); streaming
// stores (the outputs are not read again by this kernel).
__device__ __forceinline__ void store_out(const PrefillProj &e, int N, int m, int n, int32_t d,
                                          float t, int32_t xs)
{
    const int32_t acc = d - xs;
    const size_t o = size_t(m) * size_t(N) + n;
    __stcs(e.y + o, __fmul_rn(__int2float_rn(acc), t));
    if (e.acc_out)
        __stcs(e.acc_out + o, acc);
}

// 4 x 4 transpose within each quad of lanes: lane 4a + i holds m[k] = the
// value of feature 4a + i at token k (k = 0..3); on return f[j] = the value
// of feature 4a + j at token i (two exchanges, lanes i ^ 2 then i ^ 1).
__device__ __forceinline__ void quad_transpose(const int32_t (&m)[4], int32_t (&f)[4], int i)
{
    const bool b1 = i & 2, b0 = i & 1;
    // first exchange: keep the tokens whose bit 1 equals ours, trade the others
    const int32_t r0 = __shfl_xor_sync(0xffffffffu, b1 ? m[0] : m[2], 2);
    const int32_t r1 = __shfl_xor_sync(0xffffffffu, b1 ? m[1] : m[3], 2);
    const int32_t k0 = b1 ? m[2] : m[0], k1 = b1 ? m[3] : m[1];
    // w[rb][kb]: rb = bit 1 of the feature, kb = bit 0 of the token
    const int32_t w00 = b1 ? r0 : k0, w01 = b1 ? r1 : k1;
    const int32_t w10 = b1 ? k0 : r0, w11 = b1 ? k1 : r1;
    // second exchange: keep kb == bit 0 of ours, trade the other
    const int32_t u0 = __shfl_xor_sync(0xffffffffu, b0 ? w00 : w01, 1);
    const int32_t u1 = __shfl_xor_sync(0xffffffffu, b0 ? w10 : w11, 1);
    const int32_t c0 = b0 ? w01 : w00, c1 = b0 ? w11 : w10;
    f[0] = b0 ? u0 : c0;
    f[1] = b0 ? c0 : u0;
    f[2] = b0 ? u1 : c1;
    f[3] = b0 ? c1 : u1;
}

// Epilogue of columns [c_begin, c_end) (tokens tt * BN + c) of one tile's
// accumulator, by one warp of TMEM lane quarter q (plane q): lane = packed
// row prow0 + lane, feature n = that row + q N/4.
template <int BN>
__device__ __forceinline__ void drain_columns(const PrefillTable &tab, uint32_t code, int prow0,
                                              uint32_t tmem_acc, int q, int c_begin, int c_end,
                                              int lane)
{
    const int e = int(code >> 28), tt = int((code >> 14) & (kTileField - 1));
    const PrefillProj &pe = tab.e[e];
    const int N4 = pe.N4, N = 4 * N4;
    const int prow = prow0 + lane;  // packed row of this lane
    const bool row_ok = prow < N4;
    const int n = prow + q * N4;
    const uint32_t tbase = tmem_acc + (uint32_t(q * 32) << 16);
    for (int c0 = c_begin; c0 < c_end; c0 += 32) {
        const int mbase = tt * BN + c0;
        if (mbase >= tab.M)
            break;
        uint32_t v[32];
        tmem_ld32(tbase + uint32_t(c0), v);
        const int my_m = mbase + lane;
        const float my_t = my_m < tab.M ? __fmul_rn(pe.w_scale, __ldg(pe.x_scale + my_m)) : 0.0f;
        const int32_t my_s = my_m < tab.M ? __ldg(pe.x_sum + my_m) : 0;
        if (pe.vec) {
            // quads of lanes trade values so that each lane writes four
            // consecutive features of one token: a 16-byte store
            const int i4 = lane & 3;
            const int f0 = prow0 + (lane & ~3);  // first feature of the quad
            const size_t n0 = size_t(f0) + size_t(q) * N4;
#pragma unroll
            for (int k0 = 0; k0 < 32; k0 += 4) {
                const int32_t m4[4] = {int32_t(v[k0]) >> (2 * q), int32_t(v[k0 + 1]) >> (2 * q),
                                       int32_t(v[k0 + 2]) >> (2 * q), int32_t(v[k0 + 3]) >> (2 * q)};
                int32_t f4[4];
                quad_transpose(m4, f4, i4);
                const int tk = k0 + i4;  // this lane's token in the chunk
                const float ts = __shfl_sync(0xffffffffu, my_t, tk);
                const int32_t xs = __shfl_sync(0xffffffffu, my_s, tk);
                if (f0 < N4 && mbase + tk < tab.M) {
                    const size_t o = size_t(mbase + tk) * size_t(N) + n0;
                    const int4 a4 = make_int4(f4[0] - xs, f4[1] - xs, f4[2] - xs, f4[3] - xs);
                    __stcs(reinterpret_cast<float4 *>(pe.y + o),
                           make_float4(__fmul_rn(__int2float_rn(a4.x), ts),
                                       __fmul_rn(__int2float_rn(a4.y), ts),
                                       __fmul_rn(__int2float_rn(a4.z), ts),
                                       __fmul_rn(__int2float_rn(a4.w), ts)));
                    if (pe.acc_out)
                        __stcs(reinterpret_cast<int4 *>(pe.acc_out + o), a4);
                }
            }
        } else {
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                const float ts = __shfl_sync(0xffffffffu, my_t, k);
                const int32_t xs = __shfl_sync(0xffffffffu, my_s, k);
                if (row_ok && mbase + k < tab.M)
                    store_out(pe, N, mbase + k, n, int32_t(v[k]) >> (2 * q), ts, xs);
            }
        }
    }
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ PrefillTable tab)
{
    using S = PrefillShape<BN>;
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
    uint64_t *acc_full = bars + 4 * kStages;  // [2]
    uint64_t *acc_empty = acc_full + 2;       // [2]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + S::tmem_slot_off);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t_begin = tab.cta0[blockIdx.x], t_end = tab.cta0[blockIdx.x + 1];
    unsigned *err = tab.err;
    // The next grid on the stream may start its set-up now; it waits for this
    // one before it touches memory.
    pdl_launch_dependents();

    if (threadIdx.x == 0) {
        for (int j = 0; j < tab.n; ++j) {
            prefetch_tensormap(&tab.map_p[j]);
            prefetch_tensormap(&tab.map_x[j]);
        }
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&tma_full[s], 1);
            mbar_init(&a_full[s], kExpWarps);
            mbar_init(&mma_done[s], 1);
            mbar_init(&p_free[s], kExpWarps);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], kEpiWarps);
        }
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
            // every global operand may still be written by the previous grid
            // on the stream (launched with programmatic serialisation)
            pdl_wait();
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            bool ok = true;
            for (int i = t_begin; i < t_end && ok; ++i) {
                const uint32_t code = tab.tile[i];
                const int e = int(code >> 28), tt = int((code >> 14) & (kTileField - 1)),
                          ft = int(code & (kTileField - 1));
                const int KS = tab.e[e].KS;
                for (int ks = 0; ks < KS; ++ks) {
                    if (issued >= kStages) {
                        if (!mbar_wait(&mma_done[stage], phase ^ 1u, err) ||
                            !mbar_wait(&p_free[stage], phase ^ 1u, err)) {
                            ok = false;
                            break;
                        }
                    }
                    mbar_arrive_expect_tx(&tma_full[stage], kPBytes + S::kBBytes);
                    tma_load_2d(sP + stage * kPBytes, &tab.map_p[e], ks * kBK, ft * kPackedRows,
                                &tma_full[stage]);
                    tma_load_2d(sB + stage * S::kBBytes, &tab.map_x[e], ks * kBK, tt * BN,
                                &tma_full[stage]);
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
                mbar_wait(&tma_full[s], uint32_t((last / kStages) & 1), err);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int issued = 0;
            for (int i = t_begin, local = 0; i < t_end && ok; ++i, ++local) {
                const int buf = local & 1;
                // the epilogue has drained this accumulator's previous tile
                if (local >= 2 && !mbar_wait(&acc_empty[buf], uint32_t(((local - 2) >> 1) & 1), err))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + uint32_t(buf * BN);
                const int KS = tab.e[tab.tile[i] >> 28].KS;
                for (int ks = 0; ks < KS; ++ks) {
                    if (!mbar_wait(&tma_full[stage], phase, err) ||
                        !mbar_wait(&a_full[stage], phase, err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    // one descriptor per operand and stage, advanced by adds
                    const uint64_t da = umma_desc_sw128(smem_u32(sA + stage * kABytes));
                    const uint64_t db = umma_desc_sw128(smem_u32(sB + stage * S::kBBytes));
#pragma unroll
                    for (int kk = 0; kk < kBK / 32; ++kk)
                        umma_i8(d_tmem, umma_desc_advance(da, uint32_t(kk * 32)),
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
                    umma_commit(&acc_full[buf]);
            }
            // the last commit tracks every MMA this thread issued
            if (issued > 0) {
                const int s = (issued - 1) % kStages;
                mbar_wait(&mma_done[s], uint32_t(((issued - 1) / kStages) & 1), err);
            }
        }
    } else if (warp < kEpiWarp0) {
        // ------------------------------------------------ code expansion
        // thread et expands 16-byte chunk et of the stage's packed tile:
        // packed row j = et / 8, chunk c = et % 8
        const int et = threadIdx.x - kExpWarp0 * 32;  // 0..255
        const int j = et >> 3, c = et & 7;
        static_assert(kExpWarps * 32 == kPackedRows * 8, "one chunk per expansion thread");
        int stage = 0;
        uint32_t phase = 0;
        int seen = 0;
        bool ok = true;
        for (int i = t_begin; i < t_end && ok; ++i) {
            const int KS = tab.e[tab.tile[i] >> 28].KS;
            for (int ks = 0; ks < KS; ++ks) {
                const bool w1 = mbar_wait_warp(&tma_full[stage], phase, err);
                const bool w2 =
                    w1 && (seen < kStages || mbar_wait_warp(&mma_done[stage], phase ^ 1u, err));
                if (!w2) {
                    ok = false;
                    break;
                }
                const uint4 v = *reinterpret_cast<const uint4 *>(sP + stage * kPBytes + sw128_off(j, c));
                uint8_t *A = sA + stage * kABytes;
                // plane bits left in place: code c held as c * 4^pl (<= 128, a
                // u8), one AND per word; the epilogue shifts the sums back
#pragma unroll
                for (int pl = 0; pl < 4; ++pl) {
                    const uint32_t m = 0x03030303u << (2 * pl);
                    const uint4 o = make_uint4(v.x & m, v.y & m, v.z & m, v.w & m);
                    *reinterpret_cast<uint4 *>(A + sw128_off(j + 32 * pl, c)) = o;
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
        // the last tile's columns [BN/2, BN): expansion warp w drains lane
        // quarter w % 4 over one quarter of the columns
        const int local_last = t_end - 1 - t_begin;
        if (ok && local_last >= 0) {
            pdl_wait();
            const int buf = local_last & 1;
            if (mbar_wait_warp(&acc_full[buf], uint32_t((local_last >> 1) & 1), err)) {
                tc_fence_after();
                const int c_begin = BN / 2 + ((warp - kExpWarp0) >> 2) * (BN / 4);
                const uint32_t code = tab.tile[t_end - 1];
                drain_columns<BN>(tab, code, int(code & (kTileField - 1)) * kPackedRows,
                                  tmem_base + uint32_t(buf * BN), warp & 3, c_begin,
                                  c_begin + BN / 4, lane);
                tc_fence_before();
            }
        }
    } else {
        // ------------------------------------------------ epilogue
        // warp w drains lane quarter w % 4 over its half of the columns; of the
        // CTA's last tile it drains a quarter (the expansion warps, idle by
        // then, drain the other half)
        const int q = warp & 3;                    // TMEM lane quarter = plane
        const int half = (warp - kEpiWarp0) >> 2;
        pdl_wait();  // outputs and scales belong to the previous grid until it completes
        for (int i = t_begin, local = 0; i < t_end; ++i, ++local) {
            const int buf = local & 1;
            if (!mbar_wait_warp(&acc_full[buf], uint32_t((local >> 1) & 1), err))
                break;
            tc_fence_after();
            const bool last = i + 1 == t_end;
            const int c_begin = last ? half * (BN / 4) : half * (BN / 2);
            const int c_end = c_begin + (last ? BN / 4 : BN / 2);
            drain_columns<BN>(tab, tab.tile[i], int(tab.tile[i] & (kTileField - 1)) * kPackedRows,
                              tmem_base + uint32_t(buf * BN), q, c_begin, c_end, lane);
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
        tmem_dealloc(tmem_base, S::kTmemCols);
}

// ---------------------------------------------------------------------------
// The pair form: the two CTAs of a cluster run 256-row MMAs
// (tcgen05.mma.cta_group::2) on a tile of 256 features (64 packed rows: the
// even CTA expands rows 0..31, the odd one rows 32..63) x 256 tokens (each
// CTA holds 128 of them in shared memory). A K stage per CTA is 16 KB of
// codes + 16 KB of activations + 4 KB of packed bytes, so six stages fit;
// each CTA keeps its 128 rows of both accumulators in its own tensor memory.
// Barriers: the even CTA's full (the activation halves of both CTAs) and
// a_full (its own 8 expansion warps arrive; the odd CTA's 8 each complete 4
// transaction bytes with an asynchronous remote store, st.async, whose
// completion releases at cluster scope without stalling the warp -- a
// remote arrive with cluster-scope release stalls its thread ~1,000 cycles,
// too much per stage), each CTA's own pfull (its packed tile) and p_free,
// and empty / acc_full committed to both CTAs by the even CTA's MMA thread;
// acc_empty on the even CTA (its epilogue warps arrive, the odd CTA's
// complete bytes the same way).
constexpr int kPairBN = 256;              // tokens per tile
constexpr int kPairBHalf = (kPairBN / 2) * kBK;  // 16 KB: a CTA's activation rows
constexpr int kPairStage = kABytes + kPairBHalf + kPBytes;
constexpr int kPairStages =
    int((kSmemLimit - 1024 - 512) / size_t(kPairStage)) > 6 ? 6
                                                          : int((kSmemLimit - 1024 - 512) / size_t(kPairStage));
struct PairSmem {
    static constexpr size_t a_off = 0;
    static constexpr size_t b_off = a_off + size_t(kPairStages) * kABytes;
    static constexpr size_t p_off = b_off + size_t(kPairStages) * kPairBHalf;
    static constexpr size_t bar_off = p_off + size_t(kPairStages) * kPBytes;
    // full, pfull, a_full, empty, p_free per stage; acc_full[2], acc_empty[2]
    static constexpr size_t sig_off = bar_off + size_t(5 * kPairStages + 4) * 8;
    static constexpr size_t tmem_slot_off = sig_off + 64;  // 16 words written by st.async
    static constexpr size_t bytes = tmem_slot_off + 16;
    static_assert(kPairStages >= 4, "four stages at least");
    static_assert(bytes + 1024 <= kSmemLimit, "shared memory");
};
constexpr int kPairTmemCols = 2 * kPairBN;  // two accumulators

__global__ void __launch_bounds__(kThreads, 1)
prefill_pair_kernel(const __grid_constant__ PrefillTable tab)
{
    using S = PairSmem;
    constexpr int kStages = kPairStages;
    constexpr uint32_t kIdesc = idesc_i8_u8s8(2 * kGM, kPairBN);
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem + S::a_off;
    uint8_t *sB = smem + S::b_off;
    uint8_t *sP = smem + S::p_off;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S::bar_off);
    uint64_t *full = bars;                     // even CTA: activations of both CTAs
    uint64_t *pfull = bars + kStages;          // own packed tile
    uint64_t *a_full = bars + 2 * kStages;     // even CTA: 2 x 8 expansion warps
    uint64_t *empty = bars + 3 * kStages;      // MMAs of the stage done (committed to both)
    uint64_t *p_free = bars + 4 * kStages;     // own packed tile read
    uint64_t *acc_full = bars + 5 * kStages;   // [2], committed to both
    uint64_t *acc_empty = acc_full + 2;        // [2], even CTA: 2 x 8 epilogue warps
    uint32_t *sig = reinterpret_cast<uint32_t *>(smem + S::sig_off);  // st.async targets
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + S::tmem_slot_off);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = int(blockIdx.x >> 1);
    const int t_begin = tab.cta0[pair], t_end = tab.cta0[pair + 1];
    unsigned *err = tab.err;
    pdl_launch_dependents();

    if (threadIdx.x == 0) {
        for (int j = 0; j < tab.n; ++j) {
            prefetch_tensormap(&tab.map_p[j]);
            prefetch_tensormap(&tab.map_x[j]);
        }
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&pfull[s], 1);
            mbar_init(&a_full[s], kExpWarps);  // own warps; the odd CTA's by bytes
            mbar_init(&empty[s], 1);
            mbar_init(&p_free[s], kExpWarps);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], kEpiWarps);  // own warps; the odd CTA's by bytes
        }
        fence_mbar_init();
    }
    if (warp == 1)
        tmem_alloc_pair(tmem_slot, kPairTmemCols);
    tc_fence_before();
    cluster_sync_all();  // both CTAs' barriers exist before either arrives remotely
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // the even CTA's barriers, as cluster addresses
    auto lead = [&](uint64_t *b) { return map_to_rank(smem_u32(b), 0); };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            pdl_wait();
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            bool ok = true;
            for (int i = t_begin; i < t_end && ok; ++i) {
                const uint32_t code = tab.tile[i];
                const int e = int(code >> 28), tt = int((code >> 14) & (kTileField - 1)),
                          ft = int(code & (kTileField - 1));
                const int KS = tab.e[e].KS;
                for (int ks = 0; ks < KS; ++ks) {
                    if (issued >= kStages) {
                        if (!mbar_wait(&empty[stage], phase ^ 1u, err) ||
                            !mbar_wait(&p_free[stage], phase ^ 1u, err)) {
                            ok = false;
                            break;
                        }
                    }
                    if (leader)
                        mbar_arrive_expect_tx(&full[stage], 2 * kPairBHalf);
                    tma_load_2d_pair(sB + stage * kPairBHalf, &tab.map_x[e], ks * kBK,
                                     tt * kPairBN + int(rank) * (kPairBN / 2), lead(&full[stage]));
                    mbar_arrive_expect_tx(&pfull[stage], kPBytes);
                    tma_load_2d(sP + stage * kPBytes, &tab.map_p[e], ks * kBK,
                                ft * (2 * kPackedRows) + int(rank) * kPackedRows, &pfull[stage]);
                    ++issued;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // the packed tiles still in flight land before the CTA may retire
            // (the activation halves are waited for by the even CTA's MMA
            // thread, and the CTAs retire together)
            for (int s = 0; s < kStages && s < issued; ++s) {
                const int last = issued - 1 - ((issued - 1 - s) % kStages);
                mbar_wait(&pfull[s], uint32_t((last / kStages) & 1), err);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (even CTA)
        if (lane == 0 && leader) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int issued = 0;
            for (int i = t_begin, local = 0; i < t_end && ok; ++i, ++local) {
                const int buf = local & 1;
                if (local >= 2 &&
                    !mbar_wait_cluster(&acc_empty[buf], uint32_t(((local - 2) >> 1) & 1), err))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + uint32_t(buf * kPairBN);
                const int KS = tab.e[tab.tile[i] >> 28].KS;
                for (int ks = 0; ks < KS; ++ks) {
                    if (!mbar_wait(&full[stage], phase, err) ||
                        !mbar_wait_cluster(&a_full[stage], phase, err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t da = umma_desc_sw128(smem_u32(sA + stage * kABytes));
                    const uint64_t db = umma_desc_sw128(smem_u32(sB + stage * kPairBHalf));
#pragma unroll
                    for (int kk = 0; kk < kBK / 32; ++kk)
                        umma_i8_pair(d_tmem, umma_desc_advance(da, uint32_t(kk * 32)),
                                     umma_desc_advance(db, uint32_t(kk * 32)), kIdesc,
                                     (ks > 0 || kk > 0) ? 1u : 0u);
                    umma_commit_pair(&empty[stage]);
                    ++issued;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok)
                    umma_commit_pair(&acc_full[buf]);
            }
            if (issued > 0) {
                const int s = (issued - 1) % kStages;
                mbar_wait(&empty[s], uint32_t(((issued - 1) / kStages) & 1), err);
            }
        }
    } else if (warp < kEpiWarp0) {
        // ------------------------------------------------ code expansion (both CTAs)
        const int et = threadIdx.x - kExpWarp0 * 32;  // 0..255
        const int j = et >> 3, c = et & 7;
        int stage = 0;
        uint32_t phase = 0;
        int seen = 0;
        bool ok = true;
        for (int i = t_begin; i < t_end && ok; ++i) {
            const int KS = tab.e[tab.tile[i] >> 28].KS;
            for (int ks = 0; ks < KS; ++ks) {
                const bool w1 = mbar_wait_warp(&pfull[stage], phase, err);
                const bool w2 =
                    w1 && (seen < kStages || mbar_wait_warp(&empty[stage], phase ^ 1u, err));
                if (!w2) {
                    ok = false;
                    break;
                }
                const uint4 v = *reinterpret_cast<const uint4 *>(sP + stage * kPBytes + sw128_off(j, c));
                uint8_t *A = sA + stage * kABytes;
#pragma unroll
                for (int pl = 0; pl < 4; ++pl) {
                    const uint32_t m = 0x03030303u << (2 * pl);
                    const uint4 o = make_uint4(v.x & m, v.y & m, v.z & m, v.w & m);
                    *reinterpret_cast<uint4 *>(A + sw128_off(j + 32 * pl, c)) = o;
                }
                fence_proxy_async_smem();  // the codes are read by the tensor cores
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&p_free[stage]);
                    const int ew = warp - kExpWarp0;
                    if (!leader)
                        st_async_signal(map_to_rank(smem_u32(&sig[ew]), 0), 1u, lead(&a_full[stage]));
                    else if (ew == 0)  // the odd CTA's 8 x 4 bytes
                        mbar_arrive_expect_tx(&a_full[stage], 4 * kExpWarps);
                    else
                        mbar_arrive(&a_full[stage]);
                }
                ++seen;
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        // the last tile's columns [128, 256) of this CTA's rows
        const int local_last = t_end - 1 - t_begin;
        if (ok && local_last >= 0) {
            pdl_wait();
            const int buf = local_last & 1;
            if (mbar_wait_warp(&acc_full[buf], uint32_t((local_last >> 1) & 1), err)) {
                tc_fence_after();
                const uint32_t code = tab.tile[t_end - 1];
                const int c_begin = kPairBN / 2 + ((warp - kExpWarp0) >> 2) * (kPairBN / 4);
                drain_columns<kPairBN>(tab, code,
                                       int(code & (kTileField - 1)) * (2 * kPackedRows) +
                                           int(rank) * kPackedRows,
                                       tmem_base + uint32_t(buf * kPairBN), warp & 3, c_begin,
                                       c_begin + kPairBN / 4, lane);
                tc_fence_before();
            }
        }
    } else {
        // ------------------------------------------------ epilogue (both CTAs)
        const int q = warp & 3;
        const int half = (warp - kEpiWarp0) >> 2;
        pdl_wait();
        for (int i = t_begin, local = 0; i < t_end; ++i, ++local) {
            const int buf = local & 1;
            if (!mbar_wait_warp(&acc_full[buf], uint32_t((local >> 1) & 1), err))
                break;
            tc_fence_after();
            const bool last = i + 1 == t_end;
            const int c_begin = last ? half * (kPairBN / 4) : half * (kPairBN / 2);
            const int c_end = c_begin + (last ? kPairBN / 4 : kPairBN / 2);
            const uint32_t code = tab.tile[i];
            drain_columns<kPairBN>(tab, code,
                                   int(code & (kTileField - 1)) * (2 * kPackedRows) +
                                       int(rank) * kPackedRows,
                                   tmem_base + uint32_t(buf * kPairBN), q, c_begin, c_end, lane);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {  // the accumulator's loads have completed (tcgen05.wait::ld)
                const int ew = warp - kEpiWarp0;
                if (!leader)
                    st_async_signal(map_to_rank(smem_u32(&sig[kExpWarps + ew]), 0), 1u,
                                    lead(&acc_empty[buf]));
                else if (ew == 0)  // the odd CTA's 8 x 4 bytes
                    mbar_arrive_expect_tx(&acc_empty[buf], 4 * kEpiWarps);
                else
                    mbar_arrive(&acc_empty[buf]);
            }
        }
    }

    __syncwarp();
    tc_fence_before();
    cluster_sync_all();  // no remote arrive or MMA operand read outlives either CTA
    tc_fence_after();
    if (warp == 1)
        tmem_dealloc_pair(tmem_base, kPairTmemCols);
}

// Deal the tiles [0, n) (costs cost[i]) to `grid` CTAs, longest first, each
// to the least-loaded CTA; fill order[] CTA by CTA and cta0[].
void schedule_lpt(const std::vector<int> &cost, int grid, std::vector<int> &order, int *cta0)
{
    const int n = int(cost.size());
    std::vector<int> idx(static_cast<size_t>(n));
    for (int i = 0; i < n; ++i)
        idx[size_t(i)] = i;
    std::stable_sort(idx.begin(), idx.end(),
                     [&](int a, int b) { return cost[size_t(a)] > cost[size_t(b)]; });
    std::vector<long long> load(static_cast<size_t>(grid), 0);
    std::vector<int> owner(static_cast<size_t>(n));
    for (int i : idx) {
        int best = 0;
        for (int b = 1; b < grid; ++b)
            if (load[size_t(b)] < load[size_t(best)])
                best = b;
        owner[size_t(i)] = best;
        load[size_t(best)] += cost[size_t(i)];
    }
    std::vector<int> count(static_cast<size_t>(grid), 0);
    for (int i = 0; i < n; ++i)
        ++count[size_t(owner[size_t(i)])];
    cta0[0] = 0;
    for (int b = 0; b < grid; ++b)
        cta0[b + 1] = cta0[b] + count[size_t(b)];
    std::vector<int> fill(cta0, cta0 + grid);
    order.assign(size_t(n), 0);
    for (int i : idx)  // longest first within each CTA too
        order[size_t(fill[size_t(owner[size_t(i)])]++)] = i;
}

PrefillTable *prefill_table()
{
    static thread_local PrefillTable t;
    return &t;
}

// How a launch tiles the work: tokens per tile, packed rows per tile (32 per
// CTA), the activation box each CTA loads, CTAs per tile.
struct TileForm {
    int tok, prows, xbox, ctas;
    void (*kernel)(PrefillTable);
    size_t smem;
};

cudaError_t configure(const TileForm &f, std::atomic<int> &configured_dev)
{
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess)
        return err;
    if (configured_dev != dev) {
        err = cudaFuncSetAttribute(f.kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   int(f.smem));
        if (err != cudaSuccess)
            return err;
        configured_dev = dev;
    }
    return cudaSuccess;
}

cudaError_t launch_tiles(const TileForm &f, const PrefillEntry *in, int n, int M,
                         cudaStream_t stream)
{
    unsigned *err_word = device_error_word();
    if (!err_word)
        return cudaErrorUnknown;
    const int tok_tiles = (M + f.tok - 1) / f.tok;
    // every tile of every projection, in projection order
    std::vector<uint32_t> codes;
    std::vector<int> cost;
    for (int j = 0; j < n; ++j) {
        const int ft_tiles = (in[j].N / 4 + f.prows - 1) / f.prows;
        const int KS = (in[j].K + kBK - 1) / kBK;
        for (int ft = 0; ft < ft_tiles; ++ft)
            for (int tt = 0; tt < tok_tiles; ++tt) {
                codes.push_back(tile_code(j, tt, ft));
                cost.push_back(KS);
            }
    }
    PrefillTable &tab = *prefill_table();
    std::memset(static_cast<void *>(&tab), 0, sizeof(tab));
    tab.n = n;
    tab.M = M;
    tab.err = err_word;
    for (int j = 0; j < n; ++j) {
        if (!make_map(&tab.map_p[j], in[j].packed, in[j].K, in[j].N / 4, kPackedRows) ||
            !make_map(&tab.map_x[j], in[j].xq, in[j].K, M, f.xbox))
            return cudaErrorInvalidValue;
        const bool vec = (in[j].N / 4) % 4 == 0 && reinterpret_cast<uintptr_t>(in[j].y) % 16 == 0 &&
                         reinterpret_cast<uintptr_t>(in[j].acc_out) % 16 == 0;
        tab.e[j] = PrefillProj{in[j].N / 4, (in[j].K + kBK - 1) / kBK, vec ? 1 : 0, in[j].w_scale,
                               in[j].x_scale, in[j].x_sum, in[j].y, in[j].acc_out};
    }
    // launches of up to kPrefillMaxTiles tiles each (any subset of tiles is a
    // valid launch); one launch for every shape this library is measured on
    const int units = std::min(device_sm_count(), kPrefillMaxGrid) / f.ctas;
    const int total = int(codes.size());
    for (int base = 0; base < total; base += kPrefillMaxTiles) {
        const int cnt = std::min(total - base, kPrefillMaxTiles);
        const int grid = std::min(cnt, units);  // CTAs (or CTA pairs) dealt tiles
        std::vector<int> sub(cost.begin() + base, cost.begin() + base + cnt), order;
        schedule_lpt(sub, grid, order, tab.cta0);
        for (int i = 0; i < cnt; ++i)
            tab.tile[i] = codes[size_t(base + order[size_t(i)])];
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(unsigned(grid * f.ctas));
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = f.smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = unsigned(f.ctas);
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = f.ctas > 1 ? 2 : 1;
        cudaError_t err = cudaLaunchKernelEx(&cfg, f.kernel, tab);
        if (err == cudaSuccess)
            err = cudaGetLastError();
        if (err != cudaSuccess)
            return err;
    }
    return cudaSuccess;
}

template <int BN>
cudaError_t launch_bn(const PrefillEntry *in, int n, int M, cudaStream_t stream)
{
    static std::atomic<int> configured_dev{-1};  // set by any host thread
    const TileForm f{BN, kPackedRows, BN, 1, prefill_tc_kernel<BN>, PrefillShape<BN>::bytes + 1024};
    const cudaError_t err = configure(f, configured_dev);
    return err != cudaSuccess ? err : launch_tiles(f, in, n, M, stream);
}

cudaError_t launch_pair(const PrefillEntry *in, int n, int M, cudaStream_t stream)
{
    static std::atomic<int> configured_dev{-1};
    const TileForm f{kPairBN, 2 * kPackedRows, kPairBN / 2, 2, prefill_pair_kernel,
                     PairSmem::bytes + 1024};
    const cudaError_t err = configure(f, configured_dev);
    return err != cudaSuccess ? err : launch_tiles(f, in, n, M, stream);
}

}  // namespace

constexpr int kPrefillMinM = 33;

cudaError_t launch_prefill_group(const PrefillEntry *e, int n, int M, cudaStream_t stream,
                                 bool *handled)
{
    *handled = false;
    if (M < kPrefillMinM || n <= 0)
        return cudaSuccess;
    if (n > kPrefillMaxGroup)
        return cudaErrorInvalidValue;
    for (int j = 0; j < n; ++j)
        if ((e[j].N / 4 + kPackedRows - 1) / kPackedRows > kTileField)
            return cudaErrorInvalidValue;
    // 128-token tiles while they waste less of the MMA than 256-token ones;
    // from 129 tokens CTA pairs on 256 x 256 tiles (TQ_PREFILL_PAIR=0 keeps
    // single CTAs on 128 x 256 tiles, for measurement)
    const bool narrow = M <= 128;
    if ((M + (narrow ? 127 : 255)) / (narrow ? 128 : 256) > kTileField)
        return cudaErrorInvalidValue;
    static const bool pairs = [] {
        const char *v = getenv("TQ_PREFILL_PAIR");
        return !(v && !strcmp(v, "0"));
    }();
    const cudaError_t err = narrow  ? launch_bn<128>(e, n, M, stream)
                            : pairs ? launch_pair(e, n, M, stream)
                                    : launch_bn<256>(e, n, M, stream);
    if (err == cudaSuccess)
        *handled = true;
    return err;
}

cudaError_t launch_prefill_tc(const uint8_t *packed, float w_scale, const int8_t *xq,
                              const float *x_scale, const int32_t *x_sum, float *y,
                              int32_t *acc_out, int M, int N, int K, cudaStream_t stream,
                              bool *handled)
{
    const PrefillEntry e{packed, w_scale, xq, x_scale, x_sum, y, acc_out, N, K};
    return launch_prefill_group(&e, 1, M, stream, handled);
}

}  // namespace tq
