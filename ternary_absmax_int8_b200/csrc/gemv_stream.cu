// gemv_stream.cu -- the decode-shaped ternary GEMV (M <= 4 tokens per launch),
// for one projection or for a whole stack of projections in one launch.
//
// Decode reads every weight byte once per token, so this kernel is bound by
// HBM bandwidth (1bit engine blog, "Qwen3.8-27B at 45.7 tok/s ...": decode
// speed is set by the bytes read per token; 1bit.systems README, "honest
// numbers": their HIP ternary GEMV at 92% of memory-bandwidth peak on
// gfx1151). Design for sm_100a:
//
//  * Persistent CTAs, one per SM, each a producer warp plus W consumer warps.
//  * The packed weights of a projection, uint8 [N/4, K] row-major, are cut
//    into tiles of R consecutive packed rows: one contiguous R*K-byte range,
//    moved by a single 1-D bulk copy (TMA engine, cp.async.bulk, no
//    multicast) into a ring of shared-memory stages guarded by mbarriers. The
//    ring keeps ~100-200 KB per SM in flight, which is what HBM3e's latency x
//    bandwidth product asks for. Tiles of all projections of a launch form one
//    sequence, dealt round-robin to the CTAs, so a stack of projections is
//    streamed back to back in projection order with no drain in between.
//  * Activations (int8, M x K) either stay resident in shared memory for the
//    whole launch (one projection) or ride along with each tile (a stack).
//  * Consumers read 16-byte words of packed weights and activations from
//    shared memory. A 32-bit word u holds, for output row i + p*N/4 (p =
//    0..3), the codes of 4 consecutive k in its bytes' bit fields 2p..2p+1;
//    u & (0x03030303 << 2p) isolates them, scaled by 4^p, and one dp4a
//    (unsigned codes x signed int8) accumulates them: acc'_p = 4^p * sum c*q.
//    No shifts are needed in the loop; the 4^p is removed once per output.
//  * Since w = c - 1, acc = sum c*q - sum q = acc' - x_sum (x_sum comes from
//    the quantiser), so no per-element subtraction is needed either.
//  * A butterfly reduction gathers each warp's 4 partial sums per token in
//    six shuffles; warps that share a row add into shared memory with integer
//    atomics (exact, order-free); one named barrier per tile, then the
//    epilogue writes y = float(acc) * (w_scale * x_scale) for the tile's rows.
//  * Every mbarrier wait is bounded (2 s of global time); on a timeout the
//    kernel records an error bit, all consumer warps agree to stop through a
//    barrier reduction, and the producer waits (bounded) for its copies in
//    flight before the CTA exits.
#include <algorithm>
#include <cstdio>
#include <cstdlib>

#include "tq_internal.h"

namespace tq {

namespace {

constexpr int kMaxStages = 8;
constexpr int kWTargetBytes = 20480;  // weight bytes per tile, aim

// Dynamic shared memory a CTA may use when `cps` CTAs share an SM (228 KB per
// SM, 1 KB of it reserved per CTA).
constexpr size_t smem_budget(int cps) { return cps == 1 ? 227 * 1024 : 112 * 1024; }

__device__ __forceinline__ void dot16(const uint4 w, const uint4 x, int32_t (&a)[4])
{
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
    const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        a[0] = dp4a_us(ws[j] & 0x03030303u, xs[j], a[0]);
        a[1] = dp4a_us(ws[j] & 0x0C0C0C0Cu, xs[j], a[1]);
        a[2] = dp4a_us(ws[j] & 0x30303030u, xs[j], a[2]);
        a[3] = dp4a_us(ws[j] & 0xC0C0C0C0u, xs[j], a[3]);
    }
}

// Sum four per-lane values over the warp; lane L returns the total of value
// (L >> 3) & 3. Six shuffles instead of twenty.
__device__ __forceinline__ int32_t reduce4(const int32_t (&v)[4], int lane)
{
    const bool hi = lane & 16;
    int32_t k0 = hi ? v[2] : v[0], k1 = hi ? v[3] : v[1];
    const int32_t s0 = hi ? v[0] : v[2], s1 = hi ? v[1] : v[3];
    k0 += __shfl_xor_sync(0xffffffffu, s0, 16);
    k1 += __shfl_xor_sync(0xffffffffu, s1, 16);
    const bool b3 = lane & 8;
    int32_t c = b3 ? k1 : k0;
    const int32_t d = b3 ? k0 : k1;
    c += __shfl_xor_sync(0xffffffffu, d, 8);
    c += __shfl_xor_sync(0xffffffffu, c, 4);
    c += __shfl_xor_sync(0xffffffffu, c, 2);
    c += __shfl_xor_sync(0xffffffffu, c, 1);
    return c;
}

struct TileInfo {
    int entry;
    int row0;
    int rows;
};

template <int MaxE>
__device__ __forceinline__ TileInfo locate(const StreamParams<MaxE> &p, int t, int &cursor)
{
    while (cursor + 1 < p.n_entries && p.e[cursor + 1].tile_begin <= t)
        ++cursor;
    const StreamEntry &e = p.e[cursor];
    TileInfo ti;
    ti.entry = cursor;
    ti.row0 = (t - e.tile_begin) * e.rows_per_tile;
    ti.rows = min(e.rows_per_tile, e.N4 - ti.row0);
    return ti;
}

template <int MT>
__device__ __forceinline__ float pick(const float (&a)[MT], int m)
{
    float r = a[0];
#pragma unroll
    for (int i = 1; i < MT; ++i)
        r = m == i ? a[i] : r;
    return r;
}

template <int MT>
__device__ __forceinline__ int32_t pick(const int32_t (&a)[MT], int m)
{
    int32_t r = a[0];
#pragma unroll
    for (int i = 1; i < MT; ++i)
        r = m == i ? a[i] : r;
    return r;
}

// Shared-memory plan of one CTA (byte offsets from the dynamic base):
//   [x_slot]              resident activations (one-projection launches only)
//   [stages * stage]      the ring; a stage is [x_slot (stack launches)][w_slot]
//   full[8], empty[8], xbar
//   part[8][16][MT][4]    int32 partial sums of rows split across warps
//   cnt[8][16]            how many warps have added into each row's partials
template <int MT>
struct SmemTail {
    static constexpr int kBars = 2 * kMaxStages + 1;
    static constexpr int kPart = kMaxStages * kStreamMaxRows * MT * 4;
    static constexpr int kCnt = kMaxStages * kStreamMaxRows;
    static constexpr size_t bytes() { return kBars * 8 + (kPart + kCnt) * 4; }
};

template <int W, int MaxE, int MT, int CPS>
__global__ void __launch_bounds__((W + 1) * 32, CPS)
stream_gemv_kernel(const __grid_constant__ StreamParams<MaxE> p)
{
    extern __shared__ __align__(128) uint8_t smem[];
    const int stages = p.stages;
    const bool resident_x = p.n_entries == 1;
    const int stage_bytes = (resident_x ? 0 : p.x_slot) + p.w_slot;
    uint8_t *xres = smem;
    uint8_t *ring = smem + (resident_x ? p.x_slot : 0);
    uint64_t *full = reinterpret_cast<uint64_t *>(ring + stages * stage_bytes);
    uint64_t *empty = full + kMaxStages;
    uint64_t *xbar = empty + kMaxStages;
    int32_t *part = reinterpret_cast<int32_t *>(xbar + 1);
    int32_t *cnt = part + SmemTail<MT>::kPart;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    for (int i = threadIdx.x; i < SmemTail<MT>::kPart + SmemTail<MT>::kCnt; i += blockDim.x)
        part[i] = 0;
    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], W);
        }
        mbar_init(xbar, 1);
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == W) {
        // ------------------------------------------------------ producer
        if (lane != 0)
            return;
        const uint64_t pol_w = policy_evict_first();  // weights: read once
        const uint64_t pol_x = policy_evict_last();   // activations: reread by many CTAs
        bool waited = !p.overlap_prev;
        if (waited)
            pdl_wait();
        if (resident_x && waited) {
            const StreamEntry &e = p.e[0];
            mbar_arrive_expect_tx(xbar, uint32_t(p.M * e.K));
            bulk_g2s(xres, e.xq, uint32_t(p.M * e.K), xbar, pol_x);
        }
        int deferred[kMaxStages];
        int n_def = 0;
        int cursor = 0, it = 0;
        for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x, ++it) {
            const TileInfo ti = locate(p, t, cursor);
            const StreamEntry &e = p.e[ti.entry];
            const int stage = it % stages;
            const int use = it / stages;
            if (!waited && it == stages) {
                // The ring is full of weight copies issued before the
                // previous grid finished; activations may be read now.
                pdl_wait();
                waited = true;
                if (resident_x) {
                    mbar_arrive_expect_tx(xbar, uint32_t(p.M * e.K));
                    bulk_g2s(xres, e.xq, uint32_t(p.M * e.K), xbar, pol_x);
                } else {
                    for (int d = 0; d < n_def; ++d) {
                        const StreamEntry &ed = p.e[deferred[d]];
                        bulk_g2s(ring + d * stage_bytes, ed.xq, uint32_t(p.M * ed.K), &full[d],
                                 pol_x);
                    }
                }
            }
            if (use > 0 && !mbar_wait(&empty[stage], uint32_t((use - 1) & 1), p.err))
                break;
            uint8_t *st = ring + stage * stage_bytes;
            const uint32_t wbytes = uint32_t(ti.rows) * uint32_t(e.K);
            const uint32_t xbytes = resident_x ? 0u : uint32_t(p.M * e.K);
            mbar_arrive_expect_tx(&full[stage], wbytes + xbytes);
            bulk_g2s(st + (resident_x ? 0 : p.x_slot), e.packed + size_t(ti.row0) * e.K, wbytes,
                     &full[stage], pol_w);
            if (!resident_x) {
                if (waited)
                    bulk_g2s(st, e.xq, xbytes, &full[stage], pol_x);
                else
                    deferred[n_def++] = ti.entry;
            }
        }
        if (!waited) {
            // Issue the activation copies still owed, even after a failed
            // wait, so that every stage barrier can complete.
            pdl_wait();
            if (resident_x) {
                const StreamEntry &e = p.e[0];
                mbar_arrive_expect_tx(xbar, uint32_t(p.M * e.K));
                bulk_g2s(xres, e.xq, uint32_t(p.M * e.K), xbar, pol_x);
            } else {
                for (int d = 0; d < n_def; ++d) {
                    const StreamEntry &ed = p.e[deferred[d]];
                    bulk_g2s(ring + d * stage_bytes, ed.xq, uint32_t(p.M * ed.K), &full[d], pol_x);
                }
            }
        }
        // Do not let the CTA retire while a copy this thread issued is in
        // flight (matters only when a wait gave up).
        const int used = min(it, stages);
        for (int s = 0; s < used; ++s)
            mbar_wait(&full[s], uint32_t(((it - 1 - s) / stages) & 1), p.err);
        if (resident_x && used > 0)
            mbar_wait(xbar, 0, p.err);
        return;
    }

    // ---------------------------------------------------------- consumers
    // Each consumer warp walks the ring on its own (no CTA barrier): it waits
    // for a stage, takes items warp, warp + W, ... of that tile, and releases
    // the stage. A row split over several warps is finished by whichever warp
    // adds the last partial sum.
    pdl_wait();  // x_scale and x_sum are read below
    if (resident_x && p.total_tiles > int(blockIdx.x) && !mbar_wait_warp(xbar, 0, p.err))
        return;

    int cursor = 0, it = 0;
    for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x, ++it) {
        const TileInfo ti = locate(p, t, cursor);
        const StreamEntry &e = p.e[ti.entry];
        const int stage = it % stages;
        const int use = it / stages;

        // Epilogue scales, fetched before the wait so their latency hides.
        float tsc[MT];
        int32_t xsm[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            tsc[m] = 0.0f;
            xsm[m] = 0;
            if (m < p.M) {
                tsc[m] = __fmul_rn(e.w_scale, __ldg(e.x_scale + m));
                xsm[m] = __ldg(e.x_sum + m);
            }
        }

        if (!mbar_wait_warp(&full[stage], uint32_t(use & 1), p.err))
            return;

        const uint8_t *st = ring + stage * stage_bytes;
        const uint8_t *sx = resident_x ? xres : st;
        const uint8_t *sw = resident_x ? st : st + p.x_slot;
        const int K = e.K;
        const int C = K >> 4;
        const int ks = e.ksplit;
        const int N = e.N4 * 4;
        const int n_items = ti.rows * ks;
        for (int item = warp; item < n_items; item += W) {
            const int r = item / ks;
            const int piece = item - r * ks;
            const int c0 = (piece * C) / ks, c1 = ((piece + 1) * C) / ks;
            const uint4 *wrow = reinterpret_cast<const uint4 *>(sw + size_t(r) * K);
            int32_t a[MT][4];
#pragma unroll
            for (int m = 0; m < MT; ++m)
                a[m][0] = a[m][1] = a[m][2] = a[m][3] = 0;
#pragma unroll 4
            for (int c = c0 + lane; c < c1; c += 32) {
                const uint4 wv = wrow[c];
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m < p.M) {
                        const uint4 xv = reinterpret_cast<const uint4 *>(sx + m * K)[c];
                        dot16(wv, xv, a[m]);
                    }
                }
            }
            const int row = ti.row0 + r;
            if (ks == 1) {
                // Whole row in this warp: lanes 0, 8, 16, 24 write planes 0..3.
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m < p.M) {
                        const int32_t v = reduce4(a[m], lane);
                        if ((lane & 7) == 0) {
                            const int plane = lane >> 3;
                            const int32_t acc = (v >> (2 * plane)) - xsm[m];
                            const size_t o = size_t(m) * N + row + plane * e.N4;
                            e.y[o] = __fmul_rn(__int2float_rn(acc), tsc[m]);
                            if (e.acc_out)
                                e.acc_out[o] = acc;
                        }
                    }
                }
            } else {
                int32_t *slot = part + (stage * kStreamMaxRows + r) * MT * 4;
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m < p.M) {
                        const int32_t v = reduce4(a[m], lane);
                        if ((lane & 7) == 0)
                            atomicAdd(&slot[m * 4 + (lane >> 3)], v);
                    }
                }
                __threadfence_block();  // partial sums before the count
                __syncwarp();
                int old = 0;
                if (lane == 0)
                    old = atomicAdd(&cnt[stage * kStreamMaxRows + r], 1);
                old = __shfl_sync(0xffffffffu, old, 0);
                if (old == ks - 1) {
                    __threadfence_block();
                    if (lane < 4 * p.M) {
                        const int m = lane >> 2, plane = lane & 3;
                        const int32_t v = atomicExch(&slot[m * 4 + plane], 0);
                        const int32_t acc = (v >> (2 * plane)) - pick(xsm, m);
                        const size_t o = size_t(m) * N + row + plane * e.N4;
                        e.y[o] = __fmul_rn(__int2float_rn(acc), pick(tsc, m));
                        if (e.acc_out)
                            e.acc_out[o] = acc;
                    }
                    if (lane == 0)
                        cnt[stage * kStreamMaxRows + r] = 0;
                }
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&empty[stage]);
    }
}

template <int W, int MaxE, int MT, int CPS>
cudaError_t launch_instance(const StreamParams<MaxE> &p, int grid, size_t smem, bool pdl,
                            cudaStream_t stream)
{
    auto kern = stream_gemv_kernel<W, MaxE, MT, CPS>;
    static int configured_dev = -1;  // per instantiation
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               int(smem_budget(CPS)));
        if (err != cudaSuccess)
            return err;
        configured_dev = dev;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3((W + 1) * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    cudaError_t err = cudaLaunchKernelEx(&cfg, kern, p);
    if (err != cudaSuccess)
        return err;
    return cudaGetLastError();
}

// Tuning knobs: consumer warps per CTA and CTAs per SM. TQ_STREAM_CFG="W,CPS"
// picks another instantiated variant (for measurement); default 8,1.
struct StreamCfg {
    int W = 8;
    int CPS = 1;
};

StreamCfg stream_cfg()
{
    static StreamCfg cfg = [] {
        StreamCfg c;
        if (const char *s = getenv("TQ_STREAM_CFG")) {
            int w = 0, cps = 0;
            if (sscanf(s, "%d,%d", &w, &cps) == 2 &&
                ((w == 8 && (cps == 1 || cps == 2)) || (w == 16 && cps == 1) ||
                 (w == 4 && cps == 2))) {
                c.W = w;
                c.CPS = cps;
            }
        }
        return c;
    }();
    return cfg;
}

template <int MaxE, int MT>
cudaError_t launch_variant(const StreamCfg &c, const StreamParams<MaxE> &p, int grid, size_t smem,
                           bool pdl, cudaStream_t stream)
{
    if (c.W == 8 && c.CPS == 2)
        return launch_instance<8, MaxE, MT, 2>(p, grid, smem, pdl, stream);
    if (c.W == 16)
        return launch_instance<16, MaxE, MT, 1>(p, grid, smem, pdl, stream);
    if (c.W == 4)
        return launch_instance<4, MaxE, MT, 2>(p, grid, smem, pdl, stream);
    return launch_instance<8, MaxE, MT, 1>(p, grid, smem, pdl, stream);
}

template <int MaxE>
cudaError_t launch_sized(StreamEntry *entries, int n, int M, bool overlap_prev, bool single,
                         cudaStream_t stream)
{
    StreamParams<MaxE> p;  // host staging of the launch parameters
    static_assert(sizeof(StreamParams<MaxE>) <= 32000, "kernel parameters exceed 32 KB");
    const StreamCfg cfg = stream_cfg();
    const int sms = device_sm_count();
    const int W = cfg.W;
    int total = 0, kmax = 0, wmax = 0;
    for (int j = 0; j < n; ++j) {
        StreamEntry &e = entries[j];
        const int K = e.K;
        int R = kStreamMaxRows;
        while (R > 1 && R * K > kWTargetBytes)
            R >>= 1;
        if (single)
            while (R > 1 && (e.N4 + R - 1) / R < 2 * sms * cfg.CPS)
                R >>= 1;
        const int C = K >> 4;
        int ks = std::max(1, W / R);
        ks = std::min(ks, std::max(1, C / 16));
        e.rows_per_tile = R;
        e.ksplit = ks;
        e.tile_begin = total;
        total += (e.N4 + R - 1) / R;
        kmax = std::max(kmax, K);
        wmax = std::max(wmax, R * K);
        p.e[j] = e;
    }
    p.n_entries = n;
    p.total_tiles = total;
    p.M = M;
    p.x_slot = (M * kmax + 127) / 128 * 128;
    p.w_slot = (wmax + 127) / 128 * 128;
    p.overlap_prev = overlap_prev ? 1 : 0;
    p.err = device_error_word();
    if (!p.err)
        return cudaErrorUnknown;
    const bool resident = n == 1;
    const int mt = M == 1 ? 1 : (M == 2 ? 2 : 4);
    const size_t tail = mt == 1 ? SmemTail<1>::bytes()
                                : (mt == 2 ? SmemTail<2>::bytes() : SmemTail<4>::bytes());
    const size_t fixed = tail + (resident ? p.x_slot : 0);
    const int stage_bytes = (resident ? 0 : p.x_slot) + p.w_slot;
    const size_t budget = smem_budget(cfg.CPS);
    int stages = budget > fixed ? int((budget - fixed) / size_t(stage_bytes)) : 0;
    stages = std::min(stages, kMaxStages);
    if (total == 0)
        return cudaSuccess;
    if (stages < 2)
        return cudaErrorInvalidValue;
    p.stages = stages;
    const size_t smem = fixed + size_t(stages) * stage_bytes;
    const int grid = std::min(total, sms * cfg.CPS);
    switch (mt) {
    case 1: return launch_variant<MaxE, 1>(cfg, p, grid, smem, overlap_prev, stream);
    case 2: return launch_variant<MaxE, 2>(cfg, p, grid, smem, overlap_prev, stream);
    default: return launch_variant<MaxE, 4>(cfg, p, grid, smem, overlap_prev, stream);
    }
}

}  // namespace

cudaError_t launch_stream_gemv(StreamEntry *entries, int n, int M, bool overlap_prev, bool single,
                               cudaStream_t stream)
{
    if (n <= 0)
        return cudaSuccess;
    if (M < 1 || M > kStreamMaxTokens || n > kStreamStackMax)
        return cudaErrorInvalidValue;
    if (n == 1)
        return launch_sized<1>(entries, n, M, overlap_prev, single, stream);
    if (n <= 16)
        return launch_sized<16>(entries, n, M, overlap_prev, single, stream);
    return launch_sized<kStreamStackMax>(entries, n, M, overlap_prev, single, stream);
}

}  // namespace tq
