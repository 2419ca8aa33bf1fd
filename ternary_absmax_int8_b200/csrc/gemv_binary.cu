// gemv_binary.cu -- decode GEMV over binary g128 weights (M <= 4 tokens), one
// projection or a table of projections per launch.
//
// The format (baguaai "BitNet" tag page, Bonsai 27B item: a true 1-bit
// binary scheme, 128 weights sharing one fp16 scale, about 1.125 bits per
// weight), as this library stores it:
//   bits   uint8 [N/8, K]: bit p of byte (i, k) is the weight of output row
//          i + p N/8 at column k, 1 meaning +1 and 0 meaning -1 (the plane
//          layout of the ternary format, eight planes instead of four);
//   scales fp16 [N/8, K/128, 8]: entry (i, g, p) scales row i + p N/8 on
//          columns 128 g .. 128 g + 127.
// With int8 activations q (per-token absmax) and x_scale:
//   S[n, g] = sum_{k in g} b[n, k] q[k],   Q[g] = sum_{k in g} q[k],
//   acc[n, g] = 2 S[n, g] - Q[g]  (since w = 2 b - 1; exact int32),
//   y[n] = fl32(x_scale * sum_g scale[n, g] acc[n, g]), the products exact in
//   fp64 (an int32 below 2^15 times an fp16) and the sum in fp64 (exact unless
//   a row's scales span more than ~2^20), so the order of the additions does
//   not change the result.
//
// The weight stream is read once per token and dominates the bytes, so the
// kernel streams like the ternary decode kernel: persistent CTAs, one per SM;
// tiles of R whole packed rows (their bits and their scales, two 1-D bulk
// copies through the TMA engine, no multicast) in a ring of shared-memory
// stages guarded by mbarriers; two groups of eight consumer warps take
// alternate tiles; the CTA's activations are resident in shared memory.
//
// Consumer arithmetic. A warp item is one packed row (or one of 2^lg pieces
// of its groups); lane (seg, sub) = (lane >> 2, lane & 3) takes two of the
// eight 16-byte chunks of groups g0 + seg, g0 + seg + 8, ... For a 32-bit
// word u of bits (four columns, eight planes per byte), dp4a of the nested
// masks u & 0x01.., u & 0x03.., ..., u & 0x7F.. and u itself (unsigned bytes
// x signed int8) gives the nested sums T_j = sum_{p <= j} 2^p S_p: seven
// logic ops and eight dp4a per word. A transposing butterfly over the
// segment's four lanes (six shuffles) leaves lane `sub` holding the group's
// T_{2 sub} and T_{2 sub + 1}; with T_{2 sub - 1} from its neighbour,
// S_p = (T_p - T_{p-1}) >> p. Each lane so owns planes 2 sub and 2 sub + 1
// of its row: it scales the group's acc in fp64 and adds, and after the row
// the eight segments' sums are added.
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <algorithm>
#include <vector>

#include <cuda_fp16.h>

#include "mma_common.cuh"
#include "tq_internal.h"

namespace tq {

namespace {

constexpr int kBinW = 8;                  // consumer warps per group
constexpr int kBinG = 2;                  // groups (take alternate tiles)
constexpr int kBinWC = kBinW * kBinG;     // consumer warps
constexpr int kBinMaxStages = 8;
constexpr int kBinMaxRows = 16;           // packed rows per tile
constexpr int kBinSplitRows = 4;          // rows per tile when rows are cut into pieces
constexpr int kBinTileBytes = 40960;      // bit bytes per tile, aim
constexpr int kBinGroup = 128;

struct BinStageDesc {
    int entry, row0, rows, pad_;
};

template <int MT>
struct BinTail {
    static constexpr int kDesc = kBinMaxStages * int(sizeof(BinStageDesc));
    static constexpr int kBars = 2 * kBinMaxStages + 1;
    static constexpr int kSlots = kBinMaxStages * kBinSplitRows * MT * 8;
    static constexpr int kCnt = kBinMaxStages * kBinSplitRows;
    static constexpr size_t bytes()
    {
        return kDesc + kBars * 8 + size_t(kSlots) * 8 + size_t(kSlots) * 4 + size_t(kCnt) * 4 + 64;
    }
};

// Eight int32 values per lane over the four lanes of a segment: on return
// lane `sub` holds the segment's totals of values 2 sub and 2 sub + 1 (six
// shuffles).
__device__ __forceinline__ int2 transpose_reduce8x4(const int32_t (&v)[8], int sub)
{
    const bool b1 = sub & 2, b0 = sub & 1;
    int32_t k[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int32_t keep = b1 ? v[4 + i] : v[i];
        const int32_t send = b1 ? v[i] : v[4 + i];
        k[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
    int32_t l[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int32_t keep = b0 ? k[2 + i] : k[i];
        const int32_t send = b0 ? k[i] : k[2 + i];
        l[i] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
    }
    return make_int2(l[0], l[1]);
}

// Nested-mask sums of one 16-byte chunk of bits against 16 activations.
__device__ __forceinline__ void dot_bits16(const uint4 w, const uint4 x, int32_t (&t)[8])
{
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
    const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        t[0] = dp4a_us(ws[j] & 0x01010101u, xs[j], t[0]);
        t[1] = dp4a_us(ws[j] & 0x03030303u, xs[j], t[1]);
        t[2] = dp4a_us(ws[j] & 0x07070707u, xs[j], t[2]);
        t[3] = dp4a_us(ws[j] & 0x0F0F0F0Fu, xs[j], t[3]);
        t[4] = dp4a_us(ws[j] & 0x1F1F1F1Fu, xs[j], t[4]);
        t[5] = dp4a_us(ws[j] & 0x3F3F3F3Fu, xs[j], t[5]);
        t[6] = dp4a_us(ws[j] & 0x7F7F7F7Fu, xs[j], t[6]);
        t[7] = dp4a_us(ws[j], xs[j], t[7]);
    }
}

template <int MaxE, int MT>
__global__ void __launch_bounds__((kBinWC + 1) * 32, 1)
binary_gemv_kernel(const __grid_constant__ BinParams<MaxE> p)
{
    extern __shared__ __align__(128) uint8_t smem[];
    const int t_begin = p.cta_tile0[blockIdx.x], t_end = p.cta_tile0[blockIdx.x + 1];
    const int e_first = p.cta_entry0[blockIdx.x];
    const int n_ent = p.cta_nent[blockIdx.x];
    BinEntry *tab = reinterpret_cast<BinEntry *>(smem);
    float *xsc = reinterpret_cast<float *>(tab + n_ent);  // [n_ent][MT]
    int *xoff = reinterpret_cast<int *>(xsc + n_ent * MT);
    int *qoff = xoff + n_ent;
    uint8_t *xcache = smem + p.head_bytes;
    int32_t *qsum = reinterpret_cast<int32_t *>(xcache + p.x_slot);
    uint8_t *ring = xcache + p.x_slot + p.q_slot;
    BinStageDesc *desc = reinterpret_cast<BinStageDesc *>(ring + size_t(p.stages) * p.w_slot);
    uint64_t *full = reinterpret_cast<uint64_t *>(desc + kBinMaxStages);
    uint64_t *empty = full + kBinMaxStages;
    uint64_t *xbar = empty + kBinMaxStages;
    double *dpart = reinterpret_cast<double *>(xbar + 1);
    int32_t *ipart = reinterpret_cast<int32_t *>(dpart + BinTail<MT>::kSlots);
    int32_t *cnt = ipart + BinTail<MT>::kSlots;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    for (int i = threadIdx.x; i < BinTail<MT>::kSlots; i += blockDim.x) {
        dpart[i] = 0.0;
        ipart[i] = 0;
    }
    for (int i = threadIdx.x; i < BinTail<MT>::kCnt; i += blockDim.x)
        cnt[i] = 0;
    {
        static_assert(sizeof(BinEntry) % 8 == 0, "entry size");
        const uint64_t *src = reinterpret_cast<const uint64_t *>(&p.e[e_first]);
        uint64_t *dst = reinterpret_cast<uint64_t *>(tab);
        const int n64 = n_ent * int(sizeof(BinEntry) / 8);
        for (int i = threadIdx.x; i < n64; i += blockDim.x)
            dst[i] = src[i];
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int xo = 0, qo = 0;
        for (int j = 0; j < n_ent; ++j) {
            xoff[j] = xo;
            qoff[j] = qo;
            xo += (p.M * tab[j].K + 127) & ~127;
            qo += p.M * (tab[j].K / kBinGroup);
        }
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kBinW);
        }
        mbar_init(xbar, 1);
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kBinWC) {
        // ------------------------------------------------------ producer
        if (lane != 0)
            return;
        const uint64_t pol_w = policy_evict_first();
        const uint64_t pol_x = policy_evict_last();
        if (t_end > t_begin) {
            uint32_t total = 0;
            for (int j = 0; j < n_ent; ++j)
                total += uint32_t(p.M * tab[j].K);
            mbar_arrive_expect_tx(xbar, total);
            for (int j = 0; j < n_ent; ++j)
                bulk_g2s(xcache + xoff[j], tab[j].xq, uint32_t(p.M * tab[j].K), xbar, pol_x);
        } else {
            mbar_arrive(xbar);
        }
        int cursor = 0, it = 0, stage = 0;
        uint32_t phase = 0;
        for (int t = t_begin; t < t_end; ++t, ++it) {
            while (cursor + 1 < n_ent && tab[cursor + 1].tile_begin <= t)
                ++cursor;
            const BinEntry &e = tab[cursor];
            const int K = e.K, ng = K / kBinGroup;
            const int row0 = (t - e.tile_begin) * e.rows_per_tile;
            const int rows = min(e.rows_per_tile, e.N8 - row0);
            if (it >= p.stages && !mbar_wait(&empty[stage], phase ^ 1u, p.err))
                break;
            const uint32_t bbytes = uint32_t(rows) * uint32_t(K);
            const uint32_t sbytes = uint32_t(rows) * uint32_t(ng) * 16u;
            desc[stage] = BinStageDesc{cursor, row0, rows, 0};
            uint8_t *dst = ring + size_t(stage) * p.w_slot;
            mbar_arrive_expect_tx(&full[stage], bbytes + sbytes);
            bulk_g2s(dst, e.bits + size_t(row0) * K, bbytes, &full[stage], pol_w);
            bulk_g2s(dst + size_t(e.rows_per_tile) * K, e.scales + size_t(row0) * ng * 8, sbytes,
                     &full[stage], pol_w);
            if (++stage == p.stages) {
                stage = 0;
                phase ^= 1u;
            }
        }
        // Do not retire while a copy this thread issued is in flight.
        for (int s = 0; s < p.stages; ++s) {
            if (s < stage)
                mbar_wait(&full[s], phase, p.err);
            else if (it >= p.stages)
                mbar_wait(&full[s], phase ^ 1u, p.err);
        }
        mbar_wait(xbar, 0, p.err);
        return;
    }

    // ---------------------------------------------------------- consumers
    if (t_end > t_begin && !mbar_wait_warp(xbar, 0, p.err))
        return;
    // Per token and group, Q[g] = sum of the group's 128 codes.
    for (int j = 0; j < n_ent; ++j) {
        const int K = tab[j].K, ng = K / kBinGroup;
        for (int i = threadIdx.x; i < p.M * ng; i += kBinWC * 32) {
            const int m = i / ng, g = i - m * ng;
            const uint4 *xv = reinterpret_cast<const uint4 *>(xcache + xoff[j] + m * K + g * kBinGroup);
            int32_t s = 0;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 v = xv[c];
                s = __dp4a(int(v.x), 0x01010101, s);
                s = __dp4a(int(v.y), 0x01010101, s);
                s = __dp4a(int(v.z), 0x01010101, s);
                s = __dp4a(int(v.w), 0x01010101, s);
            }
            qsum[qoff[j] + i] = s;
        }
        for (int m = threadIdx.x; m < p.M; m += kBinWC * 32)
            xsc[j * MT + m] = __ldg(tab[j].x_scale + m);
    }
    named_bar_sync(1, kBinWC * 32);

    const int grp = warp / kBinW, wg = warp - grp * kBinW;
    const int seg = lane >> 2, sub = lane & 3;
    int stage = grp;  // stages % kBinG == 0: the group keeps to stages grp + k G
    uint32_t phase = 0;
    int rot = 0;
    for (int t = t_begin + grp; t < t_end; t += kBinG) {
        if (!mbar_wait_warp(&full[stage], phase, p.err))
            return;
        const BinStageDesc d = desc[stage];
        const BinEntry &e = tab[d.entry];
        const int K = e.K, ng = K / kBinGroup, N8 = e.N8;
        const int lg = e.lg;
        const uint8_t *sb = ring + size_t(stage) * p.w_slot;
        const __half *ss = reinterpret_cast<const __half *>(sb + size_t(e.rows_per_tile) * K);
        const uint8_t *sx = xcache + xoff[d.entry];
        const int32_t *sq = qsum + qoff[d.entry];
        float xs[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m)
            xs[m] = m < p.M ? xsc[d.entry * MT + m] : 0.0f;

        const int n_items = d.rows << lg;
        bool released = false;
        const int first_item = (wg - rot + kBinW) % kBinW;
        const int last_item = n_items - 1 - ((n_items - 1 - first_item) % kBinW + kBinW) % kBinW;
        rot = (rot + n_items) % kBinW;
        for (int item = first_item; item < n_items; item += kBinW) {
            const int r = item >> lg, piece = item & ((1 << lg) - 1);
            const int g0 = (piece * ng) >> lg, g1 = ((piece + 1) * ng) >> lg;
            const uint8_t *wrow = sb + size_t(r) * K;
            // planes 2 sub and 2 sub + 1 of this lane's segment groups
            double accd[MT][2];
            int32_t itot[MT][2];
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                accd[m][0] = accd[m][1] = 0.0;
                itot[m][0] = itot[m][1] = 0;
            }
            // The lane's two chunks of a group, rotated by segment so that a
            // warp's 16-byte reads hit each bank slot four times (the
            // minimum of four wavefronts per 512 bytes).
            const int c0 = (2 * sub + seg) & 7, c1 = c0 ^ 1;
            for (int gb = g0; gb < g1; gb += 8) {
                const int g = gb + seg;
                const bool valid = g < g1;
                int32_t tt[MT][8];
#pragma unroll
                for (int m = 0; m < MT; ++m)
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        tt[m][j] = 0;
                if (valid) {
                    const uint8_t *wg = wrow + g * kBinGroup;
                    const uint4 w0 = *reinterpret_cast<const uint4 *>(wg + c0 * 16);
                    const uint4 w1 = *reinterpret_cast<const uint4 *>(wg + c1 * 16);
#pragma unroll
                    for (int m = 0; m < MT; ++m)
                        if (MT == 1 || m < p.M) {
                            const uint8_t *xg = sx + m * K + g * kBinGroup;
                            dot_bits16(w0, *reinterpret_cast<const uint4 *>(xg + c0 * 16), tt[m]);
                            dot_bits16(w1, *reinterpret_cast<const uint4 *>(xg + c1 * 16), tt[m]);
                        }
                }
                // the fp16 scales of planes 2 sub, 2 sub + 1 (one 32-bit word)
                const __half2 sc2 = valid ? *reinterpret_cast<const __half2 *>(
                                                ss + (r * ng + g) * 8 + 2 * sub)
                                          : __float2half2_rn(0.0f);
                const float2 scf = __half22float2(sc2);
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (MT == 1 || m < p.M) {
                        const int2 t = transpose_reduce8x4(tt[m], sub);  // T_{2sub}, T_{2sub+1}
                        int32_t tprev = __shfl_up_sync(0xffffffffu, t.y, 1, 4);  // T_{2sub-1}
                        if (sub == 0)
                            tprev = 0;
                        if (valid) {
                            // exact: each difference is a multiple of 2^plane
                            const int32_t s_lo = (t.x - tprev) >> (2 * sub);
                            const int32_t s_hi = (t.y - t.x) >> (2 * sub + 1);
                            const int32_t q = sq[m * ng + g];
                            const int32_t a_lo = 2 * s_lo - q, a_hi = 2 * s_hi - q;
                            itot[m][0] += a_lo;
                            itot[m][1] += a_hi;
                            accd[m][0] = __dadd_rn(accd[m][0], __dmul_rn(double(a_lo), double(scf.x)));
                            accd[m][1] = __dadd_rn(accd[m][1], __dmul_rn(double(a_hi), double(scf.y)));
                        }
                    }
                }
            }
            if (lg == 0 && item == last_item) {
                // last read of the stage by this warp (split rows still
                // read nothing more from it either, but keep their slots)
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&empty[stage]);
                released = true;
            }
            // add the eight segments' sums: lane sub of every segment then
            // holds planes 2 sub and 2 sub + 1 of the row
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (MT == 1 || m < p.M) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
#pragma unroll
                        for (int o = 4; o < 32; o <<= 1) {
                            accd[m][h] = __dadd_rn(accd[m][h],
                                                   __shfl_xor_sync(0xffffffffu, accd[m][h], o));
                            itot[m][h] += __shfl_xor_sync(0xffffffffu, itot[m][h], o);
                        }
                    }
                }
            }
            const int row = d.row0 + r;
            if (lg == 0) {
                if (seg == 0) {
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        if (MT == 1 || m < p.M) {
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                const size_t o = size_t(m) * (8 * size_t(N8)) + size_t(row) +
                                                 size_t(2 * sub + h) * N8;
                                e.y[o] = __double2float_rn(__dmul_rn(accd[m][h], double(xs[m])));
                                if (e.acc_out)
                                    e.acc_out[o] = itot[m][h];
                            }
                        }
                    }
                }
            } else {
                const int slot = (stage * kBinSplitRows + r) * MT;
                if (seg == 0) {
#pragma unroll
                    for (int m = 0; m < MT; ++m)
                        if (MT == 1 || m < p.M)
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                atomicAdd(&dpart[(slot + m) * 8 + 2 * sub + h], accd[m][h]);
                                atomicAdd(&ipart[(slot + m) * 8 + 2 * sub + h], itot[m][h]);
                            }
                }
                __threadfence_block();  // partial sums before the count
                __syncwarp();
                int old = 0;
                if (lane == 0)
                    old = atomicAdd(&cnt[stage * kBinSplitRows + r], 1);
                old = __shfl_sync(0xffffffffu, old, 0);
                if (old == (1 << lg) - 1) {
                    // the last piece of this row: finish it
                    __threadfence_block();
                    if (lane < 8) {  // lane = plane
#pragma unroll
                        for (int m = 0; m < MT; ++m) {
                            if (MT == 1 || m < p.M) {
                                volatile double *dv = dpart + (slot + m) * 8 + lane;
                                const double v = *dv;
                                *dv = 0.0;
                                const int32_t iv = atomicExch(&ipart[(slot + m) * 8 + lane], 0);
                                const size_t o = size_t(m) * (8 * size_t(N8)) + size_t(row) +
                                                 size_t(lane) * N8;
                                e.y[o] = __double2float_rn(__dmul_rn(v, double(xs[m])));
                                if (e.acc_out)
                                    e.acc_out[o] = iv;
                            }
                        }
                    }
                    __syncwarp();
                    if (lane == 0)
                        cnt[stage * kBinSplitRows + r] = 0;
                }
            }
        }
        __syncwarp();
        if (lane == 0 && !released)
            mbar_arrive(&empty[stage]);
        stage += kBinG;
        if (stage >= p.stages) {
            stage -= p.stages;
            phase ^= 1u;
        }
    }
}

template <int MaxE, int MT>
cudaError_t launch_bin_instance(const BinParams<MaxE> &p, int grid, size_t smem,
                                cudaStream_t stream)
{
    auto kern = binary_gemv_kernel<MaxE, MT>;
    static std::atomic<int> configured_dev{-1};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess)
        return err;
    if (configured_dev != dev) {
        err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (err != cudaSuccess)
            return err;
        configured_dev = dev;
    }
    kern<<<grid, (kBinWC + 1) * 32, smem, stream>>>(p);
    return cudaGetLastError();
}

template <int MaxE>
cudaError_t launch_bin_sized(BinEntry *entries, int n, int M, cudaStream_t stream)
{
    BinParams<MaxE> p;
    static_assert(sizeof(BinParams<MaxE>) <= 32000, "kernel parameters exceed 32 KB");
    const int sms = std::min(device_sm_count(), kBinMaxGrid);
    const int mt = M == 1 ? 1 : (M == 2 ? 2 : 4);
    int total = 0;
    size_t w_slot = 0;
    for (int j = 0; j < n; ++j) {
        BinEntry &e = entries[j];
        const int K = e.K, ng = K / kBinGroup;
        int R = kBinMaxRows;
        while (R > 1 && R * K > kBinTileBytes)
            R >>= 1;
        // Cut rows into pieces of their groups when a tile has fewer rows
        // than a group has warps (at least four groups per piece).
        int lg = 0;
        while ((R << lg) < kBinW && (ng >> (lg + 1)) >= 4)
            ++lg;
        if (lg > 0 && R > kBinSplitRows)
            return cudaErrorInvalidValue;  // not reached: lg > 0 only when R < kBinW / 2
        e.rows_per_tile = R;
        e.lg = lg;
        e.tile_begin = total;
        total += (e.N8 + R - 1) / R;
        w_slot = std::max(w_slot, (size_t(R) * K + 127) / 128 * 128 +
                                      (size_t(R) * ng * 16 + 127) / 128 * 128);
        p.e[j] = e;
    }
    if (total == 0)
        return cudaSuccess;
    p.n_entries = n;
    p.total_tiles = total;
    p.M = M;
    p.w_slot = int(w_slot);
    const int grid = std::min(total, sms);
    // contiguous tile ranges per CTA, balanced by bytes (plus a fixed cost per tile)
    std::vector<long long> prefix(size_t(total) + 1, 0);
    {
        int t = 0;
        for (int j = 0; j < n; ++j) {
            const BinEntry &e = p.e[j];
            const int tiles = (e.N8 + e.rows_per_tile - 1) / e.rows_per_tile;
            for (int i = 0; i < tiles; ++i, ++t) {
                const int rows = std::min(e.rows_per_tile, e.N8 - i * e.rows_per_tile);
                prefix[size_t(t) + 1] = prefix[size_t(t)] + (long long)rows * e.K * 9 / 8 + 4096;
            }
        }
    }
    p.cta_tile0[0] = 0;
    for (int b = 1; b < grid; ++b) {
        const long long target = prefix[size_t(total)] * b / grid;
        int t = int(std::lower_bound(prefix.begin(), prefix.end(), target) - prefix.begin());
        t = std::max(t, p.cta_tile0[b - 1] + 1);
        t = std::min(t, total - (grid - b));
        p.cta_tile0[b] = t;
    }
    p.cta_tile0[grid] = total;
    int max_local = 1;
    size_t x_max = 0, q_max = 0;
    for (int b = 0; b < grid; ++b) {
        auto entry_of = [&](int t) {
            int lo = 0, hi = n - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) / 2;
                if (p.e[mid].tile_begin <= t)
                    lo = mid;
                else
                    hi = mid - 1;
            }
            return lo;
        };
        const int e0 = entry_of(p.cta_tile0[b]);
        const int e1 = entry_of(p.cta_tile0[b + 1] - 1);
        p.cta_entry0[b] = e0;
        p.cta_nent[b] = e1 - e0 + 1;
        max_local = std::max(max_local, e1 - e0 + 1);
        size_t xb = 0, qb = 0;
        for (int j = e0; j <= e1; ++j) {
            xb += (size_t(M) * p.e[j].K + 127) / 128 * 128;
            qb += size_t(M) * (p.e[j].K / kBinGroup) * 4;
        }
        x_max = std::max(x_max, xb);
        q_max = std::max(q_max, qb);
    }
    p.x_slot = int(x_max);
    p.q_slot = int((q_max + 127) / 128 * 128);
    p.head_bytes = int((size_t(max_local) * (sizeof(BinEntry) + size_t(mt) * 4 + 8) + 127) / 128 * 128);
    p.err = device_error_word();
    if (!p.err)
        return cudaErrorUnknown;
    const size_t tail = mt == 1 ? BinTail<1>::bytes()
                                : (mt == 2 ? BinTail<2>::bytes() : BinTail<4>::bytes());
    const size_t fixed = size_t(p.head_bytes) + p.x_slot + p.q_slot + tail;
    const size_t budget = 227 * 1024;
    int stages = budget > fixed ? int((budget - fixed) / w_slot) : 0;
    stages = std::min(stages, kBinMaxStages);
    // each consumer group must see every phase of the stages it uses
    stages -= stages % kBinG;
    if (stages < kBinG)
        return cudaErrorInvalidValue;
    p.stages = stages;
    const size_t smem = fixed + size_t(stages) * w_slot;
    switch (mt) {
    case 1: return launch_bin_instance<MaxE, 1>(p, grid, smem, stream);
    case 2: return launch_bin_instance<MaxE, 2>(p, grid, smem, stream);
    default: return launch_bin_instance<MaxE, 4>(p, grid, smem, stream);
    }
}

// ------------------------------------------------------------------------
// One token (M = 1) on the warp-level integer MMA. A byte of bits holds the
// eight planes of one column, so with the nested masks 0x01.., 0x03.., ...,
// 0x7F.. and 0xFF.. (unsigned bytes) an m16n8k32 MMA on 16 packed rows x 32
// columns gives D_j = sum_{p <= j} 2^p S_p for all 16 rows at once: eight
// MMAs and 28 logic ops per 32-column block, against 64 dp4a per lane. A
// lane's A fragment comes from 16 contiguous bytes of each of its rows (the
// column permutation of the ternary warp-MMA kernel, shared with the
// activations), streamed by cp.async into per-warp rings together with the
// 16 rows' fp16 scales of the group (so that their HBM latency is hidden as
// deep as the bits').
// A step is one 128-column group: each mask's chain of four MMAs starts from
// zero, and every column of the B fragment carries the token's codes, so the
// accumulators of all four lanes of a quad hold the group's nested sums T_j
// of rows g and g + 8. Lane t takes planes 2t and 2t + 1 -- all four lanes
// share the per-group scaling --: S_p = (T_p - T_{p-1}) >> p,
// acc = 2 S - Q_g, and the lane adds acc times the plane's fp16 scale in fp64
// (exact).
// Tiles of 16 packed rows (128 outputs) x the full K, contiguous ranges per
// CTA (16 warps, one per SM); teams of P warps split a tile's groups when
// tiles are few and add their fp64 and int32 partials in shared memory (exact,
// order-free).
constexpr int kBmW = 20;                      // warps per CTA (96 registers each)
constexpr int kBmThreads = kBmW * 32;
constexpr int kBmRing = 4;                    // stages per warp (a power of two)
constexpr int kBmBits = 2 * 2 * 32 * 16;      // [2 rows][2 halves][32 lanes][16 B]
constexpr int kBmScales = 16 * 16;            // then the scales: [16 rows][8 planes] fp16
constexpr int kBmStage = kBmBits + kBmScales + kBinGroup;  // then the group's 128 codes
constexpr int kBmRows = 16;

struct BmCursor {
    int tile, entry, step, step_end;
    int K, G;
    const uint8_t *row, *row8;  // the lane's rows g and g + 8 at column 16 t
    // lanes t = 0, 1: the scales of row g + 8 t ([group][8] fp16); t = 2: the
    // token's codes at column 16 g; advanced by `aux_step` bytes per group
    const uint8_t *aux;
    int aux_step;
    bool ok0, ok1, aux_ok;
};

struct BmWalk {
    const BinMmaEntry *tab;
    int n_ent, t_end, teams, piece, lgP, g, t;

    __device__ void start(BmCursor &c, int tl) const
    {
        c.tile = tl;
        while (c.entry + 1 < n_ent && tab[c.entry + 1].tile_begin <= tl)
            ++c.entry;
        const BinMmaEntry &e = tab[c.entry];
        c.K = e.K;
        c.G = e.K / kBinGroup;
        c.step = (c.G * piece) >> lgP;
        c.step_end = (c.G * (piece + 1)) >> lgP;
        const int r = (tl - e.tile_begin) * kBmRows + g;
        c.ok0 = r < e.N8;
        c.ok1 = r + 8 < e.N8;
        c.row = e.bits + size_t(c.ok0 ? r : 0) * e.K + 16 * t;
        // row g + 8 past the end: zero-size copies from row g's address
        c.row8 = c.ok1 ? c.row + size_t(8) * e.K : c.row;
        const int rs = t == 1 && c.ok1 ? r + 8 : (c.ok0 ? r : 0);
        if (t < 2) {
            c.aux = reinterpret_cast<const uint8_t *>(e.scales + size_t(rs) * c.G * 8);
            c.aux_step = 16;
            c.aux_ok = t == 0 ? c.ok0 : c.ok1;
        } else {
            c.aux = reinterpret_cast<const uint8_t *>(e.xq) + 16 * g;
            c.aux_step = kBinGroup;
            c.aux_ok = true;
        }
    }
    __device__ void settle(BmCursor &c) const
    {
        while (c.tile < t_end && c.step >= c.step_end) {
            if (c.tile + teams >= t_end) {
                c.tile = t_end;
                break;
            }
            start(c, c.tile + teams);
        }
    }
};

__global__ void __launch_bounds__(kBmThreads, 1)
binary_mma_kernel(const __grid_constant__ BinMmaParams p)
{
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr int kRingBytes = kBmRing * kBmStage;
    double *dslot = reinterpret_cast<double *>(smem + kBmW * kRingBytes);  // [W][16 rows][8]
    int32_t *islot = reinterpret_cast<int32_t *>(dslot + kBmW * 16 * 8);   // [W][16][8]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const uint8_t *ring = smem + warp * kRingBytes + lane * 16;
    const uint32_t ring_s = smem_u32(ring);

    const int t_begin = p.cta_tile0[blockIdx.x], t_end = p.cta_tile0[blockIdx.x + 1];
    const int lgP = p.lgP, P = 1 << lgP, teams = kBmW >> lgP;
    // teams of P warps; warps past the last whole team (kBmW not a multiple
    // of P) stay idle
    const int team = warp >> lgP, piece = warp & (P - 1);
    const int first = team < teams ? t_begin + team : t_end;
    const BmWalk wk{p.e, p.n_entries, t_end, teams, piece, lgP, g, t};

    BmCursor lc{t_end, 0, 0, 0, 0, 0, nullptr, nullptr, nullptr, 0, false, false, false};
    if (first < t_end) {
        wk.start(lc, first);
        wk.settle(lc);
    }
    int issued = 0;
    // this lane's copy target past the bits: a scale row (t < 2) or 16 codes (t = 2)
    const uint32_t sc_s = smem_u32(smem + warp * kRingBytes + kBmBits) +
                          uint32_t(t < 2 ? (g + 8 * t) * 16 : kBmScales + 16 * g);
    auto issue = [&]() {
        const uint32_t dst = ring_s + uint32_t(issued & (kBmRing - 1)) * kBmStage;
        __syncwarp();  // the slot's scales were last read by other lanes
        if (lc.tile < t_end) {
            const int k = lc.step * kBinGroup;
            cp_async16(dst, lc.row + k, lc.ok0);
            cp_async16(dst + 512, lc.row + k + 64, lc.ok0);
            cp_async16(dst + 1024, lc.row8 + k, lc.ok1);
            cp_async16(dst + 1536, lc.row8 + k + 64, lc.ok1);
            // lanes t = 0, 1: the 8 scales of row g + 8 t at this group;
            // lanes t = 2: codes 16 g .. 16 g + 15 of the group
            if (t < 3)
                cp_async16(sc_s + uint32_t(issued & (kBmRing - 1)) * kBmStage,
                           lc.aux + lc.step * lc.aux_step, lc.aux_ok);
            ++lc.step;
            wk.settle(lc);
        }
        cp_async_commit();
        ++issued;
    };
#pragma unroll
    for (int i = 0; i < kBmRing - 1; ++i)
        issue();


    double acc[2][2] = {{0.0, 0.0}, {0.0, 0.0}};  // [row g / g + 8][plane 2t / 2t + 1]
    int32_t tot[2][2] = {{0, 0}, {0, 0}};
    int consumed = 0;
    int fent = 0;
    while (fent + 1 < p.n_entries && p.e[fent + 1].tile_begin <= t_begin)
        ++fent;

    // One 128-column group from a ring stage into the lane's accumulators.
    auto group = [&](const uint8_t *stage) {
        // the token's codes for the lane's 16 + 16 columns of the group; every
        // B column carries them (lane (g, t) supplies column g), so that all
        // four lanes of a quad receive the row's sums
        const uint4 q0 = *reinterpret_cast<const uint4 *>(stage + kBmBits + kBmScales + 16 * t);
        const uint4 q1 =
            *reinterpret_cast<const uint4 *>(stage + kBmBits + kBmScales + 64 + 16 * t);
        // the group's code sum
        int32_t qs = 0;
        qs = __dp4a(int(q0.x), 0x01010101, qs);
        qs = __dp4a(int(q0.y), 0x01010101, qs);
        qs = __dp4a(int(q0.z), 0x01010101, qs);
        qs = __dp4a(int(q0.w), 0x01010101, qs);
        qs = __dp4a(int(q1.x), 0x01010101, qs);
        qs = __dp4a(int(q1.y), 0x01010101, qs);
        qs = __dp4a(int(q1.z), 0x01010101, qs);
        qs = __dp4a(int(q1.w), 0x01010101, qs);
        qs += __shfl_xor_sync(0xffffffffu, qs, 1);
        const int32_t Q = qs + __shfl_xor_sync(0xffffffffu, qs, 2);

        const uint8_t *src = stage + lane * 16;
        // planes 2 t, 2 t + 1 of rows g and g + 8 (zero past the end)
        const uint8_t *ssc = stage + kBmBits + g * 16 + 4 * t;
        const float2 s0 = __half22float2(*reinterpret_cast<const __half2 *>(ssc));
        const float2 s1 = __half22float2(*reinterpret_cast<const __half2 *>(ssc + 128));
        int32_t d[8][4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint4 lo4 = *reinterpret_cast<const uint4 *>(src + h * 512);         // row g
            const uint4 hi4 = *reinterpret_cast<const uint4 *>(src + 1024 + h * 512);  // row g + 8
            const uint4 qq = h == 0 ? q0 : q1;
            const uint32_t al[4] = {lo4.x, lo4.y, lo4.z, lo4.w};
            const uint32_t ah[4] = {hi4.x, hi4.y, hi4.z, hi4.w};
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                const uint32_t a0 = al[2 * b], a2 = al[2 * b + 1];
                const uint32_t a1 = ah[2 * b], a3 = ah[2 * b + 1];
                const uint32_t b0 = b == 0 ? qq.x : qq.z, b1 = b == 0 ? qq.y : qq.w;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    // j = 6: the raw bytes as signed, T_6 - 128 S_7 (with the
                    // unsigned T_6 + 128 S_7 of j = 7 it gives T_6, no mask)
                    const uint32_t mk = j >= 6 ? 0xFFFFFFFFu : 0x01010101u * ((2u << j) - 1u);
                    if (j == 6) {
                        if (h == 0 && b == 0)
                            mma_s8s8_z(d[j], a0, a1, a2, a3, b0, b1);
                        else
                            mma_s8s8(d[j], a0, a1, a2, a3, b0, b1);
                    } else if (h == 0 && b == 0) {
                        mma_u8s8_z(d[j], a0 & mk, a1 & mk, a2 & mk, a3 & mk, b0, b1);
                    } else {
                        mma_u8s8(d[j], a0 & mk, a1 & mk, a2 & mk, a3 & mk, b0, b1);
                    }
                }
            }
        }
        // the group's nested sums of rows g (fragment word 0) and g + 8
        // (word 2), the same in every lane of the quad: lane t takes
        // T_{2t-1}, T_{2t}, T_{2t+1}
        const bool b1 = t & 2, b0 = t & 1;
#pragma unroll
        for (int rs = 0; rs < 2; ++rs) {
            const int w = 2 * rs;
            const int32_t t6 = (d[7][w] + d[6][w]) >> 1;
            const int32_t t_lo = b1 ? (b0 ? t6 : d[4][w]) : (b0 ? d[2][w] : d[0][w]);
            const int32_t t_hi = b1 ? (b0 ? d[7][w] : d[5][w]) : (b0 ? d[3][w] : d[1][w]);
            const int32_t t_pr = b1 ? (b0 ? d[5][w] : d[3][w]) : (b0 ? d[1][w] : 0);
            const int32_t a_lo = 2 * ((t_lo - t_pr) >> (2 * t)) - Q;
            const int32_t a_hi = 2 * ((t_hi - t_lo) >> (2 * t + 1)) - Q;
            const float2 sc = rs == 0 ? s0 : s1;
            // the products are exact in fp64 (15-bit integer x 11-bit
            // significand), so one fused multiply-add rounds as the add alone
            acc[rs][0] = __fma_rn(double(a_lo), double(sc.x), acc[rs][0]);
            acc[rs][1] = __fma_rn(double(a_hi), double(sc.y), acc[rs][1]);
            tot[rs][0] += a_lo;
            tot[rs][1] += a_hi;
        }
    };

    for (int tile = first; tile < t_end; tile += teams) {
        while (fent + 1 < p.n_entries && p.e[fent + 1].tile_begin <= tile)
            ++fent;
        const BinMmaEntry &e = p.e[fent];
        // this warp's share of the tile's groups (a contiguous piece, possibly empty)
        const int G = e.K / kBinGroup;
        const int n_steps = ((G * (piece + 1)) >> lgP) - ((G * piece) >> lgP);
        for (int st = 0; st < n_steps; ++st) {
            issue();
            cp_async_wait<kBmRing - 1>();
            __syncwarp();
            group(smem + warp * kRingBytes + (consumed & (kBmRing - 1)) * kBmStage);
            ++consumed;
        }
        const int r0 = (tile - e.tile_begin) * kBmRows;
        const float xs = __ldg(e.x_scale);
        if (P == 1) {
#pragma unroll
            for (int rs = 0; rs < 2; ++rs) {
                const int row = r0 + g + 8 * rs;
                if (row < e.N8) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const size_t o = size_t(row) + size_t(2 * t + h) * e.N8;
                        e.y[o] = __double2float_rn(__dmul_rn(acc[rs][h], double(xs)));
                        if (e.acc_out)
                            e.acc_out[o] = tot[rs][h];
                    }
                }
            }
        } else {
            // the team adds its partials: slot [warp][row][plane]
            double *dm = dslot + warp * 128;
            int32_t *im = islot + warp * 128;
#pragma unroll
            for (int rs = 0; rs < 2; ++rs)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    dm[(g + 8 * rs) * 8 + 2 * t + h] = acc[rs][h];
                    im[(g + 8 * rs) * 8 + 2 * t + h] = tot[rs][h];
                }
            named_bar_sync(1 + team, 32 * P);
            const double *td = dslot + team * P * 128;
            const int32_t *ti = islot + team * P * 128;
            for (int o = piece * 32 + lane; o < 128; o += 32 * P) {
                const int row = r0 + (o >> 3), pl = o & 7;
                double a = 0.0;
                int32_t s = 0;
                for (int w = 0; w < P; ++w) {
                    a = __dadd_rn(a, td[w * 128 + o]);
                    s += ti[w * 128 + o];
                }
                if (row < e.N8) {
                    const size_t out = size_t(row) + size_t(pl) * e.N8;
                    e.y[out] = __double2float_rn(__dmul_rn(a, double(xs)));
                    if (e.acc_out)
                        e.acc_out[out] = s;
                }
            }
            named_bar_sync(1 + team, 32 * P);  // the slots are rewritten by the next tile
        }
#pragma unroll
        for (int rs = 0; rs < 2; ++rs)
            acc[rs][0] = acc[rs][1] = 0.0, tot[rs][0] = tot[rs][1] = 0;
    }
    cp_async_wait<0>();
}

BinMmaParams *bin_mma_params()
{
    static thread_local BinMmaParams p;
    return &p;
}

cudaError_t launch_binary_mma(const BinEntry *entries, int n, cudaStream_t stream)
{
    const int sms = device_sm_count();
    constexpr size_t smem = size_t(kBmW) * kBmRing * kBmStage + size_t(kBmW) * 128 * (8 + 4);
    static std::atomic<int> configured_dev{-1};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess)
        return err;
    if (configured_dev != dev) {
        err = cudaFuncSetAttribute(binary_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   int(smem));
        if (err != cudaSuccess)
            return err;
        configured_dev = dev;
    }
    for (int base = 0; base < n; base += kBinStackMax) {
        const int cnt = std::min(n - base, kBinStackMax);
        BinMmaParams &p = *bin_mma_params();
        p.n_entries = cnt;
        int total = 0;
        for (int j = 0; j < cnt; ++j) {
            const BinEntry &b = entries[base + j];
            p.e[j] = BinMmaEntry{b.bits, b.scales, b.xq, b.x_scale, b.y, b.acc_out, b.N8, b.K,
                                 total, 0};
            total += (b.N8 + kBmRows - 1) / kBmRows;
        }
        if (total == 0)
            continue;
        const int grid = std::min({total, sms, kMmaMaxGrid});
        int lgP = 0;
        while ((2 << lgP) <= kBmW && (long long)total << lgP < 2LL * kBmW * grid)
            ++lgP;
        p.lgP = lgP;
        std::vector<long long> prefix(size_t(total) + 1, 0);
        {
            int tt = 0;
            for (int j = 0; j < cnt; ++j) {
                const BinMmaEntry &e = p.e[j];
                const int tiles = (e.N8 + kBmRows - 1) / kBmRows;
                for (int i = 0; i < tiles; ++i, ++tt)
                    prefix[size_t(tt) + 1] =
                        prefix[size_t(tt)] + (long long)kBmRows * e.K * 9 / 8 + 2048;
            }
        }
        p.cta_tile0[0] = 0;
        for (int b = 1; b < grid; ++b) {
            const long long target = prefix[size_t(total)] * b / grid;
            int tt = int(std::lower_bound(prefix.begin(), prefix.end(), target) - prefix.begin());
            tt = std::max(tt, p.cta_tile0[b - 1] + 1);
            tt = std::min(tt, total - (grid - b));
            p.cta_tile0[b] = tt;
        }
        p.cta_tile0[grid] = total;
        binary_mma_kernel<<<grid, kBmThreads, smem, stream>>>(p);
        err = cudaGetLastError();
        if (err != cudaSuccess)
            return err;
    }
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_binary_gemv(BinEntry *entries, int n, int M, cudaStream_t stream)
{
    if (n <= 0)
        return cudaSuccess;
    if (M < 1 || M > kBinMaxTokens || n > kBinStackMax)
        return cudaErrorInvalidValue;
    // TQ_BINARY_KERNEL=dp4a runs one token on the dp4a kernel too (for measurement)
    static const bool force_dp4a = [] {
        const char *v = getenv("TQ_BINARY_KERNEL");
        return v && !strcmp(v, "dp4a");
    }();
    if (M == 1 && !force_dp4a)
        return launch_binary_mma(entries, n, stream);
    if (n == 1)
        return launch_bin_sized<1>(entries, n, M, stream);
    return launch_bin_sized<kBinStackMax>(entries, n, M, stream);
}

}  // namespace tq
