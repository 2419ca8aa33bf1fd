// gemv_stream.cu -- the decode-shaped ternary GEMV (M <= 4 tokens per launch),
// for one projection or for a whole stack of projections in one launch.
//
// Decode reads every weight byte once per token, so this kernel is bound by
// HBM bandwidth (1bit engine blog, "Qwen3.8-27B at 45.7 tok/s ...": decode
// speed is set by the bytes read per token; 1bit.systems README, "honest
// numbers": their HIP ternary GEMV at 92% of memory-bandwidth peak on
// gfx1151). Design for sm_100a:
//
//  * Persistent CTAs, one per SM, each a producer warp plus G groups of W
//    consumer warps.
//  * The packed weights of a projection, uint8 [N/4, K] row-major, are cut
//    into tiles of R consecutive packed rows: one contiguous R*K-byte range,
//    moved by a single 1-D bulk copy (TMA engine, cp.async.bulk, no
//    multicast) into a ring of shared-memory stages guarded by mbarriers.
//    Tiles of all projections of a launch form one sequence, cut into one
//    contiguous, byte-balanced range per CTA, so a stack of projections is
//    streamed back to back with no drain in between. Group g consumes the
//    CTA's tiles g, g + G, ...
//  * The int8 activations of the CTA's projections are copied once into a
//    resident shared-memory cache.
//  * Consumers read 16-byte words of packed weights and activations from
//    shared memory. A 32-bit word u holds, for output row i + p*N/4 (p =
//    0..3), the codes of 4 consecutive k in its bytes' bit fields 2p..2p+1.
//    Four dp4a (unsigned codes x signed int8) on nested masks of u give
//    nested sums from which 4^p * sum_k c*q follows by differences; the 4^p
//    is removed once per output.
//  * Since w = c - 1, acc = sum c*q - sum q = acc' - x_sum (x_sum comes from
//    the quantiser), so no per-element subtraction is needed either.
//  * A butterfly over the lanes of a row (8, 16 or 32) reduces the four
//    partial sums per token; the epilogue writes y = float(acc) * (w_scale *
//    x_scale). Single-projection launches may cut rows along K over several
//    warps, which then add into shared memory with integer atomics (exact,
//    order-free) and the last warp finishes the row.
//  * Every mbarrier wait is bounded (2 s of global time); on a timeout the
//    kernel records an error bit and winds down, the producer first waiting
//    (bounded) for its copies in flight.
#include <atomic>
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "quant_core.cuh"
#include "tq_internal.h"

namespace tq {

namespace {

constexpr int kMaxStages = 8;

constexpr int kWTargetBytes = 40960;  // weight bytes per tile, aim (default)

// Dynamic shared memory a CTA may use when `cps` CTAs share an SM (228 KB per
// SM, 1 KB of it reserved per CTA).
constexpr size_t smem_budget(int cps) { return cps == 1 ? 227 * 1024 : 112 * 1024; }

// Accumulators of one token: a[e][slot]. With u a packed word, byte b of u
// is c0 + 4 c1 + 16 c2 + 64 c3 (the four planes' codes at column k + b), so
// one dp4a each on u & 0x03030303, u & 0x0F0F0F0F, u & 0x3F3F3F3F and u
// itself (unsigned codes x signed int8) gives the nested sums
//   E0 = P0, E1 = P0 + 4 P1, E2 = P0 + 4 P1 + 16 P2, E3 = E2 + 64 P3,
// with P_p = sum_k c_p q. Differences recover 4^p P_p exactly (fold). Three
// logic ops and four dp4a per word; both share one half-rate pipe on sm_100,
// so the fourth mask saved is 1/8 of the inner loop. Word j of a 16-byte
// chunk goes to slot j % J, so each chunk feeds 4*J independent dp4a chains
// (J = 4 for one token, fewer when several tokens already give independent
// chains).
template <int J>
__device__ __forceinline__ void dot16(const uint4 w, const uint4 x, int32_t (&a)[4][J])
{
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
    const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int s = j % J;
        a[0][s] = dp4a_us(ws[j] & 0x03030303u, xs[j], a[0][s]);
        a[1][s] = dp4a_us(ws[j] & 0x0F0F0F0Fu, xs[j], a[1][s]);
        a[2][s] = dp4a_us(ws[j] & 0x3F3F3F3Fu, xs[j], a[2][s]);
        a[3][s] = dp4a_us(ws[j], xs[j], a[3][s]);
    }
}

// Sum the slots and turn the nested sums into out[p] = 4^p * P_p.
template <int J>
__device__ __forceinline__ void fold(const int32_t (&a)[4][J], int32_t (&out)[4])
{
    int32_t e[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        int32_t v = a[p][0];
#pragma unroll
        for (int s = 1; s < J; ++s)
            v += a[p][s];
        e[p] = v;
    }
    out[0] = e[0];
    out[1] = e[1] - e[0];
    out[2] = e[2] - e[1];
    out[3] = e[3] - e[2];
}

// What the producer tells the consumers about the tile in a stage.
struct StageDesc {
    int entry;  // index into the entry table
    int row0;   // first packed row of the tile
    int rows;   // packed rows in the tile
    int x_off;  // byte offset of the tile's activations inside the stage
};

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

// reduce4 within each 16-lane half of the warp: lane (half, sub) returns the
// half's total of value (sub >> 2) & 3. Five shuffles serve both halves.
__device__ __forceinline__ int32_t reduce4_half(const int32_t (&v)[4], int sub)
{
    const bool hi = sub & 8;
    int32_t k0 = hi ? v[2] : v[0], k1 = hi ? v[3] : v[1];
    const int32_t s0 = hi ? v[0] : v[2], s1 = hi ? v[1] : v[3];
    k0 += __shfl_xor_sync(0xffffffffu, s0, 8);
    k1 += __shfl_xor_sync(0xffffffffu, s1, 8);
    const bool b2 = sub & 4;
    int32_t c = b2 ? k1 : k0;
    const int32_t d = b2 ? k0 : k1;
    c += __shfl_xor_sync(0xffffffffu, d, 4);
    c += __shfl_xor_sync(0xffffffffu, c, 2);
    c += __shfl_xor_sync(0xffffffffu, c, 1);
    return c;
}

// Sum four per-lane values over each group of lpr lanes (8, 16 or 32; the
// groups are aligned). On return, `plane` is the value index whose group total
// this lane holds and should write, or -1 if another lane of the group writes
// it. 8 lanes: 4 shuffles; 16 lanes: 5; 32 lanes: 6.
__device__ __forceinline__ int32_t reduce4_rows(const int32_t (&v)[4], int lane, int lpr,
                                                int &plane)
{
    if (lpr == 8) {
        const int sub = lane & 7;
        const bool hi = sub & 4;
        int32_t k0 = hi ? v[2] : v[0], k1 = hi ? v[3] : v[1];
        const int32_t s0 = hi ? v[0] : v[2], s1 = hi ? v[1] : v[3];
        k0 += __shfl_xor_sync(0xffffffffu, s0, 4);
        k1 += __shfl_xor_sync(0xffffffffu, s1, 4);
        const bool b1 = sub & 2;
        int32_t c = b1 ? k1 : k0;
        const int32_t d = b1 ? k0 : k1;
        c += __shfl_xor_sync(0xffffffffu, d, 2);
        c += __shfl_xor_sync(0xffffffffu, c, 1);
        plane = (sub & 1) ? -1 : (sub >> 1);
        return c;
    }
    int32_t c = reduce4_half(v, lane & 15);
    if (lpr == 32) {
        c += __shfl_xor_sync(0xffffffffu, c, 16);
        plane = (lane < 16 && (lane & 3) == 0) ? (lane >> 2) : -1;
    } else {
        plane = (lane & 3) == 0 ? ((lane & 15) >> 2) : -1;
    }
    return c;
}

// Shared-memory plan of one CTA (byte offsets from the dynamic base):
//   [head_bytes]   this CTA's entries (copied once from the launch parameters),
//                  per entry and token w_scale * x_scale and x_sum (loaded once
//                  the previous grid is done), per entry the offset of its
//                  activations in the x cache
//   [x_slot]       the activations (M x K int8) of this CTA's entries, loaded
//                  once per launch
//   [stages * stage]  the ring of packed weight tiles
//   desc[8]        StageDesc per stage
//   full[8], empty[8], xbar
//   part[8][16][MT][4]  int32 partial sums of rows split across warps
//   cnt[8][16]     how many warps have added into each row's partials
template <int MT>
struct SmemTail {
    static constexpr int kDesc = kMaxStages * int(sizeof(StageDesc));
    static constexpr int kBars = 2 * kMaxStages + 1;
    static constexpr int kPart = kMaxStages * kStreamMaxRows * MT * 4;
    static constexpr int kCnt = kMaxStages * kStreamMaxRows;
    static constexpr int kRed = 32;
    static constexpr size_t bytes() { return kDesc + kBars * 8 + (kPart + kCnt + kRed) * 4; }
};

// Max / sum over the WC consumer warps (named barrier 1). Every thread gets
// the result; `red` holds one slot per warp. Both are exact in any order
// (max of non-NaN floats, integer sum).
template <int WC, typename T, typename Op>
__device__ __forceinline__ T consumer_reduce(T v, Op op, T *red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
    if ((threadIdx.x & 31) == 0)
        red[threadIdx.x >> 5] = v;
    named_bar_sync(1, WC * 32);
    T r = red[0];
#pragma unroll
    for (int w = 1; w < WC; ++w)
        r = op(r, red[w]);
    named_bar_sync(1, WC * 32);  // red is reused by the next reduction
    return r;
}

struct FMax {
    __device__ float operator()(float a, float b) const { return fmaxf(a, b); }
};
struct IAdd {
    __device__ int operator()(int a, int b) const { return a + b; }
};
struct DAdd {
    __device__ double operator()(double a, double b) const { return a + b; }
};


// W consumer warps per group, G groups: group g consumes the CTA's tiles
// g, g + G, ... (stages g, g + G, ...).
template <int W, int G, int MaxE, int MT, int CPS>
__global__ void __launch_bounds__((W * G + 1) * 32, CPS)
stream_gemv_kernel(const __grid_constant__ StreamParams<MaxE> p)
{
    constexpr int WC = W * G;  // consumer warps
    extern __shared__ __align__(128) uint8_t smem[];
    const int stages = p.stages;
    const int stage_bytes = p.w_slot;
    // This CTA's tiles and the entries they belong to.
    const int t_begin = p.cta_tile0[blockIdx.x], t_end = p.cta_tile0[blockIdx.x + 1];
    const int e_first = p.cta_entry0[blockIdx.x];
    const int n_entries = p.cta_nent[blockIdx.x];  // local table size
    StreamEntry *tab = reinterpret_cast<StreamEntry *>(smem);
    float2 *scl = reinterpret_cast<float2 *>(smem + n_entries * sizeof(StreamEntry));
    int *xoff = reinterpret_cast<int *>(scl + n_entries * MT);
    uint8_t *xcache = smem + p.head_bytes;
    uint8_t *ring = xcache + p.x_slot;
    StageDesc *desc = reinterpret_cast<StageDesc *>(ring + stages * stage_bytes);
    uint64_t *full = reinterpret_cast<uint64_t *>(desc + kMaxStages);
    uint64_t *empty = full + kMaxStages;
    uint64_t *xbar = empty + kMaxStages;
    int32_t *part = reinterpret_cast<int32_t *>(xbar + 1);
    int32_t *cnt = part + SmemTail<MT>::kPart;
    int32_t *red = cnt + SmemTail<MT>::kCnt;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // A dependent grid launched with programmatic serialisation (the next
    // call's stack GEMV) may start its prologue and weight copies as soon as
    // SMs free up; it reads nothing this grid writes before its own
    // griddepcontrol.wait.
    if (threadIdx.x == 0)
        pdl_launch_dependents();

    for (int i = threadIdx.x; i < SmemTail<MT>::kPart + SmemTail<MT>::kCnt + SmemTail<MT>::kRed;
         i += blockDim.x)
        part[i] = 0;
    {
        static_assert(sizeof(StreamEntry) % 8 == 0, "entry size");
        const uint64_t *src = reinterpret_cast<const uint64_t *>(&p.e[e_first]);
        uint64_t *dst = reinterpret_cast<uint64_t *>(tab);
        const int n64 = n_entries * int(sizeof(StreamEntry) / 8);
        for (int i = threadIdx.x; i < n64; i += blockDim.x)
            dst[i] = src[i];
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int off = 0;
        for (int j = 0; j < n_entries; ++j) {
            xoff[j] = off;
            off += (p.M * tab[j].K + 127) & ~127;
        }
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], W);
        }
        mbar_init(xbar, 1);
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == WC) {
        // ------------------------------------------------------ producer
        if (lane != 0)
            return;
        const uint64_t pol_w = policy_evict_first();  // weights: read once
        const uint64_t pol_x = policy_evict_last();   // activations: reread by many CTAs
        auto load_x = [&]() {
            if (p.quant) {
                // The consumers write the activation cache themselves.
                mbar_arrive(xbar);
                return;
            }
            uint32_t total = 0;
            for (int j = 0; j < n_entries; ++j)
                total += uint32_t(p.M * tab[j].K);
            mbar_arrive_expect_tx(xbar, total);
            for (int j = 0; j < n_entries; ++j)
                bulk_g2s(xcache + xoff[j], tab[j].xq, uint32_t(p.M * tab[j].K), xbar, pol_x);
        };
        bool waited = !p.overlap_prev;
        if (waited) {
            pdl_wait();
            load_x();
        }
        int cursor = 0, it = 0, stage = 0;
        uint32_t phase = 0;
        for (int t = t_begin; t < t_end; ++t, ++it) {
            if (!waited && it == stages) {
                // The ring is full of weight copies issued before the
                // previous grid finished; activations may be read now.
                pdl_wait();
                waited = true;
                load_x();
            }
            while (cursor + 1 < n_entries && tab[cursor + 1].tile_begin <= t)
                ++cursor;
            const StreamEntry &e = tab[cursor];
            const int K = e.K;
            const int row0 = (t - e.tile_begin) * e.rows_per_tile;
            const int rows = min(e.rows_per_tile, e.N4 - row0);
            if (it >= stages && !mbar_wait(&empty[stage], phase ^ 1u, p.err))
                break;
            const uint32_t wbytes = uint32_t(rows) * uint32_t(K);
            desc[stage] = StageDesc{cursor, row0, rows, 0};
            mbar_arrive_expect_tx(&full[stage], wbytes);
            bulk_g2s(ring + stage * stage_bytes, e.packed + size_t(row0) * K, wbytes, &full[stage],
                     pol_w);
            if (++stage == stages) {
                stage = 0;
                phase ^= 1u;
            }
        }
        if (!waited) {
            pdl_wait();  // also after a failed wait: the x barrier must complete
            load_x();
        }
        // Do not let the CTA retire while a copy this thread issued is in
        // flight (matters only when a wait gave up). Stage s was last used
        // in this round (parity phase) if s < stage, else in the previous one.
        for (int s = 0; s < stages; ++s) {
            if (s < stage)
                mbar_wait(&full[s], phase, p.err);
            else if (it >= stages)
                mbar_wait(&full[s], phase ^ 1u, p.err);
        }
        mbar_wait(xbar, 0, p.err);
        return;
    }

    // ---------------------------------------------------------- consumers
    // Each consumer warp walks the ring on its own (no CTA barrier in the
    // loop): for each of its items it reads the packed words from the stage
    // while it computes, and hands the stage back after its last item's K
    // loop (rows split over warps: after their partial sums are in).
    pdl_wait();  // activations, x_scale and x_sum are read below
    if (MT == 1 && p.quant == 1) {
        // Quantise the CTA's activations (one token per projection) straight
        // into the activation cache. The CTA that streams a projection's
        // first tile also writes xq, x_scale and x_sum to global memory.
        for (int j = 0; j < n_entries; ++j) {
            const StreamEntry &e = tab[j];
            const uint4 *xv = reinterpret_cast<const uint4 *>(e.xin);
            const int nvec = e.K >> 3;  // 8 bf16 per 16-byte vector
            float amax = 0.0f;
            for (int v = threadIdx.x; v < nvec; v += WC * 32)
                amax = fmaxf(amax, absmax8(__ldg(xv + v)));
            amax = consumer_reduce<WC>(amax, FMax(), reinterpret_cast<float *>(red));
            const float s = quant_inv_scale(amax);
            const bool owner = e.tile_begin >= t_begin;
            uint2 *qc = reinterpret_cast<uint2 *>(xcache + xoff[j]);
            uint2 *qg = reinterpret_cast<uint2 *>(e.xq);
            int sum = 0;
            for (int v = threadIdx.x; v < nvec; v += WC * 32) {
                const uint2 o = quant8(__ldg(xv + v), s, &sum);
                qc[v] = o;
                if (owner)
                    qg[v] = o;
            }
            sum = consumer_reduce<WC>(sum, IAdd(), red);
            if (threadIdx.x == 0) {
                const float xs = quant_scale(amax);
                scl[j * MT] = make_float2(__fmul_rn(e.w_scale, xs), __int_as_float(sum));
                if (owner) {
                    *e.x_scale = xs;
                    *e.x_sum = sum;
                }
            }
        }
    } else if (MT == 1 && p.quant >= 2) {
        // RMSNorm (gain, eps) of the token -- of bf16 x (mode 2) or of
        // relu(gate)^2 * up from fp32 rows (mode 3) -- then the same
        // quantiser, with the arithmetic of the standalone normalising
        // kernels: r = fl32(1 / sqrt(sum v^2 / K + eps)) from an fp64 sum,
        // h = fl32(fl32(v * r) * gain). Three passes over the row: sum of
        // squares, largest |h|, codes.
        static_assert(WC <= 16, "one fp64 reduction slot per consumer warp");
        for (int j = 0; j < n_entries; ++j) {
            const StreamEntry &e = tab[j];
            const int K = e.K;
            auto v4 = [&](int k) -> float4 {
                if (p.quant == 2) {
                    const uint2 u = __ldg(reinterpret_cast<const uint2 *>(
                        static_cast<const uint16_t *>(e.xin) + k));
                    return make_float4(bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y));
                }
                const float4 a = __ldg(reinterpret_cast<const float4 *>(
                    static_cast<const float *>(e.xin) + k));
                const float4 b = __ldg(reinterpret_cast<const float4 *>(e.up + k));
                auto r2 = [](float g, float u) {
                    const float r = fmaxf(g, 0.0f);
                    return __fmul_rn(__fmul_rn(r, r), u);
                };
                return make_float4(r2(a.x, b.x), r2(a.y, b.y), r2(a.z, b.z), r2(a.w, b.w));
            };
            // Each thread keeps its first kNV groups of four inputs, and
            // their gains, in registers across the three passes (all of a
            // row up to K = 4 kNV x 32 WC); a tail beyond that is re-read.
            constexpr int kNV = 4;
            constexpr int stride = 4 * WC * 32;
            auto g4 = [&](int k) {
                return make_float4(__ldg(e.gain + k), __ldg(e.gain + k + 1),
                                   __ldg(e.gain + k + 2), __ldg(e.gain + k + 3));
            };
            float4 vr[kNV], gr[kNV];
            double ss = 0.0;
            auto add_sq = [&](const float4 &v) {
                ss += double(v.x) * v.x;  // each square exact in fp64
                ss += double(v.y) * v.y;
                ss += double(v.z) * v.z;
                ss += double(v.w) * v.w;
            };
#pragma unroll
            for (int i = 0; i < kNV; ++i) {
                const int k = 4 * threadIdx.x + i * stride;
                if (k < K) {
                    vr[i] = v4(k);
                    gr[i] = g4(k);
                    add_sq(vr[i]);
                }
            }
            for (int k = 4 * threadIdx.x + kNV * stride; k < K; k += stride)
                add_sq(v4(k));
            ss = consumer_reduce<WC>(ss, DAdd(), reinterpret_cast<double *>(red));
            const float r = __double2float_rn(1.0 / sqrt(ss / double(K) + double(e.eps)));
            auto h4 = [&](const float4 &v, const float4 &g) {
                return make_float4(__fmul_rn(__fmul_rn(v.x, r), g.x), __fmul_rn(__fmul_rn(v.y, r), g.y),
                                   __fmul_rn(__fmul_rn(v.z, r), g.z), __fmul_rn(__fmul_rn(v.w, r), g.w));
            };
            auto amax4 = [](float m, const float4 &h) {
                return fmaxf(fmaxf(fmaxf(m, fabsf(h.x)), fabsf(h.y)), fmaxf(fabsf(h.z), fabsf(h.w)));
            };
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < kNV; ++i)
                if (4 * threadIdx.x + i * stride < K)
                    amax = amax4(amax, h4(vr[i], gr[i]));
            for (int k = 4 * threadIdx.x + kNV * stride; k < K; k += stride)
                amax = amax4(amax, h4(v4(k), g4(k)));
            amax = consumer_reduce<WC>(amax, FMax(), reinterpret_cast<float *>(red));
            const float s = quant_inv_scale(amax);
            const bool owner = e.tile_begin >= t_begin;
            uint32_t *qc = reinterpret_cast<uint32_t *>(xcache + xoff[j]);
            uint32_t *qg = reinterpret_cast<uint32_t *>(e.xq);
            int sum = 0;
            auto put = [&](int k, const float4 &h) {
                const int a = code_of(h.x, s), b = code_of(h.y, s);
                const int c = code_of(h.z, s), d = code_of(h.w, s);
                sum += a + b + c + d;
                const uint32_t word = (uint32_t(a) & 0xFFu) | ((uint32_t(b) & 0xFFu) << 8) |
                                      ((uint32_t(c) & 0xFFu) << 16) | ((uint32_t(d) & 0xFFu) << 24);
                qc[k >> 2] = word;
                if (owner)
                    qg[k >> 2] = word;
            };
#pragma unroll
            for (int i = 0; i < kNV; ++i) {
                const int k = 4 * threadIdx.x + i * stride;
                if (k < K)
                    put(k, h4(vr[i], gr[i]));
            }
            for (int k = 4 * threadIdx.x + kNV * stride; k < K; k += stride)
                put(k, h4(v4(k), g4(k)));
            sum = consumer_reduce<WC>(sum, IAdd(), red);
            if (threadIdx.x == 0) {
                const float xs = quant_scale(amax);
                scl[j * MT] = make_float2(__fmul_rn(e.w_scale, xs), __int_as_float(sum));
                if (owner) {
                    *e.x_scale = xs;
                    *e.x_sum = sum;
                }
            }
        }
    } else {
        for (int i = threadIdx.x; i < n_entries * p.M; i += WC * 32) {
            const int j = i / p.M, m = i - j * p.M;
            const StreamEntry &e = tab[j];
            scl[j * MT + m] = make_float2(__fmul_rn(e.w_scale, __ldg(e.x_scale + m)),
                                          __int_as_float(__ldg(e.x_sum + m)));
        }
    }
    named_bar_sync(1, WC * 32);
    if (t_end > t_begin && !mbar_wait_warp(xbar, 0, p.err))
        return;

    const int grp = warp / W, wg = warp - grp * W;
    int stage = grp;  // stages % G == 0, so the group keeps to stages grp + k*G
    uint32_t phase = 0;
    // Items are dealt to the group's warps round-robin across tiles (a tile
    // with fewer items than warps leaves different warps idle each time):
    // item i of a tile goes to warp (rot + i) % W, rot advancing by the
    // tile's item count.
    int rot = 0;
    for (int t = t_begin + grp; t < t_end; t += G) {
        if (!mbar_wait_warp(&full[stage], phase, p.err))
            return;
        const StageDesc d = desc[stage];
        const StreamEntry &e = tab[d.entry];
        const int K = e.K;
        const int C = K >> 4;
        const int N4 = e.N4;
        const int N = N4 * 4;
        float *const y = e.y;
        int32_t *const acc_out = e.acc_out;
        float tsc[MT];
        int32_t xsm[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const float2 v = scl[d.entry * MT + m];
            tsc[m] = v.x;
            xsm[m] = __float_as_int(v.y);
        }
        const uint8_t *sw = ring + stage * stage_bytes;
        const uint8_t *sx = xcache + xoff[d.entry];

        // A work item is 32 / lpr rows (lpr lanes each: 8, 16 or 32) times
        // one of 2^lg pieces of K. Fewer lanes per row means fewer shuffle
        // levels per row in the reduction and a longer loop per lane.
        const int lg = e.ksplit & 0xFF;
        const int lpr = 8 << ((e.ksplit >> 8) & 3);  // lanes per row
        const int grp_in = lane / lpr;               // row of the item this lane serves
        const int sub = lane & (lpr - 1);
        const int rpi = 32 / lpr;                    // rows per item
        const int n_items = ((d.rows + rpi - 1) / rpi) << lg;
        bool released = false;
        const int first_item = (wg - rot + W) % W;
        const int last_item = n_items - 1 - ((n_items - 1 - first_item) % W + W) % W;
        rot = (rot + n_items) % W;
        for (int item = first_item; item < n_items; item += W) {
            const int pr = item >> lg;
            const int piece = item & ((1 << lg) - 1);
            const int r = rpi * pr + grp_in;
            const bool valid = r < d.rows;
            const int c0 = (piece * C) >> lg;
            const int c1 = valid ? ((piece + 1) * C) >> lg : c0;
            const uint4 *wrow = reinterpret_cast<const uint4 *>(sw + size_t(r) * K);
            constexpr int J = 4 / MT;
            int32_t a[MT][4][J];
#pragma unroll
            for (int m = 0; m < MT; ++m)
#pragma unroll
                for (int q = 0; q < 4; ++q)
#pragma unroll
                    for (int s2 = 0; s2 < J; ++s2)
                        a[m][q][s2] = 0;
#pragma unroll 4
            for (int c = c0 + sub; c < c1; c += lpr) {
                const uint4 wv = wrow[c];
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (MT == 1 || m < p.M) {
                        const uint4 xv = reinterpret_cast<const uint4 *>(sx + m * K)[c];
                        dot16<J>(wv, xv, a[m]);
                    }
                }
            }
            if (lg == 0 && item == last_item) {
                // This warp's last read of the stage is done; the partial-sum
                // slots are used only by split rows: hand the stage back
                // before the reduction and epilogue.
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&empty[stage]);
                released = true;
            }
            const int row = d.row0 + r;
            if (lg == 0) {
                // Whole rows: lane 4 q (+16 for the second row of a pair)
                // writes plane q of its row.
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (MT == 1 || m < p.M) {
                        int32_t f[4];
                        fold<J>(a[m], f);
                        int plane;
                        const int32_t v = reduce4_rows(f, lane, lpr, plane);
                        if (valid && plane >= 0) {
                            const int32_t acc = (v >> (2 * plane)) - xsm[m];
                            const size_t o = size_t(m) * N + row + plane * N4;
                            y[o] = __fmul_rn(__int2float_rn(acc), tsc[m]);
                            if (acc_out)
                                acc_out[o] = acc;
                        }
                    }
                }
            } else {
                int32_t *slot = part + (stage * kStreamMaxRows + r) * MT * 4;
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (MT == 1 || m < p.M) {
                        int32_t f[4];
                        fold<J>(a[m], f);
                        int plane;
                        const int32_t v = reduce4_rows(f, lane, lpr, plane);
                        if (valid && plane >= 0)
                            atomicAdd(&slot[m * 4 + plane], v);
                    }
                }
                __threadfence_block();  // partial sums before the count
                __syncwarp();
                int old = 0;
                if (lane == 0)
                    old = atomicAdd(&cnt[stage * kStreamMaxRows + pr], 1);
                old = __shfl_sync(0xffffffffu, old, 0);
                if (old == (1 << lg) - 1) {
                    // Last piece of this item's rows: finish them.
                    __threadfence_block();
                    for (int oi = sub; valid && oi < 4 * p.M; oi += lpr) {
                        const int m = oi >> 2, plane = oi & 3;
                        const int32_t v = atomicExch(&slot[m * 4 + plane], 0);
                        const int32_t acc = (v >> (2 * plane)) - pick(xsm, m);
                        const size_t o = size_t(m) * N + row + plane * N4;
                        y[o] = __fmul_rn(__int2float_rn(acc), pick(tsc, m));
                        if (acc_out)
                            acc_out[o] = acc;
                    }
                    if (lane == 0)
                        cnt[stage * kStreamMaxRows + pr] = 0;
                }
            }
        }
        __syncwarp();
        if (lane == 0 && !released)
            mbar_arrive(&empty[stage]);
        stage += G;
        if (stage >= stages) {
            stage -= stages;
            phase ^= 1u;
        }
    }
}

template <int W, int G, int MaxE, int MT, int CPS>
cudaError_t launch_instance(const StreamParams<MaxE> &p, int grid, size_t smem, bool pdl,
                            cudaStream_t stream)
{
    auto kern = stream_gemv_kernel<W, G, MaxE, MT, CPS>;
    static std::atomic<int> configured_dev{-1};  // per instantiation, any host thread
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
    cfg.blockDim = dim3((W * G + 1) * 32);
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

// Tuning knobs: warps per consumer group, groups, CTAs per SM and the tile
// size aim. TQ_STREAM_CFG="W,G,CPS[,tile_bytes]" picks another instantiated
// variant (for measurement).
struct StreamCfg {
    int W = 8;
    int G = 2;
    int CPS = 1;
    int tile = kWTargetBytes;
};

StreamCfg stream_cfg()
{
    static StreamCfg cfg = [] {
        StreamCfg c;
        if (const char *s = getenv("TQ_STREAM_CFG")) {
            int w = 0, g = 0, cps = 0, tile = 0;
            const int n = sscanf(s, "%d,%d,%d,%d", &w, &g, &cps, &tile);
            const bool known = cps == 1 && ((g == 2 && (w == 4 || w == 6 || w == 7 || w == 8)) ||
                                            (g == 3 && w == 4) || (g == 4 && w == 4));
            if (n >= 3 && known) {
                c.W = w;
                c.G = g;
                c.CPS = cps;
            }
            if (n == 4 && tile >= 4096 && tile <= 65536)
                c.tile = tile;
        }
        return c;
    }();
    return cfg;
}

template <int MaxE, int MT>
cudaError_t launch_variant(const StreamCfg &c, const StreamParams<MaxE> &p, int grid, size_t smem,
                           bool pdl, cudaStream_t stream)
{
    if (c.G == 2 && c.W == 8)
        return launch_instance<8, 2, MaxE, MT, 1>(p, grid, smem, pdl, stream);
    if (c.G == 2 && c.W == 7)
        return launch_instance<7, 2, MaxE, MT, 1>(p, grid, smem, pdl, stream);
    if (c.G == 2 && c.W == 6)
        return launch_instance<6, 2, MaxE, MT, 1>(p, grid, smem, pdl, stream);
    if (c.G == 3)
        return launch_instance<4, 3, MaxE, MT, 1>(p, grid, smem, pdl, stream);
    if (c.G == 4)
        return launch_instance<4, 4, MaxE, MT, 1>(p, grid, smem, pdl, stream);
    return launch_instance<4, 2, MaxE, MT, 1>(p, grid, smem, pdl, stream);
}

template <int MaxE>
cudaError_t launch_sized(StreamEntry *entries, int n, int M, bool overlap_prev, bool single,
                         int quant, cudaStream_t stream)
{
    StreamParams<MaxE> p;  // host staging of the launch parameters
    static_assert(sizeof(StreamParams<MaxE>) <= 32000, "kernel parameters exceed 32 KB");
    const StreamCfg cfg = stream_cfg();
    const int sms = device_sm_count();
    const int W = cfg.W;
    int total = 0, stage_max = 0;
    for (int j = 0; j < n; ++j) {
        StreamEntry &e = entries[j];
        const int K = e.K;
        int R = kStreamMaxRows;
        while (R > 1 && R * K > cfg.tile)
            R >>= 1;
        if (single)
            while (R > 1 && (e.N4 + R - 1) / R < 2 * sms * cfg.CPS)
                R >>= 1;
        // Lanes per row: the fewest (8, 16, 32) that still give every warp
        // of a consumer group an item of 32 / lpr rows. Rows are cut into
        // pieces along K only if even 32 lanes per row leave warps idle.
        const int C = K >> 4;
        auto items_of = [&](int lsel) {
            const int rpi = 4 >> lsel;  // rows per item at 8 << lsel lanes per row
            return (R + rpi - 1) / rpi;
        };
        int lsel = 0;  // lanes per row = 8 << lsel
        while (lsel < 2 && items_of(lsel) < W)
            ++lsel;
        const int items = items_of(lsel);
        // Rows are cut into pieces along K only in single-projection
        // launches, where a CTA holds too few tiles for the round-robin deal
        // to keep its warps busy.
        int lg = 0;
        while (single && (items << lg) < W && (C >> (lg + 1)) >= 16)
            ++lg;
        e.rows_per_tile = R;
        e.ksplit = lg | (lsel << 8);
        e.tile_begin = total;
        total += (e.N4 + R - 1) / R;
        stage_max = std::max(stage_max, R * K);
        p.e[j] = e;
    }
    p.n_entries = n;
    p.total_tiles = total;
    p.M = M;
    p.w_slot = (stage_max + 127) / 128 * 128;
    p.overlap_prev = overlap_prev ? 1 : 0;
    p.quant = quant;
    const int mt = M == 1 ? 1 : (M == 2 ? 2 : 4);
    if (total == 0)
        return cudaSuccess;

    // Contiguous tile ranges per CTA, balanced by bytes (plus a fixed cost per
    // tile), so that every CTA streams about the same amount and finishes at
    // about the same time.
    const int grid = std::min({total, sms * cfg.CPS, kStreamMaxGrid});
    std::vector<long long> prefix(size_t(total) + 1, 0);
    {
        int t = 0;
        for (int j = 0; j < n; ++j) {
            const StreamEntry &e = p.e[j];
            const int tiles = (e.N4 + e.rows_per_tile - 1) / e.rows_per_tile;
            for (int i = 0; i < tiles; ++i, ++t) {
                const int rows = std::min(e.rows_per_tile, e.N4 - i * e.rows_per_tile);
                prefix[size_t(t) + 1] = prefix[size_t(t)] + (long long)rows * e.K + 4096;
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
    size_t x_max = 0;
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
        size_t xb = 0;
        for (int j = e0; j <= e1; ++j)
            xb += (size_t(M) * p.e[j].K + 127) / 128 * 128;
        x_max = std::max(x_max, xb);
    }
    p.x_slot = int(x_max);
    p.head_bytes = int((size_t(max_local) * (sizeof(StreamEntry) + size_t(mt) * sizeof(float2) +
                                             sizeof(int)) +
                        127) /
                       128 * 128);
    p.err = device_error_word();
    if (!p.err)
        return cudaErrorUnknown;
    const size_t tail = mt == 1 ? SmemTail<1>::bytes()
                                : (mt == 2 ? SmemTail<2>::bytes() : SmemTail<4>::bytes());
    const size_t fixed = tail + p.head_bytes + p.x_slot;
    const size_t budget = smem_budget(cfg.CPS);
    int stages = budget > fixed ? int((budget - fixed) / size_t(p.w_slot)) : 0;
    stages = std::min(stages, kMaxStages);
    // Each consumer group must see every phase of the stages it uses: with
    // stages % G != 0 a group would wait for phase k of a stage whose phase
    // k - 1 (another group's tile) has not completed yet, and a parity wait
    // cannot tell those apart.
    stages -= stages % cfg.G;
    if (stages < std::max(2, cfg.G))
        return cudaErrorInvalidValue;
    p.stages = stages;
    const size_t smem = fixed + size_t(stages) * p.w_slot;
    switch (mt) {
    case 1: return launch_variant<MaxE, 1>(cfg, p, grid, smem, overlap_prev, stream);
    case 2: return launch_variant<MaxE, 2>(cfg, p, grid, smem, overlap_prev, stream);
    default: return launch_variant<MaxE, 4>(cfg, p, grid, smem, overlap_prev, stream);
    }
}

}  // namespace

cudaError_t launch_stream_gemv(StreamEntry *entries, int n, int M, bool overlap_prev, bool single,
                               int quant, cudaStream_t stream)
{
    if (n <= 0)
        return cudaSuccess;
    if (M < 1 || M > kStreamMaxTokens || n > kStreamStackMax || quant < 0 || quant > 3 ||
        (quant && M != 1))
        return cudaErrorInvalidValue;
    if (n == 1)
        return launch_sized<1>(entries, n, M, overlap_prev, single, quant, stream);
    if (n <= 16)
        return launch_sized<16>(entries, n, M, overlap_prev, single, quant, stream);
    return launch_sized<kStreamStackMax>(entries, n, M, overlap_prev, single, quant, stream);
}

}  // namespace tq
