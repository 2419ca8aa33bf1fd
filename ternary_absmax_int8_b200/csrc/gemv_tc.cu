// gemv_tc.cu -- batched-decode ternary GEMV on the tensor cores (5 <= M <= 32
// tokens), tcgen05 with the code operand in tensor memory.
//
// Many concurrent requests turn decode into a skinny contraction (1bit engine
// blog, "One GPU, many users"): each weight byte now feeds M tokens, so
// unpacking with dp4a on the CUDA cores runs out of issue slots long before
// HBM does, while the work is still far too small for a prefill tile.
//
//   D[r, m] = sum_k c[r, k] * xq[m, k]     (u8 codes, s8 activations, s32)
//   acc = D - x_sum[m],  y = float(acc) * (w_scale * x_scale[m])
//
// * Tile: 32 packed rows = 128 MMA rows with row r = 4 j + p holding plane p
//   of packed row j (feature i0 + j + p N/4); BN = 16 or 32 token columns.
//   With this order a warp's 32 tensor-memory lanes are 8 packed rows x 4
//   planes, so each packed byte is read from shared memory once. A lane
//   keeps its plane's bits in place (code c stored as c * 4^p, one AND per
//   word): the MMA sums are 4^p times the code sums, exactly, and the
//   epilogue shifts them back.
// * The expansion warps unpack codes in registers and store them straight
//   into tensor memory (tcgen05.st): the A operand never passes through shared
//   memory, which at small N would otherwise bound the kernel (16 KB written
//   and 16 KB read back per 4 KB of weights).
// * K advances in 256-byte units; a unit is one TMA box pair of packed bytes
//   (32 rows) plus activations (BN rows), 128B swizzled. A CTA works through
//   segments (tile, first unit, end unit); two plans decide which:
//   - cluster plan (tq_gemv): with fewer tiles than SMs, the C CTAs of a
//     thread-block cluster split one tile's K range; the other CTAs store
//     their int32 partial sums into slots in the leader CTA's shared memory
//     (16-byte st.shared::cluster) and signal its mbarrier; the leader adds
//     them (exact, order-free) and applies the epilogue. With many tiles, C = 1 and each CTA takes
//     whole tiles.
//   - stream-K plan (tq_gemv_noalloc): the (tile, unit) sequence is cut into
//     one contiguous, balanced range per CTA; a tile split across CTAs adds
//     its partial sums into a global scratch with integer atomics, and the
//     CTA whose contribution completes the tile applies the epilogue and
//     zeroes the scratch for the next call.
//   - group plan (tq_gemv_stack_batch): the stream-K plan over the
//     concatenated (projection, tile, unit) sequence of up to 16 projections
//     of different shapes, one tensor map pair per projection, so that one
//     launch balances, say, the 10-unit tiles of a 2560-wide projection
//     against the 27-unit tiles of a 6912-wide one.
// * Warp roles (16 warps): 0 TMA producer, 1..3 MMA issuers (1 also
//   allocates tensor memory), 4..11 expansion (two sets of four warps, one
//   TMEM lane quarter each, taking alternate units), 12..15 epilogue. All
//   mbarrier waits are bounded.
// * A thread blocks on each tcgen05.mma it issues for about 117 cycles
//   whatever N is (measured on B200, 16 <= N <= 64), while the tensor core
//   would finish a 128 x 16 x 32 product in a few: one issuing thread caps a
//   CTA at 8 KB of weights per ~0.5 us. So three threads issue, taking units
//   in turn, each into its own accumulator; the epilogue adds the partial
//   accumulators of the issuers that had units in the segment.
#include <atomic>
#include <algorithm>
#include <mutex>
#include <utility>
#include <vector>

#include "tc_common.cuh"

namespace tq {

namespace {

constexpr int kRows = 128;             // MMA M (32 packed rows x 4 planes)
constexpr int kPRows = kRows / 4;      // packed rows per tile
constexpr int kUnitK = 256;            // bytes of K per unit (two 128-byte boxes)
// Shared-memory stages (packed bytes + activations): fewer at BN = 32, whose
// stages and cluster slots are twice as large.
template <int BN>
constexpr int kStagesOf = BN == 16 ? 10 : 6;
constexpr int kSA = 4;                 // tensor-memory A slots
// Units whose copies thread 0 issues before the CTA barrier (their latency
// overlaps the tensor-memory allocation); the producer warp issues the rest.
// Few: every copy issued here delays the barrier the whole CTA waits on.
constexpr int kEarlyUnits = 2;
constexpr int kIssuers = 3;            // MMA-issuing warps 1..3, one accumulator each
// "A slot filled" barriers, one per unit modulo lcm(kIssuers, kSA): each then
// has a single MMA issuer and a single expansion set, so its waiter has
// always seen the phase before the one it waits for. (With one barrier per
// A slot, an issuer could wait for unit i's phase while unit i - kSA, which
// another issuer consumes, was still being expanded: the parity wait then
// matched the phase before that one and passed early.)
constexpr int kAFull = 12;
constexpr int kACols = kUnitK / 4;     // TMEM columns per A slot (4 bytes per column)
constexpr int kThreads = 512;
constexpr int kExpandWarp0 = 4;        // expansion warps 4..11: two sets of four
constexpr int kExpandSets = 2;         // set s expands the CTA's units s, s + 2, ...
constexpr int kEpiWarp0 = 4 + 4 * kExpandSets;  // epilogue warps 12..15
static_assert(kAFull % kIssuers == 0 && kAFull % kSA == 0 && kAFull % kExpandSets == 0,
              "a_full barrier ownership");
constexpr int kMaxGrid = 512;

constexpr int kPlanStreamK = 0;
constexpr int kPlanCluster = 1;
constexpr int kMaxCluster = 8;
constexpr int kMaxGroup = 64;          // projections per group launch

struct SmallMParams {
    int N4, K, M;
    int tiles, units_per_tile, total_units, grid;
    int plan;   // kPlanStreamK or kPlanCluster
    int csize;  // CTAs per cluster (cluster plan)
    float w_scale;
    const float *x_scale;
    const int32_t *x_sum;
    float *y;
    int32_t *acc_out;
    int32_t *ws;    // stream-K: [tiles][BN][128] int32 partial sums (all zero between calls)
    int32_t *cnt;   // stream-K: [tiles] arrivals (all zero between calls)
    unsigned *err;
};

// One projection of a group launch: its shape, where its tiles and units
// start in the launch's sequence, and its epilogue operands.
struct GroupProj {
    int N4, U, tiles;    // packed rows, K units per tile, tiles
    int tile0, unit0;    // first tile / unit of this projection in the launch
    float w_scale;
    const float *x_scale;
    const int32_t *x_sum;
    float *y;
    int32_t *acc_out;
};

// The group launch's table (a kernel parameter; tensor maps 64-byte aligned).
struct GroupTable {
    CUtensorMap map_p[kMaxGroup];
    CUtensorMap map_x[kMaxGroup];
    GroupProj g[kMaxGroup];
    int n;
};

// A run of consecutive K units [k0, k1) of one tile (of projection `proj`
// in a group launch, else 0).
struct Seg {
    int tile, k0, k1, proj;
};

// The segments one CTA works through, in order.
struct CtaWork {
    int nseg;
    int u_begin, u_end;  // stream-K: this CTA's global unit range
    int rank;            // cluster plan: rank in the cluster

    __device__ Seg seg(const SmallMParams &p, int s) const
    {
        const int U = p.units_per_tile;
        if (p.plan == kPlanStreamK) {
            const int t = u_begin / U + s;
            return Seg{t, s == 0 ? u_begin - t * U : 0, min(U, u_end - t * U), 0};
        }
        if (p.csize == 1)
            return Seg{int(blockIdx.x) + s * int(gridDim.x), 0, U, 0};
        return Seg{int(blockIdx.x) / p.csize, U * rank / p.csize, U * (rank + 1) / p.csize, 0};
    }

    // Group plan: the CTA's first segment, and the one after `g` (the next
    // tile of the sequence, crossing into the next projection; every
    // projection of the table has at least one tile).
    __device__ Seg group_first(const GroupTable &t) const
    {
        int j = 0;
        while (j + 1 < t.n && t.g[j + 1].unit0 <= u_begin)
            ++j;
        const GroupProj &q = t.g[j];
        const int tile = (u_begin - q.unit0) / q.U;
        const int u0 = q.unit0 + tile * q.U;
        return Seg{tile, u_begin - u0, min(q.U, u_end - u0), j};
    }

    __device__ Seg group_next(const GroupTable &t, const Seg &g) const
    {
        int j = g.proj, tile = g.tile + 1;
        if (tile == t.g[j].tiles) {
            ++j;
            tile = 0;
        }
        if (j >= t.n)
            return Seg{0, 0, 0, j};
        const GroupProj &q = t.g[j];
        const int u0 = q.unit0 + tile * q.U;
        return Seg{tile, 0, min(q.U, u_end - u0), j};
    }
};

template <int BN>
struct SmallMSmem {
    static constexpr int kSP = kStagesOf<BN>;
    static constexpr int kPBytes = kPRows * kUnitK;  // 8 KB
    static constexpr int kBBytes = BN * kUnitK;
    static constexpr size_t p_off = 0;
    static constexpr size_t b_off = p_off + size_t(kSP) * kPBytes;
    // cluster plan: one slot per other CTA of the cluster for its partial
    // sums, [rank - 1][BN / 4][128 rows] x 16 bytes, in the leader
    static constexpr size_t slot_off = b_off + size_t(kSP) * kBBytes;
    static constexpr size_t kSlotBytes = size_t(kRows) * BN * 4;
    static constexpr size_t bar_off = slot_off + size_t(kMaxCluster - 1) * kSlotBytes;
    // tma_full[SP], p_free[SP], mma_done[SP], a_full[kAFull], acc_full[2],
    // acc_empty[2], red_done
    static constexpr int kBars = 3 * kSP + kAFull + 5;
    static constexpr size_t misc_off = bar_off + kBars * 8;  // tmem slot, finisher flag
    static constexpr size_t bytes = misc_off + 16;
};

// Unit u of the whole call belongs to CTA b with U(b) <= u < U(b+1).
__device__ __forceinline__ int unit_start(int b, int total, int grid)
{
    return int((long long)total * b / grid);
}

__device__ __forceinline__ int cta_of_unit(int u, int total, int grid)
{
    // largest b with unit_start(b) <= u
    int b = int(((long long)u * grid) / total);
    while (b + 1 < grid && unit_start(b + 1, total, grid) <= u)
        ++b;
    while (b > 0 && unit_start(b, total, grid) > u)
        --b;
    return b;
}

// Tile counter of the stream-K plans: release (the epilogue threads' partial
// sums, ordered before this by the named barrier) and acquire (the other
// CTAs' sums, for the CTA that completes the tile), at GPU scope.
__device__ __forceinline__ int atom_add_acq_rel_gpu(int *p, int v)
{
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;"
                 : "=r"(old)
                 : "l"(p), "r"(v)
                 : "memory");
    return old;
}

// Barrier over the 128 epilogue threads (named barrier 2) that ORs a predicate.
__device__ __forceinline__ bool epilogue_any(bool pred)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 2, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(uint32_t(pred))
        : "memory");
    return r != 0;
}

// The kernel body. maps_p / maps_x point at the launch's tensor maps in
// parameter space (one pair, or one per projection of a group launch, gt).
template <int BN, bool Group>
__device__ __forceinline__ void smallm_body(const CUtensorMap *maps_p, const CUtensorMap *maps_x,
                                            const SmallMParams &p, const GroupTable *gt)
{
    using L = SmallMSmem<BN>;
    constexpr int kSP = L::kSP;
    constexpr uint32_t kIdesc = idesc_i8_u8s8(kRows, BN);
    constexpr int kTmemCols = 512;  // kSA * kACols + 2 * kIssuers * BN, rounded to a power of two
    static_assert(kSA * kACols + 2 * kIssuers * BN <= kTmemCols, "tensor memory plan");

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sP = smem + L::p_off;
    uint8_t *sB = smem + L::b_off;
    uint4 *slots = reinterpret_cast<uint4 *>(smem + L::slot_off);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::bar_off);
    uint64_t *tma_full = bars;
    uint64_t *p_free = bars + kSP;
    uint64_t *mma_done = bars + 2 * kSP;
    uint64_t *a_full = bars + 3 * kSP;
    uint64_t *acc_full = a_full + kAFull;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *red_done = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::misc_off);
    int *fin_flag = reinterpret_cast<int *>(smem + L::misc_off + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int U = p.units_per_tile;
    const bool split_cluster = p.plan == kPlanCluster && p.csize > 1;
    CtaWork cw;
    cw.rank = split_cluster ? int(cluster_ctarank()) : 0;
    if (p.plan == kPlanStreamK) {
        cw.u_begin = unit_start(blockIdx.x, p.total_units, p.grid);
        cw.u_end = unit_start(blockIdx.x + 1, p.total_units, p.grid);
        if constexpr (Group) {
            cw.nseg = 0;
            if (cw.u_end > cw.u_begin) {
                for (Seg g = cw.group_first(*gt); g.proj < gt->n; g = cw.group_next(*gt, g)) {
                    ++cw.nseg;
                    const GroupProj &q = gt->g[g.proj];
                    if (q.unit0 + g.tile * q.U + g.k1 >= cw.u_end)
                        break;
                }
            }
        } else {
            cw.nseg = cw.u_end > cw.u_begin ? (cw.u_end - 1) / U - cw.u_begin / U + 1 : 0;
        }
    } else {
        cw.u_begin = cw.u_end = 0;
        cw.nseg = split_cluster ? 1
                                : (p.tiles > int(blockIdx.x)
                                       ? (p.tiles - 1 - int(blockIdx.x)) / int(gridDim.x) + 1
                                       : 0);
    }

    // The CTA's segments in order: segment 0, and the one after segment
    // sg - 1 (= g).
    auto first_seg = [&]() -> Seg {
        if constexpr (Group)
            return cw.group_first(*gt);
        else
            return cw.seg(p, 0);
    };
    auto next_seg = [&](const Seg &g, int sg) -> Seg {
        if constexpr (Group)
            return cw.group_next(*gt, g);
        else
            return cw.seg(p, sg);
    };

    // The producer's copies, unit by unit in the CTA's order: the packed
    // weights (which no earlier kernel writes) and the activations (which
    // the previous kernel on the stream may still be writing: copied only
    // after griddepcontrol.wait).
    auto issue_w = [&](int issued, const Seg &g, int k) {
        const int s = issued % kSP;
        const int k0 = k * kUnitK;
        mbar_arrive_expect_tx(&tma_full[s], L::kPBytes + L::kBBytes);
        uint8_t *P = sP + s * L::kPBytes;
        const CUtensorMap *mp = maps_p + g.proj;
        tma_load_2d(P, mp, k0, g.tile * kPRows, &tma_full[s]);
        tma_load_2d(P + L::kPBytes / 2, mp, k0 + 128, g.tile * kPRows, &tma_full[s]);
    };
    auto issue_x = [&](int issued, const Seg &g, int k) {
        const int s = issued % kSP;
        const int k0 = k * kUnitK;
        uint8_t *B = sB + s * L::kBBytes;
        const CUtensorMap *mx = maps_x + g.proj;
        tma_load_2d(B, mx, k0, 0, &tma_full[s]);
        tma_load_2d(B + L::kBBytes / 2, mx, k0 + 128, 0, &tma_full[s]);
    };
    int early = 0;  // weight copies thread 0 issued before the CTA barrier
    if (threadIdx.x == 0) {
        // A following kernel launched with programmatic serialisation may
        // start its own set-up and weight copies as SMs free up; it touches
        // nothing this grid reads or writes before its griddepcontrol.wait.
        pdl_launch_dependents();
        {
            const int j0 = cw.nseg > 0 ? first_seg().proj : 0;
            prefetch_tensormap(maps_p + j0);
            prefetch_tensormap(maps_x + j0);
        }
        for (int s = 0; s < kSP; ++s) {
            mbar_init(&tma_full[s], 1);
            mbar_init(&p_free[s], 4);
            mbar_init(&mma_done[s], 1);
        }
        for (int s = 0; s < kAFull; ++s)
            mbar_init(&a_full[s], 4);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], kIssuers);  // every issuer commits every segment
            mbar_init(&acc_empty[b], 4);
        }
        // every epilogue thread of every other CTA of the cluster arrives once
        mbar_init(red_done, split_cluster ? uint32_t(kRows * (p.csize - 1)) : 1u);
        fence_mbar_init();
        // Start the first stages' copies now: their latency overlaps the
        // tensor-memory allocation and the barriers below.
        Seg g = first_seg();
        for (int sg = 0; sg < cw.nseg && early < kEarlyUnits; ++sg, g = next_seg(g, sg)) {
            for (int k = g.k0; k < g.k1 && early < kEarlyUnits; ++k)
                issue_w(early++, g, k);
        }
    }
    if (warp == 1)
        tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // The leader's barrier and zeroed sum must exist before any CTA of the
    // cluster touches them.
    if (split_cluster)
        cluster_sync_all();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t tmem_a = tmem_base;                    // kSA slots of kACols
    // accumulators: [2 buffers][kIssuers][BN columns]
    const uint32_t tmem_d = tmem_base + kSA * kACols;

    if (warp == 0) {
        // -------------------------------------------------- TMA producer
        if (lane == 0) {
            int issued = 0;
            bool ok = true;
            pdl_wait();  // activations of the previous kernel on the stream
            Seg g = first_seg();
            for (int sg = 0; sg < cw.nseg && ok; ++sg, g = next_seg(g, sg)) {
                for (int k = g.k0; k < g.k1; ++k, ++issued) {
                    if (issued < early) {
                        issue_x(issued, g, k);  // its weights went before the CTA barrier
                        continue;
                    }
                    const int s = issued % kSP;
                    const uint32_t use = uint32_t(issued / kSP);
                    if (use > 0 && (!mbar_wait(&p_free[s], (use - 1) & 1, p.err) ||
                                    !mbar_wait(&mma_done[s], (use - 1) & 1, p.err))) {
                        ok = false;
                        break;
                    }
                    issue_w(issued, g, k);
                    issue_x(issued, g, k);
                }
            }
            for (int s = 0; s < kSP && s < issued; ++s) {
                const int last = issued - 1 - ((issued - 1 - s) % kSP);
                mbar_wait(&tma_full[s], uint32_t((last / kSP) & 1), p.err);
            }
        }
    } else if (warp >= 1 && warp <= kIssuers) {
        // -------------------------------------------------- MMA issuers
        // issuer t = warp - 1 takes the CTA's units i with i % kIssuers == t
        const int t = warp - 1;
        if (lane == 0) {
            int i = 0, last = -1;
            bool ok = true;
            Seg g = first_seg();
            for (int sg = 0; sg < cw.nseg && ok; ++sg, g = next_seg(g, sg)) {
                const int buf = sg & 1;
                if (sg >= 2 && !mbar_wait(&acc_empty[buf], uint32_t(((sg >> 1) - 1) & 1), p.err))
                    break;
                tc_fence_after();
                const uint32_t d = tmem_d + uint32_t((buf * kIssuers + t) * BN);
                bool fresh = true;  // this issuer's first unit of the segment
                for (int k = g.k0; k < g.k1; ++k, ++i) {
                    if (i % kIssuers != t)
                        continue;
                    const int s = i % kSP, sa = i % kSA;
                    if (!mbar_wait(&tma_full[s], uint32_t((i / kSP) & 1), p.err) ||
                        !mbar_wait(&a_full[i % kAFull], uint32_t((i / kAFull) & 1), p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    // one descriptor per unit, advanced by adds
                    const uint64_t db = umma_desc_sw128(smem_u32(sB + s * L::kBBytes));
                    const uint32_t ta = tmem_a + uint32_t(sa * kACols);
#pragma unroll
                    for (int kk = 0; kk < kUnitK / 32; ++kk)
                        umma_i8_ts(d, ta + uint32_t(kk * 8),
                                   umma_desc_advance(db, uint32_t((kk >> 2) * (L::kBBytes / 2) +
                                                                  (kk & 3) * 32)),
                                   kIdesc, (fresh && kk == 0) ? 0u : 1u);
                    umma_commit(&mma_done[s]);
                    fresh = false;
                    last = i;
                }
                if (ok)
                    umma_commit(&acc_full[buf]);
            }
            if (last >= 0) {
                const int s = last % kSP;
                mbar_wait(&mma_done[s], uint32_t((last / kSP) & 1), p.err);
            }
        }
    } else if (warp >= kExpandWarp0 && warp < kEpiWarp0) {
        // -------------------------------------------------- expansion
        const int q = warp & 3;                      // TMEM lane quarter
        const int set = (warp - kExpandWarp0) >> 2;  // this warp's units: set, set + 2, ...
        const int j = 8 * q + (lane >> 2), pl = lane & 3;  // packed row, plane of this lane
        const uint32_t lane_base = uint32_t(q * 32) << 16;
        int i = 0;
        bool ok = true;
        Seg g = first_seg();
        for (int sg = 0; sg < cw.nseg && ok; ++sg, g = next_seg(g, sg)) {
            for (int k = g.k0; k < g.k1; ++k, ++i) {
                if (i % kExpandSets != set)
                    continue;
                const int s = i % kSP, sa = i % kSA;
                ok = mbar_wait_warp(&tma_full[s], uint32_t((i / kSP) & 1), p.err);
                if (ok && i >= kSA) {
                    const int pi = i - kSA;  // the unit that last used this A slot
                    ok = mbar_wait_warp(&mma_done[pi % kSP], uint32_t((pi / kSP) & 1), p.err);
                }
                if (!ok)
                    break;
                tc_fence_after();
                const uint8_t *P = sP + s * L::kPBytes;
                // The lane's plane bits stay in place: each byte holds c * 4^pl
                // (at most 128, still a u8), one AND per word; the epilogue
                // shifts the exact int32 sums back down.
                const uint32_t mask = 0x03030303u << (2 * pl);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t v[32];
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint4 w = *reinterpret_cast<const uint4 *>(P + h * (L::kPBytes / 2) +
                                                                         sw128_off(j, c));
                        v[4 * c + 0] = w.x & mask;
                        v[4 * c + 1] = w.y & mask;
                        v[4 * c + 2] = w.z & mask;
                        v[4 * c + 3] = w.w & mask;
                    }
                    tmem_st32_async(tmem_a + lane_base + uint32_t(sa * kACols + h * 32), v);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&a_full[i % kAFull]);
                    mbar_arrive(&p_free[s]);
                }
            }
        }
    } else if (warp >= kEpiWarp0) {
        // -------------------------------------------------- epilogue
        const int q = warp & 3;
        const int r = 32 * q + lane;                 // accumulator row = TMEM lane
        const int jr = r >> 2, pl = r & 3;
        const uint32_t lane_base = uint32_t(q * 32) << 16;
        // the single projection of a plain launch, in the group's form
        const GroupProj self{p.N4, U, p.tiles, 0, 0, p.w_scale, p.x_scale, p.x_sum, p.y,
                             p.acc_out};
        pdl_wait();  // x_scale, x_sum, the outputs and the scratch
        Seg g = first_seg();
        int i0 = 0;  // the CTA's unit counter at the start of segment sg
        // Once a wait has given up (the error word is set and the outputs are
        // void), the remaining segments skip their waits and accumulator
        // reads but still count their split tiles in, so that every split
        // tile's finisher still runs and leaves the scratch zeroed.
        bool failed = false;
        for (int sg = 0; sg < cw.nseg; ++sg, i0 += g.k1 - g.k0, g = next_seg(g, sg)) {
            const GroupProj *pj;
            if constexpr (Group)
                pj = &gt->g[g.proj];
            else
                pj = &self;
            const int N = 4 * pj->N4;
            const int tile = g.tile;
            const bool whole = g.k0 == 0 && g.k1 == pj->U;
            const int buf = sg & 1;
            if (!failed) {
                const bool got = mbar_wait_warp(&acc_full[buf], uint32_t((sg >> 1) & 1), p.err);
                // The four epilogue warps meet at named barriers below: decide
                // together.
                failed = epilogue_any(!got);
            }
            // The segment's units i0, i0 + 1, ... went to issuers i0 % kIssuers,
            // then the next ones in turn: add the partial accumulators of the
            // issuers that had one (warp-uniform), 16 columns at a time.
            uint32_t v[32];
#pragma unroll
            for (int c = 0; c < 32; ++c)
                v[c] = 0;
            if (!failed) {
                tc_fence_after();
                const int n_u = g.k1 - g.k0, r0 = i0 % kIssuers;
                const uint32_t dcol = tmem_d + lane_base + uint32_t(buf * kIssuers * BN);
#pragma unroll
                for (int h = 0; h < BN / 16; ++h) {
                    uint32_t tmp[16];
                    tmem_ld16(dcol + uint32_t(r0 * BN + h * 16), tmp);
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        v[h * 16 + c] = tmp[c];
#pragma unroll
                    for (int j = 1; j < kIssuers; ++j) {
                        if (j < n_u) {
                            const int tt = (r0 + j) % kIssuers;
                            tmem_ld16(dcol + uint32_t(tt * BN + h * 16), tmp);
#pragma unroll
                            for (int c = 0; c < 16; ++c)
                                v[h * 16 + c] += tmp[c];
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&acc_empty[buf]);  // the accumulator is in registers now
            }

            const int prow = tile * kPRows + jr;
            const bool row_ok = prow < pj->N4;
            const int n = prow + pl * pj->N4;
            if (split_cluster) {
                if (cw.rank != 0) {
                    // Store this CTA's partial sums into its slot in the
                    // leader, then tell the leader (release: the stores come
                    // first).
                    const uint32_t base = map_to_rank(smem_u32(slots), 0u) +
                                          uint32_t((cw.rank - 1) * L::kSlotBytes);
#pragma unroll
                    for (int c4 = 0; c4 < BN / 4; ++c4)
                        st_cluster_v4(base + uint32_t((c4 * kRows + r) * 16),
                                      make_uint4(v[4 * c4], v[4 * c4 + 1], v[4 * c4 + 2],
                                                 v[4 * c4 + 3]));
                    mbar_arrive_remote(map_to_rank(smem_u32(red_done), 0u));
                    continue;
                }
                // Leader: wait for the other CTAs' sums, add them (integer
                // adds, exact in any order), then finish the tile.
                if (!mbar_wait_cluster_warp(red_done, 0u, p.err))
                    continue;
                for (int k = 0; k < p.csize - 1; ++k) {
                    const uint4 *sl = slots + size_t(k) * (L::kSlotBytes / 16);
#pragma unroll
                    for (int c4 = 0; c4 < BN / 4; ++c4) {
                        const uint4 a = sl[c4 * kRows + r];
                        v[4 * c4] += a.x;
                        v[4 * c4 + 1] += a.y;
                        v[4 * c4 + 2] += a.z;
                        v[4 * c4 + 3] += a.w;
                    }
                }
            }
            if (whole || split_cluster) {
#pragma unroll
                for (int c = 0; c < BN; ++c) {
                    if (c < p.M && row_ok && !failed) {
                        // sums of c * 4^pl * x: exact, |.| <= 128 * 127 * 32768
                        const int32_t acc = (int32_t(v[c]) >> (2 * pl)) - __ldg(pj->x_sum + c);
                        const float t = __fmul_rn(pj->w_scale, __ldg(pj->x_scale + c));
                        const size_t o = size_t(c) * N + n;
                        pj->y[o] = __fmul_rn(__int2float_rn(acc), t);
                        if (pj->acc_out)
                            pj->acc_out[o] = acc;
                    }
                }
                continue;
            }
            // Stream-K partial tile: add into the workspace, then count this
            // CTA in. (Tiles and units of a group launch are numbered across
            // its projections.)
            // Scratch slot: the tile's index for a single projection; in a
            // group launch the index of the CTA holding the tile's first unit
            // (each CTA's range ends in at most one split tile, so the
            // slots are unique and the scratch is sized by the grid, not by
            // the tiles).
            const int wtile = pj->tile0 + tile;
            const int wunit = pj->unit0 + tile * pj->U;
            const int first = cta_of_unit(wunit, p.total_units, p.grid);
            const int slot = Group ? first : wtile;
            int32_t *wt = p.ws + size_t(slot) * BN * kRows;
#pragma unroll
            for (int c = 0; c < BN; ++c)
                if (c < p.M)
                    atomicAdd(wt + c * kRows + r, int32_t(v[c]));
            // One thread counts the CTA in once every epilogue thread has
            // issued its adds (the barrier orders them before its release).
            named_bar_sync(2, 128);
            if (threadIdx.x == kEpiWarp0 * 32) {
                const int last = cta_of_unit(wunit + pj->U - 1, p.total_units, p.grid);
                const int old = atom_add_acq_rel_gpu(p.cnt + slot, 1);
                *fin_flag = (old == last - first) ? 1 : 0;
            }
            named_bar_sync(2, 128);
            if (*fin_flag) {
                // Every CTA of the tile has added its sums (acquired above):
                // read them all at once from L2, then leave the slots zeroed.
#pragma unroll
                for (int h = 0; h < BN / 16; ++h) {
                    int32_t d[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        d[c] = h * 16 + c < p.M ? __ldcg(wt + (h * 16 + c) * kRows + r) : 0;
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        if (h * 16 + c < p.M)
                            __stcg(wt + (h * 16 + c) * kRows + r, 0);
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const int m = h * 16 + c;
                        if (m < p.M && row_ok) {
                            const int32_t acc = (d[c] >> (2 * pl)) - __ldg(pj->x_sum + m);
                            const float t = __fmul_rn(pj->w_scale, __ldg(pj->x_scale + m));
                            const size_t o = size_t(m) * N + n;
                            pj->y[o] = __fmul_rn(__int2float_rn(acc), t);
                            if (pj->acc_out)
                                pj->acc_out[o] = acc;
                        }
                    }
                }
                if (threadIdx.x == kEpiWarp0 * 32)
                    p.cnt[slot] = 0;
            }
            named_bar_sync(2, 128);  // fin_flag is reused by the next segment
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        tmem_dealloc(tmem_base, kTmemCols);
    // No CTA leaves while another may still address its shared memory.
    if (split_cluster)
        cluster_sync_all();
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
smallm_tc_kernel(const __grid_constant__ CUtensorMap map_p, const __grid_constant__ CUtensorMap map_x,
                 const __grid_constant__ SmallMParams p)
{
    smallm_body<BN, false>(&map_p, &map_x, p, nullptr);
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
smallm_group_kernel(const __grid_constant__ GroupTable gt, const __grid_constant__ SmallMParams p)
{
    smallm_body<BN, true>(gt.map_p, gt.map_x, p, &gt);
}

template <int BN>
cudaError_t configure_bn()
{
    static std::atomic<int> configured_dev{-1};  // set by any host thread
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (configured_dev != dev) {
        e = cudaFuncSetAttribute(smallm_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(SmallMSmem<BN>::bytes + 1024));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(smallm_group_kernel<BN>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     int(SmallMSmem<BN>::bytes + 1024));
        if (e != cudaSuccess)
            return e;
        configured_dev = dev;
    }
    return cudaSuccess;
}

template <int BN>
cudaError_t launch_bn(const CUtensorMap &mp, const CUtensorMap &mx, const SmallMParams &prm,
                      cudaStream_t stream)
{
    cudaError_t e = configure_bn<BN>();
    if (e != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(prm.grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = SmallMSmem<BN>::bytes + 1024;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    if (prm.plan == kPlanCluster && prm.csize > 1) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = unsigned(prm.csize);
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    e = cudaLaunchKernelEx(&cfg, smallm_tc_kernel<BN>, mp, mx, prm);
    return e != cudaSuccess ? e : cudaGetLastError();
}

// Largest cluster size C <= min(8, units per tile) such that tiles x C CTAs
// fit the GPU in one wave as whole clusters (the occupancy API counts how
// many clusters of C CTAs can be resident at once); 1 if none does.
template <int BN>
int pick_cluster(int tiles, int units)
{
    struct Key {
        int dev, tiles, units;
    };
    static std::mutex mu;
    static std::vector<std::pair<Key, int>> memo;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return 1;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (const auto &kv : memo)
            if (kv.first.dev == dev && kv.first.tiles == tiles && kv.first.units == units)
                return kv.second;
    }
    int best = 1;
    const int sms = device_sm_count();
    if (configure_bn<BN>() == cudaSuccess) {
        for (int c = std::min(kMaxCluster, units); c >= 2; --c) {
            if (tiles * c > sms)
                continue;
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(tiles * c);
            cfg.blockDim = dim3(kThreads);
            cfg.dynamicSmemBytes = SmallMSmem<BN>::bytes + 1024;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = unsigned(c);
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int active = 0;
            if (cudaOccupancyMaxActiveClusters(&active, smallm_tc_kernel<BN>, &cfg) ==
                    cudaSuccess &&
                active >= tiles) {
                best = c;
                break;
            }
            cudaGetLastError();  // an unsupported size is not an error of the call
        }
    }
    std::lock_guard<std::mutex> lock(mu);
    memo.push_back({Key{dev, tiles, units}, best});
    return best;
}

bool fill_params(SmallMParams &prm, CUtensorMap &map_p, CUtensorMap &map_x,
                 const uint8_t *packed, float w_scale, const int8_t *xq, const float *x_scale,
                 const int32_t *x_sum, float *y, int32_t *acc_out, int M, int N, int K)
{
    const int BN = M <= 16 ? 16 : 32;
    if (!make_map(&map_p, packed, K, N / 4, kPRows) || !make_map(&map_x, xq, K, M, BN))
        return false;
    prm = SmallMParams{};
    prm.N4 = N / 4;
    prm.K = K;
    prm.M = M;
    prm.tiles = (prm.N4 + kPRows - 1) / kPRows;
    prm.units_per_tile = (K + kUnitK - 1) / kUnitK;
    prm.total_units = prm.tiles * prm.units_per_tile;
    prm.w_scale = w_scale;
    prm.x_scale = x_scale;
    prm.x_sum = x_sum;
    prm.y = y;
    prm.acc_out = acc_out;
    prm.err = device_error_word();
    return prm.err != nullptr;
}

// The stream-K plan on caller-provided, zero-filled scratch.
cudaError_t launch_smallm_streamk(const uint8_t *packed, float w_scale, const int8_t *xq,
                                  const float *x_scale, const int32_t *x_sum, float *y,
                                  int32_t *acc_out, int M, int N, int K, void *workspace,
                                  cudaStream_t stream)
{
    if (M < 1 || M > 32)
        return cudaErrorInvalidValue;
    const int BN = M <= 16 ? 16 : 32;
    CUtensorMap map_p, map_x;
    SmallMParams prm;
    if (!fill_params(prm, map_p, map_x, packed, w_scale, xq, x_scale, x_sum, y, acc_out, M, N, K))
        return cudaErrorInvalidValue;
    prm.plan = kPlanStreamK;
    prm.csize = 1;
    prm.grid = std::min({prm.total_units, device_sm_count(), kMaxGrid});
    prm.ws = static_cast<int32_t *>(workspace);
    prm.cnt = prm.ws + size_t(prm.tiles) * BN * kRows;
    return BN == 16 ? launch_bn<16>(map_p, map_x, prm, stream) : launch_bn<32>(map_p, map_x, prm, stream);
}

// Fixed scratch for tq_gemv_noalloc: the stream-K partial sums and tile
// counters live here instead of in library-allocated memory. Every GPU that
// loads the library holds these bytes until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
static __device__ __align__(256) int32_t g_noalloc_scratch[kNoAllocScratchBytes / sizeof(int32_t)];

// Fixed scratch of the group plan: one slot of partial sums (BN = 32 at most)
// and one counter per CTA of the largest grid. Unlike tq_gemv_noalloc's it
// is not zero-filled before every call: every launch leaves the parts it
// used zero (the CTA that completes a split tile zeroes its partial sums and
// counter, also after a wait gave up), so only the first call on a device,
// and the first one after a device error was reported, fill it.
constexpr size_t kGroupSlotBytes = size_t(32) * kRows * 4;
constexpr size_t kGroupScratchBytes =
    (size_t(kMaxGrid) * (kGroupSlotBytes + 4) + 255) / 256 * 256;
static __device__ __align__(256) int32_t g_group_scratch[kGroupScratchBytes / sizeof(int32_t)];

struct GroupScratch {
    std::mutex mu;
    void *ptr[64] = {};
    bool clean[64] = {};
};

GroupScratch &group_scratch()
{
    static GroupScratch gs;
    return gs;
}

// Host staging of a group launch's table, one per calling thread.
GroupTable *group_table()
{
    static thread_local GroupTable t;
    return &t;
}

static_assert(sizeof(GroupTable) + sizeof(SmallMParams) <= 32000, "kernel parameters exceed 32 KB");

// With `pdl` the launch may begin (set-up, tensor memory, weight copies)
// while the previous kernel on the stream drains; the kernel reads
// activations and scales and touches outputs and scratch only after
// griddepcontrol.wait.
template <int BN>
cudaError_t launch_group_bn(const GroupTable &gt, const SmallMParams &prm, bool pdl,
                            cudaStream_t stream)
{
    cudaError_t e = configure_bn<BN>();
    if (e != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(prm.grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = SmallMSmem<BN>::bytes + 1024;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, smallm_group_kernel<BN>, gt, prm);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

size_t smallm_workspace_bytes(int N, int M)
{
    const int BN = M <= 16 ? 16 : 32;
    const size_t tiles = (size_t(N / 4) + kPRows - 1) / kPRows;
    return tiles * BN * kRows * sizeof(int32_t) + tiles * sizeof(int32_t);
}

cudaError_t launch_smallm_tc(const uint8_t *packed, float w_scale, const int8_t *xq,
                             const float *x_scale, const int32_t *x_sum, float *y,
                             int32_t *acc_out, int M, int N, int K, cudaStream_t stream)
{
    if (M < 1 || M > 32)
        return cudaErrorInvalidValue;
    const int BN = M <= 16 ? 16 : 32;
    CUtensorMap map_p, map_x;
    SmallMParams prm;
    if (!fill_params(prm, map_p, map_x, packed, w_scale, xq, x_scale, x_sum, y, acc_out, M, N, K))
        return cudaErrorInvalidValue;
    prm.plan = kPlanCluster;
    prm.csize = BN == 16 ? pick_cluster<16>(prm.tiles, prm.units_per_tile)
                         : pick_cluster<32>(prm.tiles, prm.units_per_tile);
    prm.grid = prm.csize > 1 ? prm.tiles * prm.csize
                             : std::min({prm.tiles, device_sm_count(), kMaxGrid});
    return BN == 16 ? launch_bn<16>(map_p, map_x, prm, stream) : launch_bn<32>(map_p, map_x, prm, stream);
}

size_t noalloc_scratch_capacity() { return kNoAllocScratchBytes; }

void group_scratch_mark_dirty()
{
    GroupScratch &gs = group_scratch();
    std::lock_guard<std::mutex> lock(gs.mu);
    for (bool &c : gs.clean)
        c = false;
}

cudaError_t launch_smallm_group(const GroupEntry *e, int n, int M, bool overlap_prev,
                                cudaStream_t stream)
{
    if (M < 5 || M > 32 || n < 0)
        return cudaErrorInvalidValue;
    if (n == 0)
        return cudaSuccess;
    const int BN = M <= 16 ? 16 : 32;
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess)
        return err;
    if (dev < 0 || dev >= 64)
        return cudaErrorInvalidDevice;
    const int sms = device_sm_count();
    int32_t *scratch = nullptr;
    {
        GroupScratch &gs = group_scratch();
        std::lock_guard<std::mutex> lock(gs.mu);
        if (!gs.ptr[dev]) {
            err = cudaGetSymbolAddress(&gs.ptr[dev], g_group_scratch);
            if (err != cudaSuccess)
                return err;
        }
        if (!gs.clean[dev]) {
            err = cudaMemsetAsync(gs.ptr[dev], 0, kGroupScratchBytes, stream);
            if (err != cudaSuccess)
                return err;
            gs.clean[dev] = true;
        }
        scratch = static_cast<int32_t *>(gs.ptr[dev]);
    }
    int i = 0;
    bool first = true;
    while (i < n) {
        GroupTable &gt = *group_table();
        int j = 0, tiles = 0, units = 0;
        while (i < n && j < kMaxGroup) {
            const GroupEntry &x = e[i];
            const int t = (x.N / 4 + kPRows - 1) / kPRows;
            const int U = (x.K + kUnitK - 1) / kUnitK;
            if ((long long)units + (long long)t * U > (1 << 30))
                break;
            if (!make_map(&gt.map_p[j], x.packed, x.K, x.N / 4, kPRows) ||
                !make_map(&gt.map_x[j], x.xq, x.K, M, BN))
                return cudaErrorInvalidValue;
            gt.g[j] = GroupProj{x.N / 4, U, t, tiles, units, x.w_scale, x.x_scale, x.x_sum,
                                x.y, x.acc_out};
            tiles += t;
            units += t * U;
            ++j;
            ++i;
        }
        if (j == 0)
            return cudaErrorInvalidValue;
        gt.n = j;
        SmallMParams prm = {};
        prm.M = M;
        prm.K = 0;
        prm.plan = kPlanStreamK;
        prm.csize = 1;
        prm.tiles = tiles;
        prm.units_per_tile = 1;  // unused by the group plan
        prm.total_units = units;
        prm.grid = std::min({units, sms, kMaxGrid});
        // slots of partial sums, one per CTA, then one counter per CTA
        if (size_t(prm.grid) * (size_t(BN) * kRows * 4 + 4) > kGroupScratchBytes)
            return cudaErrorInvalidValue;
        prm.ws = scratch;
        prm.cnt = scratch + size_t(prm.grid) * BN * kRows;
        prm.err = device_error_word();
        if (!prm.err)
            return cudaErrorUnknown;
        // consecutive group launches of one call may overlap; the first one
        // overlaps the previous kernel only if the caller allows it
        const bool pdl = first ? overlap_prev : true;
        err = BN == 16 ? launch_group_bn<16>(gt, prm, pdl, stream)
                       : launch_group_bn<32>(gt, prm, pdl, stream);
        if (err != cudaSuccess)
            return err;
        first = false;
    }
    return cudaSuccess;
}

// The stream-K plan with the fixed scratch above. The device address of the
// scratch array is looked up once per device (on that device's first call)
// with cudaGetSymbolAddress; host code cannot use the array's name as a
// device pointer. The part the call uses is zero-filled on `stream` before
// the kernel, so a call never depends on what an earlier call left there.
cudaError_t launch_smallm_tc_noalloc(const uint8_t *packed, float w_scale, const int8_t *xq,
                                     const float *x_scale, const int32_t *x_sum, float *y,
                                     int32_t *acc_out, int M, int N, int K, cudaStream_t stream)
{
    static std::atomic<void *> scratch[64] = {};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess)
        return err;
    if (dev < 0 || dev >= 64)
        return cudaErrorInvalidDevice;
    const size_t need = smallm_workspace_bytes(N, M);
    if (need > kNoAllocScratchBytes)
        return cudaErrorInvalidValue;
    if (!scratch[dev]) {
        void *ptr = nullptr;
        err = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (err != cudaSuccess)
            return err;
        scratch[dev] = ptr;
    }
    err = cudaMemsetAsync(scratch[dev], 0, need, stream);
    if (err != cudaSuccess)
        return err;
    return launch_smallm_streamk(packed, w_scale, xq, x_scale, x_sum, y, acc_out, M, N, K,
                                 scratch[dev], stream);
}

}  // namespace tq
