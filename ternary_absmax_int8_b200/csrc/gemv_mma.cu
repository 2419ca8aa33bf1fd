// gemv_mma.cu -- small-batch ternary decode (2 <= M <= 32 tokens) on the
// warp-level integer MMA (mma.sync m16n8k32, u8 x s8 -> s32), one projection
// or a table of projections per launch.
//
// Many concurrent requests turn decode into a skinny contraction (1bit engine
// blog, "One GPU, many users"). Each weight byte then feeds M tokens: dp4a on
// the CUDA cores spends one instruction per 4 bytes per token, while one
// m16n8k32 MMA covers 16 packed rows x 32 columns x 8 tokens. Measured on a
// B200: 0.48 MMA per clock per SM, against 64 dp4a lanes per clock.
//
// The MMA takes the packed bytes themselves, masked. Byte (i, k) of the
// packed tensor is c0 + 4 c1 + 16 c2 + 64 c3 (the codes of rows i + p N/4),
// so with the nested masks 0x03, 0x0F, 0x3F and 0xFF (unsigned bytes) the
// products with the int8 activations give
//   D_j = sum_k (P & mask_j) q = sum_{p <= j} 4^p C_p,   C_p = sum_k c_p q,
// and 4^p C_p = D_p - D_{p-1} exactly; acc = C_p - x_sum (since w = c - 1).
// Three logic ops per 32-bit word make the operands; nothing is expanded.
//
// Operand layout. A lane's A fragment (rows g and g + 8, columns 4t..4t+3
// and 16+4t..16+4t+3 of a 32-column block) is filled from 16 contiguous
// bytes of each row: the kernel maps the physical columns
// k0 + 16t + 8b + {0..7} of each 64-column half of a step to the fragment
// columns of block b (the same permutation for both operands, so the sums
// are unchanged).
// The packed rows therefore stream with 16-byte loads (cp.async into a
// per-warp ring of shared-memory stages; each lane reads back only what it
// loaded), and the activations with 16-byte loads from L1/L2.
//
// Work split. Tiles of 16 packed rows (64 outputs) x the full K, numbered
// across the projections of a launch; each CTA (one per SM, 12 or 16 warps)
// takes a contiguous, byte-balanced range of tiles. Its warps form teams of
// P (any P up to the warp count) that take the range's tiles in turn; the P
// warps of a team split a tile's steps. With many tiles P = 1: a warp owns
// whole tiles and applies the epilogue y = float(acc) * (w_scale * x_scale)
// from its registers, no barrier. With few tiles (one projection, one FFN)
// the team adds its accumulators in shared memory (integer adds, exact in
// any order) behind a named barrier. A warp's loads for its next tile are
// in flight while it finishes the current one.
#include <atomic>
#include <algorithm>
#include <vector>

#include "mma_common.cuh"
#include "tq_internal.h"

namespace tq {

namespace {

// Warps per CTA: 16 up to 8 tokens, 12 for 9..24 (up to 170 registers a
// thread for two or three token groups), 16 beyond; three ring stages of
// 256-column steps up to 16 tokens (what fits next to the warps' accumulator
// slots), four beyond.
template <int NT>
constexpr int kMmaW = NT == 1 ? 16 : (NT <= 3 ? 12 : 16);
// cp.async stages per warp
template <int NT>
constexpr int kRing = NT <= 2 ? 3 : 4;
constexpr int kMmaRows = 16;      // packed rows per tile
// A step is H pieces of 64 columns (H = 4 up to 16 tokens, 2 for 17..24, 1
// beyond, where the accumulators and the prefetched activations take more
// registers and the accumulator slots more shared memory); a stage holds
// [2 rows][H pieces][32 lanes][16 bytes]. Wide steps keep the number of
// separate row streams per SM low: 16-row tiles read as 256-byte row pieces
// by 12 warps move ~6.1 TB/s in a copy-only test, 128-byte pieces by 16 or
// 20 warps 5.1 or 4.2 TB/s (DRAM page locality).
template <int NT>
constexpr int kHalves = NT <= 2 ? 4 : (NT == 3 ? 2 : 1);
template <int NT>
constexpr int kStep = 64 * kHalves<NT>;
template <int NT>
constexpr int kStageBytes = 2 * kHalves<NT> * 32 * 16;

// A warp's walk over the (tile, step) pairs it computes: the tiles of its
// team (t_begin + team, + teams, ...) and, in each, its piece
// [S piece / P, S (piece + 1) / P) of the tile's S steps. The per-tile state
// a lane needs is set once per tile.
struct Cursor {
    int tile;      // global tile index (t_end when done)
    int entry;     // its projection
    int step, step_end;
    int K;
    const uint8_t *row, *row8;  // this lane's rows g and g + 8 at column 16 t
    bool ok0, ok1;              // rows g, g + 8 exist
};

template <int STEP>
struct Walk {
    const MmaEntry *tab;
    int n_ent, t_end, teams, piece, P;
    int t16;  // 16 t: the lane's column offset

    __device__ void start(Cursor &c, int tl, int g) const
    {
        c.tile = tl;
        while (c.entry + 1 < n_ent && tab[c.entry + 1].tile_begin <= tl)
            ++c.entry;
        const MmaEntry &e = tab[c.entry];
        c.K = e.K;
        const int S = (e.K + STEP - 1) / STEP;
        c.step = S * piece / P;
        c.step_end = S * (piece + 1) / P;
        const int r = (tl - e.tile_begin) * kMmaRows + g;
        c.ok0 = r < e.N4;
        c.ok1 = r + 8 < e.N4;
        c.row = e.packed + size_t(r) * e.K + t16;
        c.row8 = c.row + size_t(8) * e.K;
    }
    // from c's current step on, the next pair with a step to compute
    __device__ void settle(Cursor &c, int g) const
    {
        while (c.tile < t_end && c.step >= c.step_end) {
            if (c.tile + teams >= t_end) {
                c.tile = t_end;
                break;
            }
            start(c, c.tile + teams, g);
        }
    }
};

// The epilogue of one output: plane pl of row `row`, token m, from the
// nested sums hi = D_pl and lo = D_{pl - 1}.
__device__ __forceinline__ void store_out(const MmaEntry &e, int M, int row, int m, int pl,
                                          int32_t hi, int32_t lo)
{
    if (m >= M || row >= e.N4)
        return;
    const int32_t acc = ((hi - lo) >> (2 * pl)) - __ldg(e.x_sum + m);
    const float sc = __fmul_rn(e.w_scale, __ldg(e.x_scale + m));
    const size_t out = size_t(m) * (4 * size_t(e.N4)) + size_t(row) + size_t(pl) * e.N4;
    e.y[out] = __fmul_rn(__int2float_rn(acc), sc);
    if (e.acc_out)
        e.acc_out[out] = acc;
}

template <int NT>
__global__ void __launch_bounds__(kMmaW<NT> * 32, 1)
mma_gemv_kernel(const __grid_constant__ MmaParams p)
{
    // per-warp rings: [W][RING] stages of [2 rows][H pieces][32 lanes][16
    // bytes] (16-byte lane slots keep the reads free of bank conflicts),
    // then the teams' accumulator slots [W][4 masks][16 rows][8 NT tokens]
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr int H = kHalves<NT>, STEP = kStep<NT>, SB = kStageBytes<NT>, RING = kRing<NT>;
    constexpr int kRingBytes = RING * SB;
    constexpr int kCols = 8 * NT;
    constexpr int W = kMmaW<NT>;
    int32_t *slots = reinterpret_cast<int32_t *>(smem + W * kRingBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const uint8_t *ring = smem + warp * kRingBytes + lane * 16;
    const uint32_t ring_s = smem_u32(ring);

    const int t_begin = p.cta_tile0[blockIdx.x], t_end = p.cta_tile0[blockIdx.x + 1];
    const int P = p.P, teams = W / P;
    // teams of P warps; warps past the last whole team (W not a multiple of
    // P) stay idle
    const int team = warp / P, piece = warp - team * P;
    const int first = team < teams ? t_begin + team : t_end;
    const Walk<STEP> wk{p.e, p.n_entries, t_end, teams, piece, P, 16 * t};

    if (threadIdx.x == 0)
        pdl_launch_dependents();

    // the load cursor runs RING - 1 steps ahead of the compute cursor
    Cursor lc{t_end, 0, 0, 0, 0, nullptr, nullptr, false, false};
    if (first < t_end) {
        wk.start(lc, first, g);
        wk.settle(lc, g);
    }
    int issued = 0;  // ring slot of the next copy
    auto issue = [&]() {
        const uint32_t dst = ring_s + uint32_t(issued) * SB;
        if (lc.tile < t_end) {
            const int k = lc.step * STEP;  // + 16 t already in the row pointers
            const uint8_t *s0 = lc.row + k, *s1 = lc.row8 + k;
            if (k + STEP <= lc.K) {  // a whole step (warp-uniform)
#pragma unroll
                for (int h = 0; h < H; ++h) {
                    cp_async16(dst + h * 512, s0 + 64 * h, lc.ok0);
                    cp_async16(dst + (H + h) * 512, s1 + 64 * h, lc.ok1);
                }
            } else {
#pragma unroll
                for (int h = 0; h < H; ++h) {
                    const bool kin = k + 64 * h + 16 * t < lc.K;
                    cp_async16(dst + h * 512, s0 + 64 * h, lc.ok0 && kin);
                    cp_async16(dst + (H + h) * 512, s1 + 64 * h, lc.ok1 && kin);
                }
            }
            ++lc.step;
            wk.settle(lc, g);
        }
        cp_async_commit();  // (possibly empty) group per step keeps the count uniform
        issued = issued + 1 == RING ? 0 : issued + 1;
    };
#pragma unroll
    for (int i = 0; i < RING - 1; ++i)
        issue();

    pdl_wait();  // activations, scales, outputs of the previous kernel

    int32_t d[4][NT][4];
    auto zero_acc = [&]() {
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int r = 0; r < 4; ++r)
                    d[j][n][r] = 0;
    };
    zero_acc();
    int consumed = 0;  // ring slot of the next step to compute
    Cursor cc{t_end, 0, 0, 0, 0, nullptr, nullptr, false, false};
    if (first < t_end) {
        wk.start(cc, first, g);
        wk.settle(cc, g);
    }

    int fent = 0;  // projection of `tile`, advanced with it
    while (fent + 1 < p.n_entries && p.e[fent + 1].tile_begin <= t_begin)
        ++fent;
    // The activations of a step (token n 8 + g, the lane's 16 columns of each
    // half), loaded one step ahead so their latency overlaps the MMAs of the
    // step before. A lane whose token n 8 + g is past M reads token M - 1
    // instead: its MMA column only feeds outputs that are never stored.
    // Columns past K read the row's first 16 columns instead (K >= 16): the
    // weights there are zero-filled, so the products vanish.
    uint4 qn[H][NT];
    const int8_t *xrow[NT];  // the lane's token rows at column 16 t, for entry xent
    int xent = -1;
    auto load_q = [&](const Cursor &c) {
        if (c.tile >= t_end)
            return;
        if (c.entry != xent) {
            xent = c.entry;
            const MmaEntry &ce = p.e[xent];
#pragma unroll
            for (int n = 0; n < NT; ++n)
                xrow[n] = ce.xq + size_t(min(n * 8 + g, p.M - 1)) * ce.K + 16 * t;
        }
        const int k = c.step * STEP;
        if (k + STEP <= c.K) {
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int h = 0; h < H; ++h)
                    qn[h][n] = __ldg(reinterpret_cast<const uint4 *>(xrow[n] + k + 64 * h));
        } else {
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int h = 0; h < H; ++h) {
                    const int kk = k + 64 * h + 16 * t < c.K ? k + 64 * h : -16 * t;
                    qn[h][n] = __ldg(reinterpret_cast<const uint4 *>(xrow[n] + kk));
                }
        }
    };
    load_q(cc);

    for (int tile = first; tile < t_end; tile += teams) {
        while (fent + 1 < p.n_entries && p.e[fent + 1].tile_begin <= tile)
            ++fent;
        const MmaEntry &e = p.e[fent];
        while (cc.tile == tile) {
            issue();
            uint4 q[H][NT];
#pragma unroll
            for (int h = 0; h < H; ++h)
#pragma unroll
                for (int n = 0; n < NT; ++n)
                    q[h][n] = qn[h][n];
            ++cc.step;
            wk.settle(cc, g);
            load_q(cc);  // the next step's activations
            cp_async_wait<RING - 1>();
            __syncwarp();
            const uint8_t *src = ring + consumed * SB;
#pragma unroll
            for (int h = 0; h < H; ++h) {
                const uint4 lo4 = *reinterpret_cast<const uint4 *>(src + h * 512);        // row g
                const uint4 hi4 = *reinterpret_cast<const uint4 *>(src + (H + h) * 512);  // row g + 8
                const uint32_t al[4] = {lo4.x, lo4.y, lo4.z, lo4.w};
                const uint32_t ah[4] = {hi4.x, hi4.y, hi4.z, hi4.w};
#pragma unroll
                for (int b = 0; b < 2; ++b) {
                    const uint32_t a0 = al[2 * b], a2 = al[2 * b + 1];
                    const uint32_t a1 = ah[2 * b], a3 = ah[2 * b + 1];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t mk = j == 0 ? 0x03030303u
                                                   : (j == 1 ? 0x0F0F0F0Fu
                                                             : (j == 2 ? 0x3F3F3F3Fu : 0xFFFFFFFFu));
#pragma unroll
                        for (int n = 0; n < NT; ++n) {
                            const uint32_t b0 = b == 0 ? q[h][n].x : q[h][n].z;
                            const uint32_t b1 = b == 0 ? q[h][n].y : q[h][n].w;
                            mma_u8s8(d[j][n], a0 & mk, a1 & mk, a2 & mk, a3 & mk, b0, b1);
                        }
                    }
                }
            }
            consumed = consumed + 1 == RING ? 0 : consumed + 1;
        }
        const int r0 = (tile - e.tile_begin) * kMmaRows;
        if (P == 1) {
            // the warp holds the whole tile: epilogue from registers, the
            // token's scale and sum loaded once for its eight outputs
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int par = 0; par < 2; ++par) {
                    const int m = n * 8 + 2 * t + par;
                    if (m >= p.M)
                        continue;
                    const int32_t xs = __ldg(e.x_sum + m);
                    const float sc = __fmul_rn(e.w_scale, __ldg(e.x_scale + m));
                    const size_t ob = size_t(m) * (4 * size_t(e.N4));
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const int row = r0 + g + 8 * half, hh = 2 * half + par;
                        if (row >= e.N4)
                            continue;
#pragma unroll
                        for (int pl = 0; pl < 4; ++pl) {
                            const int32_t lo = pl > 0 ? d[pl - 1][n][hh] : 0;
                            const int32_t acc = ((d[pl][n][hh] - lo) >> (2 * pl)) - xs;
                            const size_t out = ob + size_t(row) + size_t(pl) * e.N4;
                            e.y[out] = __fmul_rn(__int2float_rn(acc), sc);
                            if (e.acc_out)
                                e.acc_out[out] = acc;
                        }
                    }
                }
            zero_acc();
            continue;
        }
        // the team's P warps add their accumulators: each warp stores its
        // fragments, then the team sums them word by word into the first
        // warp's slot and applies the epilogue
        int32_t *my = slots + warp * (4 * 16 * kCols);
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const int col = n * 8 + 2 * t;
                *reinterpret_cast<int2 *>(my + (j * 16 + g) * kCols + col) =
                    make_int2(d[j][n][0], d[j][n][1]);
                *reinterpret_cast<int2 *>(my + (j * 16 + g + 8) * kCols + col) =
                    make_int2(d[j][n][2], d[j][n][3]);
            }
        zero_acc();
        named_bar_sync(1 + team, 32 * P);
        int32_t *ts = slots + team * P * (4 * 16 * kCols);
        constexpr int kWords = 4 * 16 * kCols;  // per warp slot
        for (int i = (piece * 32 + lane) * 4; i < kWords; i += 32 * P * 4) {
            int4 a = *reinterpret_cast<const int4 *>(ts + i);
            for (int w = 1; w < P; ++w) {
                const int4 b = *reinterpret_cast<const int4 *>(ts + w * kWords + i);
                a.x += b.x;
                a.y += b.y;
                a.z += b.z;
                a.w += b.w;
            }
            *reinterpret_cast<int4 *>(ts + i) = a;
        }
        named_bar_sync(1 + team, 32 * P);
        // output (token m, plane pl, row r), r fastest: 16 consecutive floats
        for (int o = piece * 32 + lane; o < 16 * 4 * p.M; o += 32 * P) {
            const int r = o & 15, pl = (o >> 4) & 3, m = o >> 6;
            store_out(e, p.M, r0 + r, m, pl, ts[(pl * 16 + r) * kCols + m],
                      pl > 0 ? ts[((pl - 1) * 16 + r) * kCols + m] : 0);
        }
        named_bar_sync(1 + team, 32 * P);  // the slots are rewritten by the next tile
    }
    cp_async_wait<0>();
}

template <int NT>
cudaError_t launch_nt(const MmaParams &p, int grid, cudaStream_t stream, bool pdl)
{
    constexpr int W = kMmaW<NT>;
    constexpr size_t smem = size_t(W) * kRing<NT> * kStageBytes<NT> + size_t(W) * 4 * 16 * 8 * NT * 4;
    static_assert(smem <= 227 * 1024, "shared memory");
    static std::atomic<int> configured_dev{-1};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (configured_dev != dev) {
        e = cudaFuncSetAttribute(mma_gemv_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(smem));
        if (e != cudaSuccess)
            return e;
        configured_dev = dev;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(W * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, mma_gemv_kernel<NT>, p);
    return e != cudaSuccess ? e : cudaGetLastError();
}

MmaParams *mma_params()
{
    static thread_local MmaParams p;
    return &p;
}

}  // namespace

cudaError_t launch_mma_gemv(const MmaEntry *entries, int n, int M, bool overlap_prev,
                            cudaStream_t stream)
{
    if (n <= 0)
        return cudaSuccess;
    if (M < 1 || M > kMmaMaxTokens)
        return cudaErrorInvalidValue;
    const int sms = device_sm_count();
    bool first = true;
    for (int base = 0; base < n; base += kMmaStackMax) {
        const int cnt = std::min(n - base, kMmaStackMax);
        MmaParams &p = *mma_params();
        p.n_entries = cnt;
        p.M = M;
        int total = 0;
        for (int j = 0; j < cnt; ++j) {
            p.e[j] = entries[base + j];
            p.e[j].tile_begin = total;
            total += (p.e[j].N4 + kMmaRows - 1) / kMmaRows;
        }
        if (total == 0)
            continue;
        // contiguous tile ranges per CTA, balanced by bytes (plus a fixed
        // cost per tile), one CTA per SM
        const int grid = std::min({total, sms, kMmaMaxGrid});
        const int W = M <= 8 ? kMmaW<1> : (M <= 16 ? kMmaW<2> : (M <= 24 ? kMmaW<3> : kMmaW<4>));
        std::vector<long long> prefix(size_t(total) + 1, 0);
        {
            int tt = 0;
            for (int j = 0; j < cnt; ++j) {
                const MmaEntry &e = p.e[j];
                const int tiles = (e.N4 + kMmaRows - 1) / kMmaRows;
                for (int i = 0; i < tiles; ++i, ++tt)
                    prefix[size_t(tt) + 1] = prefix[size_t(tt)] + (long long)kMmaRows * e.K + 2048;
            }
        }
        p.cta_tile0[0] = 0;
        int max_tiles = 0;
        for (int b = 1; b <= grid; ++b) {
            int tt = total;
            if (b < grid) {
                const long long target = prefix[size_t(total)] * b / grid;
                tt = int(std::lower_bound(prefix.begin(), prefix.end(), target) - prefix.begin());
                tt = std::max(tt, p.cta_tile0[b - 1] + 1);
                tt = std::min(tt, total - (grid - b));
            }
            p.cta_tile0[b] = tt;
            max_tiles = std::max(max_tiles, tt - p.cta_tile0[b - 1]);
        }
        // The warps of a CTA form teams of P that take the range's tiles in
        // turn, splitting each tile's steps. Teams: up to 8 tokens, one per
        // two tiles of the longest range (a team's next tile loads while it
        // finishes the current one); beyond, one per tile, whose steps carry
        // twice the MMAs. With many tiles P = 1 (whole tiles per warp). B200,
        // the FFN projections at 4, 8 and 16 tokens: 2 teams of 8 warps
        // 6.7 / 7.3 us against 8.2 / 8.5 us for one team of 16, 3 teams of
        // 4 warps 9.6 us against 13.0 for one of 8 (12 warps).
        const int teams = std::min(W, M <= 8 ? (max_tiles + 1) / 2 : max_tiles);
        p.P = W / std::max(teams, 1);
        const bool pdl = first ? overlap_prev : true;
        cudaError_t e;
        if (M <= 8)
            e = launch_nt<1>(p, grid, stream, pdl);
        else if (M <= 16)
            e = launch_nt<2>(p, grid, stream, pdl);
        else if (M <= 24)
            e = launch_nt<3>(p, grid, stream, pdl);
        else
            e = launch_nt<4>(p, grid, stream, pdl);
        if (e != cudaSuccess)
            return e;
        first = false;
    }
    return cudaSuccess;
}

}  // namespace tq
