// tq_internal.h -- launch-parameter structs and launchers shared between the
// C ABI (tq_api.cu) and the kernel files. Not installed; not part of the ABI.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "tq_device.cuh"

namespace tq {

// ---------------------------------------------------------------- quantise
constexpr int kMaxQuantStack = 512;  // projections per stack quantiser launch

// One projection's M token rows ([M, K] bf16 in, [M, K] codes and [M] scales
// and sums out); row0 = the launch's index of its first row.
struct QuantStackEntry {
    const uint16_t *x;
    int8_t *xq;
    float *x_scale;
    int32_t *x_sum;
    int K, M;
    int row0, pad_;
};

struct QuantStackParams {
    int n;     // entries
    int rows;  // sum of their M
    QuantStackEntry e[kMaxQuantStack];
};

cudaError_t launch_quant_rows(const uint16_t *x, int8_t *xq, float *x_scale, int32_t *x_sum,
                              int M, int K, cudaStream_t stream);
// One CTA per row while rows are few, one warp per row from 8 rows per SM.
cudaError_t launch_quant_stack(const QuantStackParams &p, cudaStream_t stream);

// ------------------------------------------------- streaming GEMV (M <= 4)
// One entry = one projection. The projection's packed rows are cut into
// tiles of `rows_per_tile` consecutive packed rows (a contiguous byte range);
// global tile t of the launch belongs to the entry with the largest
// tile_begin <= t. Each row of a tile is cut into 2^ksplit pieces along K,
// so that rows_per_tile << ksplit work items keep every consumer warp busy.
struct StreamEntry {
    const uint8_t *packed;  // [N4, K]
    const void *xin;        // [M, K] bf16 (quantising modes 1, 2) or fp32 gate (mode 3)
    const float *gain;      // [K] RMSNorm gain (modes 2, 3)
    const float *up;        // [M, K] fp32 up (mode 3)
    int8_t *xq;             // [M, K] (written when the launch quantises, else read)
    float *x_scale;         // [M]    (likewise)
    int32_t *x_sum;         // [M]    (likewise)
    float *y;               // [M, 4*N4]
    int32_t *acc_out;       // [M, 4*N4] or null
    float w_scale;
    float eps;              // RMSNorm epsilon (modes 2, 3)
    int N4;
    int K;
    int rows_per_tile;
    int ksplit;             // bits 0-7: log2 of the pieces each row is cut into
                            // along K; bits 8-9: lanes per row = 8 << value
    int tile_begin;
};

constexpr int kStreamMaxTokens = 4;     // tokens per launch of the streaming kernel
constexpr int kStreamMaxRows = 16;      // rows_per_tile upper bound
constexpr int kStreamMaxK = 32768;

constexpr int kStreamMaxGridFwd = 320;

template <int MaxE>
struct StreamParams {
    int n_entries;
    int total_tiles;
    int M;             // tokens, 1..kStreamMaxTokens
    int x_slot;        // bytes of resident activations (one-entry launches), else 0
    int w_slot;        // bytes of a ring stage (a tile's packed rows + activations)
    int stages;
    int overlap_prev;  // start weight copies before the previous grid completes
    int quant;         // the launch quantises (M == 1): 0 no (xq is an input); 1 absmax of
                       // bf16 x; 2 RMSNorm of bf16 x, then absmax; 3 relu(gate)^2 * up, then
                       // RMSNorm and absmax
    int head_bytes;    // shared memory for the entry table and the per-token scales
    unsigned *err;     // the library's device error word
    // Work split: CTA b streams tiles cta_tile0[b] .. cta_tile0[b+1]-1 (a
    // contiguous range, balanced by bytes), which belong to entries
    // cta_entry0[b] .. cta_entry0[b] + cta_nent[b] - 1.
    int cta_tile0[kStreamMaxGridFwd + 1];
    int cta_entry0[kStreamMaxGridFwd];
    int cta_nent[kStreamMaxGridFwd];
    StreamEntry e[MaxE];
};

constexpr int kStreamStackMax = 256;  // entries per launch (kernel parameters <= 32 KB)
constexpr int kStreamMaxGrid = kStreamMaxGridFwd;  // CTAs per launch

struct StreamLaunch {
    int grid;
    int consumer_warps;
    size_t smem_bytes;
};

// Plan tiles for a set of entries (fills rows_per_tile, ksplit, tile_begin,
// total_tiles, x_slot, w_slot, stages) and launch. `single` selects the
// small-launch heuristics for one projection. With `quant` (M == 1 only; the
// modes of StreamParams::quant) the kernel computes each entry's activation
// codes itself and writes xq, x_scale and x_sum as the standalone kernels
// would.
cudaError_t launch_stream_gemv(StreamEntry *entries, int n, int M, bool overlap_prev,
                               bool single, int quant, cudaStream_t stream);

int device_sm_count();

// ---------------------------------------- batched decode on the tensor cores
// 1 <= M <= 32. Thread-block clusters split a tile's K range when there are
// fewer tiles than SMs; no scratch memory is involved.
cudaError_t launch_smallm_tc(const uint8_t *packed, float w_scale, const int8_t *xq,
                             const float *x_scale, const int32_t *x_sum, float *y,
                             int32_t *acc_out, int M, int N, int K, cudaStream_t stream);

// Bytes of zero-filled scratch the stream-K formulation of the same kernel
// needs (its split-K partial sums and per-tile counters).
size_t smallm_workspace_bytes(int N, int M);

// The stream-K formulation on a fixed, statically allocated device scratch
// (no allocation by anyone); cudaErrorInvalidValue when the shape needs more
// than noalloc_scratch_capacity() bytes of it.
size_t noalloc_scratch_capacity();

// Group plan of the batched-decode kernel: several projections (N > 0,
// K > 0) at 5 <= M <= 32 tokens, up to 64 per launch, one stream-K partition
// over all of their tiles; split tiles finish through a fixed device scratch
// (one slot per CTA) that every launch leaves zeroed. With overlap_prev the
// first launch may start while the previous kernel on the stream drains
// (programmatic dependent launch); later launches of the call always may.
struct GroupEntry {
    const uint8_t *packed;
    float w_scale;
    const int8_t *xq;
    const float *x_scale;
    const int32_t *x_sum;
    float *y;
    int32_t *acc_out;
    int N, K;
};
cudaError_t launch_smallm_group(const GroupEntry *e, int n, int M, bool overlap_prev,
                                cudaStream_t stream);
// After a device error was reported: the next group call refills the scratch.
void group_scratch_mark_dirty();
cudaError_t launch_smallm_tc_noalloc(const uint8_t *packed, float w_scale, const int8_t *xq,
                                     const float *x_scale, const int32_t *x_sum, float *y,
                                     int32_t *acc_out, int M, int N, int K, cudaStream_t stream);

// ------------------------------- small-batch decode on the warp MMA (M <= 32)
// One entry = one projection (packed [N4, K], activations [M, K], outputs
// [M, 4 N4]); tile_begin is filled by the launcher.
struct MmaEntry {
    const uint8_t *packed;
    const int8_t *xq;
    const float *x_scale;
    const int32_t *x_sum;
    float *y;
    int32_t *acc_out;
    float w_scale;
    int N4, K;
    int tile_begin;
};

constexpr int kMmaMaxTokens = 32;
constexpr int kMmaStackMax = 256;  // entries per launch
constexpr int kMmaMaxGrid = 320;   // CTAs per launch

struct MmaParams {
    int n_entries, M;
    int P;  // warps per team (each tile's K is split over a team)
    int cta_tile0[kMmaMaxGrid + 1];
    MmaEntry e[kMmaStackMax];
};

// One launch per 256 projections; with overlap_prev the first may start
// while the previous kernel on the stream drains (its weights are not being
// written), later ones always may.
cudaError_t launch_mma_gemv(const MmaEntry *entries, int n, int M, bool overlap_prev,
                            cudaStream_t stream);

// ----------------------------------------- prompt processing (M >= 33)
// One projection of a prefill launch: packed [N/4, K], activations [M, K],
// outputs [M, N]. A launch takes up to kPrefillMaxGroup projections; their
// 128-feature x BN-token tiles are dealt to persistent CTAs longest first.
struct PrefillEntry {
    const uint8_t *packed;
    float w_scale;
    const int8_t *xq;
    const float *x_scale;
    const int32_t *x_sum;
    float *y;
    int32_t *acc_out;
    int N, K;
};

constexpr int kPrefillMaxGroup = 16;    // projections per call
constexpr int kPrefillMaxTiles = 4096;  // tiles per launch (more: several launches)
constexpr int kPrefillMaxGrid = 160;    // CTAs per launch

// *handled = false (and nothing launched) for M < 33; cudaErrorInvalidValue
// for more than kPrefillMaxGroup projections or shapes beyond the tile
// fields (N > 2^21 or M > 2^22).
cudaError_t launch_prefill_group(const PrefillEntry *e, int n, int M, cudaStream_t stream,
                                 bool *handled);
cudaError_t launch_prefill_tc(const uint8_t *packed, float w_scale, const int8_t *xq,
                              const float *x_scale, const int32_t *x_sum, float *y,
                              int32_t *acc_out, int M, int N, int K, cudaStream_t stream,
                              bool *handled);

// ------------------------------------------ decoder-layer neighbours, absmean
// input: 0 = bf16 x, 1 = fp32 x, 2 = relu(x_f32)^2 * up. One CTA per row.
cudaError_t launch_rms_quant(int input, const uint16_t *x_bf16, const float *x_f32,
                             const float *up, const float *gain, float eps, int8_t *xq,
                             float *x_scale, int32_t *x_sum, int M, int K, cudaStream_t stream);
cudaError_t launch_absmean_pack(const uint16_t *w, uint8_t *packed, float *w_scale, int N, int K,
                                cudaStream_t stream);

// ------------------------------------------- Hadamard-rotated 4-bit codes
// One CTA per token row; n (the rotation's block size) in {32, ..., 1024}
// dividing K (cudaErrorInvalidValue otherwise).
cudaError_t launch_hadamard_quant4(const uint16_t *x, int8_t *xq, float *x_scale,
                                   int32_t *x_sum, int M, int K, int n, cudaStream_t stream);
// The same over a table of projections' rows in one launch (entries as the
// stack quantiser's; every K a multiple of n, max_k their largest K).
cudaError_t launch_hadamard_quant4_stack(const QuantStackParams &p, int max_k, int n,
                                         cudaStream_t stream);

// --------------------------------------------- binary g128 GEMV (M <= 4)
// One entry = one projection: bits uint8 [N8, K] (bit p of byte (i, k) = row
// i + p N8, 1 = +1), scales fp16 [N8, K/128, 8]. Tiles of rows_per_tile whole
// packed rows; each row is cut into 2^lg pieces of its groups.
struct BinEntry {
    const uint8_t *bits;
    const uint16_t *scales;
    const int8_t *xq;       // [M, K]
    const float *x_scale;   // [M]
    float *y;               // [M, 8 N8]
    int32_t *acc_out;       // [M, 8 N8] or null: sum_k w q
    int N8, K;
    int rows_per_tile, lg, tile_begin, pad_;
};

constexpr int kBinMaxTokens = 4;
constexpr int kBinStackMax = 128;   // entries per launch
constexpr int kBinMaxGrid = 160;    // CTAs per launch

template <int MaxE>
struct BinParams {
    int n_entries, total_tiles, M, stages;
    int w_slot;      // bytes of a ring stage (a tile's bits, then its scales)
    int x_slot;      // bytes of the CTA's resident activations
    int q_slot;      // bytes of the per-token group sums of the activations
    int head_bytes;  // shared memory for the entry table and per-entry offsets
    unsigned *err;
    int cta_tile0[kBinMaxGrid + 1];
    int cta_entry0[kBinMaxGrid];
    int cta_nent[kBinMaxGrid];
    BinEntry e[MaxE];
};

// The one-token (M = 1) form on the warp-level MMA: 16-row tiles over all
// projections, per-CTA ranges balanced by bytes, teams of 2^lgP warps.
struct BinMmaEntry {
    const uint8_t *bits;
    const uint16_t *scales;
    const int8_t *xq;
    const float *x_scale;
    float *y;
    int32_t *acc_out;
    int N8, K;
    int tile_begin, pad_;
};

struct BinMmaParams {
    int n_entries, lgP;
    int cta_tile0[kBinMaxGrid * 2 + 1];
    BinMmaEntry e[kBinStackMax];
};

// M == 1: the warp-MMA kernel; M = 2..4: the dp4a kernel.
cudaError_t launch_binary_gemv(BinEntry *entries, int n, int M, cudaStream_t stream);

// Device address of the library's error word on the current device.
unsigned *device_error_word();

}  // namespace tq
