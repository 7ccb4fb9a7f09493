// Internal declarations shared by the C-ABI host code and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "skv.h"

namespace skv {

// ---------------------------------------------------------------------------
// coarsening
// ---------------------------------------------------------------------------
constexpr int kTileRows = 512;              // rows a projection tile computes (1 halo + outputs)
constexpr int kTileOut = kTileRows - 1;     // middle tokens per projection tile

// Per-sequence plan, computed on the host and copied into the workspace.
struct SeqRow {
    int64_t row_off;   // first row of the sequence in the packed [rows][d] view of k / v
    int64_t mid_off;   // first index of the sequence in the per-middle-token scratch arrays
    int32_t T, N;      // tokens, middle segments
    int32_t s_eff, w_eff, M;
    int32_t tiles;     // projection tiles per head: ceil(M / kTileOut)
    int32_t bnd_off;   // first index of the sequence in the boundary scratch (Hkv * (N + 1) each)
    int32_t ent_off;   // first index of the sequence in the entry scratch (Hkv * emax each)
    int32_t emax;      // entries a head can produce: s_eff + (M > 0 ? N : 0) + w_eff
    int32_t pad;
};
static_assert(sizeof(SeqRow) == 56, "SeqRow layout");

struct SeqTable {
    SeqRow rows[SKV_MAX_SEQS];
};

// Projection transposed for the kernels: pt[j][i] = P[i][j], j < 2d, i < 16.
struct ProjT {
    float pt[2 * 128 * SKV_PROJ_DIM];
};

// The tensor-core projection's B operand: P16 = bf16(P) (round to nearest even) as the image the
// MMAs read from shared memory: for each 32-feature chunk c (features 32 c .. 32 c + 31 of [k; v]),
// 16 rows of 64 bytes (row n = output n), the row's four 16-byte granules g (features 32 c + 8 g ..
// + 7) stored at granule position g ^ ((n >> 1) & 3) -- the 64-byte swizzle of the TMA-loaded
// token chunks. Chunk c's image starts at byte 1024 c; d = 64 uses the first half.
struct alignas(16) ProjFrag {
    uint32_t w[(2 * 128 / 32) * 16 * 64 / 4];
};

struct CoarsenArgs {
    const void *k, *v;
    int B, Hkv, d, dtype;
    int max_tiles;   // largest tiles per head over the batch
    int max_emax;    // largest emax over the batch
    int Nmax;        // largest N over the batch
    const SeqRow *seq;
    int64_t *tile_total, *unit_total, *local_scan;
    int32_t *bounds;
    int2 *ents;
    uint32_t *flags;
    uint8_t *pages;  // node pool: [num_pages][2 * 16 * d * elem + 128]
    int64_t num_pages;
    const int32_t *page_table;
    int max_pages;
    int32_t *lens;
    int32_t *user_bounds;
    int64_t *cumvar;
    int representative;  // skv_representative of the middle segments' stored key and value
    int closure;         // skv_closure: SKV_CLOSURE_DIAGONAL also writes per-dimension variances
    int center;          // 1: keys enter every stage with the unit's mean key removed
    int projection;      // skv_projection: SKV_PROJECTION_TENSOR_BF16 selects k_project_tc
    int max_blk;         // largest ceil(T / kMeanBlock) over the batch
    float *key_blk;      // [units][max_blk][d] per-block key sums (centring only)
    float *key_mu;       // [units][d] mean key of each unit (centring only)
};

constexpr int kMeanBlock = 256;   // tokens per block of the centring mean's fixed summation order

// Workspace carve-up (offsets in bytes from the workspace start).
struct CoarsenLayout {
    size_t seq, tile_total, unit_total, local_scan, bounds, ents, key_blk, key_mu, total;
};

// Host-side launchers (coarsen.cu).
// ---------------------------------------------------------------------------
// streaming coarsening state (per unit, one block of unit_bytes in the caller's state buffer)
// ---------------------------------------------------------------------------
struct StreamHdr {
    long long cT;      // cumulative quantised variation of the middle
    int n_nodes;       // middle nodes
    int T;             // tokens so far
    int ring;          // recent ring position of the oldest recent token
    int n_ent;         // entries (= lens)
    int N, S, W;       // segment count, sinks, recent window
    int open;          // entry of the open (last) middle node
    int open_page;     // its page id
    int pad[5];
    float z_last[16];  // feature of the last middle token
};
static_assert(sizeof(StreamHdr) == 128, "StreamHdr layout");

struct StreamArgs {
    const void *k_new, *v_new;   // [B][Hkv][d] (append)
    int B, Hkv, d, dtype;
    uint8_t *pages;
    int64_t num_pages;
    const int32_t *page_table;
    int max_pages;
    int32_t *lens;
    uint8_t *state;              // the units' blocks (after the projection block)
    float *pt;                   // P^T [2d][16] kept in the state buffer's first block
    int64_t unit_bytes;          // state bytes per unit
    int NM, Ecap;                // node-order capacity, entry capacity per unit
    int64_t off_order, off_recent, off_owner, off_m, off_start, off_V, off_M2, off_mk, off_mv;
    // kept so that an append finds everything it needs one round trip after the header:
    int64_t off_vord;     // [NM] int64 V of the middle nodes in node order (beside order)
    int64_t off_rpage;    // [W] int32 page id of each recent ring position's pool slot
    int64_t off_ring;     // [W][2][d] fp32 raw key and value of each recent ring position
    uint32_t *flags;
};

// Byte layout of one unit's state for entry capacity Ecap and recent window W (offsets 256-aligned).
void stream_layout(int d, int Ecap, int W, StreamArgs *s);

cudaError_t launch_stream_init(const CoarsenArgs &a, const StreamArgs &s, const ProjT &proj, cudaStream_t st);
cudaError_t launch_stream_append(const StreamArgs &s, cudaStream_t st);

// bytes at the start of a streaming state buffer that hold P^T (then the units' blocks)
constexpr int64_t kStreamProjBytes = 2 * 128 * SKV_PROJ_DIM * 4;

cudaError_t launch_coarsen(const CoarsenArgs &a, const SeqTable &table, const ProjT &proj, const ProjFrag &frag,
                           const CUtensorMap &map_k, const CUtensorMap &map_v, cudaStream_t s);

// ---------------------------------------------------------------------------
// decode
// ---------------------------------------------------------------------------
constexpr int kRowsPerPass = 32;    // query rows one pass over a unit's pages serves
constexpr int kMaxDecodeCtas = 1024;
constexpr int kMaxVUnits = 8192;

struct DecodeArgs {
    const void *q;
    const uint8_t *pages;  // node pool: [num_pages][2 * 16 * d * elem + 128]
    int64_t num_pages;
    const int32_t *page_table;
    int max_pages;
    const int32_t *lens;
    void *out;
    float *lse;
    int B, R, Hq, Hkv, G, d, dtype;
    int rows;         // R * G query rows per unit
    int row_passes;   // ceil(rows / kRowsPerPass)
    int pass_rows;    // rows a pass holds: min(kRowsPerPass, rows rounded up to 8)
    int n_vunits;     // B * Hkv * row_passes
    int ncta;         // CTAs of the split kernel
    int cluster;      // CTAs per thread-block cluster (1: no clusters)
    float *part_v;    // [ncta][2][pass_rows][d] split partial outputs (normalised)
    float *part_l;    // [ncta][2][pass_rows] split partial log2-partitions
    int32_t *counters;   // [n_vunits] pieces finished per virtual unit (zero between calls)
    uint32_t *flags;
    int closure;         // skv_closure of the pool (SKV_CLOSURE_DIAGONAL: pages carry variances)
};

struct DecodeLayout {
    size_t counters, part_v, part_l, total;
};

// Query-row geometry of one decode call and its workspace layout (split partials sized for the
// largest grid, kMaxDecodeCtas).
struct DecodePlan {
    int rows, row_passes, pass_rows, n_vunits;
    DecodeLayout lay;
};

// Host-side checks and geometry shared by every decode entry point (skv_api.cu).
skv_status plan_decode(int dtype, int B, int R, int Hq, int Hkv, int d, int max_pages, DecodePlan *plan);
// Workspace layout for a grid of ncta CTAs (flags header, counters, split partials).
DecodeLayout decode_layout(int dtype, int d, const DecodePlan &plan, int ncta);
// plan_decode plus the buffer checks; fills every DecodeArgs field except the workspace pointers
// (part_v, part_l, counters, flags) and the grid (ncta, cluster).
skv_status decode_args(const void *q, int dtype, int B, int R, int Hq, int Hkv, int d, const skv_node_pool *pool,
                       const int32_t *page_table, int max_pages, const int32_t *lens, void *out, float *lse,
                       int closure, DecodePlan *plan, DecodeArgs *args);

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s);
cudaError_t decode_split_ctas(const DecodeArgs &a, int *ncta);

}  // namespace skv
