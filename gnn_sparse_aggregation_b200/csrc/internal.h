// internal.h -- private declarations of libaggraph (host + device).
#pragma once

#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "aggraph.h"

namespace ag {

// Per-call kernels walk the CSR in tiles of `tile_edges` consecutive
// positions (a power of two between kMinTileEdges and kMaxTileEdges, chosen
// at lowering so that there are enough tiles to fill the GPU).  A row cut by
// a tile boundary leaves one fp32 partial row per tile, and a second kernel
// adds a row's partials in tile order.  Rows cut into more than
// kLongSpanTiles + 1 tiles are added up by a whole CTA.  (At R-MAT-22 tiles
// of 256 positions ran the step 0.6 % and the weight gradient 6 % faster
// than tiles of 512 with the 128-thread ring blocks; 1024 was slower.)
constexpr int kMaxTileEdges = 256;
constexpr int kMinTileEdges = 32;
constexpr int kFillGroups = 148 * 64;  // tiles wanted: SMs x resident lane groups
constexpr int kLongSpanTiles = 8;
// Weights (and the weight gradient) are regrouped per call into windows of
// 2^kWindowShift consecutive CSR positions (4 MB of fp32), so that the
// per-edge weight lookups of a tile stay inside one L2-resident window.
#ifndef AG_WINDOW_SHIFT
#define AG_WINDOW_SHIFT 20
#endif
constexpr int kWindowShift = AG_WINDOW_SHIFT;
// The per-call regrouping passes move the weights of kStageChunk consecutive
// COO ordinals at a time; stage_delta[c * windows + b] turns the slot of an
// ordinal of chunk c in window b into its position in the chunk sorted by
// window (slot + delta).  Built when the graph has at most kStageMaxWindows
// windows.
constexpr int kStageChunk = 2048;  // (R-MAT-22 step 1 % faster than with 4096; 1024 slower)
constexpr int kStageMaxWindows = 256;

constexpr size_t kAlign = 256;

inline size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }

// Schedule of one CSR direction.
struct Direction {
    int32_t *rowptr = nullptr;     // [N+1]
    int32_t *col = nullptr;        // [E] the other endpoint of each CSR position
    int32_t *order = nullptr;      // [E] CSR position -> COO ordinal
    int32_t *nz_rows = nullptr;    // [n_nz] rows with at least one edge, ascending
    int32_t *nz_rowptr = nullptr;  // [n_nz + 1] first CSR position of each, then E
    int32_t *zero_rows = nullptr;  // [N - n_nz] rows without edges, ascending
    int32_t *tile_nz = nullptr;    // [n_tiles] index into nz_rows of the row holding the tile's first position
    int4 *spans = nullptr;         // [n_span] {row, first tile, last tile, 0}: long spans first
    // window-bucketed weight layout: bucket_of_coo[e] is the slot of COO
    // ordinal e, bucket_of_pos[p] the slot read at CSR position p (slots of a
    // window are that window's CSR positions, filled in COO order)
    int32_t *bucket_of_coo = nullptr;  // [E]
    int32_t *bucket_of_pos = nullptr;  // [E]
    int32_t *stage_delta = nullptr;    // [chunks * windows] or null
    int64_t n_nz = 0, n_span = 0, n_span_long = 0, max_degree = 0;
};

}  // namespace ag

struct ag_graph {
    int device = 0;
    int64_t N = 0, E = 0;
    int tile_edges = ag::kMaxTileEdges;
    int64_t n_tiles = 0;
    size_t ws_used = 0;
    int32_t *coo_src = nullptr;  // [E] copies of the COO endpoints (edge identity)
    int32_t *coo_dst = nullptr;
    // fraction of transpose-CSR positions whose COO ordinal shares a 32-byte
    // dw sector with the previous position's: high when the COO list is
    // (nearly) sorted by source, ~0 for an arbitrary edge order
    double dw_locality = 0.0;
    ag::Direction dir[2];  // 0: forward CSR (owned by destination), 1: transpose CSR (by source)
};

namespace ag {

// Records a message for ag_last_error() and returns `status`.
int fail(int status, const char *fmt, ...);
int cuda_fail(cudaError_t err, const char *what);
void clear_error();

// AG_OK if p is device (or managed) memory usable on `device`.
int check_device_ptr(const void *p, int device, const char *name);
// AG_OK if the calling thread's current device is the graph's device.
int check_current_device(const ag_graph *g, const char *fn);

// Lowering-time workspace layout (shared by the size query and the lowering).
struct Layout {
    size_t rowptr[2], col[2], order[2], nz_rows[2], nz_rowptr[2], zero_rows[2], tile_nz[2], spans[2];
    size_t bucket_a[2], bucket_b[2], stage_delta[2];
    size_t coo_src, coo_dst;
    size_t keys_a, vals_a, keys_b, vals_b, hist, scan_tmp, aux, counters;
    size_t total;
};
bool make_layout(int64_t N, int64_t E, Layout *L);
inline int64_t n_windows(int64_t E) { return E > 0 ? ((E - 1) >> kWindowShift) + 1 : 0; }
inline int64_t n_stage_chunks(int64_t E) { return (E + kStageChunk - 1) / kStageChunk; }
inline bool staged_regroup(int64_t E) { return E > 0 && n_windows(E) <= kStageMaxWindows; }
int pick_tile_edges(int64_t E);
inline int64_t n_tiles_for(int64_t E, int T) { return (E + T - 1) / T; }

// Shared with the attention kernels (defined in aggregate.cu).
// Byte offsets, inside the per-call SpMM scratch of width H, of its two
// per-edge float arrays (after the partial rows of rows cut by tiles).
size_t spmm_scratch_edge_offset(const ag_graph *g, int64_t H, int which);
// out_b[bucket slot of COO edge e] = in[e] for the walk direction d: COO
// order into the window-bucketed order the walks read through bucket_of_pos.
void regroup_to_buckets(const ag_graph *g, int d, const float *in, float *out_b, cudaStream_t st);
// out_b[bucket slot of COO edge e] = a[e] * b[e] for the walk direction d.
void regroup_product_to_buckets(const ag_graph *g, int d, const float *a, const float *b, float *out_b,
                                cudaStream_t st);
// out[e] = in_b[bucket slot of COO edge e]: back to COO order.
void regroup_from_buckets(const ag_graph *g, int d, const float *in_b, float *out, cudaStream_t st);
// out[r].x = sum of a_b over the forward-CSR positions of every row r with
// edges (a_b in the forward walk's window slots), in a fixed order; rows
// without edges are not written.  partial: float2 [2 * tiles].
int row_sums(const ag_graph *g, const float *a_b, float2 *partial, float2 *out, cudaStream_t st);
// The SDDMM of direction d: out_b[slot of CSR position p] = dot(R[row of p], F[col[p]]).
int sddmm_bucketed(const ag_graph *g, int d, const void *R, const void *F, float *out_b, int64_t H, int dtype,
                   cudaStream_t st);


}  // namespace ag
