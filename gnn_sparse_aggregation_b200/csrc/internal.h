// internal.h -- private declarations of libaggraph (host + device).
#pragma once

#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "aggraph.h"

namespace ag {

// Rows with more than kHeavyThreshold edges are split into chunks of
// kChunkEdges edges; each chunk writes an fp32 partial row to scratch, and a
// second kernel adds a heavy row's partials in chunk order.
constexpr int kChunkEdges = 256;
constexpr int64_t kHeavyThreshold = 256;

constexpr size_t kAlign = 256;

inline size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }

// Row schedule of one CSR direction.  `rows` lists every row as
// {row, csr_begin, csr_end, first_chunk} in order of decreasing degree (ties
// by ascending row id): the first n_heavy entries are the split rows, then
// the other non-empty rows, then the empty rows.
struct Direction {
    int32_t *rowptr = nullptr;  // [N+1]
    int32_t *col = nullptr;     // [E] the other endpoint of each CSR position
    int32_t *order = nullptr;   // [E] CSR position -> COO ordinal
    int4 *rows = nullptr;       // [N]
    int4 *chunks = nullptr;     // [n_chunks] {csr_begin, csr_end, row, split-row index}
    int64_t n_heavy = 0, n_chunks = 0, n_nonempty = 0, max_degree = 0;
};

}  // namespace ag

struct ag_graph {
    int device = 0;
    int64_t N = 0, E = 0;
    size_t ws_used = 0;
    ag::Direction dir[2];  // 0: forward CSR (owned by destination), 1: transpose CSR (by source)
};

namespace ag {

// Records a message for ag_last_error() and returns `status`.
int fail(int status, const char *fmt, ...);
int cuda_fail(cudaError_t err, const char *what);
void clear_error();

// AG_OK if p is device (or managed) memory usable on `device`.
int check_device_ptr(const void *p, int device, const char *name);

// Lowering-time workspace layout (shared by the size query and the lowering).
struct Layout {
    size_t rowptr[2], col[2], order[2], rows[2], chunks[2];
    size_t keys_a, vals_a, keys_b, vals_b, hist, scan_tmp, aux, counters;
    size_t total;
};
bool make_layout(int64_t N, int64_t E, Layout *L);
int64_t max_chunks(int64_t E);

}  // namespace ag
