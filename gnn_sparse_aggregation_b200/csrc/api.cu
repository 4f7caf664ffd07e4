// api.cu -- status handling, pointer checks, workspace layout and handle
// accessors of libaggraph.  The lowering lives in lower.cu, the per-call
// kernels in aggregate.cu and attention.cu.
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "internal.h"

namespace ag {

static thread_local char g_err[512] = "";

int fail(int status, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return status;
}

int cuda_fail(cudaError_t err, const char *what) {
    return fail(AG_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(err), cudaGetErrorName(err));
}

void clear_error() { g_err[0] = '\0'; }

int check_current_device(const ag_graph *g, const char *fn) {
    int cur = -1;
    cudaError_t err = cudaGetDevice(&cur);
    if (err != cudaSuccess) return cuda_fail(err, fn);
    if (cur != g->device)
        return fail(AG_ERR_DEVICE, "%s: current device %d, but the graph lives on device %d", fn, cur, g->device);
    return AG_OK;
}

int check_device_ptr(const void *p, int device, const char *name) {
    cudaPointerAttributes attr;
    cudaError_t err = cudaPointerGetAttributes(&attr, p);
    if (err != cudaSuccess) {
        cudaGetLastError();  // this query's error is not sticky; clear it
        return fail(AG_ERR_DEVICE, "%s: pointer %p is not known to CUDA (%s)", name, p,
                    cudaGetErrorString(err));
    }
    if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
        return fail(AG_ERR_DEVICE, "%s: pointer %p is not device memory", name, p);
    if (attr.type == cudaMemoryTypeDevice && attr.device != device)
        return fail(AG_ERR_DEVICE, "%s: pointer %p lives on device %d, graph is on device %d",
                    name, p, attr.device, device);
    return AG_OK;
}

int pick_tile_edges(int64_t E) {
    int T = kMaxTileEdges;
    while (T > kMinTileEdges && n_tiles_for(E, T) < kFillGroups) T >>= 1;
    return T;
}

static size_t scan_tmp_elems(size_t n) {
    // one exclusive-scan level per 2048-element tile, recursively, each with a total slot
    size_t total = 0;
    while (n > 2048) {
        n = (n + 2047) / 2048;
        total += align_up(n + 1, 64);
    }
    return total + 64;
}

bool make_layout(int64_t N, int64_t E, Layout *L) {
    if (N < 1 || N >= (int64_t(1) << 31) || E < 0 || E >= (int64_t(1) << 31)) return false;
    const size_t n = size_t(N), e = size_t(E);
    const size_t m = n > e ? n : e;
    const size_t tile = 4096;  // radix tile: 256 threads x 16 keys
    const size_t nblk = (m + tile - 1) / tile;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t at = off;
        off += align_up(bytes ? bytes : 1);
        return at;
    };
    const size_t tiles = size_t(n_tiles_for(E, pick_tile_edges(E)));
    for (int d = 0; d < 2; ++d) {
        L->rowptr[d] = take((n + 1) * 4);
        L->col[d] = take(e * 4);
        L->order[d] = take(e * 4);
        L->nz_rows[d] = take(n * 4);
        L->nz_rowptr[d] = take((n + 1) * 4);
        L->zero_rows[d] = take(n * 4);
        L->tile_nz[d] = take(tiles * 4);
        L->spans[d] = take((tiles < n ? tiles : n) * 16);  // a tile boundary cuts at most one row
        L->bucket_a[d] = take(e * 4);
        L->bucket_b[d] = take(e * 4);
        L->stage_delta[d] = take(staged_regroup(E) ? size_t(n_stage_chunks(E) * n_windows(E)) * 4 : 0);
    }
    L->coo_src = take(e * 4);
    L->coo_dst = take(e * 4);
    // lowering temporaries (unused after ag_graph_lower returns); +1 for scan totals
    L->keys_a = take((m + 1) * 4);
    L->vals_a = take((m + 1) * 4);
    L->keys_b = take((m + 1) * 4);
    L->vals_b = take((m + 1) * 4);
    L->hist = take((256 * nblk + 1) * 4);  // +1: the in-place scan writes its total at [n]
    size_t scan_n = 256 * nblk + 1 > n + 1 ? 256 * nblk + 1 : n + 1;
    L->scan_tmp = take(scan_tmp_elems(scan_n) * 4);
    L->aux = take((n + 1) * 4);
    L->counters = take(64 * 8);
    L->total = off;
    return true;
}

}  // namespace ag

using namespace ag;

extern "C" {

size_t ag_graph_workspace_bytes(int64_t N, int64_t E) {
    Layout L;
    if (!make_layout(N, E, &L)) return 0;
    return L.total;
}

int ag_graph_arrays(const ag_graph *g, const int32_t **rowptr_f, const int32_t **col_f,
                    const int32_t **edge_order, const int32_t **rowptr_t, const int32_t **col_t,
                    const int32_t **transpose_order) {
    if (!g) return fail(AG_ERR_INVALID_ARG, "ag_graph_arrays: null graph");
    if (rowptr_f) *rowptr_f = g->dir[0].rowptr;
    if (col_f) *col_f = g->dir[0].col;
    if (edge_order) *edge_order = g->dir[0].order;
    if (rowptr_t) *rowptr_t = g->dir[1].rowptr;
    if (col_t) *col_t = g->dir[1].col;
    if (transpose_order) *transpose_order = g->dir[1].order;
    return AG_OK;
}

int ag_graph_get_stats(const ag_graph *g, ag_graph_stats *out) {
    if (!g || !out) return fail(AG_ERR_INVALID_ARG, "ag_graph_get_stats: null argument");
    memset(out, 0, sizeof *out);
    out->N = g->N;
    out->E = g->E;
    out->device = g->device;
    out->tile_edges = g->tile_edges;
    out->tiles = g->n_tiles;
    out->max_degree_f = g->dir[0].max_degree;
    out->max_degree_t = g->dir[1].max_degree;
    out->nonempty_rows_f = g->dir[0].n_nz;
    out->spanning_rows_f = g->dir[0].n_span;
    out->long_spanning_rows_f = g->dir[0].n_span_long;
    out->nonempty_rows_t = g->dir[1].n_nz;
    out->spanning_rows_t = g->dir[1].n_span;
    out->long_spanning_rows_t = g->dir[1].n_span_long;
    out->workspace_bytes_used = g->ws_used;
    out->dw_locality = g->dw_locality;
    return AG_OK;
}

void ag_graph_free(ag_graph *g) { delete g; }

const char *ag_last_error(void) { return g_err; }

const char *ag_status_string(int status) {
    switch (status) {
        case AG_OK: return "AG_OK";
        case AG_ERR_INVALID_ARG: return "AG_ERR_INVALID_ARG";
        case AG_ERR_SHAPE: return "AG_ERR_SHAPE";
        case AG_ERR_DTYPE: return "AG_ERR_DTYPE";
        case AG_ERR_DEVICE: return "AG_ERR_DEVICE";
        case AG_ERR_INDEX_RANGE: return "AG_ERR_INDEX_RANGE";
        case AG_ERR_CUDA: return "AG_ERR_CUDA";
        case AG_ERR_WORKSPACE: return "AG_ERR_WORKSPACE";
        default: return "AG_ERR_UNKNOWN";
    }
}

int ag_abi_version(void) { return 102; }  // 1.02: ag_step added

}  // extern "C"
