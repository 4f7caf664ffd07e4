// Edge-softmax attention over the forward adjacency (PyTorch Geometric
// reading guide, Step 4 "SDDMM: the second primitive, forced by attention":
// a per-edge score from both endpoints' features, a softmax over each
// destination row, then the SpMM with the normalised scores).
//
//   s_e     = scale * dot(Q[dst_e], K[src_e])           (SDDMM)
//   alpha_e = exp(s_e - m_r) / l_r,  r = dst_e           (row softmax)
//   Y[r]    = sum over edges e into r of alpha_e V[src_e] (SpMM)
//
// The scores come from the SDDMM walk of the forward CSR (owner Q[dst],
// gathered K[src]) straight into the forward walk's window slots, where the
// row statistics m_r (maximum) and l_r (sum of exp(s - m_r)) read them: one
// segmented reduction over the forward CSR, walked in the same edge-balanced
// tiles as the SpMM (one warp per tile, each lane reducing its own run of
// consecutive positions in registers, one Hillis-Steele segmented scan over
// the 32 lanes' open rows, rows cut by a tile boundary finished by a fixup
// pass in tile order); the scores then go back to COO order once, for the
// softmax pass, and the SpMMs run through this library's own entry points
// (ag_spmm_fwd, ag_spmm_dx, and ag_backward for dV with dalpha in one walk).
// Backward: c_r = sum over r's edges of alpha dalpha by the same segmented
// reduction over the products, regrouped into the forward walk's windows, then
// ds_e = scale alpha_e (dalpha_e - c_dst) in one elementwise pass.  Every
// reduction tree is fixed by the positions alone, so results are
// deterministic.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "aggraph.h"
#include "internal.h"

namespace ag {
namespace {

constexpr int kWarpsPerBlock = 8;
constexpr unsigned kFull = 0xffffffffu;

enum ReduceOp { kSoftmaxStats = 0, kSum = 1 };

// (m, l) pairs: l is a sum of exp(value - m).  (-inf, 0) is the identity.
__device__ __forceinline__ float2 combine_stats(float2 a, float2 b) {
    if (a.x == -INFINITY) return b;
    if (b.x == -INFINITY) return a;
    const float M = fmaxf(a.x, b.x);
    return make_float2(M, a.y * expf(a.x - M) + b.y * expf(b.x - M));
}

template <int OP>
__device__ __forceinline__ float2 combine(float2 a, float2 b) {
    if (OP == kSoftmaxStats) return combine_stats(a, b);
    return make_float2(a.x + b.x, 0.f);
}
template <int OP>
__device__ __forceinline__ float2 identity() {
    return OP == kSoftmaxStats ? make_float2(-INFINITY, 0.f) : make_float2(0.f, 0.f);
}

struct ReduceParams {
    const int32_t *order;      // forward CSR position -> slot of its edge in `a` and `b`
    const float *a;            // per-edge inputs, in the forward walk's window-bucketed order
    const float *b;
    float scale;
    int T;                     // positions per tile
    int64_t E, n_tiles, n_nz;
    const int32_t *tile_nz, *nz_rows, *nz_rowptr;
    float2 *partial;           // [2 * n_tiles]: slot 2t (row continued from the previous tile), 2t + 1 (continues)
    float2 *out;               // [N] per row
};

__device__ __forceinline__ float2 shfl2_up(float2 v, int d) {
    return make_float2(__shfl_up_sync(kFull, v.x, d), __shfl_up_sync(kFull, v.y, d));
}

// Adds one leaf value to a segment's aggregate: kSoftmaxStats keeps the
// maximum m and the sum l of exp(s - m), rescaling l when m grows (one
// exponential per value; (-inf, 0) is the empty segment); kSum adds.
template <int OP>
__device__ __forceinline__ void absorb(float2 &run, float s) {
    if (OP == kSoftmaxStats) {
        if (s > run.x) {
            run.y = run.y * expf(run.x - s) + 1.f;
            run.x = s;
        } else {
            run.y += expf(s - run.x);
        }
    } else {
        run.x += s;
    }
}

// Leaf value of COO edge e: kSoftmaxStats the score scale * a_e, kSum a_e * b_e
// (a_e alone when there is no b).
template <int OP>
__device__ __forceinline__ float leaf_value(const ReduceParams &P, int e) {
    // the rounded product (no contraction into a later subtraction): the
    // softmax pass forms the same value, so exp(value - maximum) is exactly 1
    // at the row's maximum
    return OP == kSoftmaxStats ? __fmul_rn(P.scale, P.a[e]) : (P.b ? P.a[e] * P.b[e] : P.a[e]);
}

// One warp per tile of T consecutive forward-CSR positions.  Lane l owns the
// T / 32 consecutive positions [l T/32, (l + 1) T/32) of the tile and reduces
// them in order in registers: every row that starts and ends inside the lane
// is finished there; the lane's head (the positions before its first row
// start) and its tail (the row open at its end) are combined across lanes
// with one segmented scan over the 32 tails.  All leaves are loaded before
// the reduction (the order map, then the values: two round trips per tile);
// while the values are in flight the tile's row starts are staged in shared
// memory, where a lane finds its first row by a binary search.
// kSoftmaxStats keeps (max, sum of exp(s - max)) per segment, rescaling the
// sum when the maximum grows; kSum keeps a sum.  Every combination order is
// fixed by the positions alone.
constexpr int kMaxChunks = kMaxTileEdges / 32;  // positions per lane at most
constexpr int kStageUnroll = 8;                  // row starts in flight per lane while staging
static_assert(kMaxChunks % 4 == 0, "16-byte loads of the order map");

template <int OP>
__global__ void __launch_bounds__(kWarpsPerBlock * 32) k_row_reduce(const ReduceParams P) {
    // the first positions of the rows after the tile's first row, up to the
    // last row that starts in the tile (at most T of them)
    __shared__ int row_start[kWarpsPerBlock][kMaxTileEdges + 1];
    const int64_t t = (int64_t(blockIdx.x) * kWarpsPerBlock) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (t >= P.n_tiles) return;  // whole warps
    int *rs = row_start[threadIdx.x >> 5];
    const int64_t p0 = t * P.T;
    const int len = int(P.E - p0 < P.T ? P.E - p0 : P.T);
    const int ppl = P.T / 32;  // positions per lane (T is a power of two >= 32)
    const int a0 = lane * ppl;
    int e[kMaxChunks];
    float x[kMaxChunks];
    if ((ppl & 3) == 0 && a0 + ppl <= len) {
        // whole runs of a multiple of 4 positions: 16-byte loads (p0 and a0
        // are multiples of 4 positions)
#pragma unroll
        for (int k = 0; k < kMaxChunks; k += 4) {
            int4 v = make_int4(-1, -1, -1, -1);
            if (k < ppl) v = __ldg(reinterpret_cast<const int4 *>(P.order + p0 + a0 + k));
            e[k] = v.x, e[k + 1] = v.y, e[k + 2] = v.z, e[k + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int k = 0; k < kMaxChunks; ++k) e[k] = (k < ppl && a0 + k < len) ? __ldg(P.order + p0 + a0 + k) : -1;
    }
    const int64_t r0 = P.tile_nz[t];
    // rows r0 + 1 .. r_last: the row holding the next tile's first position
    // closes the range (the last tile: the last row)
    const int64_t r_last = t + 1 < P.n_tiles ? P.tile_nz[t + 1] : P.n_nz - 1;
    const int nrs = int(r_last - r0);  // <= T: at most one row starts per position
    const int64_t first_start = P.nz_rowptr[r0];  // start of the tile's first row
    // the leaves (their gathers in flight while the row starts are staged)
#pragma unroll
    for (int k = 0; k < kMaxChunks; ++k) x[k] = e[k] >= 0 ? leaf_value<OP>(P, e[k]) : 0.f;
    // kStageUnroll loads in flight per lane before their stores (a tile of
    // short rows stages up to T starts: one round trip per 8 x 32 of them)
    for (int i0 = 0; i0 < nrs; i0 += 32 * kStageUnroll) {
        int v[kStageUnroll];
#pragma unroll
        for (int u = 0; u < kStageUnroll; ++u) {
            const int i = i0 + 32 * u + lane;
            v[u] = i < nrs ? __ldg(P.nz_rowptr + r0 + 1 + i) : 0;
        }
#pragma unroll
        for (int u = 0; u < kStageUnroll; ++u) {
            const int i = i0 + 32 * u + lane;
            if (i < nrs) rs[i] = v[u];
        }
    }
    const bool before = first_start < p0;
    __syncwarp();

    // the row holding this lane's first position: r0 + the number of staged
    // starts at or before it
    const bool has_pos = a0 < len;
    int lo = 0, hi = nrs;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (rs[mid] <= p0 + a0) lo = mid + 1;
        else hi = mid;
    }
    const int64_t row_a0 = r0 + lo;
    const bool starts_first = has_pos && (lo == 0 ? first_start : int64_t(rs[lo - 1])) == p0 + a0;
    int64_t row_i = row_a0;
    int64_t next = lo < nrs ? int64_t(rs[lo]) : INT64_MAX;  // start of row row_i + 1
    bool inner = false;                                        // a row starts after the first position
    float2 head = identity<OP>(), run = identity<OP>();
#pragma unroll
    for (int k = 0; k < kMaxChunks; ++k) {
        if (k >= ppl || a0 + k >= len) break;
        if (p0 + a0 + k == next) {  // a row starts here: close the open segment
            if (!inner && !starts_first) head = run;
            else P.out[P.nz_rows[row_i]] = run;  // started and ended in this lane
            inner = true;
            run = identity<OP>();
            ++row_i;
            const int m = int(row_i - r0);
            next = m < nrs ? int64_t(rs[m]) : INT64_MAX;
        }
        absorb<OP>(run, x[k]);
    }

    // segmented inclusive scan of the lanes' tails: a lane whose open segment
    // starts inside it (at or after its first position) begins a segment
    float2 v = run;  // identity for lanes without positions
    bool f = starts_first || inner;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float2 pv = shfl2_up(v, o);
        const bool pf = __shfl_up_sync(kFull, f, o);
        if (lane >= o) {
            if (!f) v = combine<OP>(pv, v);
            f = f || pf;
        }
    }
    float2 excl = shfl2_up(v, 1);
    if (lane == 0) excl = identity<OP>();
    const bool next_starts = __shfl_down_sync(kFull, starts_first, 1);
    const bool next_has = __shfl_down_sync(kFull, has_pos, 1);
    auto write_row = [&](int64_t ri, float2 total, bool continues) {
        if (ri == r0 && before) P.partial[2 * t] = total;        // row continued from the previous tile
        else if (continues) P.partial[2 * t + 1] = total;        // row continued in the next tile
        else P.out[P.nz_rows[ri]] = total;
    };
    // the row continued into this lane ends inside it
    if (has_pos && !starts_first && inner) write_row(row_a0, combine<OP>(excl, head), false);
    if (has_pos && lane < 31 && next_has) {
        // the open row ends at this lane's last position
        if (next_starts) write_row(row_i, v, false);
    } else if (has_pos) {
        // the last lane with positions: the row open at the tile's end
        const int m = int(row_i - r0);
        const int64_t end = m < nrs ? int64_t(rs[m]) : int64_t(P.nz_rowptr[row_i + 1]);
        write_row(row_i, v, end > p0 + len);
    }
}

// Rows cut by tile boundaries: out[row] = slot(2 first + 1) combined with
// the slots 2t of tiles t = first + 1 .. last.  The n_long long spans (listed
// first) take one warp each: lane l combines the tiles first + 1 + l + 32 i
// in order, then a butterfly of fixed shape combines the lanes, so no thread
// waits on a chain of hundreds of loads; every other span takes one thread
// and combines in tile order.
template <int OP>
__global__ void k_row_reduce_fixup(const int4 *__restrict__ spans, int64_t n_span, int64_t n_long,
                                   const float2 *__restrict__ partial, float2 *__restrict__ out) {
    const int64_t gt = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (gt < n_long * 32) {  // whole warps (n_long * 32 is a multiple of 32)
        const int lane = threadIdx.x & 31;
        const int4 sp = spans[gt >> 5];
        float2 v = identity<OP>();
        for (int64_t t = int64_t(sp.y) + 1 + lane; t <= sp.z; t += 32) v = combine<OP>(v, partial[2 * t]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float2 u = make_float2(__shfl_xor_sync(kFull, v.x, o), __shfl_xor_sync(kFull, v.y, o));
            v = (lane & o) ? combine<OP>(u, v) : combine<OP>(v, u);
        }
        if (lane == 0) out[sp.x] = combine<OP>(partial[2 * int64_t(sp.y) + 1], v);
        return;
    }
    const int64_t s = n_long + (gt - n_long * 32);
    if (s >= n_span) return;
    const int4 sp = spans[s];
    float2 v = partial[2 * int64_t(sp.y) + 1];
    for (int64_t t = int64_t(sp.y) + 1; t <= sp.z; ++t) v = combine<OP>(v, partial[2 * t]);
    out[sp.x] = v;
}

// The two per-edge passes below gather one per-row value per edge from an
// L2-resident table: each thread keeps kEdgeUnroll edges in flight (strided
// by the grid, so every load of the warp stays coalesced), loading all
// their inputs before the gathers and all gathers before the arithmetic.
constexpr int kEdgeUnroll = 4;

// alpha_e = exp(scale * s_e - m_r) / l_r (in place over s)
__global__ void k_softmax_alpha(float *__restrict__ s, const int32_t *__restrict__ dst, const float2 *__restrict__ ml,
                                float scale, int64_t E) {
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t e0 = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e0 < E; e0 += stride * kEdgeUnroll) {
        int d[kEdgeUnroll];
        float v[kEdgeUnroll];
        float2 r[kEdgeUnroll];
#pragma unroll
        for (int k = 0; k < kEdgeUnroll; ++k) {
            const int64_t e = e0 + k * stride;
            d[k] = e < E ? __ldcs(dst + e) : 0;
            v[k] = e < E ? s[e] : 0.f;
        }
#pragma unroll
        for (int k = 0; k < kEdgeUnroll; ++k) r[k] = e0 + k * stride < E ? ml[d[k]] : make_float2(0.f, 1.f);
#pragma unroll
        for (int k = 0; k < kEdgeUnroll; ++k) {
            const int64_t e = e0 + k * stride;
            if (e < E) s[e] = expf(__fmul_rn(scale, v[k]) - r[k].x) / r[k].y;
        }
    }
}

// ds_e = scale * alpha_e * (dalpha_e - c_r) (in place over dalpha)
__global__ void k_attn_ds(const float *__restrict__ alpha, float *__restrict__ da, const int32_t *__restrict__ dst,
                          const float2 *__restrict__ c, float scale, int64_t E) {
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t e0 = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e0 < E; e0 += stride * kEdgeUnroll) {
        int d[kEdgeUnroll];
        float a[kEdgeUnroll], g[kEdgeUnroll], cr[kEdgeUnroll];
#pragma unroll
        for (int k = 0; k < kEdgeUnroll; ++k) {
            const int64_t e = e0 + k * stride;
            d[k] = e < E ? __ldcs(dst + e) : 0;
            a[k] = e < E ? __ldcs(alpha + e) : 0.f;
            g[k] = e < E ? da[e] : 0.f;
        }
#pragma unroll
        for (int k = 0; k < kEdgeUnroll; ++k) cr[k] = e0 + k * stride < E ? c[d[k]].x : 0.f;
#pragma unroll
        for (int k = 0; k < kEdgeUnroll; ++k) {
            const int64_t e = e0 + k * stride;
            if (e < E) da[e] = scale * a[k] * (g[k] - cr[k]);
        }
    }
}

unsigned flat_blocks(int64_t n) {
    const int64_t b = (n + 255) / 256;
    return unsigned(b < 1 ? 1 : (b > 148 * 32 ? 148 * 32 : b));
}

// scratch: SpMM scratch | per-row float2 [N] | tile partials float2 [2 tiles] | float [E]
struct AttnLayout {
    size_t spmm, rows, partial, edges, total;
};
AttnLayout attn_layout(const ag_graph *g, int64_t H) {
    AttnLayout L;
    L.spmm = 0;
    L.rows = align_up(ag_spmm_scratch_bytes(g, H));
    L.partial = L.rows + align_up(size_t(g->N) * sizeof(float2));
    L.edges = L.partial + align_up(size_t(2) * size_t(g->n_tiles) * sizeof(float2));
    L.total = L.edges + align_up(size_t(g->E) * 4);
    return L;
}

// a_b, b_b: per-edge inputs already regrouped into the forward walk's
// window-bucketed order, so that the walk's reads stay inside L2-sized
// windows instead of one random sector per edge.
template <int OP>
int row_reduce(const ag_graph *g, const float *a_b, const float *b_b, float scale, float2 *partial, float2 *out,
               cudaStream_t st) {
    const Direction &D = g->dir[0];
    ReduceParams P;
    P.order = D.bucket_of_pos;
    P.a = a_b;
    P.b = b_b;
    P.scale = scale;
    P.T = g->tile_edges;
    P.E = g->E;
    P.n_tiles = g->n_tiles;
    P.n_nz = D.n_nz;
    P.tile_nz = D.tile_nz;
    P.nz_rows = D.nz_rows;
    P.nz_rowptr = D.nz_rowptr;
    P.partial = partial;
    P.out = out;
    if (g->n_tiles > 0) {
        const unsigned grid = unsigned((g->n_tiles + kWarpsPerBlock - 1) / kWarpsPerBlock);
        k_row_reduce<OP><<<grid, kWarpsPerBlock * 32, 0, st>>>(P);
    }
    if (D.n_span > 0) {
        const int64_t threads = D.n_span_long * 32 + (D.n_span - D.n_span_long);
        k_row_reduce_fixup<OP><<<unsigned((threads + 255) / 256), 256, 0, st>>>(D.spans, D.n_span, D.n_span_long,
                                                                                partial, out);
    }
    cudaError_t err = cudaGetLastError();
    return err == cudaSuccess ? AG_OK : cuda_fail(err, "row reduction");
}

}  // namespace

// out[r].x = sum of a_b over the forward-CSR positions of every row r with
// edges (a_b in the forward walk's window slots); rows without edges are not
// written.  partial: float2 [2 * tiles].
int row_sums(const ag_graph *g, const float *a_b, float2 *partial, float2 *out, cudaStream_t st) {
    return row_reduce<kSum>(g, a_b, nullptr, 1.f, partial, out, st);
}

namespace {

int check_common(const ag_graph *g, int64_t H, int dtype, const void *scratch, size_t scratch_bytes, const char *fn,
                 AttnLayout *L) {
    if (!g) return fail(AG_ERR_INVALID_ARG, "%s: null graph", fn);
    if (H < 1 || H > (int64_t(1) << 24)) return fail(AG_ERR_SHAPE, "%s: H = %lld outside [1, 2^24]", fn, (long long)H);
    if (dtype != AG_F32 && dtype != AG_BF16) return fail(AG_ERR_DTYPE, "%s: unknown dtype %d", fn, dtype);
    if (int rc = check_current_device(g, fn)) return rc;
    *L = attn_layout(g, H);
    if (!scratch || scratch_bytes < L->total)
        return fail(AG_ERR_WORKSPACE, "%s: scratch of %zu bytes, need %zu", fn, scratch_bytes, L->total);
    if (reinterpret_cast<uintptr_t>(scratch) % kAlign != 0)
        return fail(AG_ERR_WORKSPACE, "%s: scratch must be 256-byte aligned", fn);
    return check_device_ptr(scratch, g->device, "scratch");
}

}  // namespace
}  // namespace ag

using namespace ag;

extern "C" {

size_t ag_attn_scratch_bytes(const ag_graph *g, int64_t H) {
    if (!g || H < 1) return 0;
    return attn_layout(g, H).total;
}

int ag_attn_fwd(const ag_graph *g, const void *Q, const void *K, const void *V, float scale, void *Y, float *alpha,
                int64_t H, int dtype, void *scratch, size_t scratch_bytes, void *stream) {
    const char *fn = "ag_attn_fwd";
    clear_error();
    AttnLayout L;
    int rc = check_common(g, H, dtype, scratch, scratch_bytes, fn, &L);
    if (rc != AG_OK) return rc;
    if (!Q || !K || !V || !Y || (g->E > 0 && !alpha)) return fail(AG_ERR_INVALID_ARG, "%s: null Q, K, V, Y or alpha", fn);
    if (!isfinite(scale)) return fail(AG_ERR_INVALID_ARG, "%s: scale must be finite", fn);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *scr = static_cast<char *>(scratch);
    const size_t spmm_bytes = L.rows - L.spmm;
    if (g->E > 0) {
        // raw scores dot(Q[dst], K[src]) by the SDDMM walk of the forward CSR,
        // straight into the forward walk's window slots (the SpMM scratch's
        // weight-gradient array is free until the aggregation below)
        float *s_b = reinterpret_cast<float *>(scr + L.spmm + spmm_scratch_edge_offset(g, H, 1));
        if ((rc = sddmm_bucketed(g, 0, Q, K, s_b, H, dtype, st)) != AG_OK) return rc;
        float2 *ml = reinterpret_cast<float2 *>(scr + L.rows);
        rc = row_reduce<kSoftmaxStats>(g, s_b, nullptr, scale, reinterpret_cast<float2 *>(scr + L.partial), ml, st);
        if (rc != AG_OK) return rc;
        // the scores to COO order (into alpha), then alpha in place
        regroup_from_buckets(g, 0, s_b, alpha, st);
        k_softmax_alpha<<<flat_blocks(g->E), 256, 0, st>>>(alpha, g->coo_dst, ml, scale, g->E);
        cudaError_t err = cudaGetLastError();
        if (err != cudaSuccess) return cuda_fail(err, fn);
    }
    return ag_spmm_fwd(g, alpha, V, Y, H, dtype, scr + L.spmm, spmm_bytes, stream);
}

int ag_attn_backward(const ag_graph *g, const void *Q, const void *K, const void *V, float scale, const float *alpha,
                     const void *dY, void *dQ, void *dK, void *dV, int64_t H, int dtype, void *scratch,
                     size_t scratch_bytes, void *stream) {
    const char *fn = "ag_attn_backward";
    clear_error();
    AttnLayout L;
    int rc = check_common(g, H, dtype, scratch, scratch_bytes, fn, &L);
    if (rc != AG_OK) return rc;
    if (!Q || !K || !V || !dY || !dQ || !dK || !dV || (g->E > 0 && !alpha))
        return fail(AG_ERR_INVALID_ARG, "%s: null argument", fn);
    if (!isfinite(scale)) return fail(AG_ERR_INVALID_ARG, "%s: scale must be finite", fn);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *scr = static_cast<char *>(scratch);
    const size_t spmm_bytes = L.rows - L.spmm;
    void *sp = scr + L.spmm;
    float *ds = reinterpret_cast<float *>(scr + L.edges);
    if (g->E == 0) {
        if ((rc = ag_spmm_dx(g, alpha, dY, dV, H, dtype, sp, spmm_bytes, stream)) != AG_OK) return rc;
    } else {
        // dV = A_alpha^T dY and dalpha_e = dot(V[src], dY[dst]) in one transpose
        // walk (the weighted-sum backward with weights alpha and "features" V)
        if ((rc = ag_backward(g, alpha, V, dY, dV, ds, H, dtype, sp, spmm_bytes, stream)) != AG_OK) return rc;
        // c_r = sum over r's edges of alpha dalpha: the products, formed while
        // regrouping into the forward windows (the SpMM scratch's per-edge
        // arrays are free between the walks), summed per row
        float2 *c = reinterpret_cast<float2 *>(scr + L.rows);
        float *p_b = reinterpret_cast<float *>(scr + L.spmm + spmm_scratch_edge_offset(g, H, 0));
        regroup_product_to_buckets(g, 0, alpha, ds, p_b, st);
        rc = row_reduce<kSum>(g, p_b, nullptr, 1.f, reinterpret_cast<float2 *>(scr + L.partial), c, st);
        if (rc != AG_OK) return rc;
        k_attn_ds<<<flat_blocks(g->E), 256, 0, st>>>(alpha, ds, g->coo_dst, c, scale, g->E);
        cudaError_t err = cudaGetLastError();
        if (err != cudaSuccess) return cuda_fail(err, fn);
    }
    // dQ = A_ds K (scale folded into ds), dK = A_ds^T Q
    if ((rc = ag_spmm_fwd(g, g->E > 0 ? ds : nullptr, K, dQ, H, dtype, sp, spmm_bytes, stream)) != AG_OK) return rc;
    return ag_spmm_dx(g, g->E > 0 ? ds : nullptr, Q, dK, H, dtype, sp, spmm_bytes, stream);
}

}  // extern "C"
