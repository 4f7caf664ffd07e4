// aggregate.cu -- per-call kernels: weighted SpMM (forward Y = A_w X and
// feature gradient dX = A_w^T dY), the per-edge SDDMM weight gradient
// dw_e = dot(X[src_e], dY[dst_e]), both gradients in one walk, the mean
// aggregation and the GCN-normalised weights.
//
// tinymesh "Weighted aggregation experiment", section "Decision": forward and
// dX use owner-row CSR traversals, dw has one output per edge reduced over the
// feature width, and none of them needs atomics or an [E, H] intermediate.
// Section "Limits" names the two weak spots of that design: a serial
// reduction over the feature width per edge, and degree skew in the CSR
// directions.  Here:
//   * the CSR positions are cut into edge-balanced tiles of T positions; a
//     group of G lanes walks one tile, each lane owning 16-byte vectors of
//     the feature width, gathered rows in flight through a per-lane
//     shared-memory ring filled with cp.async, fp32 accumulation in
//     registers;
//   * a row cut by tile boundaries leaves fp32 partial rows in caller scratch
//     that a second kernel adds in tile order -- deterministic, no float
//     atomics;
//   * the per-call weights (COO order) are first regrouped into windows of
//     2^20 CSR positions, so the walk reads them from L2, and the weight
//     gradient leaves through the same windows back to COO order;
//   * dw walks the transpose CSR: the owner's X row is held in registers,
//     every dY row gathered once feeds one dot product, and the dots of a
//     chunk of positions are reduced across the group with one
//     reduce-scatter.
#include <cuda_bf16.h>

#include <atomic>
#include <climits>
#include <mutex>

#include "device_common.cuh"
#include "internal.h"

namespace ag {
namespace {

// Tunables (compile-time; the defaults are the measured best on B200).
#ifndef AG_RING_DEPTH
#define AG_RING_DEPTH 8   // gathered rows in flight per lane group (shared-memory ring)
#endif
#ifndef AG_W_STREAM
#define AG_W_STREAM 0     // 1: weight lookups loaded evict-first; 0: normal caching (the bucketed
                          // weights of a window are reused from L2 by the window's tiles)
#endif
#ifndef AG_RING_STEP
#define AG_RING_STEP 1    // positions per cp.async wait/commit in the ring SpMM (1 or 2)
#endif
#ifndef AG_BUCKET_STAGED
#define AG_BUCKET_STAGED 1  // 1: weight regrouping passes stage a chunk in shared memory (coalesced)
#endif
#ifndef AG_CHUNK
#define AG_CHUNK 8        // positions per unrolled chunk of a gradient-walk batch (the rest is rolled)
#endif
#ifndef AG_WALK
#define AG_WALK 1         // 1: rows of 1024 bytes take the warp walk (k_walk)
#endif
#ifndef AG_MAX_LANES
#define AG_MAX_LANES 16   // lanes that share one row (fewer lanes: more 16-byte vectors per lane)
#endif

constexpr int kThreads = 256;
// Blocks of the ring walk: tiles vary in length, and a smaller block frees
// its share of an SM as soon as its few slowest groups finish (at R-MAT-22
// the step took 4 % less time with 128 threads than with 256, the fused
// backward walk 5 % less; 64 and 512 were slower); occupancy per SM is the
// same.  The row-scaled forward walk of the mean measured 0.3 ms slower with
// 128 threads and keeps 256.
#ifndef AG_RING_THREADS
#define AG_RING_THREADS 128
#endif
constexpr int kRingThreads = AG_RING_THREADS;
#ifndef AG_WALK_THREADS
#define AG_WALK_THREADS 256  // blocks of the one-warp-per-tile walk (1 KB rows)
#endif
constexpr int kWalkThreads = AG_WALK_THREADS;
constexpr int kUnroll = 4;     // gathered rows in flight per lane (register path)
constexpr int kMinBlocks = 4;  // resident CTAs per SM the register path is compiled for
constexpr int kRingDepth = AG_RING_DEPTH;
constexpr int kChunk = AG_CHUNK;

// kBoth: feature and weight gradient in one walk.  Mean flags (ring walks
// only): kRowScale multiplies every finished output row by inv_cnt[row]
// (forward mean); kEdgeScale multiplies every edge's weight and dot product
// by inv_cnt of its gathered column (the destination, in the transpose walk).
enum Mode { kSpmm = 1, kSddmm = 2, kBoth = 3, kRowScale = 4, kEdgeScale = 8 };
constexpr int ring_threads(int MODE) { return (MODE & kRowScale) ? 256 : kRingThreads; }

// A weight looked up through the bucketed layout: each 128-byte line of a
// window is used by about 32 positions of that window's tiles, so it is kept
// in L2 with the default policy.
__device__ __forceinline__ float load_w(const float *p) {
#if AG_W_STREAM
    return __ldcs(p);
#else
    return __ldg(p);
#endif
}

// fp32 partial rows (scratch): VEC floats at p, aligned to VEC * 4 bytes.
template <int VEC>
__device__ __forceinline__ void store_partial(float *p, const float (&v)[VEC]) {
    if constexpr (VEC % 4 == 0) {
#pragma unroll
        for (int i = 0; i < VEC; i += 4)
            *reinterpret_cast<float4 *>(p + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
    } else if constexpr (VEC == 2) {
        *reinterpret_cast<float2 *>(p) = make_float2(v[0], v[1]);
    } else {
        p[0] = v[0];
    }
}
template <int VEC>
__device__ __forceinline__ void add_partial(const float *p, float (&v)[VEC]) {
    if constexpr (VEC % 4 == 0) {
#pragma unroll
        for (int i = 0; i < VEC; i += 4) {
            float4 t = __ldcs(reinterpret_cast<const float4 *>(p + i));
            v[i] += t.x; v[i + 1] += t.y; v[i + 2] += t.z; v[i + 3] += t.w;
        }
    } else if constexpr (VEC == 2) {
        float2 t = __ldcs(reinterpret_cast<const float2 *>(p));
        v[0] += t.x; v[1] += t.y;
    } else {
        v[0] += __ldcs(p);
    }
}

struct Params {
    const int32_t *col;        // other endpoint per CSR position
    const int32_t *order;      // CSR position -> COO ordinal
    const float *w;            // COO weights (SpMM)
    const int32_t *nz_rows;    // non-empty rows, ascending
    const int32_t *nz_rowptr;  // their first position, then E
    const int32_t *tile_nz;    // row (index into nz_rows) holding each tile's first position
    const int32_t *zero_rows;  // rows without edges (SpMM writes zeros)
    const void *F;             // gathered feature rows
    const void *R;             // owner feature rows (SDDMM)
    void *out;                 // SpMM output [N, H]
    float *partial;            // [2 * n_tiles, H]: slot 2t = row continued from tile t-1, 2t+1 = row continued in tile t+1
    float *dw;                 // SDDMM output, COO order
    const float *inv_cnt;      // mean modes: 1 / in-degree per node (forward CSR row lengths)
    int64_t E, H, n_nz;
    int64_t n_tiles;           // lane groups [0, n_tiles) walk one tile each
    int64_t n_zero;            // lane groups [n_tiles, n_tiles + n_zero) zero one empty row each
    int T;                     // positions per tile
    int G, log2G, col_tiles;
};

template <typename T, int VEC, int NV>
__device__ __forceinline__ void store_row(T *row, int64_t vbase, int G, const bool (&ok)[NV],
                                          const float (&acc)[NV][VEC]) {
#pragma unroll
    for (int k = 0; k < NV; ++k)
        if (ok[k]) Vec<T, VEC>::store(row + (vbase + int64_t(k) * G) * VEC, acc[k]);
}

template <int VEC, int NV>
__device__ __forceinline__ void store_slot(float *slot, int64_t vbase, int G, const bool (&ok)[NV],
                                           const float (&acc)[NV][VEC]) {
#pragma unroll
    for (int k = 0; k < NV; ++k)
        if (ok[k]) store_partial<VEC>(slot + (vbase + int64_t(k) * G) * VEC, acc[k]);
}

// One group of G lanes (G a power of two <= 32) walks the T consecutive CSR
// positions of one tile in order.  Each lane owns the column vectors
// j = tile * G * NV + k * G + lane (k < NV) of the rows it touches.
//   kSpmm : out[row] = sum w[order[p]] * F[col[p]] over the row's positions
//   kSddmm: dw[order[p]] = dot(R[row], F[col[p]])
// A row that starts and ends inside the tile is written whole; the segment
// of a row continued from the previous tile goes to partial slot 2t, the
// segment of a row continued in the next tile to slot 2t+1.
template <typename T, int VEC, int NV, int MODE, bool ONE_TILE>
__global__ void __launch_bounds__(kThreads, NV == 1 ? kMinBlocks : (NV == 2 ? 3 : 2))
k_tiles(const Params P) {
    const int G = P.G;
    const int64_t gid = (int64_t(blockIdx.x) * kThreads + threadIdx.x) >> P.log2G;
    if (gid >= P.n_tiles + P.n_zero) return;
    const int gl = threadIdx.x & (G - 1);
    const int lane = threadIdx.x & 31;
    const unsigned gmask = (G == 32) ? 0xffffffffu : (((1u << G) - 1u) << (lane & ~(G - 1)));
    const int64_t H = P.H;
    const int64_t HV = H / VEC;

    if (gid >= P.n_tiles) {  // an empty row: zeros
        T *row = static_cast<T *>(P.out) + int64_t(P.zero_rows[gid - P.n_tiles]) * H;
        float z[VEC];
#pragma unroll
        for (int v = 0; v < VEC; ++v) z[v] = 0.f;
        for (int64_t j = gl; j < HV; j += G) Vec<T, VEC>::store(row + j * VEC, z);
        return;
    }

    const int64_t p0 = gid * P.T;
    const int64_t p1 = min(p0 + int64_t(P.T), P.E);
    const int i0 = P.tile_nz[gid];
    const T *__restrict__ F = static_cast<const T *>(P.F);
    float *slot_head = P.partial + (2 * gid) * H;
    float *slot_tail = P.partial + (2 * gid + 1) * H;

    for (int tile = 0; tile < (ONE_TILE ? 1 : P.col_tiles); ++tile) {
        const int64_t vbase = int64_t(tile) * G * NV + gl;
        bool colok[NV];
#pragma unroll
        for (int k = 0; k < NV; ++k) colok[k] = vbase + int64_t(k) * G < HV;

        // current row and a look-ahead window of the next G rows (one per lane)
        int row = P.nz_rows[i0];
        int64_t rend = P.nz_rowptr[i0 + 1];
        bool before = P.nz_rowptr[i0] < p0;
        int64_t la_base = int64_t(i0) + 1;
        int la_row = 0, la_end = INT_MAX;
        if (la_base + gl < P.n_nz) {
            la_row = P.nz_rows[la_base + gl];
            la_end = P.nz_rowptr[la_base + gl + 1];
        }
        int la_k = 0;

        float acc[NV][VEC];
        float own[NV][VEC];
#pragma unroll
        for (int k = 0; k < NV; ++k)
#pragma unroll
            for (int v = 0; v < VEC; ++v) acc[k][v] = 0.f, own[k][v] = 0.f;
        if (MODE == kSddmm) {
            const T *Rrow = static_cast<const T *>(P.R) + int64_t(row) * H;
#pragma unroll
            for (int k = 0; k < NV; ++k)
                if (colok[k]) load_vec<T, VEC>(Rrow + (vbase + int64_t(k) * G) * VEC, own[k]);
        }

        // indices of the first batch
        int c_cur = 0, e_cur = 0;
        float w_cur = 0.f;
        {
            const int64_t p = p0 + gl;
            if (p < p1) {
                c_cur = __ldcs(P.col + p);
                e_cur = __ldcs(P.order + p);
                if (MODE == kSpmm) w_cur = load_w(P.w + e_cur);
            }
        }
        for (int64_t base = p0; base < p1; base += G) {
            // prefetch the next batch's indices while this batch gathers
            int c_nxt = 0, e_nxt = 0;
            const int64_t pn = base + G + gl;
            if (pn < p1) {
                c_nxt = __ldcs(P.col + pn);
                e_nxt = __ldcs(P.order + pn);
            }
            const int n = int(p1 - base < G ? p1 - base : G);
            for (int j = 0; j < n; j += kUnroll) {
                typename Vec<T, VEC>::raw x[kUnroll][NV];
                float wv[kUnroll];
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    const int src = __shfl_sync(gmask, c_cur, (j + u) & (G - 1), G);
                    wv[u] = (MODE == kSpmm) ? __shfl_sync(gmask, w_cur, (j + u) & (G - 1), G) : 0.f;
                    const T *Frow = F + int64_t(src) * H;
#pragma unroll
                    for (int k = 0; k < NV; ++k)
                        x[u][k] = (j + u < n && colok[k]) ? Vec<T, VEC>::load_raw(Frow + (vbase + int64_t(k) * G) * VEC)
                                                          : Vec<T, VEC>::zero();
                }
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    if (j + u >= n) break;
                    if (base + j + u == rend) {
                        // the current row ended: write it, move to the next row
                        if (MODE == kSpmm) {
                            if (before) store_slot<VEC, NV>(slot_head, vbase, G, colok, acc);
                            else store_row<T, VEC, NV>(static_cast<T *>(P.out) + int64_t(row) * H, vbase, G,
                                                       colok, acc);
#pragma unroll
                            for (int k = 0; k < NV; ++k)
#pragma unroll
                                for (int v = 0; v < VEC; ++v) acc[k][v] = 0.f;
                        }
                        before = false;
                        row = __shfl_sync(gmask, la_row, la_k, G);
                        rend = __shfl_sync(gmask, la_end, la_k, G);
                        if (++la_k == G) {
                            la_base += G;
                            la_k = 0;
                            la_row = 0;
                            la_end = INT_MAX;
                            if (la_base + gl < P.n_nz) {
                                la_row = P.nz_rows[la_base + gl];
                                la_end = P.nz_rowptr[la_base + gl + 1];
                            }
                        }
                        if (MODE == kSddmm) {
                            const T *Rrow = static_cast<const T *>(P.R) + int64_t(row) * H;
#pragma unroll
                            for (int k = 0; k < NV; ++k)
                                if (colok[k]) load_vec<T, VEC>(Rrow + (vbase + int64_t(k) * G) * VEC, own[k]);
                        }
                    }
                    if (MODE == kSpmm) {
#pragma unroll
                        for (int k = 0; k < NV; ++k) {
                            float xf[VEC];
                            Vec<T, VEC>::unpack(x[u][k], xf);
#pragma unroll
                            for (int v = 0; v < VEC; ++v) acc[k][v] = fmaf(wv[u], xf[v], acc[k][v]);
                        }
                    } else {
                        float dot = 0.f;
#pragma unroll
                        for (int k = 0; k < NV; ++k) {
                            float xf[VEC];
                            Vec<T, VEC>::unpack(x[u][k], xf);
#pragma unroll
                            for (int v = 0; v < VEC; ++v) dot = fmaf(own[k][v], xf[v], dot);
                        }
                        for (int o = G >> 1; o > 0; o >>= 1) dot += __shfl_xor_sync(gmask, dot, o, G);
                        if (gl == ((j + u) & (G - 1))) {
                            if (ONE_TILE) P.dw[e_cur] = dot;
                            else P.dw[e_cur] = tile == 0 ? dot : P.dw[e_cur] + dot;
                        }
                    }
                }
            }
            c_cur = c_nxt;
            e_cur = e_nxt;
            if (MODE == kSpmm) w_cur = pn < p1 ? load_w(P.w + e_nxt) : 0.f;
        }
        if (MODE == kSpmm) {
            // the row open at the tile's end
            if (before) store_slot<VEC, NV>(slot_head, vbase, G, colok, acc);
            else if (rend > p1) store_slot<VEC, NV>(slot_tail, vbase, G, colok, acc);
            else store_row<T, VEC, NV>(static_cast<T *>(P.out) + int64_t(row) * H, vbase, G, colok, acc);
        }
    }
}

// ---------------------------------------------------------------------------- shared-memory ring path

template <typename T, int VEC>
__device__ __forceinline__ typename Vec<T, VEC>::raw lds_raw(const uint4 *p) {
    if constexpr (sizeof(typename Vec<T, VEC>::raw) == 16) {
        return *reinterpret_cast<const typename Vec<T, VEC>::raw *>(p);
    } else {
        return typename Vec<T, VEC>::raw{};
    }
}

// Recursive-halving reduce-scatter over the G lanes of a group: on entry lane
// l holds v[j] = its partial sum for item j (j < G); on exit v[0] of lane l is
// the total of item l.  G - 1 shuffles for G items.
template <int G>
__device__ __forceinline__ float reduce_scatter(float (&v)[G], int gl, unsigned gmask) {
#pragma unroll
    for (int s = G / 2; s >= 1; s >>= 1) {
        const bool upper = gl & s;
#pragma unroll
        for (int i = 0; i < s; ++i) {
            const float send = upper ? v[i] : v[i + s];
            const float keep = upper ? v[i + s] : v[i];
            v[i] = keep + __shfl_xor_sync(gmask, send, s, G);
        }
    }
    return v[0];
}

// Positions per unrolled chunk of a ring batch of G with depth D: the largest
// power of two <= min(kChunk, G) that divides G - D, so that a chunk never
// straddles the switch from this batch's column indices to the next batch's.
constexpr int chunk_of(int G, int D) {
    int u = kChunk < G ? kChunk : G;
    while (u > 1 && u < G && (G - D) % u != 0) u >>= 1;
    return u;
}

// The same for a chunk of U <= G items spread over G lanes: U - 1 halving
// exchanges leave lane l with item (l mod U) summed over its U-lane block,
// then log2(G / U) butterfly steps add the blocks, so that every lane l holds
// the total of item (l mod U).  For U == G this is reduce_scatter<G>.
template <int U, int G>
__device__ __forceinline__ float reduce_chunk(float (&v)[U], int gl, unsigned gmask) {
#pragma unroll
    for (int s = U / 2; s >= 1; s >>= 1) {
        const bool upper = gl & s;
#pragma unroll
        for (int i = 0; i < s; ++i) {
            const float send = upper ? v[i] : v[i + s];
            const float keep = upper ? v[i + s] : v[i];
            v[i] = keep + __shfl_xor_sync(gmask, send, s, G);
        }
    }
#pragma unroll
    for (int o = U; o < G; o <<= 1) v[0] += __shfl_xor_sync(gmask, v[0], o, G);
    return v[0];
}

// Row accumulator of one lane: NV vectors of VEC fp32 sums updated with
// fmaf.  (Packed fma.rn.f32x2 pairs round the same way per element but cost
// register moves to form the pairs; measured slower here.)
template <typename T, int NV, int VEC> struct RowAcc {
    float a[NV][VEC];
    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int k = 0; k < NV; ++k)
#pragma unroll
            for (int v = 0; v < VEC; ++v) a[k][v] = 0.f;
    }
    __device__ __forceinline__ void fma(int k, float w, typename Vec<T, VEC>::raw x) {
        float xf[VEC];
        Vec<T, VEC>::unpack(x, xf);
#pragma unroll
        for (int v = 0; v < VEC; ++v) a[k][v] = fmaf(w, xf[v], a[k][v]);
    }
    __device__ __forceinline__ void get(float (&o)[NV][VEC]) const {
#pragma unroll
        for (int k = 0; k < NV; ++k)
#pragma unroll
            for (int v = 0; v < VEC; ++v) o[k][v] = a[k][v];
    }
};

// Same contract as k_tiles for 16-byte vectors (fp32 x 4, bf16 x 8) and a
// single column tile, with the lane-group width G and the ring depth D fixed
// at compile time.  The gathered rows travel global -> shared memory with
// cp.async: every lane group keeps the rows of the next D positions in flight
// in its own ring of D slots.  A lane copies, and later reads, only its own
// 16-byte pieces, so no barrier is needed between copy and read:
// cp.async.wait_group orders them for the issuing thread.
//
// Control flow is uniform across the warp: tile groups fill whole warps
// (groups [n_tiles, n_tiles_pad) are idle fillers), every group of a warp
// runs the warp's longest tile length in batches of G positions with its own
// bounds as predicates, and the shuffles of the common path use the full
// warp mask.  A batch inside every group's tile runs without bounds checks:
// fully unrolled in the forward walk, in rolled chunks of U unrolled
// positions in the gradient walks (slots, shuffle lanes and refill sources
// are constants within a chunk).  Indices are prefetched two batches ahead
// and weights one batch ahead.  kSddmm reduces the U dot products of a chunk
// with one reduce-scatter, after which the lane of each position writes its
// weight gradient.  kBoth does both on one walk of the transpose CSR: each
// gathered dY row feeds the feature-gradient row of its source and the dot
// product of its edge.  Rows are accumulated with scalar fp32 FMAs.
template <typename T, int VEC, int NV, int G, int MODE, int D>
__global__ void __launch_bounds__(ring_threads(MODE))
k_tiles_ring(const Params P) {
    using raw_t = typename Vec<T, VEC>::raw;
    static_assert(sizeof(raw_t) == 16, "ring path moves 16-byte vectors");
    static_assert(G >= D && G % D == 0, "ring depth must divide the batch");
    constexpr unsigned FULL = 0xffffffffu;
    extern __shared__ uint4 ring[];
    constexpr int LOG2G = G == 32 ? 5 : G == 16 ? 4 : G == 8 ? 3 : G == 4 ? 2 : G == 2 ? 1 : 0;
    const int64_t gid = (int64_t(blockIdx.x) * ring_threads(MODE) + threadIdx.x) >> LOG2G;
    const int64_t n_tiles_pad = (P.n_tiles + (32 / G) - 1) / (32 / G) * (32 / G);
    const int gl = threadIdx.x & (G - 1);
    const int lane = threadIdx.x & 31;
    const unsigned gmask = (G == 32) ? FULL : (((1u << G) - 1u) << (lane & ~(G - 1)));
    const int H = int(P.H);
    const int HV = H / VEC;
    // the ring path runs only for rows of exactly G x NV 16-byte vectors, so
    // every lane's vectors are in range (constant-folded away)
    bool colok[NV];
#pragma unroll
    for (int k = 0; k < NV; ++k) colok[k] = true;
    (void)HV;

    if (gid >= n_tiles_pad) {  // warps of empty rows: zeros
        const int64_t z = gid - n_tiles_pad;
        if (z >= P.n_zero) return;
        T *row = static_cast<T *>(P.out) + int64_t(P.zero_rows[z]) * H + gl * VEC;
        float zero[VEC];
#pragma unroll
        for (int v = 0; v < VEC; ++v) zero[v] = 0.f;
#pragma unroll
        for (int k = 0; k < NV; ++k)
            if (colok[k]) Vec<T, VEC>::store(row + k * G * VEC, zero);
        return;
    }

    // this lane's pieces of the ring: slot s, vector k at my[(s * NV + k) * G]
    const uint4 *my = ring + (threadIdx.x >> LOG2G) * (D * NV * G) + gl;
    const uint32_t my_s = smem_addr(my);
    const bool active = gid < P.n_tiles;
    const int p0 = active ? int(gid) * P.T : 0;
    const int len = active ? min(P.T, int(P.E) - p0) : 0;
    const int len_max = __reduce_max_sync(FULL, len);
    const int len_min = __reduce_min_sync(FULL, len);
    const T *__restrict__ F = static_cast<const T *>(P.F) + gl * VEC;
    float *slot_head = P.partial + (2 * gid) * P.H + gl * VEC;
    float *slot_tail = P.partial + (2 * gid + 1) * P.H + gl * VEC;
    T *out = static_cast<T *>(P.out) + gl * VEC;
    const T *R = static_cast<const T *>(P.R) + gl * VEC;

    // the row open at the current position, and the next G rows (one per lane)
    int row = 0, rend = INT_MAX, la_base = 0;
    bool before = false;
    if (active) {
        const int i0 = P.tile_nz[gid];
        row = P.nz_rows[i0];
        rend = P.nz_rowptr[i0 + 1];
        before = P.nz_rowptr[i0] < p0;
        la_base = i0 + 1;
    }
    int la_row = 0, la_end = INT_MAX;
    if (active && la_base + gl < P.n_nz) {
        la_row = P.nz_rows[la_base + gl];
        la_end = P.nz_rowptr[la_base + gl + 1];
    }
    int la_k = 0;
    // kRowScale: the open row's factor, and those of the look-ahead rows
    // (fetched with the window, so that no row end waits on a load)
    float row_inv = 0.f, la_inv = 0.f;
    if constexpr ((MODE & kRowScale) != 0) {
        if (active) row_inv = P.inv_cnt[row];
        if (active && la_base + gl < P.n_nz) la_inv = P.inv_cnt[la_row];
    }

    // indices: batch b (cur), b + 1 (nxt), b + 2 (nn); weights of b and b + 1
    int c_cur = 0, e_cur = 0, c_nxt = 0, e_nxt = 0, c_nn = 0, e_nn = 0;
    float w_cur = 0.f, w_nxt = 0.f;
    // kEdgeScale: inv_cnt of the gathered column of this lane's position in
    // batch b and b + 1 (loaded with the weights, used by weight and dot)
    float sc_cur = 1.f, sc_nxt = 1.f;
    if (gl < len) { c_cur = __ldcs(P.col + p0 + gl); e_cur = __ldcs(P.order + p0 + gl); }
    if (G + gl < len) { c_nxt = __ldcs(P.col + p0 + G + gl); e_nxt = __ldcs(P.order + p0 + G + gl); }
    if constexpr ((MODE & kEdgeScale) != 0)
        if (gl < len) sc_cur = P.inv_cnt[c_cur];
    if ((MODE & kSpmm) && gl < len) {
        w_cur = load_w(P.w + e_cur);
        if constexpr ((MODE & kEdgeScale) != 0) w_cur *= sc_cur;
    }

    const uint32_t row_bytes = uint32_t(H) * sizeof(T);
    auto issue = [&](int slot, int src) {
        const char *Frow = reinterpret_cast<const char *>(F) + uint64_t(uint32_t(src)) * row_bytes;
#pragma unroll
        for (int k = 0; k < NV; ++k)
            if (colok[k]) cp_async16(my_s + uint32_t((slot * NV + k) * G * 16), Frow + k * G * 16);
    };
    constexpr int STEP = AG_RING_STEP;
    static_assert(D % STEP == 0 && G % STEP == 0, "ring step");
#pragma unroll
    for (int s = 0; s < D; ++s) {
        const int src = __shfl_sync(FULL, c_cur, s, G);
        if (s < len) issue(s, src);
        if (s % STEP == STEP - 1) cp_async_commit();
    }

    RowAcc<T, NV, VEC> acc;
    acc.zero();
    raw_t own[NV], own_next[NV];
#pragma unroll
    for (int k = 0; k < NV; ++k) own[k] = own_next[k] = Vec<T, VEC>::zero();
    if ((MODE & kSddmm) && active) {
        const T *Rrow = R + int64_t(row) * H;
        const T *Rnext = R + int64_t(__shfl_sync(gmask, la_row, 0, G)) * H;
        const bool has_next = la_base < P.n_nz;
#pragma unroll
        for (int k = 0; k < NV; ++k)
            if (colok[k]) {
                own[k] = Vec<T, VEC>::load_raw(Rrow + k * G * VEC);
                if (has_next) own_next[k] = Vec<T, VEC>::load_raw(Rnext + k * G * VEC);
            }
    }

    auto write_open_row = [&](float *slot) {
        float o[NV][VEC];
        acc.get(o);
        if (slot) {
            store_slot<VEC, NV>(slot, 0, G, colok, o);
        } else {
            if constexpr ((MODE & kRowScale) != 0) {
                const float r = row_inv;
#pragma unroll
                for (int k = 0; k < NV; ++k)
#pragma unroll
                    for (int v = 0; v < VEC; ++v) o[k][v] *= r;
            }
            store_row<T, VEC, NV>(out + int64_t(row) * H, 0, G, colok, o);
        }
    };
    // the current row ended at the current position: write it, open the next
    // (runs only in the lane groups whose row ended: group-mask shuffles)
    auto next_row = [&]() {
        if ((MODE & kSpmm)) {
            write_open_row(before ? slot_head : nullptr);
            acc.zero();
        }
        before = false;
        row = __shfl_sync(gmask, la_row, la_k, G);
        rend = __shfl_sync(gmask, la_end, la_k, G);
        if constexpr ((MODE & kRowScale) != 0) row_inv = __shfl_sync(gmask, la_inv, la_k, G);
        if (++la_k == G) {
            la_base += G;
            la_k = 0;
            la_row = 0;
            la_end = INT_MAX;
            if (la_base + gl < P.n_nz) {
                la_row = P.nz_rows[la_base + gl];
                la_end = P.nz_rowptr[la_base + gl + 1];
                if constexpr ((MODE & kRowScale) != 0) la_inv = P.inv_cnt[la_row];
            }
        }
        if ((MODE & kSddmm)) {
            const T *Rnext = R + int64_t(__shfl_sync(gmask, la_row, la_k, G)) * H;
            const bool has_next = la_base + la_k < P.n_nz;
#pragma unroll
            for (int q = 0; q < NV; ++q) {
                own[q] = own_next[q];
                if (colok[q] && has_next) own_next[q] = Vec<T, VEC>::load_raw(Rnext + q * G * VEC);
            }
        }
    };
    // position p0 + base + j, held in ring slot `slot` (valid: inside this
    // group's tile); returns this lane's part of the dot (kSddmm)
    auto consume = [&](int base, int j, int slot, bool valid) -> float {
        const float wk = ((MODE & kSpmm)) ? __shfl_sync(FULL, w_cur, j, G) : 0.f;
        float d = 0.f;
        if (valid) {
            raw_t x[NV];
#pragma unroll
            for (int q = 0; q < NV; ++q) x[q] = *reinterpret_cast<const raw_t *>(my + (slot * NV + q) * G);
            // row ends are rare next to edges: keep the edge path straight-line
            if (__builtin_expect(p0 + base + j == rend, 0)) next_row();
            // slots of out-of-range column vectors were never written: skip them
            if ((MODE & kSpmm)) {
#pragma unroll
                for (int q = 0; q < NV; ++q)
                    if (colok[q]) acc.fma(q, wk, x[q]);
            }
            if ((MODE & kSddmm)) {
#pragma unroll
                for (int q = 0; q < NV; ++q)
                    if (colok[q]) d = dot_raw(own[q], x[q], d);
            }
        }
        return d;
    };
    // refill `slot` (= j mod D) with position base + j + D, whose column
    // index lane (j + D) mod G holds in `cols` (c_cur: this batch, c_nxt: the next)
    auto refill = [&](int base, int j, int slot, int cols, bool check) {
        const int src = __shfl_sync(FULL, cols, (j + D) & (G - 1), G);
        if (!check || base + j + D < len) issue(slot, src);
        if (j % STEP == STEP - 1) cp_async_commit();
    };
    // the unguarded batch of the gradient walks runs in chunks of U positions
    // (rolled), so that their longer row-switch code is inlined U times rather
    // than G times; the forward walk keeps the whole batch unrolled
    constexpr int U = (MODE & kSddmm) ? chunk_of(G, D) : G;
    static_assert(U % STEP == 0 && (U == G || (G - D) % U == 0) && (U >= D ? U % D == 0 : D % U == 0),
                  "chunk shape");

    for (int base = 0; base < len_max; base += G) {
        if (base > 0) {
            c_cur = c_nxt; e_cur = e_nxt; w_cur = w_nxt; sc_cur = sc_nxt;
            c_nxt = c_nn; e_nxt = e_nn;
        }
        // weights of the next batch, indices of the one after
        if ((MODE & kSpmm)) w_nxt = (base + G + gl < len) ? load_w(P.w + e_nxt) : 0.f;
        if constexpr ((MODE & kEdgeScale) != 0) {
            sc_nxt = (base + G + gl < len) ? P.inv_cnt[c_nxt] : 1.f;
            w_nxt *= sc_nxt;
        }
        c_nn = 0;
        e_nn = 0;
        if (base + 2 * G + gl < len) {
            c_nn = __ldcs(P.col + p0 + base + 2 * G + gl);
            e_nn = __ldcs(P.order + p0 + base + 2 * G + gl);
        }
        if (base + G + D <= len_min) {
#pragma unroll 1
            for (int c = 0; c < G / U; ++c) {
                float dots[U];
                const int j0 = U == G ? 0 : c * U;
                const int slot0 = U >= D ? 0 : j0 % D;
#pragma unroll
                for (int t = 0; t < U; t += STEP) {
                    cp_async_wait<D / STEP - 1>();
#pragma unroll
                    for (int u = 0; u < STEP; ++u)
                        dots[t + u] = consume(base, j0 + t + u, U >= D ? (t + u) % D : slot0 + t + u, true);
                    // (G - D) is a multiple of U: one source batch per chunk
#pragma unroll
                    for (int u = 0; u < STEP; ++u)
                        refill(base, j0 + t + u, U >= D ? (t + u) % D : slot0 + t + u,
                               (U == G ? t + u + D < G : j0 + D < G) ? c_cur : c_nxt, false);
                }
                if ((MODE & kSddmm)) {
                    const float d = reduce_chunk<U, G>(dots, gl, FULL);
                    if ((gl & ~(U - 1)) == j0)  // lane j0 + t: position j0 + t
                        P.dw[e_cur] = (MODE & kEdgeScale) ? d * sc_cur : d;
                }
            }
        } else {
#pragma unroll 1
            for (int j = 0; j < G; ++j) {
                if (j % STEP == 0) cp_async_wait<D / STEP - 1>();
                float d = consume(base, j, j % D, base + j < len);
                if ((MODE & kSddmm)) {
#pragma unroll
                    for (int o = G / 2; o > 0; o >>= 1) d += __shfl_xor_sync(FULL, d, o, G);
                    if (gl == j && base + j < len) P.dw[e_cur] = (MODE & kEdgeScale) ? d * sc_cur : d;
                }
                refill(base, j, j % D, j + D < G ? c_cur : c_nxt, true);
            }
        }
    }
    if ((MODE & kSpmm) && active) {
        if (before) write_open_row(slot_head);
        else if (rend > p0 + len) write_open_row(slot_tail);
        else write_open_row(nullptr);
    }
    cp_async_wait<0>();
}

// ---------------------------------------------------------------------------- warp walk: one warp per tile

// The walk for rows of 1024 bytes (fp32 H = 256, bf16 H = 512), which the
// ring walk would hold as four 16-byte vectors per lane.  One warp walks one
// tile, one CSR position at a time, and every lane owns 32 bytes of each row
// (two 16-byte segments).  Gathered rows travel global -> shared memory with
// cp.async into a per-warp ring of D = 4 rows (4 KB per warp), so that a warp
// keeps D rows in flight without holding them in registers; each lane copies,
// and later reads, only its own bytes of every row, so no barrier is needed
// between copy and read.  (Rows are not moved by the tensor memory
// accelerator: on B200, tile::gather4 copies gathered random 256-byte rows
// with R-MAT-distributed ids from a 1 GiB table at 6 TB/s even with ten
// CTAs per SM, per-row cp.async.bulk copies slower still, and plain loads at
// about 15 TB/s.)
// All 32 lanes work on the same position, so the row-end test, the weight
// and the column index are warp-uniform: a batch of 32 positions that lies
// inside one row runs without any test, in unrolled chunks of 8 positions;
// the others run one position at a time with the row-end test.
//   kSpmm : out[row] = sum w[slot(p)] * F[col[p]] over the row's positions
//   kSddmm: dw[slot(p)] = dot(R[row], F[col[p]]); the per-lane partial dots of
//           a chunk of 8 positions are reduced with one reduce-scatter (one
//           butterfly per position in the batches with row ends), after which
//           lane p % 32 writes the weight gradient of position p
//   kBoth : both on one walk of the transpose CSR
// Owner rows (kSddmm) are loaded kOwnAhead rows ahead of their first use;
// the next 64 rows' ids and ends are held in two 32-row windows, one lane per
// row, the second loaded while the first is used.  Rows cut by a tile
// boundary leave partial rows exactly as in k_tiles (slot 2t: continued from
// the previous tile, 2t + 1: continued in the next), summed by k_fixup.

// This lane's LB bytes of a row: NSEG segments of SEGB bytes, segment q of
// lane l at byte q * 32 * SEGB + l * SEGB, so that a warp-wide access of one
// segment touches 32 * SEGB consecutive bytes.
template <int LB> struct Slice {
    static_assert(LB % 16 == 0, "16-byte segments");
    static constexpr int SEGB = 16;
    static constexpr int NSEG = LB / SEGB;
    static constexpr int NW = LB / 4;
    uint32_t w[NW];
};

template <int LB>
__device__ __forceinline__ void load_slice(const char *p, Slice<LB> &s) {
#pragma unroll
    for (int q = 0; q < Slice<LB>::NSEG; ++q) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p + q * 32 * 16));
        s.w[4 * q] = v.x;
        s.w[4 * q + 1] = v.y;
        s.w[4 * q + 2] = v.z;
        s.w[4 * q + 3] = v.w;
    }
}
// the same from this lane's bytes of a ring slot
template <int LB>
__device__ __forceinline__ void lds_slice(const char *p, Slice<LB> &s) {
#pragma unroll
    for (int q = 0; q < Slice<LB>::NSEG; ++q) {
        const uint4 v = *reinterpret_cast<const uint4 *>(p + q * 32 * 16);
        s.w[4 * q] = v.x;
        s.w[4 * q + 1] = v.y;
        s.w[4 * q + 2] = v.z;
        s.w[4 * q + 3] = v.w;
    }
}
// copy this lane's bytes of a row (src: row start + lane offset) to a ring slot
template <int LB>
__device__ __forceinline__ void cp_async_slice(uint32_t dst, const char *src) {
#pragma unroll
    for (int q = 0; q < Slice<LB>::NSEG; ++q) cp_async16(dst + q * 32 * 16, src + q * 32 * 16);
}

// fp32 values of a slice, in feature order within each segment
template <typename T, int LB>
__device__ __forceinline__ void unpack_slice(const Slice<LB> &s, float (&v)[LB / sizeof(T)]) {
    if constexpr (sizeof(T) == 4) {
#pragma unroll
        for (int k = 0; k < Slice<LB>::NW; ++k) v[k] = __uint_as_float(s.w[k]);
    } else {
#pragma unroll
        for (int k = 0; k < Slice<LB>::NW; ++k) {
            v[2 * k] = bf16_lo(s.w[k]);
            v[2 * k + 1] = bf16_hi(s.w[k]);
        }
    }
}

// Output row slice in the feature dtype (streaming stores: written once).
template <typename T, int LB>
__device__ __forceinline__ void store_slice(char *p, const float (&v)[LB / sizeof(T)]) {
    uint32_t w[Slice<LB>::NW];
#pragma unroll
    for (int k = 0; k < Slice<LB>::NW; ++k)
        w[k] = sizeof(T) == 4 ? __float_as_uint(v[k]) : pack_bf16(v[2 * k], v[2 * k + 1]);
#pragma unroll
    for (int q = 0; q < Slice<LB>::NSEG; ++q)
        __stcs(reinterpret_cast<uint4 *>(p + q * 32 * 16), make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]));
}

// The same slice as fp32 partial sums, at the same feature indices of a
// partial row [H] (what k_fixup adds up).
template <typename T, int LB>
__device__ __forceinline__ void store_slice_partial(float *row, int lane, const float (&v)[LB / sizeof(T)]) {
    constexpr int SEGB = Slice<LB>::SEGB, VPS = SEGB / int(sizeof(T));
#pragma unroll
    for (int q = 0; q < Slice<LB>::NSEG; ++q) {
        float *d = row + (q * 32 * SEGB + lane * SEGB) / int(sizeof(T));
#pragma unroll
        for (int i = 0; i < VPS; i += 4)
            *reinterpret_cast<float4 *>(d + i) =
                make_float4(v[q * VPS + i], v[q * VPS + i + 1], v[q * VPS + i + 2], v[q * VPS + i + 3]);
    }
}

constexpr int kZeroRowsPerWarp = 8;  // empty rows zeroed by each of the trailing warps
constexpr int kOwnAhead = 2;         // owner rows loaded ahead of their first use (gradient walks)
constexpr int kWalkRingBytes = 4096;  // ring bytes per warp: D = kWalkRingBytes / row bytes rows in flight

// ids and ends of the non-empty rows base .. base + 31 (one per lane);
// past the last row: row 0 (a valid address) and an end no position reaches
__device__ __forceinline__ void load_rows(const Params &P, int64_t base, int lane, int &row, int &end) {
    row = 0;
    end = INT_MAX;
    if (base + lane < P.n_nz) {
        row = __ldg(P.nz_rows + base + lane);
        end = __ldg(P.nz_rowptr + base + lane + 1);
    }
}

// resident CTAs per SM the walk is compiled for (a register budget)
// resident blocks the warp walk is compiled for: 1024 (SpMM) or 512 (with
// the dot product) threads per SM, whatever the block size
constexpr int walk_min_blocks(int MODE) { return ((MODE & kSddmm) ? 512 : 1024) / kWalkThreads; }

template <typename T, int LB, int MODE>
__global__ void __launch_bounds__(kWalkThreads, walk_min_blocks(MODE)) k_walk(const Params P) {
    using S = Slice<LB>;
    constexpr unsigned FULL = 0xffffffffu;
    constexpr int VPL = LB / int(sizeof(T));
    constexpr int RB = 32 * LB;
    constexpr int D = kWalkRingBytes / RB;  // rows in flight per warp
    constexpr int CH = 8;                   // positions per unrolled chunk (and per reduction of partial dots)
    static_assert(32 % D == 0 && (D >= CH ? D % CH == 0 : CH % D == 0), "chunk shapes");
    constexpr bool SPMM = (MODE & kSpmm) != 0, SDDMM = (MODE & kSddmm) != 0;
    constexpr bool ROW_SCALE = (MODE & kRowScale) != 0, EDGE_SCALE = (MODE & kEdgeScale) != 0;
    extern __shared__ uint4 walk_ring[];  // (kWalkThreads / 32) * kWalkRingBytes bytes
    char *ring = reinterpret_cast<char *>(walk_ring);

    const int lane = threadIdx.x & 31;
    const int64_t warp = (int64_t(blockIdx.x) * kWalkThreads + threadIdx.x) >> 5;
    const int lane_off = lane * S::SEGB;
    if (warp >= P.n_tiles) {  // trailing warps: rows without edges get zeros
        const int64_t z0 = (warp - P.n_tiles) * kZeroRowsPerWarp;
        float zero[VPL];
#pragma unroll
        for (int v = 0; v < VPL; ++v) zero[v] = 0.f;
        for (int k = 0; k < kZeroRowsPerWarp && z0 + k < P.n_zero; ++k)
            store_slice<T, LB>(static_cast<char *>(P.out) + int64_t(P.zero_rows[z0 + k]) * RB + lane_off, zero);
        return;
    }
    // this lane's bytes of ring slot s: my + s * RB (shared address my_s + s * RB)
    const char *my = ring + (threadIdx.x >> 5) * kWalkRingBytes + lane_off;
    const uint32_t my_s = smem_addr(my);

    const int p0 = int(warp * P.T);
    const int pend = int(min(int64_t(p0) + P.T, P.E));
    const char *__restrict__ F = static_cast<const char *>(P.F) + lane_off;
    const char *__restrict__ R = static_cast<const char *>(P.R) + lane_off;
    char *__restrict__ out = static_cast<char *>(P.out) + lane_off;
    float *slot_head = P.partial + (2 * warp) * P.H;
    float *slot_tail = P.partial + (2 * warp + 1) * P.H;

    // the open row, and the next 64 rows in two windows (a: next 32, b: the 32 after)
    int64_t ci = P.tile_nz[warp];
    int row = __ldg(P.nz_rows + ci);
    int rend = __ldg(P.nz_rowptr + ci + 1);
    bool before = __ldg(P.nz_rowptr + ci) < p0;
    int64_t wbase = ci + 1;
    int wa_row, wa_end, wb_row, wb_end;
    load_rows(P, wbase, lane, wa_row, wa_end);
    load_rows(P, wbase + 32, lane, wb_row, wb_end);
    int wk = 0;  // the next row is window a, lane wk

    // column index and weight slot of batch b (cur), b + 1 (nxt); weights of b
    int c_cur = 0, s_cur = 0, c_nxt = 0, s_nxt = 0;
    if (p0 + lane < pend) {
        c_cur = __ldcs(P.col + p0 + lane);
        s_cur = __ldcs(P.order + p0 + lane);
    }
    if (p0 + 32 + lane < pend) {
        c_nxt = __ldcs(P.col + p0 + 32 + lane);
        s_nxt = __ldcs(P.order + p0 + 32 + lane);
    }
    float w_cur = 0.f;
    if (SPMM && p0 + lane < pend) {
        w_cur = load_w(P.w + s_cur);
        if constexpr (EDGE_SCALE) w_cur *= __ldg(P.inv_cnt + c_cur);
    }

    // rows in flight: positions b0 + j .. b0 + j + D - 1, slot = position mod D,
    // one cp.async group per position (empty past the tile's end)
#pragma unroll
    for (int u = 0; u < D; ++u) {
        cp_async_slice<LB>(my_s + u * RB, F + int64_t(__shfl_sync(FULL, c_cur, u)) * RB);
        cp_async_commit();
    }

    float acc[VPL], own[VPL];
#pragma unroll
    for (int v = 0; v < VPL; ++v) acc[v] = 0.f, own[v] = 0.f;
    S oq[kOwnAhead];  // owner rows of window a, lanes wk .. wk + kOwnAhead - 1
    if constexpr (SDDMM) {
        S o;
        load_slice<LB>(R + int64_t(row) * RB, o);
        unpack_slice<T, LB>(o, own);
#pragma unroll
        for (int k = 0; k < kOwnAhead; ++k) load_slice<LB>(R + int64_t(__shfl_sync(FULL, wa_row, k)) * RB, oq[k]);
    }

    auto flush = [&](float *slot) {
        if (slot) {
            store_slice_partial<T, LB>(slot, lane, acc);
        } else {
            if constexpr (ROW_SCALE) {
                const float r = __ldg(P.inv_cnt + row);
#pragma unroll
                for (int v = 0; v < VPL; ++v) acc[v] *= r;
            }
            store_slice<T, LB>(out + int64_t(row) * RB, acc);
        }
    };
    // the open row ended at the current position: write it, open the next
    auto next_row = [&]() {
        if constexpr (SPMM) {
            flush(before ? slot_head : nullptr);
#pragma unroll
            for (int v = 0; v < VPL; ++v) acc[v] = 0.f;
        }
        before = false;
        if constexpr (SDDMM) {
            unpack_slice<T, LB>(oq[0], own);
#pragma unroll
            for (int k = 0; k + 1 < kOwnAhead; ++k) oq[k] = oq[k + 1];
            const int k = wk + kOwnAhead;
            const int r = __shfl_sync(FULL, k < 32 ? wa_row : wb_row, k & 31);
            load_slice<LB>(R + int64_t(r) * RB, oq[kOwnAhead - 1]);
        }
        row = __shfl_sync(FULL, wa_row, wk);
        rend = __shfl_sync(FULL, wa_end, wk);
        if (++wk == 32) {
            wa_row = wb_row;
            wa_end = wb_end;
            wk = 0;
            wbase += 32;
            load_rows(P, wbase + 32, lane, wb_row, wb_end);
        }
    };

    float dots[CH];
#pragma unroll
    for (int t = 0; t < CH; ++t) dots[t] = 0.f;
    // Position b0 + j (held in ring slot `slot`): returns this lane's part of
    // its dot product (SDDMM); CHECK: test the tile end and the row end.
    auto position = [&](int b0, int j, int slot, bool check) -> float {
        const bool valid = !check || b0 + j < pend;
        cp_async_wait<D - 1>();  // the group of this position has landed
        if (check && valid && b0 + j == rend) next_row();
        S xs;
        lds_slice<LB>(my + slot * RB, xs);
        float xv[VPL];
        unpack_slice<T, LB>(xs, xv);
        if constexpr (SPMM) {
            const float wj = __shfl_sync(FULL, w_cur, j & 31);
            if (valid) {
#pragma unroll
                for (int v = 0; v < VPL; ++v) acc[v] = fmaf(wj, xv[v], acc[v]);
            }
        }
        float d = 0.f;
        if constexpr (SDDMM) {
#pragma unroll
            for (int v = 0; v < VPL; ++v) d = fmaf(own[v], xv[v], d);
        }
        // refill the slot with position b0 + j + D (the column of a position
        // past the tile's end is 0: a valid row, never read)
        const int jn = j + D;
        const int src = __shfl_sync(FULL, jn < 32 ? c_cur : c_nxt, jn & 31);
        cp_async_slice<LB>(my_s + slot * RB, F + int64_t(src) * RB);
        cp_async_commit();
        return valid ? d : 0.f;
    };

    for (int b0 = p0; b0 < pend; b0 += 32) {
        // indices of batch b + 2 (prefetched, consumed next batch), weights of batch b + 1
        int c_nn = 0, s_nn = 0;
        if (b0 + 64 + lane < pend) {
            c_nn = __ldcs(P.col + b0 + 64 + lane);
            s_nn = __ldcs(P.order + b0 + 64 + lane);
        }
        float w_nxt = 0.f;
        if (SPMM && b0 + 32 + lane < pend) {
            w_nxt = load_w(P.w + s_nxt);
            if constexpr (EDGE_SCALE) w_nxt *= __ldg(P.inv_cnt + c_nxt);
        }
        if (b0 + 32 <= pend && rend >= b0 + 32) {
            // the whole batch lies in the open row: chunks of CH positions
            // without tests; the CH partial dots of a chunk are reduced with
            // one reduce-scatter, after which lane j of the chunk's lane block
            // holds the dot of position b0 + lane and writes it
#pragma unroll 1
            for (int c = 0; c < 32; c += CH) {
                const int sb = c % D;  // slots sb .. sb + CH - 1 (mod D) hold the chunk
#pragma unroll
                for (int t = 0; t < CH; ++t) dots[t] = position(b0, c + t, D >= CH ? sb + t : t % D, false);
                if constexpr (SDDMM) {
                    const float d = reduce_chunk<CH, 32>(dots, lane, FULL);
                    if ((lane & ~(CH - 1)) == c) P.dw[s_cur] = EDGE_SCALE ? d * __ldg(P.inv_cnt + c_cur) : d;
                }
            }
        } else {
            // one position at a time with the row-end test; each dot is
            // reduced over the warp on its own and written by lane j
#pragma unroll 1
            for (int j = 0; j < 32; ++j) {
                float d = position(b0, j, j % D, true);
                if constexpr (SDDMM) {
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(FULL, d, o);
                    if (lane == j && b0 + j < pend) P.dw[s_cur] = EDGE_SCALE ? d * __ldg(P.inv_cnt + c_cur) : d;
                }
            }
        }
        c_cur = c_nxt;
        s_cur = s_nxt;
        w_cur = w_nxt;
        c_nxt = c_nn;
        s_nxt = s_nn;
    }
    if constexpr (SPMM) {
        if (before) flush(slot_head);
        else if (rend > pend) flush(slot_tail);
        else flush(nullptr);
    }
    cp_async_wait<0>();
}

template <int VEC, int NV>
__device__ __forceinline__ void scale_rows(float (&acc)[NV][VEC], float r) {
#pragma unroll
    for (int k = 0; k < NV; ++k)
#pragma unroll
        for (int v = 0; v < VEC; ++v) acc[k][v] *= r;
}

// Rows cut by tile boundaries: out[row] = slot(2 * first + 1) + sum over the
// following tiles t of slot(2t), in tile order.  Blocks [0, n_long) take one
// long span each with the whole CTA: lane group q < kStripes adds the tiles
// t = first + 1 + q, first + 1 + q + kStripes, ... in order, and group 0 then
// adds the stripes in order.  The stripe count is fixed, so the result does
// not depend on the lane-group width.  The remaining blocks take one span per
// lane group, added sequentially.
constexpr int kStripes = 8;

template <typename T, int VEC, int NV>
__global__ void __launch_bounds__(kThreads)
k_fixup(const int4 *__restrict__ spans, int64_t n_long, int64_t n_span, const float *__restrict__ partial,
        void *out, int64_t H, int G, int log2G, int col_tiles, const float *__restrict__ row_scale) {
    __shared__ float red[kStripes * 32 * NV * VEC];
    const int gl = threadIdx.x & (G - 1);
    const int gi = threadIdx.x >> log2G;
    const int ng = kThreads >> log2G;
    const int64_t HV = H / VEC;
    if (blockIdx.x < n_long) {
        const int4 sp = spans[blockIdx.x];
        for (int tile = 0; tile < col_tiles; ++tile) {
            const int64_t vbase = int64_t(tile) * G * NV + gl;
            bool ok[NV];
#pragma unroll
            for (int k = 0; k < NV; ++k) ok[k] = vbase + int64_t(k) * G < HV;
            float acc[NV][VEC];
#pragma unroll
            for (int k = 0; k < NV; ++k)
#pragma unroll
                for (int v = 0; v < VEC; ++v) acc[k][v] = 0.f;
            if (gi < kStripes) {
                if (gi == 0) {
                    const float *s0 = partial + (2 * int64_t(sp.y) + 1) * H;
#pragma unroll
                    for (int k = 0; k < NV; ++k)
                        if (ok[k]) add_partial<VEC>(s0 + (vbase + int64_t(k) * G) * VEC, acc[k]);
                }
                for (int64_t t = sp.y + 1 + gi; t <= sp.z; t += kStripes) {
                    const float *s1 = partial + (2 * t) * H;
#pragma unroll
                    for (int k = 0; k < NV; ++k)
                        if (ok[k]) add_partial<VEC>(s1 + (vbase + int64_t(k) * G) * VEC, acc[k]);
                }
#pragma unroll
                for (int k = 0; k < NV; ++k)
#pragma unroll
                    for (int v = 0; v < VEC; ++v) red[(gi * G * NV + k * G + gl) * VEC + v] = acc[k][v];
            }
            __syncthreads();
            if (gi == 0) {
                for (int q = 1; q < kStripes; ++q)
#pragma unroll
                    for (int k = 0; k < NV; ++k)
#pragma unroll
                        for (int v = 0; v < VEC; ++v) acc[k][v] += red[(q * G * NV + k * G + gl) * VEC + v];
                T *row = static_cast<T *>(out) + int64_t(sp.x) * H;
                if (row_scale) scale_rows<VEC, NV>(acc, row_scale[sp.x]);
                store_row<T, VEC, NV>(row, vbase, G, ok, acc);
            }
            __syncthreads();
        }
        return;
    }
    const int64_t s = n_long + (int64_t(blockIdx.x) - n_long) * ng + gi;
    if (s >= n_span) return;
    const int4 sp = spans[s];
    for (int tile = 0; tile < col_tiles; ++tile) {
        const int64_t vbase = int64_t(tile) * G * NV + gl;
        bool ok[NV];
#pragma unroll
        for (int k = 0; k < NV; ++k) ok[k] = vbase + int64_t(k) * G < HV;
        float acc[NV][VEC];
#pragma unroll
        for (int k = 0; k < NV; ++k)
#pragma unroll
            for (int v = 0; v < VEC; ++v) acc[k][v] = 0.f;
        const float *s0 = partial + (2 * int64_t(sp.y) + 1) * H;
#pragma unroll
        for (int k = 0; k < NV; ++k)
            if (ok[k]) add_partial<VEC>(s0 + (vbase + int64_t(k) * G) * VEC, acc[k]);
        for (int64_t t = sp.y + 1; t <= sp.z; ++t) {
            const float *s1 = partial + (2 * t) * H;
#pragma unroll
            for (int k = 0; k < NV; ++k)
                if (ok[k]) add_partial<VEC>(s1 + (vbase + int64_t(k) * G) * VEC, acc[k]);
        }
        if (row_scale) scale_rows<VEC, NV>(acc, row_scale[sp.x]);
        store_row<T, VEC, NV>(static_cast<T *>(out) + int64_t(sp.x) * H, vbase, G, ok, acc);
    }
}

// ---------------------------------------------------------------------------- host side

struct Shape {
    int vec, G, log2G, nv, col_tiles;
    int lb;  // > 0: bytes per lane of the register walk (rows of 32 * lb bytes)
};

int log2i(int v) {
    int l = 0;
    while ((1 << l) < v) ++l;
    return l;
}

bool aligned(const void *p, size_t a) { return p == nullptr || reinterpret_cast<uintptr_t>(p) % a == 0; }

// Widest vector whose width divides H and whose alignment all pointers meet.
Shape pick_shape(int64_t H, int dtype, const void *a, const void *b, const void *c) {
    const int elem = dtype == AG_F32 ? 4 : 2;
    const int cands_f32[] = {4, 1};
    const int cands_bf16[] = {8, 2, 1};
    const int *cands = dtype == AG_F32 ? cands_f32 : cands_bf16;
    const int ncand = dtype == AG_F32 ? 2 : 3;
    int vec = 1;
    for (int i = 0; i < ncand; ++i) {
        int v = cands[i];
        size_t al = size_t(v) * elem;
        if (H % v == 0 && aligned(a, al) && aligned(b, al) && aligned(c, al)) {
            vec = v;
            break;
        }
    }
    Shape s;
    s.vec = vec;
    const int64_t HV = H / vec;
    int G = 1;
    while (G < AG_MAX_LANES && G < HV) G <<= 1;
    s.G = G;
    s.log2G = log2i(G);
    const int64_t per_lane = (HV + G - 1) / G;
    s.nv = per_lane <= 1 ? 1 : (per_lane <= 2 ? 2 : 4);
    s.col_tiles = int((HV + int64_t(G) * s.nv - 1) / (int64_t(G) * s.nv));
    // the warp walk: rows of 1024 bytes (fp32 H = 256, bf16 H = 512), every
    // pointer 16-byte aligned; narrower rows take the shared-memory ring walk
    const int64_t row_bytes = H * elem;
    s.lb = 0;
    if (AG_WALK && row_bytes == 1024 && aligned(a, 16) && aligned(b, 16) && aligned(c, 16)) s.lb = 32;
    return s;
}

template <typename T, int VEC, int NV, int G, int MODE>
void launch_ring(const Params &P, cudaStream_t st) {
    constexpr int D = kRingDepth < G ? kRingDepth : G;
    // tile groups padded to whole warps, then the empty-row groups
    const int64_t per_warp = 32 / G;
    const int64_t groups = (P.n_tiles + per_warp - 1) / per_warp * per_warp + P.n_zero;
    constexpr int TPB = ring_threads(MODE);
    const unsigned grid = unsigned((groups + TPB / G - 1) / (TPB / G));
    // ring: D slots x NV vectors x 16 bytes for every lane of the block
    const size_t smem = size_t(TPB) * D * NV * 16;
    // the shared-memory limit is an attribute of the function in each device's
    // context: set it once per device (a race only repeats the same call)
    static std::atomic<uint64_t> configured{0};
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = uint64_t(1) << (dev & 63);
    if (!(configured.load(std::memory_order_relaxed) & bit)) {
        cudaFuncSetAttribute(k_tiles_ring<T, VEC, NV, G, MODE, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem));
        configured.fetch_or(bit, std::memory_order_relaxed);
    }
    k_tiles_ring<T, VEC, NV, G, MODE, D><<<grid, TPB, smem, st>>>(P);
}

template <typename T, int VEC, int NV, int MODE>
void launch_main(const Params &P, const Shape &s, cudaStream_t st) {
    const int64_t groups_per_block = kThreads / s.G;
    const int64_t groups = P.n_tiles + P.n_zero;
    const unsigned grid = unsigned((groups + groups_per_block - 1) / groups_per_block);
    if constexpr (sizeof(typename Vec<T, VEC>::raw) == 16 && NV <= 2) {
        if (s.col_tiles == 1 && s.G >= 4 && int64_t(s.G) * NV * VEC == P.H) {
            switch (s.G) {
                case 4: launch_ring<T, VEC, NV, 4, MODE>(P, st); return;
                case 8: launch_ring<T, VEC, NV, 8, MODE>(P, st); return;
                case 16: launch_ring<T, VEC, NV, 16, MODE>(P, st); return;
                default: launch_ring<T, VEC, NV, 32, MODE>(P, st); return;
            }
        }
    }
    if constexpr (MODE != kBoth && (MODE & (kRowScale | kEdgeScale)) == 0) {
        if (s.col_tiles == 1) k_tiles<T, VEC, NV, MODE, true><<<grid, kThreads, 0, st>>>(P);
        else k_tiles<T, VEC, NV, MODE, false><<<grid, kThreads, 0, st>>>(P);
    }
}

template <typename T, int VEC, int NV>
void launch_fixup(const ag::Direction &D, const float *partial, void *out, int64_t H, const Shape &s,
                  const float *row_scale, cudaStream_t st) {
    const int64_t groups_per_block = kThreads / s.G;
    const int64_t short_spans = D.n_span - D.n_span_long;
    const unsigned grid = unsigned(D.n_span_long + (short_spans + groups_per_block - 1) / groups_per_block);
    k_fixup<T, VEC, NV><<<grid, kThreads, 0, st>>>(D.spans, D.n_span_long, D.n_span, partial, out, H, s.G,
                                                   s.log2G, s.col_tiles, row_scale);
}

template <int MODE, typename T, int VEC>
void dispatch_nv(const Params &P, const Shape &s, cudaStream_t st) {
    switch (s.nv) {
        case 1: launch_main<T, VEC, 1, MODE>(P, s, st); break;
        case 2: launch_main<T, VEC, 2, MODE>(P, s, st); break;
        default: launch_main<T, VEC, 4, MODE>(P, s, st); break;
    }
}

template <typename T, int LB, int MODE>
void launch_walk(const Params &P, cudaStream_t st) {
    const int64_t warps = P.n_tiles + (P.n_zero + kZeroRowsPerWarp - 1) / kZeroRowsPerWarp;
    const unsigned grid = unsigned((warps + kWalkThreads / 32 - 1) / (kWalkThreads / 32));
    const size_t smem = size_t(kWalkThreads / 32) * kWalkRingBytes;
    // the shared-memory limit is an attribute of the function in each device's
    // context: set it once per device (a race only repeats the same call)
    static std::atomic<uint64_t> configured{0};
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = uint64_t(1) << (dev & 63);
    if (!(configured.load(std::memory_order_relaxed) & bit)) {
        cudaFuncSetAttribute(k_walk<T, LB, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        configured.fetch_or(bit, std::memory_order_relaxed);
    }
    if (grid > 0) k_walk<T, LB, MODE><<<grid, kWalkThreads, smem, st>>>(P);
}

template <int MODE, typename T>
void dispatch_walk(const Params &P, int lb, cudaStream_t st) {
    launch_walk<T, 32, MODE>(P, st);  // pick_shape selects the warp walk for 1024-byte rows only
}

template <int MODE>
void dispatch_main(const Params &P, const Shape &s, int dtype, cudaStream_t st) {
    if (s.lb > 0) {
        if (dtype == AG_F32) dispatch_walk<MODE, float>(P, s.lb, st);
        else dispatch_walk<MODE, bf16_t>(P, s.lb, st);
        return;
    }
    if (dtype == AG_F32) {
        if (s.vec == 4) dispatch_nv<MODE, float, 4>(P, s, st);
        else dispatch_nv<MODE, float, 1>(P, s, st);
    } else {
        if (s.vec == 8) dispatch_nv<MODE, bf16_t, 8>(P, s, st);
        else if (s.vec == 2) dispatch_nv<MODE, bf16_t, 2>(P, s, st);
        else dispatch_nv<MODE, bf16_t, 1>(P, s, st);
    }
}

template <typename T, int VEC>
void fixup_nv(const ag::Direction &D, const float *partial, void *out, int64_t H, const Shape &s,
              const float *row_scale, cudaStream_t st) {
    switch (s.nv) {
        case 1: launch_fixup<T, VEC, 1>(D, partial, out, H, s, row_scale, st); break;
        case 2: launch_fixup<T, VEC, 2>(D, partial, out, H, s, row_scale, st); break;
        default: launch_fixup<T, VEC, 4>(D, partial, out, H, s, row_scale, st); break;
    }
}

// row_scale: non-null multiplies every finished row by row_scale[row] (mean)
void dispatch_fixup(const ag::Direction &D, const float *partial, void *out, int64_t H, const Shape &s,
                    int dtype, cudaStream_t st, const float *row_scale = nullptr) {
    if (dtype == AG_F32) {
        if (s.vec == 4) fixup_nv<float, 4>(D, partial, out, H, s, row_scale, st);
        else fixup_nv<float, 1>(D, partial, out, H, s, row_scale, st);
    } else {
        if (s.vec == 8) fixup_nv<bf16_t, 8>(D, partial, out, H, s, row_scale, st);
        else if (s.vec == 2) fixup_nv<bf16_t, 2>(D, partial, out, H, s, row_scale, st);
        else fixup_nv<bf16_t, 1>(D, partial, out, H, s, row_scale, st);
    }
}

Params base_params(const ag_graph *g, const ag::Direction &D, int64_t H, const Shape &s) {
    Params P{};
    P.col = D.col;
    P.order = D.order;
    P.nz_rows = D.nz_rows;
    P.nz_rowptr = D.nz_rowptr;
    P.tile_nz = D.tile_nz;
    P.zero_rows = D.zero_rows;
    P.E = g->E;
    P.H = H;
    P.n_nz = D.n_nz;
    P.n_tiles = g->n_tiles;
    P.T = g->tile_edges;
    P.G = s.G;
    P.log2G = s.log2G;
    P.col_tiles = s.col_tiles;
    return P;
}

int check_call(const ag_graph *g, int64_t H, int dtype, const char *fn) {
    if (!g) return fail(AG_ERR_INVALID_ARG, "%s: null graph", fn);
    if (dtype != AG_F32 && dtype != AG_BF16) return fail(AG_ERR_DTYPE, "%s: unknown dtype %d", fn, dtype);
    if (H < 1 || H > (int64_t(1) << 24) || g->N * H >= (int64_t(1) << 40))
        return fail(AG_ERR_SHAPE, "%s: H=%lld out of range for N=%lld", fn, (long long)H, (long long)g->N);
    return check_current_device(g, fn);
}

// Per-call scratch: [partial rows][weights, bucketed][weight gradient, bucketed]
struct ScratchLayout {
    size_t partial, w_b, dw_b, inv, total;
};
ScratchLayout scratch_layout(const ag_graph *g, int64_t H) {
    ScratchLayout L;
    const bool spans = g->dir[0].n_span > 0 || g->dir[1].n_span > 0;
    const size_t part = spans ? size_t(2) * size_t(g->n_tiles) * size_t(H) * 4 : 0;
    const size_t ev = size_t(g->E) * 4;
    L.partial = 0;
    L.w_b = align_up(part);
    L.dw_b = L.w_b + align_up(ev);
    L.inv = L.dw_b + align_up(ev);  // mean: 1 / in-degree per node
    L.total = g->E > 0 ? L.inv + align_up(size_t(g->N) * 4) : L.w_b;
    return L;
}
size_t scratch_needed(const ag_graph *g, int64_t H) {
    const ScratchLayout L = scratch_layout(g, H);
    return (g->E > 0 || L.w_b > 0) ? L.total : 0;
}

// Optional per-edge factor applied while regrouping: divide the value of COO
// edge e by the in-degree of its destination (mean aggregation).  dst = null:
// no factor.
struct EdgeScale {
    const int32_t *dst = nullptr;     // COO destinations [E]
    const int32_t *rowptr = nullptr;  // forward CSR row pointers [N + 1]
    const float *mul = nullptr;       // into buckets only: multiply edge e's value by mul[e] first
};
__device__ __forceinline__ float per_dst(float v, const EdgeScale &sc, int64_t e) {
    const int d = __ldcs(sc.dst + e);
    return __fdiv_rn(v, float(sc.rowptr[d + 1] - sc.rowptr[d]));  // >= 1: the edge itself
}

// w_b[slot[e]] = w[e] (w = null: 1): COO-ordered weights into the
// window-bucketed layout.  Reads are coalesced; the slots of consecutive
// ordinals that share a window are consecutive, so the writes land in short
// runs that L2 merges.
template <bool SCALED>
__global__ void k_bucket_scatter(const float *__restrict__ w, const int32_t *__restrict__ slot, int64_t E,
                                 EdgeScale sc, float *__restrict__ w_b) {
    for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < E; e += int64_t(gridDim.x) * blockDim.x) {
        float v = w ? __ldcs(w + e) : 1.f;
        if (sc.mul) v *= __ldcs(sc.mul + e);
        if (SCALED) v = per_dst(v, sc, e);
        w_b[__ldcs(slot + e)] = v;
    }
}
// dw[e] = dw_b[slot[e]]: the bucketed weight gradient back to COO order.
template <bool SCALED>
__global__ void k_bucket_gather(const float *__restrict__ dw_b, const int32_t *__restrict__ slot, int64_t E,
                                EdgeScale sc, float *__restrict__ dw) {
    for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < E; e += int64_t(gridDim.x) * blockDim.x) {
        float v = dw_b[__ldcs(slot + e)];
        if (SCALED) v = per_dst(v, sc, e);
        __stcs(dw + e, v);
    }
}
// Staged regrouping with the lowering's table: the ordinals of one chunk,
// sorted by window, form runs of consecutive slots (slots of a window are
// handed out in COO order), and slot + delta[window] is an ordinal's place in
// that order.  TO_BUCKETS: w_b[slot[e]] = w[e] written run by run; otherwise
// dw[e] = dw_b[slot[e]] read run by run.  Both sides coalesced, no atomics.
constexpr int kStageItems = kStageChunk / kThreads;

template <bool TO_BUCKETS, bool SCALED>
__global__ void __launch_bounds__(kThreads)
k_bucket_staged(const float *__restrict__ in, const int32_t *__restrict__ slot,
                const int32_t *__restrict__ delta_table, int64_t E, int shift, int nwin, EdgeScale sc,
                float *__restrict__ out) {
    __shared__ int delta[kStageMaxWindows];
    __shared__ int stage_slot[kStageChunk];
    __shared__ float stage_val[kStageChunk];
    const int64_t c0 = int64_t(blockIdx.x) * kStageChunk;
    const int n = int(E - c0 < kStageChunk ? E - c0 : kStageChunk);
    for (int b = threadIdx.x; b < nwin; b += kThreads) delta[b] = delta_table[int64_t(blockIdx.x) * nwin + b];
    for (int i = threadIdx.x; i < n; i += kThreads) stage_slot[i] = -1;
    __syncthreads();
    // all global loads of the chunk first (independent), then the staging
    int sl[kStageItems];
    float v[kStageItems];
    float cnt[SCALED ? kStageItems : 1];  // in-degree of each item's destination
#pragma unroll
    for (int k = 0; k < kStageItems; ++k) {
        const int i = k * kThreads + threadIdx.x;
        sl[k] = i < n ? __ldcs(slot + c0 + i) : -1;
        v[k] = (TO_BUCKETS && i < n) ? (in ? __ldcs(in + c0 + i) : 1.f) : 0.f;
    }
    if (TO_BUCKETS && sc.mul) {
#pragma unroll
        for (int k = 0; k < kStageItems; ++k) {
            const int i = k * kThreads + threadIdx.x;
            if (i < n) v[k] *= __ldcs(sc.mul + c0 + i);
        }
    }
    if constexpr (SCALED) {
        // destinations of all items, then their row lengths: two waves of
        // independent loads rather than a dependent pair per item
        int d[kStageItems];
#pragma unroll
        for (int k = 0; k < kStageItems; ++k) {
            const int i = k * kThreads + threadIdx.x;
            d[k] = i < n ? __ldcs(sc.dst + c0 + i) : 0;
        }
#pragma unroll
        for (int k = 0; k < kStageItems; ++k) {
            const int i = k * kThreads + threadIdx.x;
            cnt[k] = i < n ? float(sc.rowptr[d[k] + 1] - sc.rowptr[d[k]]) : 1.f;  // >= 1: the edge itself
        }
        if (TO_BUCKETS) {
#pragma unroll
            for (int k = 0; k < kStageItems; ++k) v[k] = __fdiv_rn(v[k], cnt[k]);
        }
    }
    int pos[kStageItems];
#pragma unroll
    for (int k = 0; k < kStageItems; ++k) {
        pos[k] = -1;
        if (sl[k] >= 0) {
            const int p = sl[k] + delta[sl[k] >> shift];
            if (p >= 0 && p < n) {  // always true for a consistent table
                pos[k] = p;
                stage_slot[p] = sl[k];
                if (TO_BUCKETS) stage_val[p] = v[k];
            }
        }
    }
    __syncthreads();
    // (every position of the chunk holds a slot in [0, E); the checks only
    // keep an inconsistent table from turning into a stray access)
    if (TO_BUCKETS) {
#pragma unroll
        for (int k = 0; k < kStageItems; ++k) {
            const int i = k * kThreads + threadIdx.x;
            const int s2 = i < n ? stage_slot[i] : -1;
            if (s2 >= 0 && s2 < E) out[s2] = stage_val[i];
        }
    } else {
        float g[kStageItems];
#pragma unroll
        for (int k = 0; k < kStageItems; ++k) {
            const int i = k * kThreads + threadIdx.x;
            const int s2 = i < n ? stage_slot[i] : -1;
            g[k] = (s2 >= 0 && s2 < E) ? in[s2] : 0.f;
        }
#pragma unroll
        for (int k = 0; k < kStageItems; ++k) {
            const int i = k * kThreads + threadIdx.x;
            if (i < n) stage_val[i] = g[k];
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < kStageItems; ++k) {
            const int i = k * kThreads + threadIdx.x;
            if (i < n && pos[k] >= 0) {
                if constexpr (SCALED) __stcs(out + c0 + i, __fdiv_rn(stage_val[pos[k]], cnt[k]));
                else __stcs(out + c0 + i, stage_val[pos[k]]);
            }
        }
    }
}

template <bool SCALED>
void regroup_as(bool to_buckets, const ag::Direction &D, const float *in, int64_t E, const EdgeScale &sc,
                float *out, cudaStream_t st) {
    if (AG_BUCKET_STAGED && D.stage_delta) {
        const unsigned grid = unsigned(n_stage_chunks(E));
        const int nwin = int(n_windows(E));
        if (to_buckets)
            k_bucket_staged<true, SCALED><<<grid, kThreads, 0, st>>>(in, D.bucket_of_coo, D.stage_delta, E,
                                                                      kWindowShift, nwin, sc, out);
        else
            k_bucket_staged<false, SCALED><<<grid, kThreads, 0, st>>>(in, D.bucket_of_coo, D.stage_delta, E,
                                                                       kWindowShift, nwin, sc, out);
        return;
    }
    const int64_t b = (E + kThreads - 1) / kThreads;
    const unsigned grid = unsigned(b < 1 ? 1 : (b > 148 * 32 ? 148 * 32 : b));
    if (to_buckets) k_bucket_scatter<SCALED><<<grid, kThreads, 0, st>>>(in, D.bucket_of_coo, E, sc, out);
    else k_bucket_gather<SCALED><<<grid, kThreads, 0, st>>>(in, D.bucket_of_coo, E, sc, out);
}
// w_b[slot[e]] = w[e] (to_buckets; w = null: 1) or dw[e] = dw_b[slot[e]],
// each divided by the in-degree of e's destination when sc.dst is set
void regroup(bool to_buckets, const ag::Direction &D, const float *in, int64_t E, float *out, cudaStream_t st,
             const EdgeScale &sc = EdgeScale{}) {
    if (sc.dst) regroup_as<true>(to_buckets, D, in, E, sc, out, st);
    else regroup_as<false>(to_buckets, D, in, E, sc, out, st);
}

int check_scratch(const ag_graph *g, size_t need, const void *scratch, size_t scratch_bytes, const char *fn) {
    if (need > 0 && (!scratch || scratch_bytes < need))
        return fail(AG_ERR_WORKSPACE, "%s: scratch of %zu bytes, need %zu", fn, scratch_bytes, need);
    if (!aligned(scratch, kAlign)) return fail(AG_ERR_WORKSPACE, "%s: scratch must be 256-byte aligned", fn);
    return AG_OK;
}

// SpMM over direction d: out = A_w X (d = 0) or A_w^T dY (d = 1).
// The shapes the shared-memory ring walks take (see launch_main).
bool ring_shape(const Shape &s, int dtype, int64_t H) {
    return s.lb > 0 || s.col_tiles == 1 && s.G >= 4 && s.nv <= 2 && (dtype == AG_F32 ? s.vec == 4 : s.vec == 8) &&
           int64_t(s.G) * s.nv * s.vec == H;
}

// inv[i] = 1 / (number of edges into i), 0 for rows without edges
__global__ void k_inv_counts(const int32_t *__restrict__ rowptr, int64_t N, float *__restrict__ inv) {
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < N; i += int64_t(gridDim.x) * blockDim.x) {
        const int c = rowptr[i + 1] - rowptr[i];
        inv[i] = c > 0 ? 1.f / float(c) : 0.f;
    }
}
float *mean_inverses(const ag_graph *g, char *scr, const ScratchLayout &SL, cudaStream_t st) {
    float *inv = reinterpret_cast<float *>(scr + SL.inv);
    const int64_t b = (g->N + kThreads - 1) / kThreads;
    k_inv_counts<<<unsigned(b < 1 ? 1 : (b > 148 * 32 ? 148 * 32 : b)), kThreads, 0, st>>>(g->dir[0].rowptr, g->N,
                                                                                          inv);
    return inv;
}

EdgeScale mean_scale(const ag_graph *g, bool mean) {
    EdgeScale sc;
    if (mean) {
        sc.dst = g->coo_dst;
        sc.rowptr = g->dir[0].rowptr;
    }
    return sc;
}

// mean: divide every edge by the in-degree of its destination (w may then be
// null for unit weights).
int spmm(const ag_graph *g, int d, const float *w, const void *F, void *out, int64_t H, int dtype,
         void *scratch, size_t scratch_bytes, void *stream, const char *fn, bool check_ptrs, bool mean = false) {
    int rc = check_call(g, H, dtype, fn);
    if (rc != AG_OK) return rc;
    if (!F || !out || (g->E > 0 && !w && !mean)) return fail(AG_ERR_INVALID_ARG, "%s: null w, input or output", fn);
    const ag::Direction &D = g->dir[d];
    const ScratchLayout SL = scratch_layout(g, H);
    const size_t need = g->E > 0 ? (mean ? SL.total : SL.w_b + align_up(size_t(g->E) * 4)) : SL.w_b;
    if ((rc = check_scratch(g, need, scratch, scratch_bytes, fn)) != AG_OK) return rc;
    if (check_ptrs) {
        if ((rc = check_device_ptr(F, g->device, "input")) != AG_OK) return rc;
        if ((rc = check_device_ptr(out, g->device, "output")) != AG_OK) return rc;
        if (g->E > 0 && w && (rc = check_device_ptr(w, g->device, "w")) != AG_OK) return rc;
        if (need > 0 && (rc = check_device_ptr(scratch, g->device, "scratch")) != AG_OK) return rc;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *scr = static_cast<char *>(scratch);
    const Shape s = pick_shape(H, dtype, F, out, nullptr);
    Params P = base_params(g, D, H, s);
    P.F = F;
    P.out = out;
    P.partial = reinterpret_cast<float *>(scr + SL.partial);
    P.n_zero = g->N - D.n_nz;
    // mean on the ring shapes: the forward walk scales finished rows, the
    // transpose walk scales each edge by its destination (other shapes divide
    // the weights while regrouping them)
    const bool ring_mean = mean && g->E > 0 && ring_shape(s, dtype, H);
    if (ring_mean) P.inv_cnt = mean_inverses(g, scr, SL, st);
    if (g->E > 0) {
        float *w_b = reinterpret_cast<float *>(scr + SL.w_b);
        regroup(true, D, w, g->E, w_b, st, mean_scale(g, mean && !ring_mean));
        P.w = w_b;
        P.order = D.bucket_of_pos;  // the kernels read w[order[p]]: here the bucketed slot
    }
    if (P.n_tiles + P.n_zero > 0) {
        if (ring_mean && d == 0) dispatch_main<kSpmm | kRowScale>(P, s, dtype, st);
        else if (ring_mean) dispatch_main<kSpmm | kEdgeScale>(P, s, dtype, st);
        else dispatch_main<kSpmm>(P, s, dtype, st);
    }
    if (D.n_span > 0) dispatch_fixup(D, P.partial, out, H, s, dtype, st, ring_mean && d == 0 ? P.inv_cnt : nullptr);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return cuda_fail(err, fn);
    return AG_OK;
}

// dw over the transpose CSR: owner = source row (X), gathered = dY[col_t];
// each edge's dot goes to its bucketed slot, then back to COO order.
int sddmm(const ag_graph *g, const void *X, const void *dY, float *dw, int64_t H, int dtype, void *scratch,
          size_t scratch_bytes, void *stream, const char *fn, bool check_ptrs, bool mean = false) {
    int rc = check_call(g, H, dtype, fn);
    if (rc != AG_OK) return rc;
    if (!X || !dY || (g->E > 0 && !dw)) return fail(AG_ERR_INVALID_ARG, "%s: null X, dY or dw", fn);
    const ScratchLayout SL = scratch_layout(g, H);
    const size_t need = g->E > 0 ? SL.total : 0;
    if ((rc = check_scratch(g, need, scratch, scratch_bytes, fn)) != AG_OK) return rc;
    if (check_ptrs) {
        if ((rc = check_device_ptr(X, g->device, "X")) != AG_OK) return rc;
        if ((rc = check_device_ptr(dY, g->device, "dY")) != AG_OK) return rc;
        if (g->E > 0 && (rc = check_device_ptr(dw, g->device, "dw")) != AG_OK) return rc;
        if (need > 0 && (rc = check_device_ptr(scratch, g->device, "scratch")) != AG_OK) return rc;
    }
    if (g->E == 0) return AG_OK;
    const ag::Direction &D = g->dir[1];
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const Shape s = pick_shape(H, dtype, X, dY, nullptr);
    float *dw_b = reinterpret_cast<float *>(static_cast<char *>(scratch) + SL.dw_b);
    Params P = base_params(g, D, H, s);
    P.order = D.bucket_of_pos;
    P.F = dY;
    P.R = X;
    P.dw = dw_b;
    P.n_zero = 0;
    dispatch_main<kSddmm>(P, s, dtype, st);
    regroup(false, D, dw_b, g->E, dw, st, mean_scale(g, mean));
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return cuda_fail(err, fn);
    return AG_OK;
}

// Feature gradient and weight gradient in one walk of the transpose CSR.
// mean: the gradients of the mean aggregation (w may be null for unit
// weights, dw null when no weight gradient is wanted).
int backward(const ag_graph *g, const float *w, const void *X, const void *dY, void *dX, float *dw, int64_t H,
             int dtype, void *scratch, size_t scratch_bytes, void *stream, const char *fn, bool check_ptrs,
             bool mean = false) {
    int rc = check_call(g, H, dtype, fn);
    if (rc != AG_OK) return rc;
    if (!X || !dY || !dX || (g->E > 0 && (!w || !dw) && !mean))
        return fail(AG_ERR_INVALID_ARG, "%s: null w, X, dY, dX or dw", fn);
    if (mean && !dw) return spmm(g, 1, w, dY, dX, H, dtype, scratch, scratch_bytes, stream, fn, check_ptrs, true);
    const ScratchLayout SL = scratch_layout(g, H);
    const size_t need = g->E > 0 ? SL.total : SL.w_b;
    if ((rc = check_scratch(g, need, scratch, scratch_bytes, fn)) != AG_OK) return rc;
    if (check_ptrs) {
        if ((rc = check_device_ptr(X, g->device, "X")) != AG_OK) return rc;
        if ((rc = check_device_ptr(dY, g->device, "dY")) != AG_OK) return rc;
        if ((rc = check_device_ptr(dX, g->device, "dX")) != AG_OK) return rc;
        if (g->E > 0 && w && (rc = check_device_ptr(w, g->device, "w")) != AG_OK) return rc;
        if (g->E > 0 && (rc = check_device_ptr(dw, g->device, "dw")) != AG_OK) return rc;
        if (need > 0 && (rc = check_device_ptr(scratch, g->device, "scratch")) != AG_OK) return rc;
    }
    const ag::Direction &D = g->dir[1];
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const Shape s = pick_shape(H, dtype, X, dY, dX);
    if (!ring_shape(s, dtype, H) || g->E == 0) {
        // shapes without the single walk: the two separate passes
        if ((rc = spmm(g, 1, w, dY, dX, H, dtype, scratch, scratch_bytes, stream, fn, false, mean)) != AG_OK)
            return rc;
        return sddmm(g, X, dY, dw, H, dtype, scratch, scratch_bytes, stream, fn, false, mean);
    }
    char *scr = static_cast<char *>(scratch);
    float *w_b = reinterpret_cast<float *>(scr + SL.w_b);
    float *dw_b = reinterpret_cast<float *>(scr + SL.dw_b);
    // mean: each edge's weight and dot scaled by its destination inside the walk
    const EdgeScale sc{};
    Params P = base_params(g, D, H, s);
    if (mean) P.inv_cnt = mean_inverses(g, scr, SL, st);
    regroup(true, D, w, g->E, w_b, st, sc);
    P.order = D.bucket_of_pos;
    P.w = w_b;
    P.F = dY;
    P.R = X;
    P.out = dX;
    P.dw = dw_b;
    P.partial = reinterpret_cast<float *>(scr + SL.partial);
    P.n_zero = g->N - D.n_nz;
    if (mean) dispatch_main<kBoth | kEdgeScale>(P, s, dtype, st);
    else dispatch_main<kBoth>(P, s, dtype, st);
    if (D.n_span > 0) dispatch_fixup(D, P.partial, dX, H, s, dtype, st);
    regroup(false, D, dw_b, g->E, dw, st, sc);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return cuda_fail(err, fn);
    return AG_OK;
}

// ---------------------------------------------------------------- GCN weights

// unit weights: the degree is the row length of the forward CSR
__global__ void k_row_counts(const int32_t *__restrict__ rowptr, int64_t N, float *__restrict__ deg) {
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < N; i += int64_t(gridDim.x) * blockDim.x)
        deg[i] = float(rowptr[i + 1] - rowptr[i]);
}
// deg^-1/2 in place (0 where deg <= 0)
__global__ void k_inv_sqrt(float *__restrict__ deg, int64_t N) {
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < N; i += int64_t(gridDim.x) * blockDim.x) {
        const float d = deg[i];
        deg[i] = d > 0.f ? 1.f / sqrtf(d) : 0.f;
    }
}
// deg[i]^-1/2 from the row sums sums[i].x (rows without edges hold 0)
__global__ void k_inv_sqrt_sums(const float2 *__restrict__ sums, int64_t N, float *__restrict__ deg) {
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < N; i += int64_t(gridDim.x) * blockDim.x) {
        const float d = sums[i].x;
        deg[i] = d > 0.f ? 1.f / sqrtf(d) : 0.f;
    }
}
__global__ void k_zero2(float2 *__restrict__ p, int64_t n) {
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x)
        p[i] = make_float2(0.f, 0.f);
}
// out[e] = dis[src_e] * w_e * dis[dst_e] in COO order (w = null: 1).  Each
// thread keeps kGcnUnroll edges in flight (strided by the grid, so the
// warp's loads stay coalesced): all endpoint and weight loads, then all
// gathers from the L2-resident dis, then the products.
constexpr int kGcnUnroll = 4;
__global__ void k_gcn_weights(const int32_t *__restrict__ src, const int32_t *__restrict__ dst,
                              const float *__restrict__ w, const float *__restrict__ dis, int64_t E,
                              float *__restrict__ out) {
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t e0 = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e0 < E; e0 += stride * kGcnUnroll) {
        int a[kGcnUnroll], b[kGcnUnroll];
        float we[kGcnUnroll], da[kGcnUnroll], db[kGcnUnroll];
#pragma unroll
        for (int k = 0; k < kGcnUnroll; ++k) {
            const int64_t e = e0 + k * stride;
            a[k] = e < E ? __ldcs(src + e) : 0;
            b[k] = e < E ? __ldcs(dst + e) : 0;
            we[k] = (w && e < E) ? __ldcs(w + e) : 1.f;
        }
#pragma unroll
        for (int k = 0; k < kGcnUnroll; ++k) {
            const bool ok = e0 + k * stride < E;
            da[k] = ok ? dis[a[k]] : 0.f;
            db[k] = ok ? dis[b[k]] : 0.f;
        }
#pragma unroll
        for (int k = 0; k < kGcnUnroll; ++k) {
            const int64_t e = e0 + k * stride;
            if (e < E) __stcs(out + e, da[k] * we[k] * db[k]);
        }
    }
}
unsigned flat_grid(int64_t n) {
    const int64_t b = (n + kThreads - 1) / kThreads;
    return unsigned(b < 1 ? 1 : (b > 148 * 32 ? 148 * 32 : b));
}

// Scratch of ag_gcn_norm: deg[N] | row sums float2[N] | tile partials
// float2[2 tiles] | weights in forward windows float[E].
struct GcnLayout {
    size_t deg, sums, partial, w_b, total;
};
GcnLayout gcn_layout(const ag_graph *g) {
    GcnLayout L;
    L.deg = 0;
    L.sums = align_up(size_t(g->N) * 4);
    L.partial = L.sums + align_up(size_t(g->N) * 8);
    L.w_b = L.partial + align_up(size_t(2) * size_t(g->n_tiles) * 8);
    L.total = L.w_b + align_up(size_t(g->E) * 4);
    return L;
}

int gcn_norm(const ag_graph *g, const float *w, float *w_norm, void *scratch, size_t scratch_bytes, void *stream) {
    const char *fn = "ag_gcn_norm";
    if (!g) return fail(AG_ERR_INVALID_ARG, "%s: null graph", fn);
    if (int rc0 = check_current_device(g, fn)) return rc0;
    if (g->E > 0 && !w_norm) return fail(AG_ERR_INVALID_ARG, "%s: null w_norm", fn);
    const GcnLayout L = gcn_layout(g);
    int rc = check_scratch(g, L.total, scratch, scratch_bytes, fn);
    if (rc != AG_OK) return rc;
    if (g->E == 0) return AG_OK;
    if ((rc = check_device_ptr(w_norm, g->device, "w_norm")) != AG_OK) return rc;
    if (w && (rc = check_device_ptr(w, g->device, "w")) != AG_OK) return rc;
    if ((rc = check_device_ptr(scratch, g->device, "scratch")) != AG_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *scr = static_cast<char *>(scratch);
    float *deg = reinterpret_cast<float *>(scr + L.deg);
    if (w) {
        // weighted in-degree: the weights summed over each forward-CSR row
        // (a segmented reduction in a fixed order, over the weights regrouped
        // into the forward walk's windows)
        float *w_b = reinterpret_cast<float *>(scr + L.w_b);
        float2 *sums = reinterpret_cast<float2 *>(scr + L.sums);
        regroup(true, g->dir[0], w, g->E, w_b, st);
        k_zero2<<<flat_grid(g->N), kThreads, 0, st>>>(sums, g->N);
        rc = row_sums(g, w_b, reinterpret_cast<float2 *>(scr + L.partial), sums, st);
        if (rc != AG_OK) return rc;
        k_inv_sqrt_sums<<<flat_grid(g->N), kThreads, 0, st>>>(sums, g->N, deg);
    } else {
        k_row_counts<<<flat_grid(g->N), kThreads, 0, st>>>(g->dir[0].rowptr, g->N, deg);
        k_inv_sqrt<<<flat_grid(g->N), kThreads, 0, st>>>(deg, g->N);
    }
    k_gcn_weights<<<flat_grid(g->E), kThreads, 0, st>>>(g->coo_src, g->coo_dst, w, deg, g->E, w_norm);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return cuda_fail(err, fn);
    return AG_OK;
}

// The SDDMM walk over direction d: out_b[slot of position p] = dot(R[row of
// p], F[col[p]]) in that direction's window slots (no regrouping).
int sddmm_bucketed_impl(const ag_graph *g, int d, const void *R, const void *F, float *out_b, int64_t H, int dtype,
                        cudaStream_t st) {
    if (g->E == 0) return AG_OK;
    const ag::Direction &D = g->dir[d];
    const Shape s = pick_shape(H, dtype, R, F, nullptr);
    Params P = base_params(g, D, H, s);
    P.order = D.bucket_of_pos;
    P.F = F;
    P.R = R;
    P.dw = out_b;
    P.n_zero = 0;
    dispatch_main<kSddmm>(P, s, dtype, st);
    cudaError_t err = cudaGetLastError();
    return err == cudaSuccess ? AG_OK : cuda_fail(err, "bucketed SDDMM");
}

}  // namespace

int sddmm_bucketed(const ag_graph *g, int d, const void *R, const void *F, float *out_b, int64_t H, int dtype,
                   cudaStream_t st) {
    return sddmm_bucketed_impl(g, d, R, F, out_b, H, dtype, st);
}
void regroup_from_buckets(const ag_graph *g, int d, const float *in_b, float *out, cudaStream_t st) {
    regroup(false, g->dir[d], in_b, g->E, out, st);
}

size_t spmm_scratch_edge_offset(const ag_graph *g, int64_t H, int which) {
    const ScratchLayout L = scratch_layout(g, H);
    return which == 0 ? L.w_b : L.dw_b;
}
void regroup_to_buckets(const ag_graph *g, int d, const float *in, float *out_b, cudaStream_t st) {
    regroup(true, g->dir[d], in, g->E, out_b, st);
}
void regroup_product_to_buckets(const ag_graph *g, int d, const float *a, const float *b, float *out_b,
                                cudaStream_t st) {
    EdgeScale sc;
    sc.mul = b;
    regroup(true, g->dir[d], a, g->E, out_b, st, sc);
}

}  // namespace ag

using namespace ag;

extern "C" {

size_t ag_spmm_scratch_bytes(const ag_graph *g, int64_t H) {
    if (!g || H < 1) return 0;
    return scratch_needed(g, H);
}

int ag_spmm_fwd(const ag_graph *g, const float *w, const void *X, void *Y, int64_t H, int dtype,
                void *scratch, size_t scratch_bytes, void *stream) {
    clear_error();
    return spmm(g, 0, w, X, Y, H, dtype, scratch, scratch_bytes, stream, "ag_spmm_fwd", true);
}

int ag_spmm_dx(const ag_graph *g, const float *w, const void *dY, void *dX, int64_t H, int dtype,
               void *scratch, size_t scratch_bytes, void *stream) {
    clear_error();
    return spmm(g, 1, w, dY, dX, H, dtype, scratch, scratch_bytes, stream, "ag_spmm_dx", true);
}

int ag_sddmm_dw(const ag_graph *g, const void *X, const void *dY, float *dw, int64_t H, int dtype,
                void *scratch, size_t scratch_bytes, void *stream) {
    clear_error();
    return sddmm(g, X, dY, dw, H, dtype, scratch, scratch_bytes, stream, "ag_sddmm_dw", true);
}

int ag_backward(const ag_graph *g, const float *w, const void *X, const void *dY, void *dX, float *dw, int64_t H,
                int dtype, void *scratch, size_t scratch_bytes, void *stream) {
    clear_error();
    return backward(g, w, X, dY, dX, dw, H, dtype, scratch, scratch_bytes, stream, "ag_backward", true);
}

int ag_mean_fwd(const ag_graph *g, const float *w, const void *X, void *Y, int64_t H, int dtype, void *scratch,
                size_t scratch_bytes, void *stream) {
    clear_error();
    return spmm(g, 0, w, X, Y, H, dtype, scratch, scratch_bytes, stream, "ag_mean_fwd", true, true);
}

int ag_mean_backward(const ag_graph *g, const float *w, const void *X, const void *dY, void *dX, float *dw,
                     int64_t H, int dtype, void *scratch, size_t scratch_bytes, void *stream) {
    clear_error();
    return backward(g, w, X, dY, dX, dw, H, dtype, scratch, scratch_bytes, stream, "ag_mean_backward", true, true);
}

size_t ag_gcn_norm_scratch_bytes(const ag_graph *g) {
    if (!g) return 0;
    return gcn_layout(g).total;
}

int ag_gcn_norm(const ag_graph *g, const float *w, float *w_norm, void *scratch, size_t scratch_bytes,
                void *stream) {
    clear_error();
    return gcn_norm(g, w, w_norm, scratch, scratch_bytes, stream);
}

}  // extern "C"

namespace {
// Two helper streams per device for ag_step_host (created once, never
// destroyed): one brings dY in while the forward pass runs, one takes the
// results out, so that host-to-device and device-to-host copies overlap.
constexpr int kStepDevices = 64;
std::mutex g_step_mu;
cudaStream_t g_step_in[kStepDevices] = {}, g_step_out[kStepDevices] = {};

int step_streams(int device, cudaStream_t *in, cudaStream_t *out) {
    if (device < 0 || device >= kStepDevices) return fail(AG_ERR_DEVICE, "ag_step_host: device %d", device);
    std::lock_guard<std::mutex> lock(g_step_mu);
    if (!g_step_in[device]) {
        cudaStream_t a = nullptr, b = nullptr;
        cudaError_t err = cudaStreamCreateWithFlags(&a, cudaStreamNonBlocking);
        if (err == cudaSuccess) err = cudaStreamCreateWithFlags(&b, cudaStreamNonBlocking);
        if (err != cudaSuccess) {
            if (a) cudaStreamDestroy(a);
            return cuda_fail(err, "ag_step_host: stream creation");
        }
        g_step_in[device] = a;
        g_step_out[device] = b;
    }
    *in = g_step_in[device];
    *out = g_step_out[device];
    return AG_OK;
}

// Events of one ag_step_host call, released when the call returns (the
// runtime keeps them alive until the work that waits on them is done).
struct StepEvents {
    cudaEvent_t e[6] = {};
    cudaError_t create() {
        for (auto &x : e) {
            cudaError_t err = cudaEventCreateWithFlags(&x, cudaEventDisableTiming);
            if (err != cudaSuccess) return err;
        }
        return cudaSuccess;
    }
    ~StepEvents() {
        for (auto &x : e)
            if (x) cudaEventDestroy(x);
    }
};

// Pipelined steps: per staging buffer, an event recorded after the last
// read of its input part (w, X, dY) by a step's fused backward pass.  The
// input copies of the next pipelined step on that buffer wait for this
// event only, so they overlap the previous step's copies out.  That is safe
// only while consecutive steps lay the buffer out the same way (the input
// part of one step must not overlap the output part of the previous one), so
// an entry holds the layout it was recorded for: a step with another graph,
// width, dtype or staging size -- or a buffer whose entry was reused, or that
// was never seen -- gets the full ordering after `stream` again.
constexpr int kStagingSlots = 16;
struct StagingKey {
    const void *staging = nullptr;
    int device = -1;
    const ag_graph *graph = nullptr;
    int64_t N = 0, E = 0, H = 0;
    int dtype = -1;
    size_t bytes = 0;
    bool operator==(const StagingKey &o) const {
        return staging == o.staging && device == o.device && graph == o.graph && N == o.N && E == o.E &&
               H == o.H && dtype == o.dtype && bytes == o.bytes;
    }
};
struct StagingOrder {
    StagingKey key;
    cudaEvent_t done = nullptr;
};
StagingOrder g_staging[kStagingSlots];
int g_staging_next = 0;

// The entry of this buffer (same address and device), whatever its layout.
StagingOrder *find_staging(const StagingKey &k) {
    for (auto &s : g_staging)
        if (s.done && s.key.staging == k.staging && s.key.device == k.device) return &s;
    return nullptr;
}

// Make `in` wait for the previous step's reads of the staging buffer's
// inputs (pipelined, same layout), or for everything on `st` so far (first
// use of the buffer, or a new layout).
cudaError_t staging_wait_inputs(const StagingKey &k, cudaStream_t st, cudaStream_t in, cudaEvent_t tmp) {
    std::lock_guard<std::mutex> lock(g_step_mu);
    StagingOrder *s = find_staging(k);
    if (s && s->key == k) return cudaStreamWaitEvent(in, s->done, 0);
    if (!s) {
        s = &g_staging[g_staging_next];
        g_staging_next = (g_staging_next + 1) % kStagingSlots;
        if (s->done) cudaEventDestroy(s->done);  // released once its pending waits are done
        *s = StagingOrder{};
        cudaError_t err = cudaEventCreateWithFlags(&s->done, cudaEventDisableTiming);
        if (err != cudaSuccess) {
            s->done = nullptr;
            return err;
        }
    }
    s->key = k;  // a new layout keeps the buffer's event, ordered after `st` below
    cudaError_t err = cudaEventRecord(tmp, st);
    return err == cudaSuccess ? cudaStreamWaitEvent(in, tmp, 0) : err;
}

// After a step's backward pass (on st): the staging buffer's inputs are read.
cudaError_t staging_mark_read(const StagingKey &k, cudaStream_t st) {
    std::lock_guard<std::mutex> lock(g_step_mu);
    StagingOrder *s = find_staging(k);
    if (s && s->key == k) return cudaEventRecord(s->done, st);
    return cudaSuccess;
}
}  // namespace

extern "C" {

// Staging layout: w | X | dY | Y | dX | dw | scratch, each 256-byte aligned.
static bool staging_layout(const ag_graph *g, int64_t H, int dtype, size_t off[7], size_t *total) {
    if (!g || H < 1 || (dtype != AG_F32 && dtype != AG_BF16)) return false;
    const size_t elem = dtype == AG_F32 ? 4 : 2;
    const size_t feat = size_t(g->N) * size_t(H) * elem;
    const size_t sizes[7] = {size_t(g->E) * 4, feat, feat, feat, feat, size_t(g->E) * 4, scratch_needed(g, H)};
    size_t at = 0;
    for (int i = 0; i < 7; ++i) {
        off[i] = at;
        at += align_up(sizes[i] ? sizes[i] : 1);
    }
    *total = at;
    return true;
}

size_t ag_step_staging_bytes(const ag_graph *g, int64_t H, int dtype) {
    size_t off[7], total = 0;
    if (!staging_layout(g, H, dtype, off, &total)) return 0;
    return total;
}

}  // extern "C"

namespace {
int step_host(const ag_graph *g, const float *w_host, const void *X_host, const void *dY_host, void *Y_host,
              void *dX_host, float *dw_host, int64_t H, int dtype, void *staging, size_t staging_bytes,
              void *stream, bool pipelined, const char *fn) {
    clear_error();
    int rc = check_call(g, H, dtype, fn);
    if (rc != AG_OK) return rc;
    if (!X_host || !dY_host || !Y_host || !dX_host || (g->E > 0 && (!w_host || !dw_host)) || !staging)
        return fail(AG_ERR_INVALID_ARG, "%s: null buffer", fn);
    size_t off[7], total = 0;
    staging_layout(g, H, dtype, off, &total);
    if (staging_bytes < total)
        return fail(AG_ERR_WORKSPACE, "%s: staging of %zu bytes, need %zu", fn, staging_bytes, total);
    if (!aligned(staging, kAlign)) return fail(AG_ERR_WORKSPACE, "%s: staging must be 256-byte aligned", fn);
    if ((rc = check_device_ptr(staging, g->device, "staging")) != AG_OK) return rc;
    char *base = static_cast<char *>(staging);
    float *w = reinterpret_cast<float *>(base + off[0]);
    void *X = base + off[1], *dY = base + off[2], *Y = base + off[3], *dX = base + off[4];
    float *dw = reinterpret_cast<float *>(base + off[5]);
    void *scratch = base + off[6];
    const size_t feat = size_t(g->N) * size_t(H) * (dtype == AG_F32 ? 4 : 2);
    const size_t wb = size_t(g->E) * 4;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaStream_t s_in = nullptr, s_out = nullptr;
    if ((rc = step_streams(g->device, &s_in, &s_out)) != AG_OK) return rc;
    StepEvents ev;
    cudaError_t err = ev.create();
    auto copy = [&](void *to, const void *from, size_t n, cudaMemcpyKind k, cudaStream_t s) {
        if (err == cudaSuccess && n > 0) err = cudaMemcpyAsync(to, from, n, k, s);
    };
    auto record = [&](cudaEvent_t e, cudaStream_t s) {
        if (err == cudaSuccess) err = cudaEventRecord(e, s);
    };
    auto wait = [&](cudaStream_t s, cudaEvent_t e) {
        if (err == cudaSuccess) err = cudaStreamWaitEvent(s, e, 0);
    };
    const size_t scr = scratch_needed(g, H);  // staging's scratch part
    StagingKey key;
    key.staging = staging;
    key.device = g->device;
    key.graph = g;
    key.N = g->N;
    key.E = g->E;
    key.H = H;
    key.dtype = dtype;
    key.bytes = staging_bytes;
    if (pipelined) {
        // all inputs on the helper stream, after the previous step's backward
        // pass on this staging buffer (not after its copies out)
        if (err == cudaSuccess) err = staging_wait_inputs(key, st, s_in, ev.e[5]);
        copy(w, w_host, wb, cudaMemcpyHostToDevice, s_in);
        copy(X, X_host, feat, cudaMemcpyHostToDevice, s_in);
        record(ev.e[0], s_in);
        wait(st, ev.e[0]);
    } else {
        // w and X first; dY follows on its own stream while the forward pass runs
        copy(w, w_host, wb, cudaMemcpyHostToDevice, st);
        copy(X, X_host, feat, cudaMemcpyHostToDevice, st);
        record(ev.e[0], st);
        wait(s_in, ev.e[0]);
    }
    copy(dY, dY_host, feat, cudaMemcpyHostToDevice, s_in);
    record(ev.e[1], s_in);
    if (err != cudaSuccess) return cuda_fail(err, fn);
    if ((rc = spmm(g, 0, w, X, Y, H, dtype, scratch, scr, stream, fn, false)) != AG_OK) return rc;
    // Y goes out (device to host) while dY still comes in (host to device)
    record(ev.e[2], st);
    wait(s_out, ev.e[2]);
    copy(Y_host, Y, feat, cudaMemcpyDeviceToHost, s_out);
    wait(st, ev.e[1]);
    if (err != cudaSuccess) return cuda_fail(err, fn);
    if ((rc = backward(g, w, X, dY, dX, dw, H, dtype, scratch, scr, stream, fn, false)) != AG_OK) return rc;
    if (err == cudaSuccess) err = staging_mark_read(key, st);
    record(ev.e[3], st);
    wait(s_out, ev.e[3]);
    copy(dX_host, dX, feat, cudaMemcpyDeviceToHost, s_out);
    copy(dw_host, dw, wb, cudaMemcpyDeviceToHost, s_out);
    // `stream` covers every copy: the caller synchronizes it alone
    record(ev.e[4], s_out);
    wait(st, ev.e[4]);
    if (err != cudaSuccess) return cuda_fail(err, fn);
    return AG_OK;
}
}  // namespace

extern "C" {

int ag_step_host(const ag_graph *g, const float *w_host, const void *X_host, const void *dY_host,
                 void *Y_host, void *dX_host, float *dw_host, int64_t H, int dtype, void *staging,
                 size_t staging_bytes, void *stream) {
    return step_host(g, w_host, X_host, dY_host, Y_host, dX_host, dw_host, H, dtype, staging, staging_bytes,
                     stream, false, "ag_step_host");
}

int ag_step_host_pipelined(const ag_graph *g, const float *w_host, const void *X_host, const void *dY_host,
                           void *Y_host, void *dX_host, float *dw_host, int64_t H, int dtype, void *staging,
                           size_t staging_bytes, void *stream) {
    return step_host(g, w_host, X_host, dY_host, Y_host, dX_host, dw_host, H, dtype, staging, staging_bytes,
                     stream, true, "ag_step_host_pipelined");
}

// ---------------------------------------------------------------------------- one step in one call

}  // extern "C"

namespace {
// Scratch of ag_step: the backward pass's SpMM scratch, then the forward
// pass's partial rows and its weights in forward windows.
struct StepLayout {
    ScratchLayout bwd;
    size_t fwd_partial, fwd_w_b, total;
};
StepLayout step_layout(const ag_graph *g, int64_t H) {
    StepLayout L;
    L.bwd = scratch_layout(g, H);
    const bool spans = g->dir[0].n_span > 0 || g->dir[1].n_span > 0;
    L.fwd_partial = align_up(L.bwd.total);
    L.fwd_w_b = L.fwd_partial + align_up(spans ? size_t(2) * size_t(g->n_tiles) * size_t(H) * 4 : 0);
    L.total = L.fwd_w_b + align_up(size_t(g->E) * 4);
    return L;
}

int step_device(const ag_graph *g, const float *w, const void *X, const void *dY, void *Y, void *dX, float *dw,
                int64_t H, int dtype, void *scratch, size_t scratch_bytes, void *stream) {
    const char *fn = "ag_step";
    int rc = check_call(g, H, dtype, fn);
    if (rc != AG_OK) return rc;
    if (!X || !dY || !Y || !dX || (g->E > 0 && (!w || !dw)))
        return fail(AG_ERR_INVALID_ARG, "%s: null w, X, dY, Y, dX or dw", fn);
    const StepLayout L = step_layout(g, H);
    if ((rc = check_scratch(g, L.total, scratch, scratch_bytes, fn)) != AG_OK) return rc;
    const void *ptrs[] = {X, dY, Y, dX, scratch};
    const char *names[] = {"X", "dY", "Y", "dX", "scratch"};
    for (int i = 0; i < 5; ++i)
        if ((rc = check_device_ptr(ptrs[i], g->device, names[i])) != AG_OK) return rc;
    if (g->E > 0) {
        if ((rc = check_device_ptr(w, g->device, "w")) != AG_OK) return rc;
        if ((rc = check_device_ptr(dw, g->device, "dw")) != AG_OK) return rc;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const Shape sf = pick_shape(H, dtype, X, Y, nullptr);
    const Shape sb = pick_shape(H, dtype, X, dY, dX);
    if (g->E == 0 || !ring_shape(sb, dtype, H)) {
        // shapes without the single backward walk: the two calls in order
        rc = spmm(g, 0, w, X, Y, H, dtype, scratch, L.bwd.total, stream, fn, false);
        if (rc == AG_OK) rc = backward(g, w, X, dY, dX, dw, H, dtype, scratch, L.bwd.total, stream, fn, false);
        return rc;
    }
    cudaStream_t side = nullptr, unused = nullptr;
    if ((rc = step_streams(g->device, &side, &unused)) != AG_OK) return rc;
    StepEvents ev;
    cudaError_t err = ev.create();
    auto record = [&](cudaEvent_t e, cudaStream_t s) {
        if (err == cudaSuccess) err = cudaEventRecord(e, s);
    };
    auto wait = [&](cudaStream_t s, cudaEvent_t e) {
        if (err == cudaSuccess) err = cudaStreamWaitEvent(s, e, 0);
    };
    char *scr = static_cast<char *>(scratch);
    float *w_b_f = reinterpret_cast<float *>(scr + L.fwd_w_b);
    float *w_b_t = reinterpret_cast<float *>(scr + L.bwd.w_b);
    float *dw_b = reinterpret_cast<float *>(scr + L.bwd.dw_b);
    // side: the forward weights into their windows, while the backward walk runs
    record(ev.e[0], st);
    wait(side, ev.e[0]);
    if (err != cudaSuccess) return cuda_fail(err, fn);
    regroup(true, g->dir[0], w, g->E, w_b_f, side);
    record(ev.e[1], side);
    // main: the fused backward walk over the transpose CSR
    const ag::Direction &Dt = g->dir[1];
    Params Pb = base_params(g, Dt, H, sb);
    regroup(true, Dt, w, g->E, w_b_t, st);
    Pb.order = Dt.bucket_of_pos;
    Pb.w = w_b_t;
    Pb.F = dY;
    Pb.R = X;
    Pb.out = dX;
    Pb.dw = dw_b;
    Pb.partial = reinterpret_cast<float *>(scr + L.bwd.partial);
    Pb.n_zero = g->N - Dt.n_nz;
    dispatch_main<kBoth>(Pb, sb, dtype, st);
    record(ev.e[2], st);
    // side: the backward's rows cut by tiles and dw back to COO order, while
    // the forward walk runs (the two passes use separate partial rows)
    wait(side, ev.e[2]);
    if (err != cudaSuccess) return cuda_fail(err, fn);
    if (Dt.n_span > 0) dispatch_fixup(Dt, Pb.partial, dX, H, sb, dtype, side);
    regroup(false, Dt, dw_b, g->E, dw, side);
    record(ev.e[3], side);
    // main: the forward walk
    const ag::Direction &Df = g->dir[0];
    Params Pf = base_params(g, Df, H, sf);
    Pf.order = Df.bucket_of_pos;
    Pf.w = w_b_f;
    Pf.F = X;
    Pf.out = Y;
    Pf.partial = reinterpret_cast<float *>(scr + L.fwd_partial);
    Pf.n_zero = g->N - Df.n_nz;
    wait(st, ev.e[1]);
    if (err != cudaSuccess) return cuda_fail(err, fn);
    if (Pf.n_tiles + Pf.n_zero > 0) dispatch_main<kSpmm>(Pf, sf, dtype, st);
    if (Df.n_span > 0) dispatch_fixup(Df, Pf.partial, Y, H, sf, dtype, st);
    // `stream` is ordered after the side stream's work
    wait(st, ev.e[3]);
    if (err == cudaSuccess) err = cudaGetLastError();
    if (err != cudaSuccess) return cuda_fail(err, fn);
    return AG_OK;
}
}  // namespace

extern "C" {

size_t ag_step_scratch_bytes(const ag_graph *g, int64_t H) {
    if (!g || H < 1) return 0;
    return step_layout(g, H).total;
}

int ag_step(const ag_graph *g, const float *w, const void *X, const void *dY, void *Y, void *dX, float *dw, int64_t H,
            int dtype, void *scratch, size_t scratch_bytes, void *stream) {
    clear_error();
    return step_device(g, w, X, dY, Y, dX, dw, H, dtype, scratch, scratch_bytes, stream);
}

// ---------------------------------------------------------------------------- forward without caller scratch

}  // extern "C"

// Built-in scratch for ag_spmm_fwd_static_scratch: a fixed device array that
// every GPU loading this library holds until the process exits.  In host code
// the name g_static_scratch only stands in for the symbol; its device address
// comes from cudaGetSymbolAddress below.
static constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) float g_static_scratch[kStaticScratchBytes / sizeof(float)];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
void *g_static_ptr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device (looked up once
// per device; the host-side name is only a stand-in for the symbol).
int static_scratch(int device, void **out) {
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (!g_static_ptr[device]) {
        void *p = nullptr;
        cudaError_t err = cudaGetSymbolAddress(&p, g_static_scratch);
        if (err != cudaSuccess) return ag::cuda_fail(err, "ag_spmm_fwd_static_scratch: cudaGetSymbolAddress");
        g_static_ptr[device] = p;
    }
    *out = g_static_ptr[device];
    return AG_OK;
}
}  // namespace

extern "C" {

size_t ag_spmm_static_scratch_capacity(void) { return kStaticScratchBytes; }

int ag_spmm_fwd_static_scratch(const ag_graph *g, const float *w, const void *X, void *Y, int64_t H, int dtype,
                               void *stream) {
    clear_error();
    if (!g) return fail(AG_ERR_INVALID_ARG, "ag_spmm_fwd_static_scratch: null graph");
    if (H < 1) return fail(AG_ERR_SHAPE, "ag_spmm_fwd_static_scratch: H=%lld", (long long)H);
    const ScratchLayout SL = scratch_layout(g, H);
    const size_t need = g->E > 0 ? SL.w_b + align_up(size_t(g->E) * 4) : SL.w_b;
    if (need > kStaticScratchBytes)
        return fail(AG_ERR_WORKSPACE,
                    "ag_spmm_fwd_static_scratch: this graph needs %zu bytes of scratch at H=%lld, more than the "
                    "built-in %zu; use ag_spmm_fwd with caller scratch",
                    need, (long long)H, kStaticScratchBytes);
    int device = -1;
    cudaError_t err = cudaGetDevice(&device);
    if (err != cudaSuccess) return cuda_fail(err, "ag_spmm_fwd_static_scratch: cudaGetDevice");
    if (device != g->device)
        return fail(AG_ERR_DEVICE, "ag_spmm_fwd_static_scratch: current device %d, graph is on device %d", device,
                    g->device);
    if (device < 0 || device >= kMaxDevices)
        return fail(AG_ERR_DEVICE, "ag_spmm_fwd_static_scratch: device %d out of range", device);
    void *scratch = nullptr;
    int rc = static_scratch(device, &scratch);
    if (rc != AG_OK) return rc;
    return spmm(g, 0, w, X, Y, H, dtype, scratch, kStaticScratchBytes, stream, "ag_spmm_fwd_static_scratch", true);
}

}  // extern "C"
