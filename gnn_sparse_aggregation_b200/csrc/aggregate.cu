// aggregate.cu -- per-call kernels: weighted SpMM (forward Y = A_w X and
// feature gradient dX = A_w^T dY) and the per-edge SDDMM weight gradient
// dw_e = dot(X[src_e], dY[dst_e]).
//
// tinymesh "Weighted aggregation experiment", section "Decision": forward and
// dX reuse one owner-row CSR traversal, dw has one output per edge reduced
// over the feature width, and none of them needs atomics or an [E, H]
// intermediate.  Section "Limits" names the two weak spots of that design:
// a serial reduction over the feature width per edge, and degree skew in the
// CSR directions.  Here:
//   * an owner row is handled by a group of G lanes that together span the
//     feature width with 16-byte vector loads (float4 / 8 x bf16), several
//     gathered rows in flight per lane, fp32 accumulation in registers;
//   * rows come in decreasing-degree order (longest work first), and rows
//     longer than kHeavyThreshold are cut into kChunkEdges-edge chunks whose
//     fp32 partial rows go to caller scratch and are summed in chunk order by
//     a second kernel -- deterministic, no float atomics;
//   * dw walks the transpose CSR: the owner's X row is held in registers and
//     every dY row gathered once feeds one dot product, reduced across the
//     group with xor shuffles.
#include <cuda_bf16.h>

#include "internal.h"

namespace ag {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;  // gathered rows in flight per lane

enum Mode { kSpmm = 1, kSddmm = 2 };

using bf16_t = uint16_t;  // bfloat16 stored as raw bits

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }
__device__ __forceinline__ uint32_t bf16_bits(float f) {
    return uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(f)));
}
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) { return bf16_bits(a) | (bf16_bits(b) << 16); }

// Read-only gathered rows: non-coherent path, keep in L1/L2.
template <typename T, int VEC> struct Vec;

template <> struct Vec<float, 4> {
    static __device__ __forceinline__ void load(const float *p, float (&v)[4]) {
        float4 t = __ldg(reinterpret_cast<const float4 *>(p));
        v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    }
    static __device__ __forceinline__ void store(float *p, const float (&v)[4]) {
        __stcs(reinterpret_cast<float4 *>(p), make_float4(v[0], v[1], v[2], v[3]));
    }
};
template <> struct Vec<float, 1> {
    static __device__ __forceinline__ void load(const float *p, float (&v)[1]) { v[0] = __ldg(p); }
    static __device__ __forceinline__ void store(float *p, const float (&v)[1]) { __stcs(p, v[0]); }
};
template <> struct Vec<bf16_t, 8> {
    static __device__ __forceinline__ void load(const bf16_t *p, float (&v)[8]) {
        uint4 t = __ldg(reinterpret_cast<const uint4 *>(p));
        v[0] = bf16_lo(t.x); v[1] = bf16_hi(t.x); v[2] = bf16_lo(t.y); v[3] = bf16_hi(t.y);
        v[4] = bf16_lo(t.z); v[5] = bf16_hi(t.z); v[6] = bf16_lo(t.w); v[7] = bf16_hi(t.w);
    }
    static __device__ __forceinline__ void store(bf16_t *p, const float (&v)[8]) {
        uint4 t = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                             pack_bf16(v[6], v[7]));
        __stcs(reinterpret_cast<uint4 *>(p), t);
    }
};
template <> struct Vec<bf16_t, 2> {
    static __device__ __forceinline__ void load(const bf16_t *p, float (&v)[2]) {
        uint32_t t = __ldg(reinterpret_cast<const unsigned int *>(p));
        v[0] = bf16_lo(t); v[1] = bf16_hi(t);
    }
    static __device__ __forceinline__ void store(bf16_t *p, const float (&v)[2]) {
        __stcs(reinterpret_cast<unsigned int *>(p), pack_bf16(v[0], v[1]));
    }
};
template <> struct Vec<bf16_t, 1> {
    static __device__ __forceinline__ void load(const bf16_t *p, float (&v)[1]) {
        v[0] = __uint_as_float(uint32_t(__ldg(reinterpret_cast<const unsigned short *>(p))) << 16);
    }
    static __device__ __forceinline__ void store(bf16_t *p, const float (&v)[1]) {
        *reinterpret_cast<unsigned short *>(p) = (unsigned short)bf16_bits(v[0]);
    }
};

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
    const int4 *rows;     // schedule {row, begin, end, first chunk}
    const int4 *chunks;   // {begin, end, row, split-row index}
    const int32_t *col;   // other endpoint per CSR position
    const int32_t *order; // CSR position -> COO ordinal
    const float *w;       // COO weights (SpMM)
    const void *F;        // gathered feature rows
    const void *R;        // owner feature rows (SDDMM)
    void *out;            // SpMM output [N, H]
    float *partial;       // [n_chunks, H] fp32
    float *dw;            // SDDMM output, COO order
    int64_t H;
    int64_t n_chunks;     // items [0, n_chunks) are chunks
    int64_t row_first;    // items [n_chunks, n_items) are rows[row_first + i]
    int64_t n_items;
    int G, log2G, col_tiles;
};

// Group of G lanes (G a power of two <= 32) per item.  Each lane owns the
// column vectors j = tile * G * NV + k * G + lane (k < NV) of the row.
template <typename T, int VEC, int NV, int MODE, bool ONE_TILE>
__global__ void __launch_bounds__(kThreads)
k_aggregate(const Params P) {
    const int G = P.G;
    const int64_t gid = (int64_t(blockIdx.x) * kThreads + threadIdx.x) >> P.log2G;
    if (gid >= P.n_items) return;
    const int gl = threadIdx.x & (G - 1);
    const int lane = threadIdx.x & 31;
    const unsigned gmask = (G == 32) ? 0xffffffffu : (((1u << G) - 1u) << (lane & ~(G - 1)));

    int64_t beg, end, row;
    float *partial_row = nullptr;
    if (gid < P.n_chunks) {
        const int4 c = P.chunks[gid];
        beg = c.x; end = c.y; row = c.z;
        if (MODE == kSpmm) partial_row = P.partial + gid * P.H;
    } else {
        const int4 r = P.rows[P.row_first + (gid - P.n_chunks)];
        row = r.x; beg = r.y; end = r.z;
    }
    const int64_t H = P.H;
    const int64_t HV = H / VEC;
    const T *__restrict__ F = static_cast<const T *>(P.F);

    for (int tile = 0; tile < (ONE_TILE ? 1 : P.col_tiles); ++tile) {
        const int64_t vbase = int64_t(tile) * G * NV + gl;
        bool colok[NV];
#pragma unroll
        for (int k = 0; k < NV; ++k) colok[k] = vbase + int64_t(k) * G < HV;

        float acc[NV][VEC];
        float own[NV][VEC];
#pragma unroll
        for (int k = 0; k < NV; ++k)
#pragma unroll
            for (int v = 0; v < VEC; ++v) acc[k][v] = 0.f, own[k][v] = 0.f;
        if (MODE == kSddmm) {
            const T *Rrow = static_cast<const T *>(P.R) + row * H;
#pragma unroll
            for (int k = 0; k < NV; ++k)
                if (colok[k]) Vec<T, VEC>::load(Rrow + (vbase + int64_t(k) * G) * VEC, own[k]);
        }

        for (int64_t base = beg; base < end; base += G) {
            const int64_t p = base + gl;
            int c = 0, e = 0;
            float wt = 0.f;
            if (p < end) {
                c = __ldcs(P.col + p);
                e = __ldcs(P.order + p);
                if (MODE == kSpmm) wt = __ldg(P.w + e);
            }
            const int n = int(end - base < G ? end - base : G);
            for (int j = 0; j < n; j += kUnroll) {
                float x[kUnroll][NV][VEC];
                float wv[kUnroll];
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    const int src = __shfl_sync(gmask, c, (j + u) & (G - 1), G);
                    wv[u] = (MODE == kSpmm) ? __shfl_sync(gmask, wt, (j + u) & (G - 1), G) : 0.f;
                    const T *Frow = F + int64_t(src) * H;
#pragma unroll
                    for (int k = 0; k < NV; ++k) {
                        if (j + u < n && colok[k]) {
                            Vec<T, VEC>::load(Frow + (vbase + int64_t(k) * G) * VEC, x[u][k]);
                        } else {
#pragma unroll
                            for (int v = 0; v < VEC; ++v) x[u][k][v] = 0.f;
                        }
                    }
                }
                if (MODE == kSpmm) {
#pragma unroll
                    for (int u = 0; u < kUnroll; ++u)
                        if (j + u < n)
#pragma unroll
                            for (int k = 0; k < NV; ++k)
#pragma unroll
                                for (int v = 0; v < VEC; ++v) acc[k][v] = fmaf(wv[u], x[u][k][v], acc[k][v]);
                } else {
                    float dot[kUnroll];
#pragma unroll
                    for (int u = 0; u < kUnroll; ++u) {
                        dot[u] = 0.f;
#pragma unroll
                        for (int k = 0; k < NV; ++k)
#pragma unroll
                            for (int v = 0; v < VEC; ++v) dot[u] = fmaf(own[k][v], x[u][k][v], dot[u]);
                    }
#pragma unroll
                    for (int u = 0; u < kUnroll; ++u)
                        for (int o = G >> 1; o > 0; o >>= 1) dot[u] += __shfl_xor_sync(gmask, dot[u], o, G);
                    if (ONE_TILE) {
#pragma unroll
                        for (int u = 0; u < kUnroll; ++u)
                            if (j + u < n && gl == ((j + u) & (G - 1))) P.dw[e] = dot[u];
                    } else {
                        // several column tiles: accumulate the partial dots in dw (this
                        // lane alone owns edge e, so the read-modify-write is race free)
#pragma unroll
                        for (int u = 0; u < kUnroll; ++u)
                            if (j + u < n && gl == ((j + u) & (G - 1)))
                                P.dw[e] = tile == 0 ? dot[u] : P.dw[e] + dot[u];
                    }
                }
            }
        }
        if (MODE == kSpmm) {
            if (partial_row) {
#pragma unroll
                for (int k = 0; k < NV; ++k)
                    if (colok[k]) store_partial<VEC>(partial_row + (vbase + int64_t(k) * G) * VEC, acc[k]);
            } else {
                T *Yrow = static_cast<T *>(P.out) + row * H;
#pragma unroll
                for (int k = 0; k < NV; ++k)
                    if (colok[k]) Vec<T, VEC>::store(Yrow + (vbase + int64_t(k) * G) * VEC, acc[k]);
            }
        }
    }
}

// Sum of the partial rows of every split row, in chunk order.
template <typename T, int VEC, int NV>
__global__ void __launch_bounds__(kThreads)
k_finish(const int4 *__restrict__ rows, int64_t n_heavy, const float *__restrict__ partial, void *out,
         int64_t H, int G, int log2G, int col_tiles) {
    const int64_t h = (int64_t(blockIdx.x) * kThreads + threadIdx.x) >> log2G;
    if (h >= n_heavy) return;
    const int gl = threadIdx.x & (G - 1);
    const int4 r = rows[h];
    const int nch = (r.z - r.y + kChunkEdges - 1) / kChunkEdges;
    const int64_t HV = H / VEC;
    for (int tile = 0; tile < col_tiles; ++tile) {
        const int64_t vbase = int64_t(tile) * G * NV + gl;
        float acc[NV][VEC];
#pragma unroll
        for (int k = 0; k < NV; ++k)
#pragma unroll
            for (int v = 0; v < VEC; ++v) acc[k][v] = 0.f;
        for (int c = 0; c < nch; ++c) {
            const float *prow = partial + (int64_t(r.w) + c) * H;
#pragma unroll
            for (int k = 0; k < NV; ++k)
                if (vbase + int64_t(k) * G < HV) add_partial<VEC>(prow + (vbase + int64_t(k) * G) * VEC, acc[k]);
        }
        T *Yrow = static_cast<T *>(out) + int64_t(r.x) * H;
#pragma unroll
        for (int k = 0; k < NV; ++k)
            if (vbase + int64_t(k) * G < HV) Vec<T, VEC>::store(Yrow + (vbase + int64_t(k) * G) * VEC, acc[k]);
    }
}

// ---------------------------------------------------------------------------- host side

struct Shape {
    int vec, G, log2G, nv, col_tiles;
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
    while (G < 32 && G < HV) G <<= 1;
    s.G = G;
    s.log2G = log2i(G);
    const int64_t per_lane = (HV + G - 1) / G;
    s.nv = per_lane <= 1 ? 1 : (per_lane <= 2 ? 2 : 4);
    s.col_tiles = int((HV + int64_t(G) * s.nv - 1) / (int64_t(G) * s.nv));
    return s;
}

template <typename T, int VEC, int NV, int MODE>
void launch_main(const Params &P, const Shape &s, cudaStream_t st) {
    const int64_t groups_per_block = kThreads / s.G;
    const unsigned grid = unsigned((P.n_items + groups_per_block - 1) / groups_per_block);
    if (s.col_tiles == 1) k_aggregate<T, VEC, NV, MODE, true><<<grid, kThreads, 0, st>>>(P);
    else k_aggregate<T, VEC, NV, MODE, false><<<grid, kThreads, 0, st>>>(P);
}

template <typename T, int VEC, int NV>
void launch_finish(const ag::Direction &D, const float *partial, void *out, int64_t H, const Shape &s,
                   cudaStream_t st) {
    const int64_t groups_per_block = kThreads / s.G;
    const unsigned grid = unsigned((D.n_heavy + groups_per_block - 1) / groups_per_block);
    k_finish<T, VEC, NV><<<grid, kThreads, 0, st>>>(D.rows, D.n_heavy, partial, out, H, s.G, s.log2G,
                                                    s.col_tiles);
}

template <int MODE, typename T, int VEC>
void dispatch_nv(const Params &P, const Shape &s, cudaStream_t st) {
    switch (s.nv) {
        case 1: launch_main<T, VEC, 1, MODE>(P, s, st); break;
        case 2: launch_main<T, VEC, 2, MODE>(P, s, st); break;
        default: launch_main<T, VEC, 4, MODE>(P, s, st); break;
    }
}

template <int MODE>
void dispatch_main(const Params &P, const Shape &s, int dtype, cudaStream_t st) {
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
void finish_nv(const ag::Direction &D, const float *partial, void *out, int64_t H, const Shape &s, cudaStream_t st) {
    switch (s.nv) {
        case 1: launch_finish<T, VEC, 1>(D, partial, out, H, s, st); break;
        case 2: launch_finish<T, VEC, 2>(D, partial, out, H, s, st); break;
        default: launch_finish<T, VEC, 4>(D, partial, out, H, s, st); break;
    }
}

void dispatch_finish(const ag::Direction &D, const float *partial, void *out, int64_t H, const Shape &s,
                     int dtype, cudaStream_t st) {
    if (dtype == AG_F32) {
        if (s.vec == 4) finish_nv<float, 4>(D, partial, out, H, s, st);
        else finish_nv<float, 1>(D, partial, out, H, s, st);
    } else {
        if (s.vec == 8) finish_nv<bf16_t, 8>(D, partial, out, H, s, st);
        else if (s.vec == 2) finish_nv<bf16_t, 2>(D, partial, out, H, s, st);
        else finish_nv<bf16_t, 1>(D, partial, out, H, s, st);
    }
}

int check_call(const ag_graph *g, int64_t H, int dtype, const char *fn) {
    if (!g) return fail(AG_ERR_INVALID_ARG, "%s: null graph", fn);
    if (dtype != AG_F32 && dtype != AG_BF16) return fail(AG_ERR_DTYPE, "%s: unknown dtype %d", fn, dtype);
    if (H < 1 || H > (int64_t(1) << 24) || g->N * H >= (int64_t(1) << 40))
        return fail(AG_ERR_SHAPE, "%s: H=%lld out of range for N=%lld", fn, (long long)H, (long long)g->N);
    return AG_OK;
}

size_t scratch_needed(const ag_graph *g, int64_t H) {
    int64_t c = g->dir[0].n_chunks > g->dir[1].n_chunks ? g->dir[0].n_chunks : g->dir[1].n_chunks;
    return size_t(c) * size_t(H) * 4;
}

// SpMM over direction d: out = A_w X (d = 0) or A_w^T dY (d = 1).
int spmm(const ag_graph *g, int d, const float *w, const void *F, void *out, int64_t H, int dtype,
         void *scratch, size_t scratch_bytes, void *stream, const char *fn, bool check_ptrs) {
    int rc = check_call(g, H, dtype, fn);
    if (rc != AG_OK) return rc;
    if (!F || !out || (g->E > 0 && !w)) return fail(AG_ERR_INVALID_ARG, "%s: null w, input or output", fn);
    const ag::Direction &D = g->dir[d];
    const size_t need = size_t(D.n_chunks) * size_t(H) * 4;
    if (need > 0 && (!scratch || scratch_bytes < need))
        return fail(AG_ERR_WORKSPACE, "%s: scratch of %zu bytes, need %zu", fn, scratch_bytes, need);
    if (!aligned(scratch, 16)) return fail(AG_ERR_WORKSPACE, "%s: scratch must be 16-byte aligned", fn);
    if (check_ptrs) {
        if ((rc = check_device_ptr(F, g->device, "input")) != AG_OK) return rc;
        if ((rc = check_device_ptr(out, g->device, "output")) != AG_OK) return rc;
        if (g->E > 0 && (rc = check_device_ptr(w, g->device, "w")) != AG_OK) return rc;
        if (need > 0 && (rc = check_device_ptr(scratch, g->device, "scratch")) != AG_OK) return rc;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const Shape s = pick_shape(H, dtype, F, out, nullptr);
    Params P{};
    P.rows = D.rows;
    P.chunks = D.chunks;
    P.col = D.col;
    P.order = D.order;
    P.w = w;
    P.F = F;
    P.out = out;
    P.partial = static_cast<float *>(scratch);
    P.H = H;
    P.n_chunks = D.n_chunks;
    P.row_first = D.n_heavy;
    P.n_items = D.n_chunks + (g->N - D.n_heavy);
    P.G = s.G;
    P.log2G = s.log2G;
    P.col_tiles = s.col_tiles;
    if (P.n_items > 0) dispatch_main<kSpmm>(P, s, dtype, st);
    if (D.n_heavy > 0) dispatch_finish(D, P.partial, out, H, s, dtype, st);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return cuda_fail(err, fn);
    return AG_OK;
}

// dw over the transpose CSR: owner = source row (X), gathered = dY[col_t].
int sddmm(const ag_graph *g, const void *X, const void *dY, float *dw, int64_t H, int dtype, void *stream,
          const char *fn, bool check_ptrs) {
    int rc = check_call(g, H, dtype, fn);
    if (rc != AG_OK) return rc;
    if (!X || !dY || (g->E > 0 && !dw)) return fail(AG_ERR_INVALID_ARG, "%s: null X, dY or dw", fn);
    if (check_ptrs) {
        if ((rc = check_device_ptr(X, g->device, "X")) != AG_OK) return rc;
        if ((rc = check_device_ptr(dY, g->device, "dY")) != AG_OK) return rc;
        if (g->E > 0 && (rc = check_device_ptr(dw, g->device, "dw")) != AG_OK) return rc;
    }
    if (g->E == 0) return AG_OK;
    const ag::Direction &D = g->dir[1];
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const Shape s = pick_shape(H, dtype, X, dY, nullptr);
    Params P{};
    P.rows = D.rows;
    P.chunks = D.chunks;
    P.col = D.col;
    P.order = D.order;
    P.F = dY;
    P.R = X;
    P.dw = dw;
    P.H = H;
    P.n_chunks = D.n_chunks;
    P.row_first = D.n_heavy;
    P.n_items = D.n_chunks + (D.n_nonempty - D.n_heavy);
    P.G = s.G;
    P.log2G = s.log2G;
    P.col_tiles = s.col_tiles;
    if (P.n_items > 0) dispatch_main<kSddmm>(P, s, dtype, st);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return cuda_fail(err, fn);
    return AG_OK;
}

}  // namespace
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
                void *stream) {
    clear_error();
    return sddmm(g, X, dY, dw, H, dtype, stream, "ag_sddmm_dw", true);
}

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

int ag_step_host(const ag_graph *g, const float *w_host, const void *X_host, const void *dY_host,
                 void *Y_host, void *dX_host, float *dw_host, int64_t H, int dtype, void *staging,
                 size_t staging_bytes, void *stream) {
    clear_error();
    int rc = check_call(g, H, dtype, "ag_step_host");
    if (rc != AG_OK) return rc;
    if (!X_host || !dY_host || !Y_host || !dX_host || (g->E > 0 && (!w_host || !dw_host)) || !staging)
        return fail(AG_ERR_INVALID_ARG, "ag_step_host: null buffer");
    size_t off[7], total = 0;
    staging_layout(g, H, dtype, off, &total);
    if (staging_bytes < total)
        return fail(AG_ERR_WORKSPACE, "ag_step_host: staging of %zu bytes, need %zu", staging_bytes, total);
    if (!aligned(staging, kAlign)) return fail(AG_ERR_WORKSPACE, "ag_step_host: staging must be 256-byte aligned");
    if ((rc = check_device_ptr(staging, g->device, "staging")) != AG_OK) return rc;
    char *base = static_cast<char *>(staging);
    float *w = reinterpret_cast<float *>(base + off[0]);
    void *X = base + off[1], *dY = base + off[2], *Y = base + off[3], *dX = base + off[4];
    float *dw = reinterpret_cast<float *>(base + off[5]);
    void *scratch = base + off[6];
    const size_t feat = size_t(g->N) * size_t(H) * (dtype == AG_F32 ? 4 : 2);
    const size_t wb = size_t(g->E) * 4;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t err = cudaSuccess;
    auto copy = [&](void *to, const void *from, size_t n, cudaMemcpyKind k) {
        if (err == cudaSuccess && n > 0) err = cudaMemcpyAsync(to, from, n, k, st);
    };
    const size_t scr = scratch_needed(g, H);
    copy(w, w_host, wb, cudaMemcpyHostToDevice);
    copy(X, X_host, feat, cudaMemcpyHostToDevice);
    if (err != cudaSuccess) return cuda_fail(err, "ag_step_host: copy in");
    if ((rc = spmm(g, 0, w, X, Y, H, dtype, scratch, scr, stream, "ag_step_host", false)) != AG_OK) return rc;
    copy(Y_host, Y, feat, cudaMemcpyDeviceToHost);
    copy(dY, dY_host, feat, cudaMemcpyHostToDevice);
    if (err != cudaSuccess) return cuda_fail(err, "ag_step_host: copy");
    if ((rc = spmm(g, 1, w, dY, dX, H, dtype, scratch, scr, stream, "ag_step_host", false)) != AG_OK) return rc;
    copy(dX_host, dX, feat, cudaMemcpyDeviceToHost);
    if ((rc = sddmm(g, X, dY, dw, H, dtype, stream, "ag_step_host", false)) != AG_OK) return rc;
    copy(dw_host, dw, wb, cudaMemcpyDeviceToHost);
    if (err != cudaSuccess) return cuda_fail(err, "ag_step_host: copy out");
    return AG_OK;
}

}  // extern "C"
