// lower.cu -- COO -> forward CSR + transpose CSR connectivity lowering.
//
// tinymesh "Weighted aggregation experiment", section "Edge order is
// explicit": connectivity is sorted by owner without detaching the weights.
// edge_order and transpose_order take a slot of the sorted CSR back to the
// edge's index in the caller's COO list; two edges with the same endpoints
// are two slots, never merged.  Section "Exact
// witness": edges 0->2, 1->2, 0->1 lower to edge_order = (2, 0, 1), i.e. ties
// between edges of one owner stay in COO order (a stable sort on the owner).
//
// Device algorithm (all integer, deterministic, no inter-block waiting):
//   1. range check of every src/dst index (sets a flag, the host returns
//      AG_ERR_INDEX_RANGE);
//   2. stable LSD radix sort of the COO ordinals by owner key, 8-bit digits,
//      one (histogram, exclusive scan, stable scatter) triple per digit;
//      the scatter ranks equal digits with __match_any_sync inside a warp
//      and in warp order across the tile, so equal keys keep COO order;
//   3. rowptr[r] = lower_bound(sorted keys, r), col = other[order];
//   4. the tile schedule of the per-call kernels: the non-empty rows
//      compacted (ids and first positions), the empty rows listed, the row
//      holding the first position of every tile, and the rows cut by a tile
//      boundary (long ones first);
//   5. the weight windows: every edge's slot in an order grouped by windows
//      of 2^20 consecutive CSR positions (COO order inside a window), the
//      slot read at every CSR position, and the per-chunk staging table that
//      lets the per-call regrouping write whole runs of slots.  An edge's
//      window comes from its row's pointers (and, for the few rows that cross
//      a window boundary, one order lookup); its slot from one ranking pass.
// The radix scatter stages each tile in digit order in shared memory and
// writes whole runs, so its global writes are coalesced.
#include <climits>
#include <cstdio>

#include "internal.h"

namespace ag {
namespace {

constexpr int kRadixThreads = 256;
constexpr int kRadixItems = 16;  // keys per thread
constexpr int kRadixTile = kRadixThreads * kRadixItems;
constexpr int kRadixWarps = kRadixThreads / 32;
constexpr int kRadix = 256;
static_assert(kRadixThreads == kRadix, "one thread per digit in the tile's digit scan");

constexpr int kScanThreads = 256;
constexpr int kScanItems = 8;
constexpr int kScanTile = kScanThreads * kScanItems;  // 2048

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

__global__ void k_check_range(const int32_t *__restrict__ src, const int32_t *__restrict__ dst,
                              int64_t E, int64_t N, unsigned *bad_first) {
    for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < E;
         e += int64_t(gridDim.x) * blockDim.x) {
        if (uint32_t(src[e]) >= uint64_t(N) || uint32_t(dst[e]) >= uint64_t(N))
            atomicMin(bad_first, unsigned(e));
    }
}

// Per-tile digit counts, stored digit-major: hist[d * nblk + tile].
__global__ void __launch_bounds__(kRadixThreads)
k_radix_hist(const int32_t *__restrict__ keys, int64_t n, int shift, int nblk,
             int32_t *__restrict__ hist) {
    __shared__ int cnt[kRadix];
    for (int i = threadIdx.x; i < kRadix; i += kRadixThreads) cnt[i] = 0;
    __syncthreads();
    const int64_t base = int64_t(blockIdx.x) * kRadixTile;
#pragma unroll 4
    for (int k = 0; k < kRadixItems; ++k) {
        int64_t i = base + int64_t(k) * kRadixThreads + threadIdx.x;
        if (i < n) atomicAdd(&cnt[(uint32_t(keys[i]) >> shift) & (kRadix - 1)], 1);
    }
    __syncthreads();
    for (int d = threadIdx.x; d < kRadix; d += kRadixThreads)
        hist[int64_t(d) * nblk + blockIdx.x] = cnt[d];
}

// Exclusive scan of v over the kRadixThreads threads of the block (one value
// each); returns this thread's prefix.  `wtot` holds kRadixWarps ints.
__device__ __forceinline__ int block_exclusive_scan(int v, int *wtot) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wtot[warp] = incl;
    __syncthreads();
    int before = 0;
#pragma unroll
    for (int w = 0; w < kRadixWarps; ++w) before += w < warp ? wtot[w] : 0;
    __syncthreads();
    return before + incl - v;
}

// Stable scatter of one digit pass.  Warp w of the tile owns the contiguous
// items [w * 32 * kRadixItems, (w + 1) * 32 * kRadixItems) and ranks them in
// order, 32 at a time (__match_any_sync inside a warp, warp order across the
// tile), which gives every item its place in the tile's digit-sorted order;
// offs holds the exclusive scan of hist (digit-major).
//   MOVE: the tile is put in digit order in shared memory and then written
//         out in that order, so that consecutive threads write consecutive
//         addresses of one digit's run (keys_out, vals_out).
//   otherwise: only the destination of every item is written, in item order:
//         pos_out[i] = where item i goes (the rank of i in the stable order).
template <bool MOVE>
__global__ void __launch_bounds__(kRadixThreads)
k_radix_scatter(const int32_t *__restrict__ keys_in, const int32_t *__restrict__ vals_in,
                int64_t n, int shift, int nblk, const int32_t *__restrict__ offs,
                int32_t *__restrict__ keys_out, int32_t *__restrict__ vals_out) {
    __shared__ int whist[kRadixWarps][kRadix];
    __shared__ int dstart[kRadix];      // first place of each digit in the tile's sorted order
    __shared__ int dbase[kRadix];       // global position of that place
    __shared__ int wtot[kRadixWarps];
    __shared__ int skey[MOVE ? kRadixTile : 1], sval[MOVE ? kRadixTile : 1];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < kRadixWarps * kRadix; i += kRadixThreads)
        (&whist[0][0])[i] = 0;
    __syncthreads();

    const int64_t tile0 = int64_t(blockIdx.x) * kRadixTile;
    const int64_t base = tile0 + int64_t(warp) * 32 * kRadixItems;
    const unsigned lt = lanemask_lt();
    int key[kRadixItems], val[kRadixItems], rank[kRadixItems];
#pragma unroll
    for (int k = 0; k < kRadixItems; ++k) {
        const int64_t i = base + k * 32 + lane;
        const bool valid = i < n;
        key[k] = valid ? keys_in[i] : 0;
        val[k] = valid ? (vals_in ? vals_in[i] : int(i)) : 0;
        rank[k] = 0;
        const unsigned vmask = __ballot_sync(0xffffffffu, valid);
        if (valid) {
            const int d = (uint32_t(key[k]) >> shift) & (kRadix - 1);
            const unsigned peers = __match_any_sync(vmask, d);
            const int prior = whist[warp][d];
            rank[k] = prior + __popc(peers & lt);
            __syncwarp(vmask);
            if (lane == __ffs(peers) - 1) whist[warp][d] = prior + __popc(peers);
            __syncwarp(vmask);
        }
    }
    __syncthreads();
    // exclusive prefix over warps, per digit (warp order = item order), and
    // the tile's count of every digit
    int count = 0;
    {
        const int d = threadIdx.x;  // kRadixThreads == kRadix
#pragma unroll
        for (int w = 0; w < kRadixWarps; ++w) {
            const int t = whist[w][d];
            whist[w][d] = count;
            count += t;
        }
    }
    const int start = block_exclusive_scan(count, wtot);
    dstart[threadIdx.x] = start;
    dbase[threadIdx.x] = offs[int64_t(threadIdx.x) * nblk + blockIdx.x];
    __syncthreads();
    if constexpr (MOVE) {
#pragma unroll
        for (int k = 0; k < kRadixItems; ++k) {
            const int64_t i = base + k * 32 + lane;
            if (i < n) {
                const int d = (uint32_t(key[k]) >> shift) & (kRadix - 1);
                const int local = dstart[d] + whist[warp][d] + rank[k];
                skey[local] = key[k];
                sval[local] = val[k];
            }
        }
        __syncthreads();
        const int m = int(n - tile0 < kRadixTile ? n - tile0 : kRadixTile);
        for (int i = threadIdx.x; i < m; i += kRadixThreads) {
            const int kk = skey[i];
            const int d = (uint32_t(kk) >> shift) & (kRadix - 1);
            const int64_t pos = int64_t(dbase[d]) + (i - dstart[d]);
            keys_out[pos] = kk;
            vals_out[pos] = sval[i];
        }
    } else {
#pragma unroll
        for (int k = 0; k < kRadixItems; ++k) {
            const int64_t i = base + k * 32 + lane;
            if (i < n) {
                const int d = (uint32_t(key[k]) >> shift) & (kRadix - 1);
                vals_out[i] = dbase[d] + whist[warp][d] + rank[k];
            }
        }
    }
}

__global__ void __launch_bounds__(kScanThreads)
k_scan_tile_sums(const int32_t *__restrict__ in, int64_t n, int32_t *__restrict__ sums) {
    __shared__ int wsum[kScanThreads / 32];
    const int64_t base = int64_t(blockIdx.x) * kScanTile;
    int s = 0;
    for (int i = threadIdx.x; i < kScanTile; i += kScanThreads) {
        int64_t g = base + i;
        if (g < n) s += in[g];
    }
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        int t = 0;
        for (int w = 0; w < kScanThreads / 32; ++w) t += wsum[w];
        sums[blockIdx.x] = t;
    }
}

// Exclusive scan of one 2048-item tile plus the tile's offset; the tile that
// reaches the end also writes the grand total to out[n].  In-place safe.
__global__ void __launch_bounds__(kScanThreads)
k_scan_tiles(const int32_t *in, int64_t n, const int32_t *__restrict__ tile_off, int32_t *out) {
    __shared__ int s[kScanTile];
    __shared__ int wtot[kScanThreads / 32];
    const int64_t base = int64_t(blockIdx.x) * kScanTile;
    for (int i = threadIdx.x; i < kScanTile; i += kScanThreads) {
        int64_t g = base + i;
        s[i] = g < n ? in[g] : 0;
    }
    __syncthreads();
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    int v[kScanItems], sum = 0;
#pragma unroll
    for (int k = 0; k < kScanItems; ++k) {
        v[k] = s[t * kScanItems + k];
        sum += v[k];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wtot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int x = lane < kScanThreads / 32 ? wtot[lane] : 0;
        int xi = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, xi, o);
            if (lane >= o) xi += y;
        }
        if (lane < kScanThreads / 32) wtot[lane] = xi - x;
    }
    __syncthreads();
    int run = incl - sum + wtot[warp] + (tile_off ? tile_off[blockIdx.x] : 0);
#pragma unroll
    for (int k = 0; k < kScanItems; ++k) {
        s[t * kScanItems + k] = run;
        run += v[k];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kScanTile; i += kScanThreads) {
        int64_t g = base + i;
        if (g < n) out[g] = s[i];
    }
    if (t == kScanThreads - 1 && base + kScanTile >= n) out[n] = run;
}

__global__ void k_iota(int32_t *out, int64_t n) {
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n;
         i += int64_t(gridDim.x) * blockDim.x)
        out[i] = int32_t(i);
}

// rowptr[r] = first position p with sorted_keys[p] >= r, for r in [0, N].
__global__ void k_rowptr_search(const int32_t *__restrict__ keys, int64_t E, int64_t N,
                                int32_t *__restrict__ rowptr) {
    for (int64_t r = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; r <= N;
         r += int64_t(gridDim.x) * blockDim.x) {
        int64_t lo = 0, hi = E;
        while (lo < hi) {
            int64_t mid = (lo + hi) >> 1;
            if (keys[mid] < r) lo = mid + 1;
            else hi = mid;
        }
        rowptr[r] = int32_t(lo);
    }
}

// out[i] = from[idx[i]]; four independent gathers in flight per thread
__global__ void k_gather(const int32_t *__restrict__ idx, const int32_t *__restrict__ from,
                         int64_t n, int32_t *__restrict__ out) {
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
    for (; i + 3 * stride < n; i += 4 * stride) {
        const int j0 = __ldcs(idx + i), j1 = __ldcs(idx + i + stride);
        const int j2 = __ldcs(idx + i + 2 * stride), j3 = __ldcs(idx + i + 3 * stride);
        const int v0 = from[j0], v1 = from[j1], v2 = from[j2], v3 = from[j3];
        __stcs(out + i, v0);
        __stcs(out + i + stride, v1);
        __stcs(out + i + 2 * stride, v2);
        __stcs(out + i + 3 * stride, v3);
    }
    for (; i < n; i += stride) out[i] = from[idx[i]];
}

__global__ void k_max_degree(const int32_t *__restrict__ rowptr, int64_t N, int *maxdeg) {
    int m = 0;
    for (int64_t r = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; r < N;
         r += int64_t(gridDim.x) * blockDim.x)
        m = max(m, rowptr[r + 1] - rowptr[r]);
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0 && m > 0) atomicMax(maxdeg, m);
}

// flags[r] = 1 if row r has at least one edge
__global__ void k_nz_flags(const int32_t *__restrict__ rowptr, int64_t N, int32_t *__restrict__ flags) {
    for (int64_t r = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; r < N;
         r += int64_t(gridDim.x) * blockDim.x)
        flags[r] = rowptr[r + 1] > rowptr[r] ? 1 : 0;
}

// pos = exclusive scan of the flags (pos[N] = number of non-empty rows).
__global__ void k_nz_scatter(const int32_t *__restrict__ rowptr, const int32_t *__restrict__ pos, int64_t N,
                             int64_t E, int32_t *__restrict__ nz_rows, int32_t *__restrict__ nz_rowptr,
                             int32_t *__restrict__ zero_rows) {
    for (int64_t r = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; r < N;
         r += int64_t(gridDim.x) * blockDim.x) {
        const int i = pos[r];
        if (rowptr[r + 1] > rowptr[r]) {
            nz_rows[i] = int32_t(r);
            nz_rowptr[i] = rowptr[r];
        } else {
            zero_rows[r - i] = int32_t(r);
        }
        if (r == N - 1) nz_rowptr[pos[N]] = int32_t(E);
    }
}

// tile_nz[t] = the non-empty row i with nz_rowptr[i] <= t*T < nz_rowptr[i+1].
__global__ void k_tile_nz(const int32_t *__restrict__ nz_rowptr, int64_t n_nz, int T,
                          int32_t *__restrict__ tile_nz) {
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n_nz;
         i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t b = nz_rowptr[i], e = nz_rowptr[i + 1];
        for (int64_t t = (b + T - 1) / T; t <= (e - 1) / T; ++t) tile_nz[t] = int32_t(i);
    }
}

// Rows whose first and last edge fall in different tiles; `lng` marks those
// that cross more than kLongSpanTiles tile boundaries.
__global__ void k_span_flags(const int32_t *__restrict__ nz_rowptr, int64_t n_nz, int T,
                             int32_t *__restrict__ lng, int32_t *__restrict__ shrt) {
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n_nz;
         i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t ta = nz_rowptr[i] / T, tb = (int64_t(nz_rowptr[i + 1]) - 1) / T;
        const bool span = ta != tb;
        const bool is_long = span && tb - ta > kLongSpanTiles;
        lng[i] = is_long ? 1 : 0;
        shrt[i] = (span && !is_long) ? 1 : 0;
    }
}

__global__ void k_span_scatter(const int32_t *__restrict__ nz_rows, const int32_t *__restrict__ nz_rowptr,
                               int64_t n_nz, int T, const int32_t *__restrict__ lpos,
                               const int32_t *__restrict__ spos, int64_t n_long, int4 *__restrict__ spans) {
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n_nz;
         i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t ta = nz_rowptr[i] / T, tb = (int64_t(nz_rowptr[i + 1]) - 1) / T;
        if (ta == tb) continue;
        const int4 v = make_int4(nz_rows[i], int(ta), int(tb), 0);
        if (tb - ta > kLongSpanTiles) spans[lpos[i]] = v;
        else spans[n_long + spos[i]] = v;
    }
}

// out[e] = the weight window (position >> shift) of COO ordinal e, found from
// its row key[e]: the row's positions [rowptr[k], rowptr[k + 1]) lie in one
// window unless the row crosses window boundaries, and inside a row the
// ordinals ascend with the position, so e lies at or past boundary B exactly
// when order[B] <= e.  Reads are sequential except the L2-resident row
// pointers.
__global__ void k_window_of(const int32_t *__restrict__ key, const int32_t *__restrict__ rowptr,
                            const int32_t *__restrict__ order, int64_t n, int shift, int32_t *__restrict__ out) {
    for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < n;
         e += int64_t(gridDim.x) * blockDim.x) {
        const int k = __ldcs(key + e);
        const int64_t a = rowptr[k], b = rowptr[k + 1];
        int w = int(a >> shift);
        for (int64_t B = (int64_t(w) + 1) << shift; B < b; B += int64_t(1) << shift) {
            if (order[B] <= e) ++w;
            else break;
        }
        __stcs(out + e, w);
    }
}

// out[order[p]] = p >> shift: the weight window of every COO ordinal.
__global__ void k_window_keys(const int32_t *__restrict__ order, int64_t n, int shift, int32_t *__restrict__ out) {
    for (int64_t p = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; p < n;
         p += int64_t(gridDim.x) * blockDim.x)
        out[order[p]] = int32_t(p >> shift);
}

// out[perm[i]] = i
__global__ void k_invert(const int32_t *__restrict__ perm, int64_t n, int32_t *__restrict__ out) {
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n;
         i += int64_t(gridDim.x) * blockDim.x)
        out[perm[i]] = int32_t(i);
}

// Per chunk of kStageChunk ordinals: for every window b that has ordinals in
// the chunk, delta = (start of b's run in the chunk sorted by window) - (the
// smallest slot of the chunk in b).  The slots of a window within a chunk are
// consecutive, so slot + delta is the ordinal's position in the sorted chunk.
__global__ void __launch_bounds__(256)
k_stage_table(const int32_t *__restrict__ slot, int64_t E, int shift, int nwin, int32_t *__restrict__ delta) {
    __shared__ int cnt[kStageMaxWindows];
    __shared__ int first[kStageMaxWindows];
    const int64_t c0 = int64_t(blockIdx.x) * kStageChunk;
    const int n = int(E - c0 < kStageChunk ? E - c0 : kStageChunk);
    for (int b = threadIdx.x; b < nwin; b += blockDim.x) {
        cnt[b] = 0;
        first[b] = INT_MAX;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int sl = slot[c0 + i];
        atomicAdd(&cnt[sl >> shift], 1);
        atomicMin(&first[sl >> shift], sl);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int b = 0; b < nwin; ++b) {
            delta[int64_t(blockIdx.x) * nwin + b] = cnt[b] ? run - first[b] : 0;
            run += cnt[b];
        }
    }
}

// Number of positions p > 0 whose ordinal lies in the same 8-ordinal
// (32-byte) sector as the ordinal at p - 1.
__global__ void k_sector_runs(const int32_t *__restrict__ order, int64_t n, unsigned long long *count) {
    unsigned c = 0;
    for (int64_t p = 1 + blockIdx.x * int64_t(blockDim.x) + threadIdx.x; p < n;
         p += int64_t(gridDim.x) * blockDim.x)
        c += (order[p] >> 3) == (order[p - 1] >> 3) ? 1u : 0u;
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if ((threadIdx.x & 31) == 0 && c) atomicAdd(count, (unsigned long long)c);
}

inline unsigned grid_for(int64_t n, int threads, int64_t cap = 148 * 64) {
    int64_t b = (n + threads - 1) / threads;
    if (b < 1) b = 1;
    if (b > cap) b = cap;
    return unsigned(b);
}

struct Tmp {
    int32_t *keys_a, *vals_a, *keys_b, *vals_b, *hist, *scan, *aux, *aux2;
};

// Exclusive scan of in[0, n) into out[0, n], out[n] = total.  `tmp` holds the
// per-tile sums of every recursion level.
void exclusive_scan(const int32_t *in, int32_t *out, int64_t n, int32_t *tmp, cudaStream_t s) {
    if (n <= kScanTile) {
        k_scan_tiles<<<1, kScanThreads, 0, s>>>(in, n, nullptr, out);
        return;
    }
    const int64_t nb = (n + kScanTile - 1) / kScanTile;
    int32_t *sums = tmp;
    k_scan_tile_sums<<<unsigned(nb), kScanThreads, 0, s>>>(in, n, sums);
    exclusive_scan(sums, sums, nb, tmp + align_up(size_t(nb) + 1, 64), s);
    k_scan_tiles<<<unsigned(nb), kScanThreads, 0, s>>>(in, n, sums, out);
}

int bit_length(int64_t v) {
    int b = 0;
    while (v > 0) {
        ++b;
        v >>= 1;
    }
    return b;
}

// Stable sort of (key, value) pairs by key, keys in [0, 2^bits).  vals_in ==
// nullptr means values 0..n-1.  The sorted values go to vals_out; the
// returned pointer holds the sorted keys (one of the two ping-pong buffers).
const int32_t *radix_sort(const int32_t *keys_in, const int32_t *vals_in, int64_t n, int bits,
                          int32_t *vals_out, const Tmp &t, cudaStream_t s) {
    const int passes = (bits + 7) / 8;
    if (passes == 0 || n == 0) {
        if (n > 0) {
            if (vals_in)
                cudaMemcpyAsync(vals_out, vals_in, size_t(n) * 4, cudaMemcpyDeviceToDevice, s);
            else
                k_iota<<<grid_for(n, 256), 256, 0, s>>>(vals_out, n);
        }
        return keys_in;
    }
    const int nblk = int((n + kRadixTile - 1) / kRadixTile);
    const int32_t *kin = keys_in, *vin = vals_in;
    int32_t *bufk[2] = {t.keys_a, t.keys_b}, *bufv[2] = {t.vals_a, t.vals_b};
    for (int p = 0; p < passes; ++p) {
        int32_t *kout = bufk[p & 1];
        int32_t *vout = (p == passes - 1) ? vals_out : bufv[p & 1];
        k_radix_hist<<<nblk, kRadixThreads, 0, s>>>(kin, n, 8 * p, nblk, t.hist);
        exclusive_scan(t.hist, t.hist, int64_t(kRadix) * nblk, t.scan, s);
        k_radix_scatter<true><<<nblk, kRadixThreads, 0, s>>>(kin, vin, n, 8 * p, nblk, t.hist, kout, vout);
        kin = kout;
        vin = vout;
    }
    return kin;
}

}  // namespace
}  // namespace ag

using namespace ag;

extern "C" int ag_graph_lower(const int32_t *src, const int32_t *dst, int64_t N, int64_t E,
                              void *workspace, size_t workspace_bytes, void *stream,
                              ag_graph **out) {
    clear_error();
    if (N < 1 || N >= (int64_t(1) << 31) || E < 0 || E >= (int64_t(1) << 31))
        return fail(AG_ERR_SHAPE, "ag_graph_lower: need 1 <= N < 2^31 and 0 <= E < 2^31 (N=%lld, E=%lld)",
                    (long long)N, (long long)E);
    if (!out || !workspace) return fail(AG_ERR_INVALID_ARG, "ag_graph_lower: null out or workspace");
    if (E > 0 && (!src || !dst)) return fail(AG_ERR_INVALID_ARG, "ag_graph_lower: null src/dst with E > 0");
    Layout L;
    make_layout(N, E, &L);
    if (workspace_bytes < L.total)
        return fail(AG_ERR_WORKSPACE, "ag_graph_lower: workspace of %zu bytes, need %zu", workspace_bytes, L.total);
    if (reinterpret_cast<uintptr_t>(workspace) % kAlign)
        return fail(AG_ERR_WORKSPACE, "ag_graph_lower: workspace must be %zu-byte aligned", kAlign);
    int device = 0;
    cudaError_t err = cudaGetDevice(&device);
    if (err != cudaSuccess) return cuda_fail(err, "cudaGetDevice");
    int rc;
    if ((rc = check_device_ptr(workspace, device, "workspace")) != AG_OK) return rc;
    if (E > 0) {
        if ((rc = check_device_ptr(src, device, "src")) != AG_OK) return rc;
        if ((rc = check_device_ptr(dst, device, "dst")) != AG_OK) return rc;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char *ws = static_cast<char *>(workspace);
    auto I = [&](size_t off) { return reinterpret_cast<int32_t *>(ws + off); };
    Tmp t{I(L.keys_a), I(L.vals_a), I(L.keys_b), I(L.vals_b), I(L.hist), I(L.scan_tmp), I(L.aux), nullptr};
    int *counters = reinterpret_cast<int *>(ws + L.counters);
    int host_counters[8];

    auto sync_read = [&](const char *what) -> int {
        cudaError_t e2 = cudaGetLastError();
        if (e2 != cudaSuccess) return cuda_fail(e2, what);
        e2 = cudaMemcpyAsync(host_counters, counters, sizeof host_counters, cudaMemcpyDeviceToHost, s);
        if (e2 == cudaSuccess) e2 = cudaStreamSynchronize(s);
        if (e2 != cudaSuccess) return cuda_fail(e2, what);
        return AG_OK;
    };

    // 1. every index in [0, N)
    err = cudaMemsetAsync(counters, 0xff, sizeof(int), s);
    if (err != cudaSuccess) return cuda_fail(err, "cudaMemsetAsync");
    if (E > 0) k_check_range<<<grid_for(E, 256), 256, 0, s>>>(src, dst, E, N, reinterpret_cast<unsigned *>(counters));
    if ((rc = sync_read("ag_graph_lower: range check")) != AG_OK) return rc;
    if (host_counters[0] != -1) {
        return fail(AG_ERR_INDEX_RANGE, "ag_graph_lower: edge %u has an index outside [0, %lld)",
                    unsigned(host_counters[0]), (long long)N);
    }

    ag_graph g;
    g.device = device;
    g.N = N;
    g.E = E;
    g.ws_used = L.total;
    g.tile_edges = pick_tile_edges(E);
    g.n_tiles = n_tiles_for(E, g.tile_edges);
    g.coo_src = I(L.coo_src);
    g.coo_dst = I(L.coo_dst);
    if (E > 0) {
        err = cudaMemcpyAsync(g.coo_src, src, size_t(E) * 4, cudaMemcpyDeviceToDevice, s);
        if (err == cudaSuccess) err = cudaMemcpyAsync(g.coo_dst, dst, size_t(E) * 4, cudaMemcpyDeviceToDevice, s);
        if (err != cudaSuccess) return cuda_fail(err, "ag_graph_lower: edge copies");
    }
    const int key_bits = bit_length(N - 1);
    for (int d = 0; d < 2; ++d) {
        Direction &D = g.dir[d];
        D.rowptr = I(L.rowptr[d]);
        D.col = I(L.col[d]);
        D.order = I(L.order[d]);
        D.nz_rows = I(L.nz_rows[d]);
        D.nz_rowptr = I(L.nz_rowptr[d]);
        D.zero_rows = I(L.zero_rows[d]);
        D.tile_nz = I(L.tile_nz[d]);
        D.spans = reinterpret_cast<int4 *>(ws + L.spans[d]);
        const int32_t *key = d == 0 ? dst : src;
        const int32_t *other = d == 0 ? src : dst;

        // 2-3. stable sort of COO ordinals by owner, rowptr, col
        const int32_t *sorted = radix_sort(key, nullptr, E, key_bits, D.order, t, s);
        k_rowptr_search<<<grid_for(N + 1, 256), 256, 0, s>>>(sorted, E, N, D.rowptr);
        if (E > 0) k_gather<<<grid_for(E, 256), 256, 0, s>>>(D.order, other, E, D.col);

        // window-bucketed weight layout (see kWindowShift): the slot of an
        // ordinal is its place in the COO ordinals sorted stably by the window
        // of their CSR position
        if (E > 0) {
            int32_t *A = I(L.bucket_a[d]), *B = I(L.bucket_b[d]);
            const int wbits = bit_length((E - 1) >> kWindowShift);
            if (wbits <= 8) {
                // windows from the row pointers (the sorted keys are dead), then
                // one ranking pass: A[ordinal] = its place in the stable order
                int32_t *win = t.keys_a;
                k_window_of<<<grid_for(E, 256), 256, 0, s>>>(key, D.rowptr, D.order, E, kWindowShift, win);
                const int nblk = int((E + kRadixTile - 1) / kRadixTile);
                k_radix_hist<<<nblk, kRadixThreads, 0, s>>>(win, E, 0, nblk, t.hist);
                exclusive_scan(t.hist, t.hist, int64_t(kRadix) * nblk, t.scan, s);
                k_radix_scatter<false><<<nblk, kRadixThreads, 0, s>>>(win, nullptr, E, 0, nblk, t.hist, nullptr, A);
            } else {
                k_window_keys<<<grid_for(E, 256), 256, 0, s>>>(D.order, E, kWindowShift, A);
                radix_sort(A, nullptr, E, wbits, B, t, s);              // B[slot] = ordinal
                k_invert<<<grid_for(E, 256), 256, 0, s>>>(B, E, A);     // A[ordinal] = slot
            }
            k_gather<<<grid_for(E, 256), 256, 0, s>>>(D.order, A, E, B);  // B[pos] = slot
            D.bucket_of_coo = A;
            D.bucket_of_pos = B;
            if (staged_regroup(E)) {
                D.stage_delta = I(L.stage_delta[d]);
                k_stage_table<<<unsigned(n_stage_chunks(E)), 256, 0, s>>>(A, E, kWindowShift, int(n_windows(E)),
                                                                         D.stage_delta);
            }
        }

        // 4. tile schedule
        err = cudaMemsetAsync(counters, 0, 8 * sizeof(int), s);
        if (err != cudaSuccess) return cuda_fail(err, "cudaMemsetAsync");
        k_max_degree<<<grid_for(N, 256), 256, 0, s>>>(D.rowptr, N, counters + 1);
        k_nz_flags<<<grid_for(N, 256), 256, 0, s>>>(D.rowptr, N, t.vals_a);
        exclusive_scan(t.vals_a, t.aux, N, t.scan, s);  // aux[N] = non-empty rows
        k_nz_scatter<<<grid_for(N, 256), 256, 0, s>>>(D.rowptr, t.aux, N, E, D.nz_rows, D.nz_rowptr,
                                                      D.zero_rows);
        cudaMemcpyAsync(counters + 2, t.aux + N, sizeof(int), cudaMemcpyDeviceToDevice, s);
        if ((rc = sync_read("ag_graph_lower: rows")) != AG_OK) return rc;
        D.max_degree = host_counters[1];
        D.n_nz = host_counters[2];
        if (D.n_nz > 0) {
            k_tile_nz<<<grid_for(D.n_nz, 256), 256, 0, s>>>(D.nz_rowptr, D.n_nz, g.tile_edges, D.tile_nz);
            k_span_flags<<<grid_for(D.n_nz, 256), 256, 0, s>>>(D.nz_rowptr, D.n_nz, g.tile_edges,
                                                              t.keys_a, t.keys_b);
            exclusive_scan(t.keys_a, t.vals_a, D.n_nz, t.scan, s);  // long spans
            exclusive_scan(t.keys_b, t.vals_b, D.n_nz, t.scan, s);  // other spans
            cudaMemcpyAsync(counters + 3, t.vals_a + D.n_nz, sizeof(int), cudaMemcpyDeviceToDevice, s);
            cudaMemcpyAsync(counters + 4, t.vals_b + D.n_nz, sizeof(int), cudaMemcpyDeviceToDevice, s);
            if ((rc = sync_read("ag_graph_lower: spans")) != AG_OK) return rc;
            D.n_span_long = host_counters[3];
            D.n_span = host_counters[3] + host_counters[4];
            if (D.n_span > 0)
                k_span_scatter<<<grid_for(D.n_nz, 256), 256, 0, s>>>(D.nz_rows, D.nz_rowptr, D.n_nz,
                                                                    g.tile_edges, t.vals_a, t.vals_b,
                                                                    D.n_span_long, D.spans);
        }
    }
    // locality of the transpose order, for ag_backward's choice of walk
    if (E > 1) {
        unsigned long long *cnt = reinterpret_cast<unsigned long long *>(counters + 8);
        cudaMemsetAsync(cnt, 0, sizeof *cnt, s);
        k_sector_runs<<<grid_for(E, 256), 256, 0, s>>>(g.dir[1].order, E, cnt);
        unsigned long long host_cnt = 0;
        err = cudaMemcpyAsync(&host_cnt, cnt, sizeof host_cnt, cudaMemcpyDeviceToHost, s);
        if (err == cudaSuccess) err = cudaStreamSynchronize(s);
        if (err != cudaSuccess) return cuda_fail(err, "ag_graph_lower: locality");
        g.dw_locality = double(host_cnt) / double(E - 1);
    }
    err = cudaGetLastError();
    if (err == cudaSuccess) err = cudaStreamSynchronize(s);
    if (err != cudaSuccess) return cuda_fail(err, "ag_graph_lower");
    *out = new ag_graph(g);
    return AG_OK;
}
