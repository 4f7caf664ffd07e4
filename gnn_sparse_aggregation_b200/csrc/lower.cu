// lower.cu -- COO -> forward CSR + transpose CSR connectivity lowering.
//
// tinymesh "Weighted aggregation experiment", section "Edge order is
// explicit": connectivity is sorted by owner without detaching the weights.
// Both order maps send a CSR position to the original COO ordinal, and
// duplicate source-target pairs keep separate positions.  Section "Exact
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
//   4. the row schedule: rows sorted by decreasing degree (the same stable
//      radix sort on maxdeg - deg), rows longer than kHeavyThreshold split
//      into kChunkEdges-edge chunks.
#include <cstdio>

#include "internal.h"

namespace ag {
namespace {

constexpr int kRadixThreads = 256;
constexpr int kRadixItems = 16;  // keys per thread
constexpr int kRadixTile = kRadixThreads * kRadixItems;
constexpr int kRadixWarps = kRadixThreads / 32;
constexpr int kRadix = 256;

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

// Stable scatter of one digit pass.  Warp w of the tile owns the contiguous
// items [w * 32 * kRadixItems, (w + 1) * 32 * kRadixItems) and walks them in
// order, 32 at a time; offs holds the exclusive scan of hist.
__global__ void __launch_bounds__(kRadixThreads)
k_radix_scatter(const int32_t *__restrict__ keys_in, const int32_t *__restrict__ vals_in,
                int64_t n, int shift, int nblk, const int32_t *__restrict__ offs,
                int32_t *__restrict__ keys_out, int32_t *__restrict__ vals_out) {
    __shared__ int whist[kRadixWarps][kRadix];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < kRadixWarps * kRadix; i += kRadixThreads)
        (&whist[0][0])[i] = 0;
    __syncthreads();

    const int64_t base = int64_t(blockIdx.x) * kRadixTile + int64_t(warp) * 32 * kRadixItems;
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
    // exclusive prefix over warps, per digit: warp order = item order
    for (int d = threadIdx.x; d < kRadix; d += kRadixThreads) {
        int run = 0;
#pragma unroll
        for (int w = 0; w < kRadixWarps; ++w) {
            int t = whist[w][d];
            whist[w][d] = run;
            run += t;
        }
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kRadixItems; ++k) {
        const int64_t i = base + k * 32 + lane;
        if (i < n) {
            const int d = (uint32_t(key[k]) >> shift) & (kRadix - 1);
            const int64_t pos = int64_t(offs[int64_t(d) * nblk + blockIdx.x]) + whist[warp][d] + rank[k];
            keys_out[pos] = key[k];
            vals_out[pos] = val[k];
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

__global__ void k_gather(const int32_t *__restrict__ idx, const int32_t *__restrict__ from,
                         int64_t n, int32_t *__restrict__ out) {
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n;
         i += int64_t(gridDim.x) * blockDim.x)
        out[i] = from[idx[i]];
}

__global__ void k_max_degree(const int32_t *__restrict__ rowptr, int64_t N, int *maxdeg) {
    int m = 0;
    for (int64_t r = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; r < N;
         r += int64_t(gridDim.x) * blockDim.x)
        m = max(m, rowptr[r + 1] - rowptr[r]);
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0 && m > 0) atomicMax(maxdeg, m);
}

__global__ void k_degree_keys(const int32_t *__restrict__ rowptr, int64_t N, int maxdeg,
                              int32_t *__restrict__ keys) {
    for (int64_t r = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; r < N;
         r += int64_t(gridDim.x) * blockDim.x)
        keys[r] = maxdeg - (rowptr[r + 1] - rowptr[r]);
}

// sched is sorted by decreasing degree; count the split rows and non-empty
// rows (both are prefixes) and the chunks of every split row.
__global__ void k_sched_counts(const int32_t *__restrict__ sched, const int32_t *__restrict__ rowptr,
                               int64_t N, int32_t *__restrict__ nch, int *n_heavy, int *n_nonempty) {
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < N;
         i += int64_t(gridDim.x) * blockDim.x) {
        const int r = sched[i];
        const int deg = rowptr[r + 1] - rowptr[r];
        int next = -1;
        if (i + 1 < N) {
            const int r2 = sched[i + 1];
            next = rowptr[r2 + 1] - rowptr[r2];
        }
        nch[i] = deg > kHeavyThreshold ? (deg + kChunkEdges - 1) / kChunkEdges : 0;
        if (deg > kHeavyThreshold && next <= kHeavyThreshold) *n_heavy = int(i + 1);
        if (deg > 0 && next <= 0) *n_nonempty = int(i + 1);
    }
}

__global__ void k_rows_fill(const int32_t *__restrict__ sched, const int32_t *__restrict__ rowptr,
                            const int32_t *__restrict__ chunk_off, int64_t N, int64_t n_heavy,
                            int4 *__restrict__ rows) {
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < N;
         i += int64_t(gridDim.x) * blockDim.x) {
        const int r = sched[i];
        rows[i] = make_int4(r, rowptr[r], rowptr[r + 1], i < n_heavy ? chunk_off[i] : 0);
    }
}

// One warp per split row writes its chunk table entries.
__global__ void k_chunks_fill(const int4 *__restrict__ rows, int64_t n_heavy, int4 *__restrict__ chunks) {
    const int64_t h = (blockIdx.x * int64_t(blockDim.x) + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (h >= n_heavy) return;
    const int4 r = rows[h];
    const int nch = (r.z - r.y + kChunkEdges - 1) / kChunkEdges;
    for (int j = lane; j < nch; j += 32) {
        const int b = r.y + j * kChunkEdges;
        chunks[int64_t(r.w) + j] = make_int4(b, min(b + kChunkEdges, r.z), r.x, int(h));
    }
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
        k_radix_scatter<<<nblk, kRadixThreads, 0, s>>>(kin, vin, n, 8 * p, nblk, t.hist, kout, vout);
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
    const int key_bits = bit_length(N - 1);
    for (int d = 0; d < 2; ++d) {
        Direction &D = g.dir[d];
        D.rowptr = I(L.rowptr[d]);
        D.col = I(L.col[d]);
        D.order = I(L.order[d]);
        D.rows = reinterpret_cast<int4 *>(ws + L.rows[d]);
        D.chunks = reinterpret_cast<int4 *>(ws + L.chunks[d]);
        const int32_t *key = d == 0 ? dst : src;
        const int32_t *other = d == 0 ? src : dst;

        // 2-3. stable sort of COO ordinals by owner, rowptr, col
        const int32_t *sorted = radix_sort(key, nullptr, E, key_bits, D.order, t, s);
        k_rowptr_search<<<grid_for(N + 1, 256), 256, 0, s>>>(sorted, E, N, D.rowptr);
        if (E > 0) k_gather<<<grid_for(E, 256), 256, 0, s>>>(D.order, other, E, D.col);

        // 4. schedule: rows by decreasing degree
        cudaMemsetAsync(counters, 0, 8 * sizeof(int), s);
        k_max_degree<<<grid_for(N, 256), 256, 0, s>>>(D.rowptr, N, counters + 1);
        if ((rc = sync_read("ag_graph_lower: degrees")) != AG_OK) return rc;
        const int maxdeg = host_counters[1];
        D.max_degree = maxdeg;
        k_degree_keys<<<grid_for(N, 256), 256, 0, s>>>(D.rowptr, N, maxdeg, t.aux);
        // The radix passes ping-pong through keys_a/b and vals_a/b and read
        // their keys from aux, so the sorted row ids go to rows[] (16 bytes
        // per row, not yet written) and are then copied to keys_b, because
        // rows[] is filled from them below.
        int32_t *sched_out = reinterpret_cast<int32_t *>(D.rows);
        radix_sort(t.aux, nullptr, N, bit_length(maxdeg), sched_out, t, s);
        int32_t *sched = t.keys_b;
        cudaMemcpyAsync(sched, sched_out, size_t(N) * 4, cudaMemcpyDeviceToDevice, s);
        k_sched_counts<<<grid_for(N, 256), 256, 0, s>>>(sched, D.rowptr, N, t.vals_a,
                                                        counters + 2, counters + 3);
        exclusive_scan(t.vals_a, t.aux, N, t.scan, s);  // chunk offsets; aux[N] = total
        cudaMemcpyAsync(counters + 4, t.aux + N, sizeof(int), cudaMemcpyDeviceToDevice, s);
        if ((rc = sync_read("ag_graph_lower: schedule")) != AG_OK) return rc;
        D.n_heavy = host_counters[2];
        D.n_nonempty = host_counters[3];
        D.n_chunks = host_counters[4];
        k_rows_fill<<<grid_for(N, 256), 256, 0, s>>>(sched, D.rowptr, t.aux, N, D.n_heavy, D.rows);
        if (D.n_heavy > 0)
            k_chunks_fill<<<unsigned((D.n_heavy * 32 + 255) / 256), 256, 0, s>>>(D.rows, D.n_heavy, D.chunks);
    }
    err = cudaGetLastError();
    if (err == cudaSuccess) err = cudaStreamSynchronize(s);
    if (err != cudaSuccess) return cuda_fail(err, "ag_graph_lower");
    *out = new ag_graph(g);
    return AG_OK;
}
