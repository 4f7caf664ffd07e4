/*
 * aggraph.h -- C ABI of the fused weighted GNN aggregation library
 * (libaggraph.so, CUDA, sm_100a).
 *
 * The operation is the weighted scalar-edge aggregation of the tinymesh page
 * "Weighted aggregation experiment" (sections "Decision" and "Edge order is
 * explicit"), which is the fused form of message passing described in the
 * reading guide "PyTorch Geometric: one abstraction, the whole GNN
 * literature" (Step 3, "message_and_aggregate is one SpMM"; Step 4, SDDMM):
 *
 *   forward          Y  = A_w   X    Y[d, :]  = sum over edges e = (s -> d) of w_e * X[s, :]
 *   feature grad     dX = A_w^T dY   dX[s, :] = sum over edges e = (s -> d) of w_e * dY[d, :]
 *   weight grad      dw_e = dot(X[s_e, :], dY[d_e, :])
 *
 * A_w[d, s] = w_e, so the forward output is owned by destination rows and the
 * feature gradient by source rows.  Weights w and their gradient dw stay in
 * the caller's COO edge order on every call; the library reaches them through
 * its edge_order / transpose_order maps.  Duplicate (s, d) pairs are separate
 * edges.  No [E, H] per-edge message tensor is ever formed, and no kernel uses
 * floating-point atomics, so every output is bitwise reproducible run to run.
 *
 * Conventions shared by every entry point
 *   - Indices are int32; 1 <= N < 2^31 and 0 <= E < 2^31.
 *   - Feature matrices are dense, row-major, contiguous [N, H] of the given
 *     dtype (AG_F32: float; AG_BF16: bfloat16 stored as uint16).  w and dw are
 *     float [E].  Arithmetic is fp32 with fp32 accumulation; bf16 outputs are
 *     rounded once (round to nearest even) from the fp32 result.
 *   - All array pointers are DEVICE pointers on the graph's device unless a
 *     name ends in _host.  The caller owns every buffer; the library never
 *     allocates device memory.  Pointers must stay valid until the work on
 *     `stream` has finished.
 *   - Per-call functions run on the calling thread's current device, which
 *     must be the device the graph was lowered on (AG_ERR_DEVICE otherwise).
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  Per-call functions only enqueue work and return; results are
 *     ready when the stream reaches that point.
 *   - Outputs are fully overwritten (never accumulated into).
 *   - Every int-returning function returns an ag_status; on failure nothing
 *     is launched and ag_last_error() describes the reason.
 */
#ifndef AGGRAPH_H
#define AGGRAPH_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define AG_API __attribute__((visibility("default")))
#else
#define AG_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct ag_graph ag_graph; /* opaque lowered topology; fixed once built */

typedef enum ag_dtype {
    AG_F32 = 0,  /* float32 features */
    AG_BF16 = 1  /* bfloat16 features (fp32 accumulation) */
} ag_dtype;

typedef enum ag_status {
    AG_OK = 0,
    AG_ERR_INVALID_ARG = 1, /* null handle or pointer, unknown enum value */
    AG_ERR_SHAPE = 2,       /* N, E or H outside the supported range */
    AG_ERR_DTYPE = 3,       /* dtype is not AG_F32 or AG_BF16 */
    AG_ERR_DEVICE = 4,      /* pointer is not device memory of the graph's device */
    AG_ERR_INDEX_RANGE = 5, /* some src/dst index lies outside [0, N) */
    AG_ERR_CUDA = 6,        /* a CUDA runtime call or launch failed */
    AG_ERR_WORKSPACE = 7    /* workspace/scratch/staging too small or misaligned */
} ag_status;

/* Schedule facts of a lowered graph, for inspection and tests. */
typedef struct ag_graph_stats {
    int64_t N, E;
    int32_t device;             /* CUDA ordinal the graph was lowered on */
    int32_t tile_edges;         /* per-call kernels walk the CSR in tiles of this many positions */
    int64_t tiles;              /* ceil(E / tile_edges) */
    int64_t max_degree_f;       /* largest in-degree (forward CSR row length) */
    int64_t max_degree_t;       /* largest out-degree (transpose CSR row length) */
    int64_t nonempty_rows_f;    /* rows with at least one in-edge */
    int64_t spanning_rows_f;    /* rows cut by a tile boundary (summed from per-tile partials) */
    int64_t long_spanning_rows_f; /* of those, rows cut into more than 9 tiles */
    int64_t nonempty_rows_t, spanning_rows_t, long_spanning_rows_t; /* same, transpose CSR */
    size_t workspace_bytes_used;
    double dw_locality;         /* share of transpose-CSR neighbours whose COO ordinals share a 32-byte sector */
} ag_graph_stats;

/*
 * Upper bound on the device workspace ag_graph_lower needs for N nodes and E
 * edges (256-byte aligned sub-arrays included).  Pure host arithmetic; no
 * CUDA call.  Returns 0 if N or E is out of range.  The bound is O(N + E):
 * the two CSRs (2E + 2(N + 1) ints, section "Edge order is explicit"), the
 * two order maps (2E ints), the row schedules, and sort temporaries.
 */
AG_API size_t ag_graph_workspace_bytes(int64_t N, int64_t E);

/*
 * Connectivity lowering ("Edge order is explicit"; witness in "Exact
 * witness": edges 0->2, 1->2, 0->1 give edge_order = (2, 0, 1)).
 *
 *   src, dst   device int32 [E], the COO edge list (edge e runs src[e] -> dst[e]);
 *              may be NULL when E == 0.  Read only; they are not retained.
 *   N, E       node and edge counts.
 *   workspace  device buffer of at least ag_graph_workspace_bytes(N, E)
 *              bytes, 256-byte aligned.  The graph lives in it: it must
 *              outlive the handle and must not be written by the caller.
 *   stream     stream for the lowering work.  The call synchronizes this
 *              stream before returning (it reads back validation flags and
 *              schedule sizes).
 *   out        receives a new handle (host memory, freed by ag_graph_free).
 *
 * Builds, bit-exactly and deterministically:
 *   rowptr_f[N+1], col_f[E] = src[edge_order], edge_order[E]     (by destination)
 *   rowptr_t[N+1], col_t[E] = dst[transpose_order], transpose_order[E] (by source)
 * where each order map sends a CSR position to its COO ordinal, sorted by the
 * owner key with ties in ascending COO ordinal (a stable sort), plus what
 * the per-call kernels walk: the edge-balanced tile schedule of each CSR
 * (rows with edges, the row holding each tile's first position, the rows cut
 * by tile boundaries) and the tables that regroup per-edge arrays into
 * windows of 2^20 consecutive CSR positions.
 *
 * Errors: AG_ERR_SHAPE for N < 1, E < 0, N or E >= 2^31; AG_ERR_INVALID_ARG
 * for null out/workspace or null src/dst with E > 0; AG_ERR_WORKSPACE if the
 * workspace is too small or not 256-byte aligned; AG_ERR_DEVICE if a pointer
 * is not device memory; AG_ERR_INDEX_RANGE if any index is outside [0, N)
 * (checked on the device; *out is left unchanged); AG_ERR_CUDA otherwise.
 */
AG_API int ag_graph_lower(const int32_t *src, const int32_t *dst, int64_t N, int64_t E,
                   void *workspace, size_t workspace_bytes, void *stream, ag_graph **out);

/* Device views of the lowered arrays (inside the workspace; any out pointer may be NULL). */
AG_API int ag_graph_arrays(const ag_graph *g, const int32_t **rowptr_f, const int32_t **col_f,
                    const int32_t **edge_order, const int32_t **rowptr_t,
                    const int32_t **col_t, const int32_t **transpose_order);

/* Fills *out with the graph's schedule facts.  AG_ERR_INVALID_ARG on NULL. */
AG_API int ag_graph_get_stats(const ag_graph *g, ag_graph_stats *out);

/*
 * Device scratch, in bytes, that the per-call functions need for feature
 * width H: two fp32 partial rows per tile for the rows that a tile boundary
 * cuts (2 x tiles x H x 4 bytes, 0 when no row is cut), plus two float [E]
 * buffers that hold the weights and the weight gradient regrouped by windows
 * of 2^20 consecutive CSR positions (the weights stay in COO order in the
 * caller's arrays; the regrouping keeps each tile's weight lookups inside
 * one window), plus one float [N] of reciprocal in-degrees for the mean.
 * O(E / tile_edges * H + E + N), never E x H.
 */
AG_API size_t ag_spmm_scratch_bytes(const ag_graph *g, int64_t H);

/*
 * Forward aggregation Y = A_w X ("Decision": the forward pass walks the CSR
 * whose rows belong to destinations; reading guide Step 3: the gather / message /
 * scatter triple reduces to one SpMM whenever each message is just the
 * source's feature row times a per-edge number, which is what PyG's GraphConv
 * sends when given edge weights, section "Reference contract").
 *
 *   w        device float [E], COO order (may be NULL when E == 0)
 *   X        device [N, H] of dtype
 *   Y        device [N, H] of dtype, fully written; rows without in-edges are 0
 *   scratch  device buffer of ag_spmm_scratch_bytes(g, H) bytes (NULL if 0),
 *            256-byte aligned; its contents are scratch only
 * Rows cut by tile boundaries are summed in fixed tile order, so results are
 * bitwise reproducible.  Errors: AG_ERR_INVALID_ARG, AG_ERR_SHAPE (H < 1 or N*H too
 * large), AG_ERR_DTYPE, AG_ERR_DEVICE, AG_ERR_WORKSPACE, AG_ERR_CUDA.
 */
AG_API int ag_spmm_fwd(const ag_graph *g, const float *w, const void *X, void *Y, int64_t H,
                int dtype, void *scratch, size_t scratch_bytes, void *stream);

/*
 * Feature gradient dX = A_w^T dY ("Decision": the same kind of CSR walk,
 * here over the source-owned transpose CSR and transpose_order).
 * Arguments and errors as ag_spmm_fwd, with dY in place of X and dX in place
 * of Y; rows without out-edges are 0.
 */
AG_API int ag_spmm_dx(const ag_graph *g, const float *w, const void *dY, void *dX, int64_t H,
               int dtype, void *scratch, size_t scratch_bytes, void *stream);

/*
 * Weight gradient dw_e = dot(X[src_e], dY[dst_e]) ("Edge order is explicit";
 * "Exact witness": exactly one value per edge, a sum over the H feature
 * positions;
 * reading guide Step 4: SDDMM, a dense product evaluated only at the
 * adjacency's nonzeros).
 *
 *   X, dY    device [N, H] of dtype
 *   dw       device float [E], written in COO order (may be NULL when E == 0)
 *   scratch  device buffer of ag_spmm_scratch_bytes(g, H) bytes (see there)
 * Every edge's value is computed independently (duplicates get equal values).
 * Errors as ag_spmm_fwd.
 */
AG_API int ag_sddmm_dw(const ag_graph *g, const void *X, const void *dY, float *dw, int64_t H,
                int dtype, void *scratch, size_t scratch_bytes, void *stream);

/*
 * Feature gradient and weight gradient in one pass over the transpose CSR:
 * dX = A_w^T dY and dw_e = dot(X[src_e], dY[dst_e]).  Both follow the
 * definitions of "Edge order is explicit" (tinymesh "Weighted aggregation
 * experiment"); the fusion is this library's: every dY row gathered for an
 * edge feeds both the dX row of the edge's source and the edge's dot
 * product, so dY is gathered once for both gradients instead of twice.
 * Results are bitwise identical to ag_spmm_dx followed by ag_sddmm_dw.
 *
 *   w        device float [E], COO order
 *   X, dY    device [N, H] of dtype
 *   dX       device [N, H] of dtype, fully written
 *   dw       device float [E], COO order
 *   scratch  as ag_spmm_dx (ag_spmm_scratch_bytes(g, H) bytes)
 * Errors as ag_spmm_fwd.
 */
AG_API int ag_backward(const ag_graph *g, const float *w, const void *X, const void *dY, void *dX, float *dw,
                       int64_t H, int dtype, void *scratch, size_t scratch_bytes, void *stream);

/*
 * One training step in one call: the forward pass Y = A_w X and the fused
 * backward pass dX = A_w^T dY, dw_e = dot(X[src_e], dY[dst_e]) (the
 * definitions of "Edge order is explicit"; the packaging is this library's).
 * Y, dX and dw are bitwise identical to ag_spmm_fwd followed by ag_backward.
 * The two passes depend only on the inputs, so the call overlaps them: the
 * backward walk runs first on `stream` while a helper stream of the device
 * (created on first use, kept until exit) regroups the forward weights; the
 * backward pass's rows cut by tiles and its dw regrouping then run on the
 * helper stream while the forward walk runs on `stream`.  `stream` is
 * ordered after all of it when the call's work is done.
 *
 *   w, X, dY, Y, dX, dw  as ag_spmm_fwd and ag_backward (device pointers)
 *   scratch  device buffer of ag_step_scratch_bytes(g, H) bytes, 256-byte
 *            aligned: ag_spmm_scratch_bytes(g, H) plus a second set of
 *            partial rows and a second float [E] for the forward pass
 * Errors as ag_backward; AG_ERR_CUDA also when an event cannot be created.
 */
AG_API size_t ag_step_scratch_bytes(const ag_graph *g, int64_t H);
AG_API int ag_step(const ag_graph *g, const float *w, const void *X, const void *dY, void *Y, void *dX, float *dw,
                   int64_t H, int dtype, void *scratch, size_t scratch_bytes, void *stream);

/*
 * Mean aggregation (PyTorch Geometric reading guide, Step 3: the sum and mean
 * reductions of spmm; "Done when": sum and mean are the reductions that keep
 * the semiring structure):
 *   Y[r] = (1 / cnt(r)) * sum over edges e into r of w_e X[src_e],
 * cnt(r) = number of edges into r (duplicates counted), Y[r] = 0 when
 * cnt(r) = 0.  The walk is that of ag_spmm_fwd; on the widths its shared-
 * memory ring serves (16-byte vectors, at most two per lane, one pass over
 * the width) every finished fp32 row sum is multiplied by the fp32
 * reciprocal of cnt(r), on the others each weight is divided by cnt(dst_e)
 * (IEEE division) while the weights are regrouped.
 *
 *   w        device float [E], COO order, or NULL for unit weights
 *   other arguments and errors as ag_spmm_fwd (same scratch size)
 */
AG_API int ag_mean_fwd(const ag_graph *g, const float *w, const void *X, void *Y, int64_t H, int dtype,
                       void *scratch, size_t scratch_bytes, void *stream);

/*
 * Gradients of ag_mean_fwd for the upstream gradient dY, in one transpose
 * walk like ag_backward (each edge's weight and dot product scaled by the
 * fp32 reciprocal of cnt(dst_e) inside the walk on the ring widths, divided
 * by cnt(dst_e) while the per-edge arrays are regrouped on the others):
 *   dX[s] = sum over edges e out of s of (w_e / cnt(dst_e)) dY[dst_e]
 *   dw_e  = dot(X[src_e], dY[dst_e]) / cnt(dst_e)
 *
 *   w        device float [E] (COO order) or NULL for unit weights
 *   dw       device float [E] (COO order), or NULL: no weight gradient
 *            (then X is not read and may be any non-NULL device pointer)
 *   other arguments and errors as ag_backward
 */
AG_API int ag_mean_backward(const ag_graph *g, const float *w, const void *X, const void *dY, void *dX,
                            float *dw, int64_t H, int dtype, void *scratch, size_t scratch_bytes, void *stream);

/*
 * GCN-normalised edge weights, D^-1/2 A_w D^-1/2 (PyTorch Geometric reading
 * guide, "Done when": GCNConv.forward runs gcn_norm to build the normalised
 * adjacency, then one SpMM):
 *   deg(i)    = sum of w_e over the edges into i (w = NULL: their number)
 *   w_norm[e] = deg(src_e)^-1/2 * w_e * deg(dst_e)^-1/2, COO order,
 * with deg^-1/2 = 0 where deg <= 0.  Self-loops are whatever the edge list
 * holds (add them to the COO before lowering for the usual GCN operator).
 * The weighted degree is a segmented fp32 sum of the weights over each
 * forward-CSR row, in an order fixed by the CSR alone (deterministic);
 * deg^-1/2 is 1 / sqrtf(deg), both IEEE-rounded.  Feed w_norm to
 * ag_spmm_fwd / ag_backward.
 *
 *   w        device float [E] (COO order) or NULL
 *   w_norm   device float [E], written (may be NULL when E == 0)
 *   scratch  device buffer, 256-byte aligned, of ag_gcn_norm_scratch_bytes(g)
 *            bytes (degrees, row sums, per-tile partial sums and the weights
 *            regrouped into the forward CSR's windows)
 * Errors: AG_ERR_INVALID_ARG (null graph or w_norm), AG_ERR_WORKSPACE
 * (scratch too small or misaligned), AG_ERR_DEVICE, AG_ERR_CUDA.
 */
AG_API size_t ag_gcn_norm_scratch_bytes(const ag_graph *g);
AG_API int ag_gcn_norm(const ag_graph *g, const float *w, float *w_norm, void *scratch, size_t scratch_bytes,
                       void *stream);

/*
 * Edge-softmax attention over the forward adjacency (PyTorch Geometric
 * reading guide, Step 4: a per-edge score from both endpoints' features,
 * a softmax over each destination row, then the SpMM with the normalised
 * scores -- SpMM and SDDMM together):
 *   s_e     = scale * dot(Q[dst_e], K[src_e])
 *   alpha_e = exp(s_e - m_r) / sum over edges e' into r of exp(s_e' - m_r),
 *             r = dst_e, m_r = max of s over r's edges
 *   Y[r]    = sum over edges e into r of alpha_e V[src_e]   (0 for rows without edges)
 * Scores are the fp32 dot products of ag_sddmm_dw; the row maximum and the
 * sum of exponentials are reduced in fp32 in a fixed order per row; alpha
 * is expf(s - m) / l; Y is ag_spmm_fwd with weights alpha.
 *
 *   Q, K, V  device [N, H] of dtype (Q gathered by destination, K and V by source)
 *   scale    finite fp32 factor of the scores (1/sqrt(H) for scaled dot-product attention)
 *   Y        device [N, H] of dtype, fully written
 *   alpha    device float [E], written in COO order (kept for the backward pass)
 *   scratch  device buffer, 256-byte aligned, of ag_attn_scratch_bytes(g, H) bytes
 * Errors as ag_spmm_fwd; AG_ERR_INVALID_ARG also for a non-finite scale.
 */
AG_API size_t ag_attn_scratch_bytes(const ag_graph *g, int64_t H);
AG_API int ag_attn_fwd(const ag_graph *g, const void *Q, const void *K, const void *V, float scale, void *Y,
                       float *alpha, int64_t H, int dtype, void *scratch, size_t scratch_bytes, void *stream);

/*
 * Gradients of ag_attn_fwd for the upstream gradient dY, by the chain rule
 * through the row softmax:
 *   dalpha_e = dot(dY[dst_e], V[src_e]),  c_r = sum over edges e into r of alpha_e dalpha_e
 *   ds_e     = scale * alpha_e * (dalpha_e - c_{dst_e})
 *   dQ[r]    = sum over edges e into r of ds_e K[src_e]        (ag_spmm_fwd with weights ds)
 *   dK[s]    = sum over edges e out of s of ds_e Q[dst_e]      (ag_spmm_dx with weights ds)
 *   dV[s]    = sum over edges e out of s of alpha_e dY[dst_e]  (with dalpha: ag_backward with
 *                                                               weights alpha and features V)
 *
 *   alpha    the alpha written by ag_attn_fwd for the same Q, K, scale
 *   dQ, dK, dV  device [N, H] of dtype, fully written
 *   other arguments and errors as ag_attn_fwd (same scratch size)
 */
AG_API int ag_attn_backward(const ag_graph *g, const void *Q, const void *K, const void *V, float scale,
                            const float *alpha, const void *dY, void *dQ, void *dK, void *dV, int64_t H,
                            int dtype, void *scratch, size_t scratch_bytes, void *stream);

/*
 * One whole aggregation step from HOST buffers: copies w, X and dY to the
 * device staging area, runs the forward pass and the fused backward pass
 * (ag_backward), and copies Y, dX and dw back.  The copy of dY and the copies
 * out run on two helper streams of the graph's device (created on first use,
 * kept until exit) and are joined to `stream` with events, so that dY comes
 * in while the forward pass runs and Y goes out while dY comes in; `stream`
 * is ordered after every one of them.
 *
 *   *_host   host buffers (page-locked memory is needed for the copies to be
 *            asynchronous); w_host/dw_host may be NULL when E == 0
 *   staging  device buffer of ag_step_staging_bytes(g, H, dtype) bytes,
 *            256-byte aligned; holds the device copies and the SpMM scratch
 * The host output buffers are valid once `stream` has been synchronized.
 */
AG_API size_t ag_step_staging_bytes(const ag_graph *g, int64_t H, int dtype);
AG_API int ag_step_host(const ag_graph *g, const float *w_host, const void *X_host,
                 const void *dY_host, void *Y_host, void *dX_host, float *dw_host,
                 int64_t H, int dtype, void *staging, size_t staging_bytes, void *stream);

/*
 * ag_step_host for a sequence of steps (an interface addition of this
 * library): the same arguments, copies and results, but this call's copies
 * in (w, X, dY, all on the helper stream) are ordered only after the previous
 * step's fused backward pass on the same staging buffer, not after that
 * step's copies out.  Back-to-back steps on one staging buffer therefore
 * bring the next step's inputs in while the previous step's dX and dw go out.
 * `stream` is still ordered after every copy of this call.  Steps that
 * alternate between two staging buffers, each with its own `stream` (and
 * its own host outputs), overlap further: a step's copies in wait only for
 * the backward pass two steps back, and its compute only for its inputs.
 *
 * The staging buffer belongs to the steps between calls: no other work may
 * read or write it.  The first call on a buffer (or on one of more than 16
 * buffers in use) is ordered after everything on `stream`, like ag_step_host;
 * an ag_step_host call on the same buffer keeps the order for the next
 * pipelined call.  The host input buffers are read until `stream` has been
 * synchronized after the call.
 *
 * Errors: those of ag_step_host (null buffers, staging too small or not
 * 256-byte aligned, staging not on the graph's device, CUDA failures);
 * AG_ERR_CUDA also when the ordering event cannot be created.
 */
AG_API int ag_step_host_pipelined(const ag_graph *g, const float *w_host, const void *X_host,
                 const void *dY_host, void *Y_host, void *dX_host, float *dw_host,
                 int64_t H, int dtype, void *staging, size_t staging_bytes, void *stream);

/*
 * Forward aggregation without caller scratch (no counterpart on the pages:
 * an interface addition of this library).
 *
 * Same result as ag_spmm_fwd, for callers that cannot allocate device memory
 * when they call -- for example code that runs while a framework owns the
 * allocator (allocating behind its back can fail or fragment its pool),
 * latency-critical paths where cudaMalloc and cudaFree may synchronize the
 * device, or plug-in hooks that are handed only their input and output
 * buffers.  The partial rows of rows cut by tile boundaries go to a fixed
 * device array built into the library instead of caller scratch.
 *
 *   - The built-in array holds ag_spmm_static_scratch_capacity() bytes
 *     (32 MiB) on every GPU that loads the library, until the process exits.
 *     A graph that needs more (the partial rows and the regrouped weights of
 *     ag_spmm_scratch_bytes) is rejected with AG_ERR_WORKSPACE; nothing is
 *     launched.
 *   - The call allocates nothing (no cudaMalloc, cudaFree or allocating
 *     library routine).  Its first call on a device looks up the array's
 *     device address there (cudaGetSymbolAddress) and keeps it for the life
 *     of the process; make that first call before any stream capture, and do
 *     not reset the device (cudaDeviceReset) while the library is loaded,
 *     since the kept address would then be stale.  Call it with the graph's
 *     device current (AG_ERR_DEVICE otherwise).
 *   - All calls share the one array: calls whose work overlaps on the GPU
 *     (different streams, different host threads) race and must be ordered
 *     by the caller.  The array keeps the previous call's contents; no part
 *     of it has to start at zero, because everything a call reads from it is
 *     written earlier in the same call.
 * Arguments and other errors as ag_spmm_fwd.
 */
AG_API int ag_spmm_fwd_static_scratch(const ag_graph *g, const float *w, const void *X, void *Y, int64_t H,
                                      int dtype, void *stream);
AG_API size_t ag_spmm_static_scratch_capacity(void);

/* Releases the host handle (the caller frees the workspace). NULL is a no-op. */
AG_API void ag_graph_free(ag_graph *g);

/* Message for the last failure on the calling thread ("" if none). */
AG_API const char *ag_last_error(void);

/* Static name of a status code. */
AG_API const char *ag_status_string(int status);

/* Version of this ABI (major * 100 + minor). */
AG_API int ag_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* AGGRAPH_H */
