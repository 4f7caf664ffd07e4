/*
 * oracle.c -- plain, slow, fp64 CPU oracle for weighted GNN aggregation.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or helper
 * with the CUDA library; it is a single-threaded host loop written to be
 * checked against the pages by eye.
 *
 * What it computes (tinymesh "Weighted aggregation experiment", sections
 * "Decision" and "Edge order is explicit"; PyTorch Geometric reading guide
 * "PyTorch Geometric: one abstraction, the whole GNN literature", Step 2
 * "the COO path" and Step 3 "the fused path"):
 *
 *   forward   Y  = A_w  X     Y[dst_e, :]  += w_e * X[src_e, :]
 *   feature   dX = A_w^T dY   dX[src_e, :] += w_e * dY[dst_e, :]
 *   weight    dw_e = dot(X[src_e, :], dY[dst_e, :])
 *
 * with A_w[dst, src] = w_e, so the forward output is owned by destinations.
 * The loops walk the raw COO edge list once, in edge order, with one fp64
 * accumulator per output element and no [E, H] message temporary (the COO
 * illustration of Step 2 with its temporary removed: the reading guide says
 * the fused path is the same result without it).
 *
 * Inputs (weights, features) are taken as fp32 arrays.  Both fp32 and bf16
 * feature values convert to fp64 exactly, so every product and sum below is
 * done in fp64 on the exact input values.
 *
 * Lowering ("Edge order is explicit"): edge_order[p] is the COO index of the
 * edge stored at slot p of the forward CSR (slots grouped by destination);
 * transpose_order[p] is the same for the transpose CSR (grouped by source).
 * Repeated (source, target) pairs occupy one slot each.  Within one owner row the order is ascending COO ordinal (a
 * stable sort on the owner key alone); this is the reading that reproduces the
 * printed witness edge_order = (2, 0, 1) of section "Exact witness".  The
 * stable sort is written out as a counting sort.
 *
 * Every function is pinned by tests against values that do not come from
 * this file: the hand-derived witness, dense matrix products, the adjoint
 * identity, finite differences and library stable sorts.
 *
 * Indices are int32: N and E must both be below 2^31.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

#define ORACLE_OK 0
#define ORACLE_BAD_SIZE 1
#define ORACLE_BAD_INDEX 2
#define ORACLE_NO_MEMORY 3

static int sizes_ok(int64_t N, int64_t E)
{
    return N >= 1 && N < ((int64_t)1 << 31) && E >= 0 && E < ((int64_t)1 << 31);
}

static int indices_ok(int64_t N, int64_t E, const int32_t *src, const int32_t *dst)
{
    for (int64_t e = 0; e < E; ++e) {
        if (src[e] < 0 || src[e] >= N || dst[e] < 0 || dst[e] >= N)
            return 0;
    }
    return 1;
}

/*
 * Stable counting sort of the COO ordinals 0..E-1 by key[e] in [0, N).
 * rowptr[r] is the first position of owner r, rowptr[N] = E;
 * order[p] is the COO ordinal found at CSR position p.
 */
static int stable_sort_by_owner(int64_t N, int64_t E, const int32_t *key,
                                int32_t *rowptr, int32_t *order)
{
    int64_t *next = (int64_t *)malloc((size_t)N * sizeof(int64_t));
    if (!next)
        return ORACLE_NO_MEMORY;
    for (int64_t r = 0; r <= N; ++r)
        rowptr[r] = 0;
    /* in-degree of every owner */
    for (int64_t e = 0; e < E; ++e)
        rowptr[key[e] + 1] += 1;
    /* exclusive prefix sum gives the first position of every owner */
    for (int64_t r = 0; r < N; ++r)
        rowptr[r + 1] += rowptr[r];
    for (int64_t r = 0; r < N; ++r)
        next[r] = rowptr[r];
    /* walking the edges in COO order keeps equal keys in COO order */
    for (int64_t e = 0; e < E; ++e) {
        int64_t p = next[key[e]]++;
        order[p] = (int32_t)e;
    }
    free(next);
    return ORACLE_OK;
}

/*
 * Forward CSR (owned by destination) and transpose CSR (owned by source):
 *   rowptr_f[N+1], col_f[E] = src[edge_order], edge_order[E]
 *   rowptr_t[N+1], col_t[E] = dst[transpose_order], transpose_order[E]
 */
int oracle_lower(int64_t N, int64_t E, const int32_t *src, const int32_t *dst,
                 int32_t *rowptr_f, int32_t *col_f, int32_t *edge_order,
                 int32_t *rowptr_t, int32_t *col_t, int32_t *transpose_order)
{
    if (!sizes_ok(N, E))
        return ORACLE_BAD_SIZE;
    if (!indices_ok(N, E, src, dst))
        return ORACLE_BAD_INDEX;
    int rc = stable_sort_by_owner(N, E, dst, rowptr_f, edge_order);
    if (rc)
        return rc;
    rc = stable_sort_by_owner(N, E, src, rowptr_t, transpose_order);
    if (rc)
        return rc;
    for (int64_t p = 0; p < E; ++p) {
        col_f[p] = src[edge_order[p]];
        col_t[p] = dst[transpose_order[p]];
    }
    return ORACLE_OK;
}

/*
 * Y[dst_e, h] = sum over edges e of w_e * X[src_e, h]   (Y is [N, H]).
 * absb (may be NULL) receives sum over the same edges of |w_e * X[src_e, h]|,
 * the scale used by the tolerance of the comparison.
 */
int oracle_fwd(int64_t N, int64_t E, int64_t H, const int32_t *src, const int32_t *dst,
               const float *w, const float *X, double *Y, double *absb)
{
    if (!sizes_ok(N, E) || H < 1)
        return ORACLE_BAD_SIZE;
    if (!indices_ok(N, E, src, dst))
        return ORACLE_BAD_INDEX;
    memset(Y, 0, (size_t)(N * H) * sizeof(double));
    if (absb)
        memset(absb, 0, (size_t)(N * H) * sizeof(double));
    for (int64_t e = 0; e < E; ++e) {
        double we = (double)w[e];
        const float *xs = X + (int64_t)src[e] * H;
        double *yd = Y + (int64_t)dst[e] * H;
        for (int64_t h = 0; h < H; ++h)
            yd[h] += we * (double)xs[h];
        if (absb) {
            double *bd = absb + (int64_t)dst[e] * H;
            for (int64_t h = 0; h < H; ++h)
                bd[h] += fabs(we * (double)xs[h]);
        }
    }
    return ORACLE_OK;
}

/* dX[src_e, h] = sum over edges e of w_e * dY[dst_e, h]   (dX is [N, H]). */
int oracle_dx(int64_t N, int64_t E, int64_t H, const int32_t *src, const int32_t *dst,
              const float *w, const float *dY, double *dX, double *absb)
{
    if (!sizes_ok(N, E) || H < 1)
        return ORACLE_BAD_SIZE;
    if (!indices_ok(N, E, src, dst))
        return ORACLE_BAD_INDEX;
    memset(dX, 0, (size_t)(N * H) * sizeof(double));
    if (absb)
        memset(absb, 0, (size_t)(N * H) * sizeof(double));
    for (int64_t e = 0; e < E; ++e) {
        double we = (double)w[e];
        const float *gd = dY + (int64_t)dst[e] * H;
        double *xs = dX + (int64_t)src[e] * H;
        for (int64_t h = 0; h < H; ++h)
            xs[h] += we * (double)gd[h];
        if (absb) {
            double *bs = absb + (int64_t)src[e] * H;
            for (int64_t h = 0; h < H; ++h)
                bs[h] += fabs(we * (double)gd[h]);
        }
    }
    return ORACLE_OK;
}

/*
 * dw_e = sum over h (ascending) of X[src_e, h] * dY[dst_e, h], written at
 * COO position e; absb_e = sum over h of |X[src_e, h] * dY[dst_e, h]|.
 */
int oracle_dw(int64_t N, int64_t E, int64_t H, const int32_t *src, const int32_t *dst,
              const float *X, const float *dY, double *dw, double *absb)
{
    if (!sizes_ok(N, E) || H < 1)
        return ORACLE_BAD_SIZE;
    if (!indices_ok(N, E, src, dst))
        return ORACLE_BAD_INDEX;
    for (int64_t e = 0; e < E; ++e) {
        const float *xs = X + (int64_t)src[e] * H;
        const float *gd = dY + (int64_t)dst[e] * H;
        double acc = 0.0, acc_abs = 0.0;
        for (int64_t h = 0; h < H; ++h) {
            double t = (double)xs[h] * (double)gd[h];
            acc += t;
            acc_abs += fabs(t);
        }
        dw[e] = acc;
        if (absb)
            absb[e] = acc_abs;
    }
    return ORACLE_OK;
}

/*
 * Sampled forms for graphs too large to evaluate whole: the same COO edge
 * loop, restricted to the output rows (or edges) listed in sel[0..nsel).
 * Row i of out / absb corresponds to row sel[i]; sel must not repeat a row.
 * by_source = 0 samples the forward output (rows are destinations, the loop
 * adds w_e * feat[src_e]); by_source = 1 samples the feature gradient (rows
 * are sources, the loop adds w_e * feat[dst_e]).
 */
int oracle_spmm_rows(int64_t N, int64_t E, int64_t H, const int32_t *src,
                     const int32_t *dst, const float *w, const float *feat,
                     int by_source, int64_t nsel, const int32_t *sel,
                     double *out, double *absb)
{
    if (!sizes_ok(N, E) || H < 1 || nsel < 0)
        return ORACLE_BAD_SIZE;
    if (!indices_ok(N, E, src, dst))
        return ORACLE_BAD_INDEX;
    int64_t *slot = (int64_t *)malloc((size_t)N * sizeof(int64_t));
    if (!slot)
        return ORACLE_NO_MEMORY;
    for (int64_t r = 0; r < N; ++r)
        slot[r] = -1;
    for (int64_t i = 0; i < nsel; ++i) {
        if (sel[i] < 0 || sel[i] >= N || slot[sel[i]] >= 0) {
            free(slot);
            return ORACLE_BAD_INDEX;
        }
        slot[sel[i]] = i;
    }
    memset(out, 0, (size_t)(nsel * H) * sizeof(double));
    if (absb)
        memset(absb, 0, (size_t)(nsel * H) * sizeof(double));
    for (int64_t e = 0; e < E; ++e) {
        int32_t owner = by_source ? src[e] : dst[e];
        int32_t other = by_source ? dst[e] : src[e];
        int64_t i = slot[owner];
        if (i < 0)
            continue;
        double we = (double)w[e];
        const float *f = feat + (int64_t)other * H;
        for (int64_t h = 0; h < H; ++h) {
            out[i * H + h] += we * (double)f[h];
            if (absb)
                absb[i * H + h] += fabs(we * (double)f[h]);
        }
    }
    free(slot);
    return ORACLE_OK;
}

/* dw for the listed COO ordinals only: out[i] = dw_{sel[i]}. */
int oracle_dw_edges(int64_t N, int64_t E, int64_t H, const int32_t *src,
                    const int32_t *dst, const float *X, const float *dY,
                    int64_t nsel, const int64_t *sel, double *out, double *absb)
{
    if (!sizes_ok(N, E) || H < 1 || nsel < 0)
        return ORACLE_BAD_SIZE;
    for (int64_t i = 0; i < nsel; ++i) {
        int64_t e = sel[i];
        if (e < 0 || e >= E)
            return ORACLE_BAD_INDEX;
        if (src[e] < 0 || src[e] >= N || dst[e] < 0 || dst[e] >= N)
            return ORACLE_BAD_INDEX;
        const float *xs = X + (int64_t)src[e] * H;
        const float *gd = dY + (int64_t)dst[e] * H;
        double acc = 0.0, acc_abs = 0.0;
        for (int64_t h = 0; h < H; ++h) {
            double t = (double)xs[h] * (double)gd[h];
            acc += t;
            acc_abs += fabs(t);
        }
        out[i] = acc;
        if (absb)
            absb[i] = acc_abs;
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------
 * Further aggregators over the same adjacency (PyTorch Geometric reading
 * guide: Step 3 "the fused path" for the degree-normalised GCN weights and
 * the sum-or-mean reductions of spmm, "Done when" on reduce='max'; Step 4
 * "SDDMM: the second primitive, forced by attention" for the edge softmax).
 * ------------------------------------------------------------------------ */

/* number of edges into every destination; NULL when out of memory */
static double *in_counts(int64_t N, int64_t E, const int32_t *dst)
{
    double *cnt = (double *)calloc((size_t)N, sizeof(double));
    if (!cnt)
        return NULL;
    for (int64_t e = 0; e < E; ++e)
        cnt[dst[e]] += 1.0;
    return cnt;
}

/*
 * Mean aggregation: Y[r, h] = (sum over edges e into r of w_e X[src_e, h]) / cnt(r),
 * cnt(r) = number of edges into r (duplicates counted); rows with no edge are 0.
 * absb receives the same sums of |w_e X[src_e, h]| / cnt(r).
 */
int oracle_mean_fwd(int64_t N, int64_t E, int64_t H, const int32_t *src, const int32_t *dst,
                    const float *w, const float *X, double *Y, double *absb)
{
    int rc = oracle_fwd(N, E, H, src, dst, w, X, Y, absb);
    if (rc)
        return rc;
    double *cnt = in_counts(N, E, dst);
    if (!cnt)
        return ORACLE_NO_MEMORY;
    for (int64_t r = 0; r < N; ++r) {
        if (cnt[r] == 0.0)
            continue;
        for (int64_t h = 0; h < H; ++h) {
            Y[r * H + h] /= cnt[r];
            if (absb)
                absb[r * H + h] /= cnt[r];
        }
    }
    free(cnt);
    return ORACLE_OK;
}

/*
 * Gradients of the mean aggregation for an upstream gradient dY:
 *   dX[src_e, h] += (w_e / cnt(dst_e)) dY[dst_e, h]
 *   dw_e = dot(X[src_e], dY[dst_e]) / cnt(dst_e)
 */
int oracle_mean_dx(int64_t N, int64_t E, int64_t H, const int32_t *src, const int32_t *dst,
                   const float *w, const float *dY, double *dX, double *absb)
{
    if (!sizes_ok(N, E) || H < 1)
        return ORACLE_BAD_SIZE;
    if (!indices_ok(N, E, src, dst))
        return ORACLE_BAD_INDEX;
    double *cnt = in_counts(N, E, dst);
    if (!cnt)
        return ORACLE_NO_MEMORY;
    memset(dX, 0, (size_t)(N * H) * sizeof(double));
    if (absb)
        memset(absb, 0, (size_t)(N * H) * sizeof(double));
    for (int64_t e = 0; e < E; ++e) {
        double a = (double)w[e] / cnt[dst[e]];
        const float *gd = dY + (int64_t)dst[e] * H;
        double *xs = dX + (int64_t)src[e] * H;
        for (int64_t h = 0; h < H; ++h) {
            xs[h] += a * (double)gd[h];
            if (absb)
                absb[(int64_t)src[e] * H + h] += fabs(a * (double)gd[h]);
        }
    }
    free(cnt);
    return ORACLE_OK;
}

int oracle_mean_dw(int64_t N, int64_t E, int64_t H, const int32_t *src, const int32_t *dst,
                   const float *X, const float *dY, double *dw, double *absb)
{
    int rc = oracle_dw(N, E, H, src, dst, X, dY, dw, absb);
    if (rc)
        return rc;
    double *cnt = in_counts(N, E, dst);
    if (!cnt)
        return ORACLE_NO_MEMORY;
    for (int64_t e = 0; e < E; ++e) {
        dw[e] /= cnt[dst[e]];
        if (absb)
            absb[e] /= cnt[dst[e]];
    }
    free(cnt);
    return ORACLE_OK;
}

/*
 * GCN normalisation of the weights, D^-1/2 A_w D^-1/2:
 *   deg(i) = sum of w_e over the edges into i (w = NULL: every w_e = 1),
 *   out_e  = w_e / sqrt(deg(src_e)) / sqrt(deg(dst_e)),
 * with deg^-1/2 taken as 0 where deg(i) <= 0 (no normalisation is defined
 * there).  Self-loops are part of the edge list given.
 */
int oracle_gcn_norm(int64_t N, int64_t E, const int32_t *src, const int32_t *dst,
                    const float *w, double *out)
{
    if (!sizes_ok(N, E))
        return ORACLE_BAD_SIZE;
    if (!indices_ok(N, E, src, dst))
        return ORACLE_BAD_INDEX;
    double *deg = (double *)calloc((size_t)N, sizeof(double));
    if (!deg)
        return ORACLE_NO_MEMORY;
    for (int64_t e = 0; e < E; ++e)
        deg[dst[e]] += w ? (double)w[e] : 1.0;
    for (int64_t i = 0; i < N; ++i)
        deg[i] = deg[i] > 0.0 ? 1.0 / sqrt(deg[i]) : 0.0;
    for (int64_t e = 0; e < E; ++e)
        out[e] = deg[src[e]] * (w ? (double)w[e] : 1.0) * deg[dst[e]];
    free(deg);
    return ORACLE_OK;
}

/*
 * Edge-softmax attention over the forward adjacency (SDDMM scores, a softmax
 * per destination row, then the SpMM with the normalised scores):
 *   s_e     = scale * dot(Q[dst_e], K[src_e])
 *   m_r     = max of s_e over the edges into r
 *   alpha_e = exp(s_e - m_r) / (sum over edges e' into r of exp(s_e' - m_r))
 *   Y[r, h] = sum over edges e into r of alpha_e V[src_e, h]
 * Rows without edges have Y = 0.  s and alpha are written in COO order;
 * absb[r, h] = sum over the same edges of |alpha_e V[src_e, h]|.
 */
int oracle_attn_fwd(int64_t N, int64_t E, int64_t H, const int32_t *src, const int32_t *dst,
                    const float *Q, const float *K, const float *V, double scale,
                    double *s, double *alpha, double *Y, double *absb)
{
    if (!sizes_ok(N, E) || H < 1)
        return ORACLE_BAD_SIZE;
    if (!indices_ok(N, E, src, dst))
        return ORACLE_BAD_INDEX;
    double *m = (double *)malloc((size_t)N * sizeof(double));
    double *z = (double *)calloc((size_t)N, sizeof(double));
    if (!m || !z) {
        free(m);
        free(z);
        return ORACLE_NO_MEMORY;
    }
    for (int64_t r = 0; r < N; ++r)
        m[r] = -INFINITY;
    for (int64_t e = 0; e < E; ++e) {
        const float *q = Q + (int64_t)dst[e] * H;
        const float *k = K + (int64_t)src[e] * H;
        double acc = 0.0;
        for (int64_t h = 0; h < H; ++h)
            acc += (double)q[h] * (double)k[h];
        s[e] = scale * acc;
        if (s[e] > m[dst[e]])
            m[dst[e]] = s[e];
    }
    for (int64_t e = 0; e < E; ++e)
        z[dst[e]] += exp(s[e] - m[dst[e]]);
    for (int64_t e = 0; e < E; ++e)
        alpha[e] = exp(s[e] - m[dst[e]]) / z[dst[e]];
    memset(Y, 0, (size_t)(N * H) * sizeof(double));
    if (absb)
        memset(absb, 0, (size_t)(N * H) * sizeof(double));
    for (int64_t e = 0; e < E; ++e) {
        const float *v = V + (int64_t)src[e] * H;
        double *y = Y + (int64_t)dst[e] * H;
        for (int64_t h = 0; h < H; ++h) {
            y[h] += alpha[e] * (double)v[h];
            if (absb)
                absb[(int64_t)dst[e] * H + h] += fabs(alpha[e] * (double)v[h]);
        }
    }
    free(m);
    free(z);
    return ORACLE_OK;
}

/*
 * Gradients of the attention for an upstream gradient dY (alpha as computed
 * by oracle_attn_fwd), from the chain rule through the row softmax:
 *   dalpha_e = dot(dY[dst_e], V[src_e])
 *   c_r      = sum over edges e into r of alpha_e dalpha_e
 *   ds_e     = alpha_e (dalpha_e - c_{dst_e})
 *   dQ[r]    = scale * sum over edges e into r   of ds_e K[src_e]
 *   dK[s]    = scale * sum over edges e out of s of ds_e Q[dst_e]
 *   dV[s]    =         sum over edges e out of s of alpha_e dY[dst_e]
 * ds (COO order) is returned too.
 */
int oracle_attn_bwd(int64_t N, int64_t E, int64_t H, const int32_t *src, const int32_t *dst,
                    const float *Q, const float *K, const float *V, double scale,
                    const double *alpha, const float *dY,
                    double *dQ, double *dK, double *dV, double *ds)
{
    if (!sizes_ok(N, E) || H < 1)
        return ORACLE_BAD_SIZE;
    if (!indices_ok(N, E, src, dst))
        return ORACLE_BAD_INDEX;
    double *c = (double *)calloc((size_t)N, sizeof(double));
    if (!c)
        return ORACLE_NO_MEMORY;
    for (int64_t e = 0; e < E; ++e) {
        const float *g = dY + (int64_t)dst[e] * H;
        const float *v = V + (int64_t)src[e] * H;
        double acc = 0.0;
        for (int64_t h = 0; h < H; ++h)
            acc += (double)g[h] * (double)v[h];
        ds[e] = acc;  /* dalpha_e for now */
        c[dst[e]] += alpha[e] * acc;
    }
    for (int64_t e = 0; e < E; ++e)
        ds[e] = alpha[e] * (ds[e] - c[dst[e]]);
    memset(dQ, 0, (size_t)(N * H) * sizeof(double));
    memset(dK, 0, (size_t)(N * H) * sizeof(double));
    memset(dV, 0, (size_t)(N * H) * sizeof(double));
    for (int64_t e = 0; e < E; ++e) {
        const int64_t r = dst[e], so = src[e];
        for (int64_t h = 0; h < H; ++h) {
            dQ[r * H + h] += scale * ds[e] * (double)K[so * H + h];
            dK[so * H + h] += scale * ds[e] * (double)Q[r * H + h];
            dV[so * H + h] += alpha[e] * (double)dY[r * H + h];
        }
    }
    free(c);
    return ORACLE_OK;
}

/*
 * Sampled form of the attention and its gradients for graphs too large to
 * evaluate whole: the definitions of oracle_attn_fwd / oracle_attn_bwd,
 * evaluated only for the destination rows sel_r (outputs Y and dQ) and the
 * source rows sel_s (outputs dK and dV).  The row statistics m_r, l_r and
 * c_r are formed for every row that one of those outputs needs (the sampled
 * destinations and every destination of an edge out of a sampled source),
 * over all of that row's edges.  Neither list may repeat a row.
 * Scales for the tolerances: absY_r = sum over edges into r of
 * |alpha_e V[src_e]|; with B_e = sum_h |dY[dst_e, h] V[src_e, h]| and
 * C_r = sum over edges into r of alpha_e B_e, the weight w_e =
 * |scale| alpha_e (B_e + C_{dst_e}) bounds |ds_e| and gives
 * absdQ_r = sum over edges into r of w_e |K[src_e]|, absdK_s = sum over
 * edges out of s of w_e |Q[dst_e]|, absdV_s = sum over edges out of s of
 * alpha_e |dY[dst_e]|.
 */
int oracle_attn_sampled(int64_t N, int64_t E, int64_t H, const int32_t *src, const int32_t *dst,
                        const float *Q, const float *K, const float *V, double scale, const float *dY,
                        int64_t nsel_r, const int32_t *sel_r, int64_t nsel_s, const int32_t *sel_s,
                        double *Y_r, double *dQ_r, double *dK_s, double *dV_s, double *absY_r,
                        double *absdQ_r, double *absdK_s, double *absdV_s)
{
    if (!sizes_ok(N, E) || H < 1 || nsel_r < 0 || nsel_s < 0)
        return ORACLE_BAD_SIZE;
    if (!indices_ok(N, E, src, dst))
        return ORACLE_BAD_INDEX;
    int64_t *slot_r = (int64_t *)malloc((size_t)N * sizeof(int64_t));
    int64_t *slot_s = (int64_t *)malloc((size_t)N * sizeof(int64_t));
    char *need = (char *)calloc((size_t)N, 1);
    double *m = (double *)malloc((size_t)N * sizeof(double));
    double *z = (double *)calloc((size_t)N, sizeof(double));
    double *c = (double *)calloc((size_t)N, sizeof(double));
    double *C = (double *)calloc((size_t)N, sizeof(double));
    int rc = ORACLE_OK;
    if (!slot_r || !slot_s || !need || !m || !z || !c || !C) {
        rc = ORACLE_NO_MEMORY;
        goto done;
    }
    for (int64_t i = 0; i < N; ++i) {
        slot_r[i] = slot_s[i] = -1;
        m[i] = -INFINITY;
    }
    for (int64_t i = 0; i < nsel_r; ++i) {
        if (sel_r[i] < 0 || sel_r[i] >= N || slot_r[sel_r[i]] >= 0) {
            rc = ORACLE_BAD_INDEX;
            goto done;
        }
        slot_r[sel_r[i]] = i;
        need[sel_r[i]] = 1;
    }
    for (int64_t i = 0; i < nsel_s; ++i) {
        if (sel_s[i] < 0 || sel_s[i] >= N || slot_s[sel_s[i]] >= 0) {
            rc = ORACLE_BAD_INDEX;
            goto done;
        }
        slot_s[sel_s[i]] = i;
    }
    for (int64_t e = 0; e < E; ++e)
        if (slot_s[src[e]] >= 0)
            need[dst[e]] = 1;
    memset(Y_r, 0, (size_t)(nsel_r * H) * sizeof(double));
    memset(dQ_r, 0, (size_t)(nsel_r * H) * sizeof(double));
    memset(absY_r, 0, (size_t)(nsel_r * H) * sizeof(double));
    memset(dK_s, 0, (size_t)(nsel_s * H) * sizeof(double));
    memset(dV_s, 0, (size_t)(nsel_s * H) * sizeof(double));
    memset(absdQ_r, 0, (size_t)(nsel_r * H) * sizeof(double));
    memset(absdK_s, 0, (size_t)(nsel_s * H) * sizeof(double));
    memset(absdV_s, 0, (size_t)(nsel_s * H) * sizeof(double));
    /* pass 1: row maxima of the scores; pass 2: sums of exponentials */
    for (int pass = 0; pass < 2; ++pass) {
        for (int64_t e = 0; e < E; ++e) {
            const int64_t r = dst[e];
            if (!need[r])
                continue;
            double acc = 0.0;
            for (int64_t h = 0; h < H; ++h)
                acc += (double)Q[r * H + h] * (double)K[(int64_t)src[e] * H + h];
            const double s = scale * acc;
            if (pass == 0) {
                if (s > m[r])
                    m[r] = s;
            } else {
                z[r] += exp(s - m[r]);
            }
        }
    }
    /* pass 3: c_r; pass 4: the outputs */
    for (int pass = 0; pass < 2; ++pass) {
        for (int64_t e = 0; e < E; ++e) {
            const int64_t r = dst[e], so = src[e];
            if (!need[r])
                continue;
            double acc = 0.0, da = 0.0, B = 0.0;
            for (int64_t h = 0; h < H; ++h) {
                acc += (double)Q[r * H + h] * (double)K[so * H + h];
                da += (double)dY[r * H + h] * (double)V[so * H + h];
                B += fabs((double)dY[r * H + h] * (double)V[so * H + h]);
            }
            const double alpha = exp(scale * acc - m[r]) / z[r];
            if (pass == 0) {
                c[r] += alpha * da;
                C[r] += alpha * B;
                continue;
            }
            const double ds = alpha * (da - c[r]);
            const double wb = fabs(scale) * alpha * (B + C[r]);
            const int64_t i = slot_r[r], j = slot_s[so];
            for (int64_t h = 0; h < H; ++h) {
                if (i >= 0) {
                    Y_r[i * H + h] += alpha * (double)V[so * H + h];
                    absY_r[i * H + h] += fabs(alpha * (double)V[so * H + h]);
                    dQ_r[i * H + h] += scale * ds * (double)K[so * H + h];
                    absdQ_r[i * H + h] += wb * fabs((double)K[so * H + h]);
                }
                if (j >= 0) {
                    dK_s[j * H + h] += scale * ds * (double)Q[r * H + h];
                    dV_s[j * H + h] += alpha * (double)dY[r * H + h];
                    absdK_s[j * H + h] += wb * fabs((double)Q[r * H + h]);
                    absdV_s[j * H + h] += alpha * fabs((double)dY[r * H + h]);
                }
            }
        }
    }
done:
    free(slot_r);
    free(slot_s);
    free(need);
    free(m);
    free(z);
    free(c);
    free(C);
    return rc;
}
