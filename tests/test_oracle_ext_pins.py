"""Pins of the oracle's further aggregators (mean, GCN-normalised weights,
edge-softmax attention) against facts that do not come from the oracle.

The PyTorch Geometric reading guide names these operations (Step 3: GCN's
normalised adjacency and the sum or mean reductions of spmm; Step 4: SDDMM
scores and a per-row softmax before the SpMM) without writing them out, so
the pins are closed forms, hand-derived values, invariants, dense matrix
formulations with library routines (numpy bincount and matmul, scipy
softmax), and finite differences of a scalar loss for every gradient.
"""
import numpy as np
import pytest
from scipy.special import softmax

import oracle


def rand_graph(rng, N, E, H, positive=False):
    src = rng.integers(0, N, E).astype(np.int32)
    dst = rng.integers(0, N, E).astype(np.int32)
    w = (rng.random(E) + 0.1 if positive else rng.standard_normal(E)).astype(np.float32)
    X = rng.standard_normal((N, H)).astype(np.float32)
    G = rng.standard_normal((N, H)).astype(np.float32)
    return src, dst, w, X, G


def dense_A(N, src, dst, w):
    A = np.zeros((N, N), np.float64)
    np.add.at(A, (np.asarray(dst), np.asarray(src)), np.asarray(w, np.float64))
    return A


def nudge(a: np.ndarray, idx, delta: float):
    """Copy of fp32 array `a` with a[idx] moved by about `delta`; returns the
    copy and the exact change after rounding to fp32."""
    b = a.copy()
    b[idx] = np.float32(np.float64(a[idx]) + delta)
    return b, np.float64(b[idx]) - np.float64(a[idx])


# ----------------------------------------------------------------------------- mean

def test_mean_star_closed_form():
    rng = np.random.default_rng(1)
    k, H = 7, 5
    N = k + 1
    src = np.arange(1, N, dtype=np.int32)
    dst = np.zeros(k, np.int32)
    w = rng.standard_normal(k).astype(np.float32)
    X = rng.standard_normal((N, H)).astype(np.float32)
    Y = oracle.mean_fwd(src, dst, N, w, X)
    want = np.mean(w.astype(np.float64)[:, None] * X[1:].astype(np.float64), axis=0)
    np.testing.assert_allclose(Y[0], want, rtol=1e-14, atol=1e-15)
    assert not Y[1:].any()


def test_mean_counts_duplicate_edges():
    # the same pair twice counts twice: (2 * w0 x + w1 x') / 3 for node 0
    src = np.array([1, 1, 2], np.int32)
    dst = np.array([0, 0, 0], np.int32)
    w = np.array([0.5, 0.5, 2.0], np.float32)
    X = np.array([[0, 0], [1, 2], [4, 8]], np.float32)
    Y = oracle.mean_fwd(src, dst, 3, w, X)
    np.testing.assert_allclose(Y[0], [(0.5 + 0.5 + 8.0) / 3, (1 + 1 + 16.0) / 3], rtol=1e-15)


@pytest.mark.parametrize("seed", [2, 3])
def test_mean_is_degree_scaled_dense_product(seed):
    rng = np.random.default_rng(seed)
    N, E, H = 17, 60, 4
    src, dst, w, X, G = rand_graph(rng, N, E, H)
    cnt = np.bincount(dst, minlength=N).astype(np.float64)
    inv = np.divide(1.0, cnt, out=np.zeros(N), where=cnt > 0)
    A = dense_A(N, src, dst, w)
    np.testing.assert_allclose(oracle.mean_fwd(src, dst, N, w, X), inv[:, None] * (A @ X), atol=1e-12)
    np.testing.assert_allclose(oracle.mean_dx(src, dst, N, w, G), A.T @ (inv[:, None] * G), atol=1e-12)
    np.testing.assert_allclose(oracle.mean_dw(src, dst, N, X, G),
                               np.einsum("eh,eh->e", X[src].astype(np.float64), G[dst]) * inv[dst],
                               atol=1e-12)


def test_mean_gradients_are_derivatives_of_the_loss():
    # L(w, X) = <mean_fwd(w, X), G> is linear in X and in w: a finite
    # difference is exact up to fp64 rounding
    rng = np.random.default_rng(4)
    N, E, H = 9, 30, 3
    src, dst, w, X, G = rand_graph(rng, N, E, H)
    L = lambda w_, X_: float(np.sum(oracle.mean_fwd(src, dst, N, w_, X_) * G))
    dX = oracle.mean_dx(src, dst, N, w, G)
    dw = oracle.mean_dw(src, dst, N, X, G)
    for idx in [(0, 0), (3, 2), (int(src[5]), 1), (int(src[11]), 0)]:
        X2, d = nudge(X, idx, 0.25)
        assert abs((L(w, X2) - L(w, X)) / d - dX[idx]) < 1e-10
    for e in [0, 7, 19, 29]:
        w2, d = nudge(w, e, 0.25)
        assert abs((L(w2, X) - L(w, X)) / d - dw[e]) < 1e-10


def test_mean_with_unit_in_degree_is_the_sum():
    rng = np.random.default_rng(5)
    N, H = 12, 4
    src = rng.permutation(N).astype(np.int32)
    dst = np.arange(N, dtype=np.int32)
    w = rng.standard_normal(N).astype(np.float32)
    X = rng.standard_normal((N, H)).astype(np.float32)
    np.testing.assert_array_equal(oracle.mean_fwd(src, dst, N, w, X), oracle.fwd(src, dst, N, w, X))


def test_mean_empty_graph_and_bounds():
    z = np.zeros(0, np.int32)
    X = np.ones((3, 2), np.float32)
    assert not oracle.mean_fwd(z, z, 3, np.zeros(0, np.float32), X).any()
    rng = np.random.default_rng(6)
    src, dst, w, X, G = rand_graph(rng, 8, 25, 3)
    _, b = oracle.mean_fwd(src, dst, 8, w, X, with_bound=True)
    cnt = np.bincount(dst, minlength=8).astype(np.float64)
    inv = np.divide(1.0, cnt, out=np.zeros(8), where=cnt > 0)
    np.testing.assert_allclose(b, inv[:, None] * (dense_A(8, src, dst, np.abs(w)) @ np.abs(X)), atol=1e-12)


# ----------------------------------------------------------------------------- gcn_norm

def test_gcn_norm_hand_example():
    # path 0 - 1 - 2, both directions, plus a self-loop on every node:
    # in-degrees 2, 3, 2
    src = np.array([0, 1, 2, 0, 1, 1, 2], np.int32)
    dst = np.array([0, 1, 2, 1, 0, 2, 1], np.int32)
    got = oracle.gcn_norm(src, dst, 3)
    r6 = 1 / np.sqrt(6.0)
    np.testing.assert_allclose(got, [0.5, 1 / 3, 0.5, r6, r6, r6, r6], rtol=1e-15)


def test_gcn_norm_regular_graph_is_one_over_degree():
    N = 11
    i = np.arange(N, dtype=np.int32)
    src = np.concatenate([i, i, (i + 3) % N]).astype(np.int32)
    dst = np.concatenate([i, (i + 1) % N, i]).astype(np.int32)
    np.testing.assert_allclose(oracle.gcn_norm(src, dst, N), np.full(3 * N, 1 / 3), rtol=1e-15)


@pytest.mark.parametrize("seed", [7, 8])
def test_gcn_norm_fixes_sqrt_degree(seed):
    # with D = weighted in-degree, (D^-1/2 A D^-1/2) D^1/2 1 = D^1/2 1 whenever
    # every node has an incoming edge (self-loops make sure of it)
    rng = np.random.default_rng(seed)
    N, E = 23, 90
    src, dst, w, _, _ = rand_graph(rng, N, E, 1, positive=True)
    src = np.concatenate([src, np.arange(N, dtype=np.int32)])
    dst = np.concatenate([dst, np.arange(N, dtype=np.int32)])
    w = np.concatenate([w, np.ones(N, np.float32)])
    norm = oracle.gcn_norm(src, dst, N, w)
    d = np.bincount(dst, weights=w.astype(np.float64), minlength=N)
    An = dense_A(N, src, dst, norm)
    np.testing.assert_allclose(An @ np.sqrt(d), np.sqrt(d), rtol=1e-13)


def test_gcn_norm_unit_weights_and_zero_degree():
    rng = np.random.default_rng(9)
    src, dst, _, _, _ = rand_graph(rng, 10, 40, 1)
    np.testing.assert_array_equal(oracle.gcn_norm(src, dst, 10),
                                  oracle.gcn_norm(src, dst, 10, np.ones(40, np.float32)))
    # node 2 has no incoming edge: its outgoing edges get weight 0
    src = np.array([2, 0], np.int32)
    dst = np.array([1, 1], np.int32)
    np.testing.assert_allclose(oracle.gcn_norm(src, dst, 3), [0.0, 0.0])
    src = np.array([0, 1], np.int32)
    dst = np.array([1, 0], np.int32)
    np.testing.assert_allclose(oracle.gcn_norm(src, dst, 3, np.array([4.0, 9.0], np.float32)),
                               [4 / np.sqrt(9 * 4), 9 / np.sqrt(4 * 9)], rtol=1e-15)


# ----------------------------------------------------------------------------- attention

def test_attn_rows_are_distributions():
    rng = np.random.default_rng(10)
    N, E, H = 15, 70, 6
    src, dst, _, X, G = rand_graph(rng, N, E, H)
    s, a, _ = oracle.attn_fwd(src, dst, N, X, G, X, 0.4)
    assert (a >= 0).all()
    sums = np.bincount(dst, weights=a, minlength=N)
    has = np.bincount(dst, minlength=N) > 0
    np.testing.assert_allclose(sums[has], 1.0, rtol=1e-14)
    # scores are scaled dot products of Q[dst] and K[src]
    np.testing.assert_allclose(s, 0.4 * np.einsum("eh,eh->e", X[dst].astype(np.float64), G[src]), rtol=1e-13)


def test_attn_single_edge_rows_copy_values():
    rng = np.random.default_rng(11)
    N, H = 9, 4
    src = rng.integers(0, N, N).astype(np.int32)
    dst = np.arange(N, dtype=np.int32)
    Q, K, V = (rng.standard_normal((N, H)).astype(np.float32) for _ in range(3))
    _, a, Y = oracle.attn_fwd(src, dst, N, Q, K, V, 1.0)
    np.testing.assert_array_equal(a, np.ones(N))
    np.testing.assert_array_equal(Y, V[src].astype(np.float64))


def test_attn_zero_queries_is_unweighted_mean():
    rng = np.random.default_rng(12)
    N, E, H = 14, 55, 5
    src, dst, _, V, K = rand_graph(rng, N, E, H)
    _, _, Y = oracle.attn_fwd(src, dst, N, np.zeros((N, H), np.float32), K, V, 0.7)
    np.testing.assert_allclose(Y, oracle.mean_fwd(src, dst, N, np.ones(E, np.float32), V), atol=1e-14)


@pytest.mark.parametrize("seed", [13, 14])
def test_attn_is_dense_masked_softmax(seed):
    rng = np.random.default_rng(seed)
    N, H = 16, 8
    pairs = rng.choice(N * N, 70, replace=False)  # distinct (dst, src) pairs
    dst, src = (pairs // N).astype(np.int32), (pairs % N).astype(np.int32)
    Q, K, V = (rng.standard_normal((N, H)).astype(np.float32) for _ in range(3))
    scale = 1 / np.sqrt(H)
    S = scale * (Q.astype(np.float64) @ K.astype(np.float64).T)
    mask = np.zeros((N, N), bool)
    mask[dst, src] = True
    P = softmax(np.where(mask, S, -np.inf), axis=1)
    P[~mask.any(axis=1)] = 0.0
    _, a, Y = oracle.attn_fwd(src, dst, N, Q, K, V, scale)
    np.testing.assert_allclose(a, P[dst, src], rtol=1e-12)
    np.testing.assert_allclose(Y, P @ V.astype(np.float64), atol=1e-12)


def test_attn_gradients_are_derivatives_of_the_loss():
    rng = np.random.default_rng(15)
    N, E, H = 8, 26, 3
    src, dst, _, _, _ = rand_graph(rng, N, E, H)
    Q, K, V, G = (rng.standard_normal((N, H)).astype(np.float32) for _ in range(4))
    scale = 0.6

    def L(Q_, K_, V_):
        return float(np.sum(oracle.attn_fwd(src, dst, N, Q_, K_, V_, scale)[2] * G))

    _, a, _ = oracle.attn_fwd(src, dst, N, Q, K, V, scale)
    dQ, dK, dV, ds = oracle.attn_bwd(src, dst, N, Q, K, V, scale, a, G)
    # the score gradient sums to zero over every row (softmax is shift-invariant)
    np.testing.assert_allclose(np.bincount(dst, weights=ds, minlength=N), 0.0, atol=1e-13)
    base = (Q, K, V)
    for which, grad in ((0, dQ), (1, dK), (2, dV)):
        for idx in [(int(dst[0]), 0), (int(src[3]), 2), (int(dst[9]), 1), (int(src[17]), 0)]:
            up, d1 = nudge(base[which], idx, 1e-3)
            dn, d2 = nudge(base[which], idx, -1e-3)
            args_up = list(base); args_up[which] = up
            args_dn = list(base); args_dn[which] = dn
            fd = (L(*args_up) - L(*args_dn)) / (d1 - d2)
            assert abs(fd - grad[idx]) <= 1e-5 * (1 + abs(grad[idx])), (which, idx, fd, grad[idx])


def test_attn_catches_planted_mistakes():
    # a softmax over the source side instead of the destination row, or a
    # missing max shift in fp32, would break the distributions above; here a
    # transposed score (Q[src] K[dst]) must differ from the oracle's
    rng = np.random.default_rng(16)
    N, E, H = 10, 40, 4
    src, dst, _, Q, K = rand_graph(rng, N, E, H)
    s, _, _ = oracle.attn_fwd(src, dst, N, Q, K, K, 1.0)
    wrong = np.einsum("eh,eh->e", Q[src].astype(np.float64), K[dst])
    assert not np.allclose(s, wrong)


def test_attn_sampled_form_matches_full():
    rng = np.random.default_rng(17)
    N, E, H = 30, 160, 5
    src, dst, _, _, _ = rand_graph(rng, N, E, H)
    Q, K, V, G = (rng.standard_normal((N, H)).astype(np.float32) for _ in range(4))
    scale = 0.45
    _, a, Y, bY = oracle.attn_fwd(src, dst, N, Q, K, V, scale, with_bound=True)
    dQ, dK, dV, _ = oracle.attn_bwd(src, dst, N, Q, K, V, scale, a, G)
    rr = np.array([0, 5, 11, int(dst[3]), 29], np.int32)
    rr = np.unique(rr)
    rs = np.unique(np.array([2, int(src[7]), 19, 28], np.int32))
    o = oracle.attn_sampled(src, dst, N, Q, K, V, scale, G, rr, rs)
    np.testing.assert_allclose(o["Y"], Y[rr], atol=1e-13)
    np.testing.assert_allclose(o["absY"], bY[rr], atol=1e-13)
    np.testing.assert_allclose(o["dQ"], dQ[rr], atol=1e-13)
    np.testing.assert_allclose(o["dK"], dK[rs], atol=1e-13)
    np.testing.assert_allclose(o["dV"], dV[rs], atol=1e-13)
    # the gradient scales dominate the gradients they bound
    assert (np.abs(o["dQ"]) <= o["absdQ"] + 1e-12).all()
    assert (np.abs(o["dK"]) <= o["absdK"] + 1e-12).all()
    assert (np.abs(o["dV"]) <= o["absdV"] + 1e-12).all()


def test_ext_pins_catch_planted_mistakes():
    """Plausible slips, planted by calling the oracle with its operands
    exchanged (on the CPU), must fail the invariants above."""
    rng = np.random.default_rng(31)
    N, E, H = 23, 90, 4
    src, dst, w, X, G = rand_graph(rng, N, E, H, positive=True)
    # GCN normalised by out-degrees (source and destination exchanged):
    # the sqrt-degree fixed point of the in-degree normalisation fails
    s2 = np.concatenate([src, np.arange(N, dtype=np.int32)])
    d2 = np.concatenate([dst, np.arange(N, dtype=np.int32)])
    w2 = np.concatenate([w, np.ones(N, np.float32)])
    d_in = np.bincount(d2, weights=w2.astype(np.float64), minlength=N)
    wrong = oracle.gcn_norm(d2, s2, N, w2)                     # degrees taken at the sources
    An = dense_A(N, s2, d2, wrong)
    assert not np.allclose(An @ np.sqrt(d_in), np.sqrt(d_in), rtol=1e-6)
    # mean divided by out-degree (source and destination exchanged in the count)
    cnt_in = np.bincount(dst, minlength=N).astype(np.float64)
    inv = np.divide(1.0, cnt_in, out=np.zeros(N), where=cnt_in > 0)
    right = inv[:, None] * (dense_A(N, src, dst, w) @ X)
    swapped = oracle.mean_dx(dst, src, N, w, X)                 # sums at destinations, counts at sources
    assert not np.allclose(swapped, right, atol=1e-9)
    # softmax taken over the edges out of a source instead of into a destination
    _, a_wrong, _ = oracle.attn_fwd(dst, src, N, X, X, X, 0.5)
    sums = np.bincount(dst, weights=a_wrong, minlength=N)
    has = np.bincount(dst, minlength=N) > 0
    assert not np.allclose(sums[has], 1.0)
