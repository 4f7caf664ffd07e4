"""Pins of the fp64 oracle against facts that do not come from the oracle.

Each pin is chosen so that a plausible slip in the oracle (a transposed
operand, a wrong index, a dropped term, a sign, an unstable sort) fails at
least one test: the hand-derived "Exact witness" of the tinymesh "Weighted
aggregation experiment" page, dense matrix products by brute force (numpy),
library stable sorts, the adjoint identity, finite differences of the linear
loss, and the edge cases listed in section "Exact witness" (two COO
orderings of one graph, repeated edges carrying unequal weights, nodes with
no edges, a graph of a single node).
"""
import numpy as np
import pytest

import oracle
from tests.golden import load


def dense_A(N, src, dst, w):
    A = np.zeros((N, N), np.float64)
    np.add.at(A, (np.asarray(dst), np.asarray(src)), np.asarray(w, np.float64))
    return A


def rand_graph(rng, N, E, H):
    src = rng.integers(0, N, E).astype(np.int32)
    dst = rng.integers(0, N, E).astype(np.int32)
    w = rng.standard_normal(E).astype(np.float32)
    X = rng.standard_normal((N, H)).astype(np.float32)
    dY = rng.standard_normal((N, H)).astype(np.float32)
    return src, dst, w, X, dY


# ----------------------------------------------------------------------------- witness

def test_witness_fixture():
    g = load("witness_3edge.txt")
    N, H = g["N"], g["H"]
    src, dst = g["src"].astype(np.int32), g["dst"].astype(np.int32)
    w = g["w"].astype(np.float32)
    X = g["X"].reshape(N, H).astype(np.float32)
    dY = g["dY"].reshape(N, H).astype(np.float32)
    low = oracle.lower(src, dst, N)
    for k in ("edge_order", "rowptr_f", "col_f", "transpose_order", "rowptr_t", "col_t"):
        np.testing.assert_array_equal(low[k], g[k].astype(np.int32), err_msg=k)
    np.testing.assert_array_equal(oracle.fwd(src, dst, N, w, X)[:, 0], g["Y"])
    np.testing.assert_array_equal(oracle.dx(src, dst, N, w, dY)[:, 0], g["dX"])
    np.testing.assert_array_equal(oracle.dw(src, dst, N, X, dY), g["dw"])


def test_witness_storage_bound():
    # "Edge order is explicit": the two CSR forms hold 2E + 2(N + 1) integers
    # and execution adds the two order maps (with src/dst: 4E device ints).
    g = load("witness_3edge.txt")
    N, E = g["N"], len(g["src"])
    low = oracle.lower(g["src"], g["dst"], N)
    csr = sum(low[k].size for k in ("rowptr_f", "col_f", "rowptr_t", "col_t"))
    assert csr == 2 * E + 2 * (N + 1)
    assert low["edge_order"].size + low["transpose_order"].size == 2 * E


# ----------------------------------------------------------------------------- planted mistakes

def test_witness_catches_planted_mistakes():
    """Oracle variants with a planted slip (run on the CPU) must fail the witness."""
    g = load("witness_3edge.txt")
    N = g["N"]
    src, dst = g["src"].astype(np.int32), g["dst"].astype(np.int32)
    w = g["w"].astype(np.float32)
    X = g["X"].reshape(N, 1).astype(np.float32)
    dY = g["dY"].reshape(N, 1).astype(np.float32)
    # transposed operand: aggregating at sources instead of destinations
    assert not np.array_equal(oracle.fwd(dst, src, N, w, X)[:, 0], g["Y"])
    # dX computed with the forward orientation
    assert not np.array_equal(oracle.fwd(src, dst, N, w, dY)[:, 0], g["dX"])
    # sign slip on the weights
    assert not np.array_equal(oracle.fwd(src, dst, N, -w, X)[:, 0], g["Y"])
    # dw with the two feature operands swapped
    assert not np.array_equal(oracle.dw(src, dst, N, dY, X), g["dw"])
    # weights read in CSR order instead of COO order
    eo = g["edge_order"].astype(np.int64)
    assert not np.array_equal(oracle.fwd(src, dst, N, w[eo], X)[:, 0], g["Y"])
    # a sort that is not stable on ties (reverse COO order inside a row)
    order = np.argsort(-np.arange(3))
    bad = order[np.argsort(dst[order], kind="stable")]
    assert not np.array_equal(bad, g["edge_order"])


# ----------------------------------------------------------------------------- dense brute force

@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("N,E,H", [(1, 3, 2), (5, 17, 3), (33, 200, 4), (64, 512, 7)])
def test_dense_bruteforce(seed, N, E, H):
    rng = np.random.default_rng(seed * 131 + N)
    src, dst, w, X, dY = rand_graph(rng, N, E, H)
    A = dense_A(N, src, dst, w)
    Y = oracle.fwd(src, dst, N, w, X)
    dX = oracle.dx(src, dst, N, w, dY)
    np.testing.assert_allclose(Y, A @ X.astype(np.float64), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dX, A.T @ dY.astype(np.float64), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("seed", range(4))
def test_dw_is_derivative_of_linear_loss(seed):
    """dw_e = dL/dw_e with L(w) = <A_w X, dY>; L is linear in w, so the
    derivative is L evaluated at the unit weight vector of edge e (dense)."""
    rng = np.random.default_rng(1000 + seed)
    N, E, H = 17, 60, 5
    src, dst, w, X, dY = rand_graph(rng, N, E, H)
    X64, dY64 = X.astype(np.float64), dY.astype(np.float64)
    got = oracle.dw(src, dst, N, X, dY)
    for e in range(E):
        unit = np.zeros(E)
        unit[e] = 1.0
        L_e = np.sum((dense_A(N, src, dst, unit) @ X64) * dY64)
        assert abs(got[e] - L_e) <= 1e-12 * max(1.0, abs(L_e))
    # and a finite difference around a non-zero w, dense all the way
    base = np.sum((dense_A(N, src, dst, w) @ X64) * dY64)
    for e in (0, E // 2, E - 1):
        wp = w.astype(np.float64).copy()
        wp[e] += 0.5
        fd = (np.sum((dense_A(N, src, dst, wp) @ X64) * dY64) - base) / 0.5
        assert abs(got[e] - fd) <= 1e-9 * max(1.0, abs(fd))


def test_abs_bound_is_dense_abs_product():
    rng = np.random.default_rng(7)
    N, E, H = 40, 300, 6
    src, dst, w, X, dY = rand_graph(rng, N, E, H)
    Y, BY = oracle.fwd(src, dst, N, w, X, with_bound=True)
    dX, BX = oracle.dx(src, dst, N, w, dY, with_bound=True)
    dw, Bw = oracle.dw(src, dst, N, X, dY, with_bound=True)
    Aabs = dense_A(N, src, dst, np.abs(w))
    np.testing.assert_allclose(BY, Aabs @ np.abs(X.astype(np.float64)), rtol=1e-12)
    np.testing.assert_allclose(BX, Aabs.T @ np.abs(dY.astype(np.float64)), rtol=1e-12)
    np.testing.assert_allclose(
        Bw, np.abs(X[src].astype(np.float64) * dY[dst].astype(np.float64)).sum(1), rtol=1e-12)
    assert np.all(np.abs(Y) <= BY + 1e-12) and np.all(np.abs(dX) <= BX + 1e-12)
    assert np.all(np.abs(dw) <= Bw + 1e-12)


# ----------------------------------------------------------------------------- lowering

@pytest.mark.parametrize("seed", range(5))
@pytest.mark.parametrize("N,E", [(1, 0), (1, 9), (7, 0), (7, 40), (300, 5000), (5000, 300)])
def test_lowering_matches_library_stable_sort(seed, N, E):
    rng = np.random.default_rng(seed + 17 * N + E)
    src = rng.integers(0, N, E).astype(np.int32)
    dst = rng.integers(0, N, E).astype(np.int32)
    low = oracle.lower(src, dst, N)
    for key, other, order, rowptr, col in ((dst, src, "edge_order", "rowptr_f", "col_f"),
                                           (src, dst, "transpose_order", "rowptr_t", "col_t")):
        ref = np.argsort(key, kind="stable")
        np.testing.assert_array_equal(low[order], ref)
        np.testing.assert_array_equal(
            low[rowptr], np.concatenate([[0], np.cumsum(np.bincount(key, minlength=N))]))
        np.testing.assert_array_equal(low[col], other[ref])
    if E <= 40:
        py = sorted(range(E), key=lambda e: int(dst[e]))   # Python's sort is stable
        np.testing.assert_array_equal(low["edge_order"], py)


def test_lowering_invariants():
    rng = np.random.default_rng(3)
    N, E = 1000, 20000
    src = rng.integers(0, N, E).astype(np.int32)
    dst = (rng.integers(0, 30, E) ** 2 % N).astype(np.int32)   # skewed rows, many empty
    low = oracle.lower(src, dst, N)
    for key, order, rowptr in ((dst, "edge_order", "rowptr_f"), (src, "transpose_order", "rowptr_t")):
        o, rp = low[order], low[rowptr]
        assert np.array_equal(np.sort(o), np.arange(E))                # a permutation
        assert rp[0] == 0 and rp[-1] == E and np.all(np.diff(rp) >= 0)
        assert np.all(np.diff(key[o]) >= 0)                             # sorted by owner
        for r in range(N):                                              # ties in COO order
            seg = o[rp[r]:rp[r + 1]]
            assert np.all(np.diff(seg) > 0)
            assert np.all(key[seg] == r)


# ----------------------------------------------------------------------------- algebra

def test_adjoint_identity():
    rng = np.random.default_rng(11)
    N, E, H = 500, 8000, 9
    src, dst, w, X, dY = rand_graph(rng, N, E, H)
    Y = oracle.fwd(src, dst, N, w, X)
    dX = oracle.dx(src, dst, N, w, dY)
    dw = oracle.dw(src, dst, N, X, dY)
    a = np.sum(Y * dY.astype(np.float64))
    b = np.sum(X.astype(np.float64) * dX)
    c = np.sum(w.astype(np.float64) * dw)
    scale = np.sum(np.abs(w.astype(np.float64))[:, None]
                   * np.abs(X[src].astype(np.float64) * dY[dst].astype(np.float64)))
    assert abs(a - b) <= 1e-12 * scale and abs(a - c) <= 1e-12 * scale


def test_linearity_in_weights():
    rng = np.random.default_rng(12)
    N, E, H = 50, 400, 3
    src, dst, w, X, dY = rand_graph(rng, N, E, H)
    for alpha in (2.0, -0.5, 0.0):
        np.testing.assert_array_equal(oracle.fwd(src, dst, N, (alpha * w).astype(np.float32), X),
                                      alpha * oracle.fwd(src, dst, N, w, X))
        np.testing.assert_array_equal(oracle.dx(src, dst, N, (alpha * w).astype(np.float32), dY),
                                      alpha * oracle.dx(src, dst, N, w, dY))


# ----------------------------------------------------------------------------- page edge cases

def test_paired_coo_permutation():
    rng = np.random.default_rng(13)
    N, E, H = 80, 700, 4
    src, dst, w, X, dY = rand_graph(rng, N, E, H)
    perm = rng.permutation(E)
    Y0, Y1 = oracle.fwd(src, dst, N, w, X), oracle.fwd(src[perm], dst[perm], N, w[perm], X)
    dX0, dX1 = oracle.dx(src, dst, N, w, dY), oracle.dx(src[perm], dst[perm], N, w[perm], dY)
    np.testing.assert_allclose(Y1, Y0, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dX1, dX0, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(oracle.dw(src[perm], dst[perm], N, X, dY),
                                  oracle.dw(src, dst, N, X, dY)[perm])
    # the maps change with the permutation but still point at the same edges
    l0, l1 = oracle.lower(src, dst, N), oracle.lower(src[perm], dst[perm], N)
    np.testing.assert_array_equal(l0["rowptr_f"], l1["rowptr_f"])
    np.testing.assert_array_equal(np.sort(perm[l1["edge_order"]]), np.arange(E))
    np.testing.assert_array_equal(dst[perm[l1["edge_order"]]], dst[l0["edge_order"]])


def test_duplicate_edges_with_different_weights():
    N, H = 4, 3
    src = np.array([1, 1, 2, 1], np.int32)
    dst = np.array([3, 3, 0, 3], np.int32)
    w = np.array([0.5, -2.0, 1.0, 4.0], np.float32)
    rng = np.random.default_rng(14)
    X = rng.standard_normal((N, H)).astype(np.float32)
    dY = rng.standard_normal((N, H)).astype(np.float32)
    merged = (np.array([1, 2], np.int32), np.array([3, 0], np.int32),
              np.array([0.5 - 2.0 + 4.0, 1.0], np.float32))
    np.testing.assert_allclose(oracle.fwd(src, dst, N, w, X), oracle.fwd(*merged[:2], N, merged[2], X),
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(oracle.dx(src, dst, N, w, dY), oracle.dx(*merged[:2], N, merged[2], dY),
                               rtol=1e-12, atol=1e-12)
    dw = oracle.dw(src, dst, N, X, dY)
    assert dw[0] == dw[1] == dw[3]                 # each duplicate keeps its own position
    low = oracle.lower(src, dst, N)
    np.testing.assert_array_equal(low["edge_order"], [2, 0, 1, 3])
    np.testing.assert_array_equal(low["rowptr_f"], [0, 1, 1, 1, 4])


def test_isolated_and_empty_rows_are_exact_zero():
    N, H = 6, 5
    src = np.array([0, 0, 2], np.int32)
    dst = np.array([1, 2, 1], np.int32)
    rng = np.random.default_rng(15)
    w = rng.standard_normal(3).astype(np.float32)
    X = rng.standard_normal((N, H)).astype(np.float32)
    dY = rng.standard_normal((N, H)).astype(np.float32)
    Y = oracle.fwd(src, dst, N, w, X)
    dX = oracle.dx(src, dst, N, w, dY)
    for r in (0, 3, 4, 5):
        assert np.all(Y[r] == 0.0)
    for r in (1, 3, 4, 5):
        assert np.all(dX[r] == 0.0)


def test_one_node_and_empty_graphs():
    X = np.array([[1.5, -2.0]], np.float32)
    dY = np.array([[0.25, 3.0]], np.float32)
    e = np.zeros(0, np.int32)
    assert np.all(oracle.fwd(e, e, 1, np.zeros(0, np.float32), X) == 0)
    assert np.all(oracle.dx(e, e, 1, np.zeros(0, np.float32), dY) == 0)
    assert oracle.dw(e, e, 1, X, dY).shape == (0,)
    low = oracle.lower(e, e, 1)
    np.testing.assert_array_equal(low["rowptr_f"], [0, 0])
    one = np.zeros(1, np.int32)
    w = np.array([-3.0], np.float32)
    np.testing.assert_array_equal(oracle.fwd(one, one, 1, w, X), [[-4.5, 6.0]])
    np.testing.assert_array_equal(oracle.dx(one, one, 1, w, dY), [[-0.75, -9.0]])
    np.testing.assert_array_equal(oracle.dw(one, one, 1, X, dY), [1.5 * 0.25 - 2.0 * 3.0])
    # an edgeless graph with many nodes
    N = 9
    Xn = np.ones((N, 3), np.float32)
    assert np.all(oracle.fwd(e, e, N, np.zeros(0, np.float32), Xn) == 0)
    np.testing.assert_array_equal(oracle.lower(e, e, N)["rowptr_t"], np.zeros(N + 1))


def test_rejects_bad_input():
    with pytest.raises(oracle.OracleError):
        oracle.lower([0, 3], [1, 1], 3)
    with pytest.raises(oracle.OracleError):
        oracle.lower([0, -1], [1, 1], 3)
    with pytest.raises(oracle.OracleError):
        oracle.lower([], [], 0)
    with pytest.raises(oracle.OracleError):
        oracle.fwd([0], [5], 2, [1.0], np.ones((2, 1), np.float32))


def test_sampled_forms_match_full():
    rng = np.random.default_rng(16)
    N, E, H = 300, 4000, 6
    src, dst, w, X, dY = rand_graph(rng, N, E, H)
    Y, BY = oracle.fwd(src, dst, N, w, X, with_bound=True)
    dX, BX = oracle.dx(src, dst, N, w, dY, with_bound=True)
    dw, Bw = oracle.dw(src, dst, N, X, dY, with_bound=True)
    rows = rng.choice(N, 37, replace=False).astype(np.int32)
    ys, bys = oracle.spmm_rows(src, dst, N, w, X, rows, by_source=False, with_bound=True)
    xs, bxs = oracle.spmm_rows(src, dst, N, w, dY, rows, by_source=True, with_bound=True)
    np.testing.assert_array_equal(ys, Y[rows])
    np.testing.assert_array_equal(bys, BY[rows])
    np.testing.assert_array_equal(xs, dX[rows])
    np.testing.assert_array_equal(bxs, BX[rows])
    edges = rng.choice(E, 50, replace=False)
    de, be = oracle.dw_edges(src, dst, N, X, dY, edges, with_bound=True)
    np.testing.assert_array_equal(de, dw[edges])
    np.testing.assert_array_equal(be, Bw[edges])
