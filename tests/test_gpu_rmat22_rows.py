"""Mean aggregation, GCN weights and edge-softmax attention on the full-size
R-MAT scale-22 graph (4,194,304 nodes, 67,108,864 edges, H = 128, bf16
features), as the benchmark runs them.

The oracle checks the GCN weights of every edge, and sampled rows and edges
of the other outputs (heavy rows split across many tiles, empty rows and
random rows); row sums of alpha are checked for every row.

Attention tolerance at this size: every score is off by at most
1e-5 * scale * sum_h |q k| <= 1e-5 * scale * max|Q_r| max|K_s| (Cauchy-
Schwarz over the row norms), so alpha is off by at most rel = exp(2 d) - 1
plus 1e-6 * (8 + max in-degree / 256) for expf, the division and the
ordered fp32 sum of exponentials; Y by (rel + TOL) * sum alpha |V|; the
softmax-gradient weights ds by (2 rel + 3e-5) of their scale, so dQ and dK
by (2 rel + 3e-5 + TOL) of the oracle's gradient scales, dV by
(rel + TOL) * sum alpha |dY|.
"""
import numpy as np
import pytest
import torch

import workloads
from tests.gpu_helpers import TOL, TOL_DW, assert_within, host, lib

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def big():
    agb = lib()
    wl = workloads.make("rmat22", seed=1, device="cuda")
    g = agb.ag_graph_lower(wl.src, wl.dst, wl.N)
    return agb, wl, g


@pytest.fixture(scope="module")
def hosted(big):
    _, wl, g = big
    src, dst = host(wl.src), host(wl.dst)
    cnt = np.bincount(dst, minlength=wl.N)
    return src, dst, cnt


def _rows(rng, deg, n_random=1500):
    top = np.argsort(-deg, kind="stable")[:24]
    empty = np.flatnonzero(deg == 0)[:24]
    rows = np.concatenate([top, empty, rng.choice(deg.size, n_random, replace=False)])
    return np.unique(rows).astype(np.int32)


def test_rmat22_mean(big, hosted):
    import oracle
    agb, wl, g = big
    src, dst, cnt = hosted
    Y = agb.ag_mean_fwd(g, wl.w, wl.X)
    dX, dw = agb.ag_mean_backward(g, wl.w, wl.X, wl.dY)
    torch.cuda.synchronize()
    w, X, dY = host(wl.w), host(wl.X), host(wl.dY)
    rng = np.random.default_rng(5)
    inv = np.divide(1.0, cnt, out=np.zeros(wl.N), where=cnt > 0)
    tol = TOL[torch.bfloat16]
    rows = _rows(rng, cnt)
    ref, bound = oracle.spmm_rows(src, dst, wl.N, w, X, rows, by_source=False, with_bound=True)
    assert_within(Y[torch.from_numpy(rows).long().cuda()], ref * inv[rows, None], bound * inv[rows, None], tol,
                  "rmat22 mean Y rows")
    # dX: the weights w_e / cnt(dst_e) are formed in fp64 and rounded once to
    # fp32 for the oracle's input (relative 2^-24, inside the tolerance)
    w_mean = (w.astype(np.float64) * inv[dst]).astype(np.float32)
    rows_s = _rows(rng, np.bincount(src, minlength=wl.N))
    ref, bound = oracle.spmm_rows(src, dst, wl.N, w_mean, dY, rows_s, by_source=True, with_bound=True)
    assert_within(dX[torch.from_numpy(rows_s).long().cuda()], ref, bound, tol, "rmat22 mean dX rows")
    edges = np.unique(rng.integers(0, wl.E, 200_000))
    ref, bound = oracle.dw_edges(src, dst, wl.N, X, dY, edges, with_bound=True)
    assert_within(dw[torch.from_numpy(edges).cuda()], ref * inv[dst[edges]], bound * inv[dst[edges]], TOL_DW,
                  "rmat22 mean dw edges")


def test_rmat22_gcn_norm_every_edge(big, hosted):
    import oracle
    agb, wl, g = big
    src, dst, _ = hosted
    got = agb.ag_gcn_norm(g)
    wpos = wl.w.abs() + 0.05
    got_w = agb.ag_gcn_norm(g, wpos)
    torch.cuda.synchronize()
    ref = oracle.gcn_norm(src, dst, wl.N)
    assert_within(got, ref, np.abs(ref), 1e-6, "rmat22 gcn unit")
    ref_w = oracle.gcn_norm(src, dst, wl.N, host(wpos))
    assert_within(got_w, ref_w, np.abs(ref_w), 1e-5, "rmat22 gcn weighted")


def test_rmat22_attention(big, hosted):
    import oracle
    agb, wl, g = big
    src, dst, cnt = hosted
    H = wl.H
    mk = lambda s: workloads.features(wl.N, H, torch.bfloat16, 11000 + s, "cuda")
    Q, K, V, G = mk(1), mk(2), mk(3), mk(4)
    scale = 1.0 / np.sqrt(H)
    Y, alpha = agb.ag_attn_fwd(g, Q, K, V, scale)
    dQ, dK, dV = agb.ag_attn_backward(g, Q, K, V, scale, alpha, G)
    torch.cuda.synchronize()
    # alpha: a distribution on every row with edges
    sums = torch.zeros(wl.N, dtype=torch.float64, device="cuda").index_add_(0, wl.dst.long(), alpha.double())
    has = torch.from_numpy(cnt > 0).cuda()
    assert (alpha >= 0).all()
    assert torch.allclose(sums[has], torch.ones_like(sums[has]), atol=1e-4)
    rng = np.random.default_rng(9)
    rows_r = _rows(rng, cnt, 600)
    outdeg = np.bincount(src, minlength=wl.N)
    rows_s = np.unique(np.concatenate([np.argsort(-outdeg, kind="stable")[:4], np.flatnonzero(outdeg == 0)[:16],
                                       rng.choice(wl.N, 150, replace=False)])).astype(np.int32)
    hQ, hK, hV, hG = host(Q), host(K), host(V), host(G)
    o = oracle.attn_sampled(src, dst, wl.N, hQ, hK, hV, scale, hG, rows_r, rows_s)
    nq = np.sqrt((hQ.astype(np.float64) ** 2).sum(1)).max()
    nk = np.sqrt((hK.astype(np.float64) ** 2).sum(1)).max()
    rel = np.expm1(2e-5 * scale * nq * nk) + 1e-6 * (8 + cnt.max() / 256)
    tol = TOL[torch.bfloat16]
    ir = torch.from_numpy(rows_r).long().cuda()
    js = torch.from_numpy(rows_s).long().cuda()
    assert_within(Y[ir], o["Y"], o["absY"] * (rel + tol), 1.0, "rmat22 attention Y rows")
    assert_within(dQ[ir], o["dQ"], o["absdQ"] * (2 * rel + 3e-5 + tol), 1.0, "rmat22 attention dQ rows")
    assert_within(dK[js], o["dK"], o["absdK"] * (2 * rel + 3e-5 + tol), 1.0, "rmat22 attention dK rows")
    assert_within(dV[js], o["dV"], o["absdV"] * (rel + tol), 1.0, "rmat22 attention dV rows")
