"""Parity of the mean aggregation and the GCN-normalised weights (CUDA path
through the C ABI) with the fp64 oracle.

Mean: the CUDA path scales by 1 / in-degree once per row (forward) or per
edge (backward), either as a product with the fp32 reciprocal (two
roundings, relative 2^-23) or as an IEEE division while regrouping (one,
2^-24), around the weighted-sum walks, so the weighted-sum tolerances apply
unchanged to the degree-scaled bounds the oracle returns.  GCN weights: with unit weights
the degrees are exact integers and the result carries four fp32 roundings
(sqrt, division, two products): relative 1e-6.  With weights, the degree is
an fp32 sum over the row (the width-1 SpMM, error within 1e-5 of the sum of
the positive weights), so 1e-5 relative.
"""
import numpy as np
import pytest
import torch

import workloads
from tests.gpu_helpers import TOL, TOL_DW, assert_within, bits, host, lib

pytestmark = pytest.mark.gpu

DEV = "cuda"
TOL_GCN_UNIT = 1e-6
TOL_GCN_WEIGHTED = 1e-5


@pytest.fixture(scope="module")
def agb():
    return lib()


def _bf16_twin(wl):
    return workloads.Workload(wl.name + "-bf16", wl.N, wl.E, wl.H, torch.bfloat16, wl.src, wl.dst, wl.w,
                              wl.X.bfloat16(), wl.dY.bfloat16())


@pytest.fixture(scope="module", params=["uniform", "sbm", "rmat16", "twohop", "rmat16-bf16"])
def config(request, agb):
    name = request.param.replace("-bf16", "")
    wl = workloads.make(name, seed=2, device=DEV)
    if request.param.endswith("-bf16"):
        wl = _bf16_twin(wl)
    return wl, agb.ag_graph_lower(wl.src, wl.dst, wl.N)


def test_mean_forward_and_gradients(agb, config):
    import oracle
    wl, g = config
    src, dst, w, X, dY = host(wl.src), host(wl.dst), host(wl.w), host(wl.X), host(wl.dY)
    tol = TOL[wl.feature_dtype]
    Y = agb.ag_mean_fwd(g, wl.w, wl.X)
    dX, dw = agb.ag_mean_backward(g, wl.w, wl.X, wl.dY)
    torch.cuda.synchronize()
    rY, bY = oracle.mean_fwd(src, dst, wl.N, w, X, with_bound=True)
    rX, bX = oracle.mean_dx(src, dst, wl.N, w, dY, with_bound=True)
    rw, bw = oracle.mean_dw(src, dst, wl.N, X, dY, with_bound=True)
    assert_within(Y, rY, bY, tol, f"{wl.name} mean Y")
    assert_within(dX, rX, bX, tol, f"{wl.name} mean dX")
    assert_within(dw, rw, bw, TOL_DW, f"{wl.name} mean dw")
    # without the weight gradient: the same dX bit for bit
    dX2, none = agb.ag_mean_backward(g, wl.w, wl.X, wl.dY, want_dw=False)
    torch.cuda.synchronize()
    assert none is None
    assert torch.equal(bits(dX2), bits(dX))


def test_mean_unit_weights(agb, config):
    import oracle
    wl, g = config
    src, dst, X, dY = host(wl.src), host(wl.dst), host(wl.X), host(wl.dY)
    ones = np.ones(wl.E, np.float32)
    tol = TOL[wl.feature_dtype]
    Y = agb.ag_mean_fwd(g, None, wl.X)
    dX, dw = agb.ag_mean_backward(g, None, wl.X, wl.dY)
    torch.cuda.synchronize()
    rY, bY = oracle.mean_fwd(src, dst, wl.N, ones, X, with_bound=True)
    rX, bX = oracle.mean_dx(src, dst, wl.N, ones, dY, with_bound=True)
    rw, bw = oracle.mean_dw(src, dst, wl.N, X, dY, with_bound=True)
    assert_within(Y, rY, bY, tol, f"{wl.name} unit mean Y")
    assert_within(dX, rX, bX, tol, f"{wl.name} unit mean dX")
    assert_within(dw, rw, bw, TOL_DW, f"{wl.name} unit mean dw")


@pytest.mark.parametrize("H,dtype", [(1, torch.float32), (5, torch.bfloat16), (17, torch.float32),
                                     (96, torch.bfloat16)])
def test_mean_narrow_and_ragged_widths(agb, H, dtype):
    import oracle
    rng = np.random.default_rng(100 + H)
    N, E = 800, 7000
    src = np.concatenate([rng.integers(0, N, E), np.full(1200, 9)])
    dst = np.concatenate([rng.integers(0, N, E), rng.integers(0, 40, 1200)])
    wl = workloads.custom(N, src, dst, H, seed=H, feature_dtype=dtype, device=DEV)
    g = agb.ag_graph_lower(wl.src, wl.dst, N)
    Y = agb.ag_mean_fwd(g, wl.w, wl.X)
    dX, dw = agb.ag_mean_backward(g, wl.w, wl.X, wl.dY)
    torch.cuda.synchronize()
    s, d = host(wl.src), host(wl.dst)
    hw, hX, hdY = host(wl.w), host(wl.X), host(wl.dY)
    tol = TOL[dtype]
    rY, bY = oracle.mean_fwd(s, d, N, hw, hX, with_bound=True)
    rX, bX = oracle.mean_dx(s, d, N, hw, hdY, with_bound=True)
    rw, bw = oracle.mean_dw(s, d, N, hX, hdY, with_bound=True)
    assert_within(Y, rY, bY, tol, f"H={H} mean Y")
    assert_within(dX, rX, bX, tol, f"H={H} mean dX")
    assert_within(dw, rw, bw, TOL_DW, f"H={H} mean dw")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_mean_of_unit_in_degree_equals_weighted_sum(agb, dtype):
    # every node receives exactly one edge: mean == sum, bit for bit
    N, H = 3000, 64
    rng = np.random.default_rng(3)
    src = rng.permutation(N)
    dst = np.arange(N)
    wl = workloads.custom(N, src, dst, H, seed=5, feature_dtype=dtype, device=DEV)
    g = agb.ag_graph_lower(wl.src, wl.dst, N)
    Y1 = agb.ag_mean_fwd(g, wl.w, wl.X)
    Y2 = agb.ag_spmm_fwd(g, wl.w, wl.X)
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2)


def _with_self_loops(wl):
    n = torch.arange(wl.N, dtype=torch.int32, device=wl.src.device)
    src = torch.cat([wl.src, n])
    dst = torch.cat([wl.dst, n])
    w = torch.cat([wl.w.abs() + 0.05, torch.ones(wl.N, device=wl.w.device)])
    return src, dst, w


@pytest.mark.parametrize("name", ["uniform", "sbm", "rmat16", "twohop"])
def test_gcn_norm_matches_oracle(agb, name):
    import oracle
    wl = workloads.make(name, seed=3, device=DEV)
    src, dst, w = _with_self_loops(wl)
    g = agb.ag_graph_lower(src, dst, wl.N)
    hs, hd, hw = host(src), host(dst), host(w)
    unit = agb.ag_gcn_norm(g)
    weighted = agb.ag_gcn_norm(g, w)
    torch.cuda.synchronize()
    ru = oracle.gcn_norm(hs, hd, wl.N)
    rw = oracle.gcn_norm(hs, hd, wl.N, hw)
    assert_within(unit, ru, np.abs(ru), TOL_GCN_UNIT, f"{name} gcn unit")
    assert_within(weighted, rw, np.abs(rw), TOL_GCN_WEIGHTED, f"{name} gcn weighted")
    # the normalised weights feed the ordinary SpMM: GCN's A_hat X
    Y = agb.ag_spmm_fwd(g, weighted, wl.X)
    torch.cuda.synchronize()
    rY, bY = oracle.fwd(hs, hd, wl.N, rw.astype(np.float32), host(wl.X), with_bound=True)
    assert_within(Y, rY, bY, TOL[wl.feature_dtype], f"{name} gcn Y")


def test_gcn_norm_without_self_loops_zeroes_sources_without_inputs(agb):
    import oracle
    src = np.array([0, 1, 2, 3, 3], np.int32)
    dst = np.array([1, 2, 1, 1, 2], np.int32)   # nodes 0 and 3 receive nothing
    s_t = torch.tensor(src, device=DEV)
    d_t = torch.tensor(dst, device=DEV)
    g = agb.ag_graph_lower(s_t, d_t, 4)
    got = agb.ag_gcn_norm(g)
    torch.cuda.synchronize()
    want = oracle.gcn_norm(src, dst, 4)
    assert_within(got, want, np.abs(want) + 1e-30, TOL_GCN_UNIT, "gcn zero-degree")
    assert got[0].item() == 0.0 and got[3].item() == 0.0 and got[4].item() == 0.0


def test_mean_and_gcn_empty_graph(agb):
    z = torch.zeros(0, dtype=torch.int32, device=DEV)
    g = agb.ag_graph_lower(z, z, 5)
    X = torch.randn(5, 8, device=DEV)
    Y = agb.ag_mean_fwd(g, torch.zeros(0, device=DEV), X)
    dX, dw = agb.ag_mean_backward(g, torch.zeros(0, device=DEV), X, X)
    out = agb.ag_gcn_norm(g)
    torch.cuda.synchronize()
    assert not Y.any() and not dX.any() and dw.numel() == 0 and out.numel() == 0


def test_mean_rejects_bad_arguments(agb):
    wl = workloads.make("uniform", seed=1, device=DEV)
    g = agb.ag_graph_lower(wl.src, wl.dst, wl.N)
    with pytest.raises(agb.AggraphError):
        agb.ag_mean_fwd(g, wl.w[:-1], wl.X)
    with pytest.raises(agb.AggraphError):
        agb.ag_gcn_norm(g, wl.w.double())
