"""Full-size R-MAT scale-22 graph (4,194,304 nodes, 67,108,864 edges, H = 128,
bf16 features with fp32 accumulation), run exactly as the benchmark runs it.

The oracle checks the whole lowering bit-exactly, and the floating-point
outputs on sampled rows and edges it computes one by one: the heaviest rows
(split into chunks), empty rows and random rows of Y and dX, and random edges
of dw.  The adjoint identity <Y, dY> = <X, dX> = sum_e w_e dw_e checks every
output at once.
"""
import numpy as np
import pytest
import torch

import workloads
from tests.gpu_helpers import TOL, TOL_DW, assert_within, check_lowering, host, lib, run_path

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def big():
    agb = lib()
    wl = workloads.make("rmat22", seed=1, device="cuda")
    g = agb.ag_graph_lower(wl.src, wl.dst, wl.N)
    outs = run_path(g, wl)
    return wl, g, outs


@pytest.fixture(scope="module")
def host_inputs(big):
    wl, _, _ = big
    return host(wl.src), host(wl.dst), host(wl.w), host(wl.X), host(wl.dY)


def test_rmat22_shape_and_schedule(big):
    wl, g, _ = big
    assert (wl.N, wl.E, wl.H, wl.feature_dtype) == (1 << 22, 1 << 26, 128, torch.bfloat16)
    s = g.stats
    assert s["tile_edges"] == 256 and s["tiles"] == wl.E // 256
    assert s["long_spanning_rows_f"] > 100 and s["max_degree_f"] > 100_000
    assert 0 < s["nonempty_rows_f"] < wl.N


def test_rmat22_lowering_bit_exact(big):
    wl, g, _ = big
    check_lowering(g, wl)


def _sample_rows(rowptr: np.ndarray, rng, n_random=3000):
    deg = np.diff(rowptr.astype(np.int64))
    top = np.argsort(-deg, kind="stable")[:48]
    empty = np.flatnonzero(deg == 0)[:48]
    light = np.flatnonzero((deg > 0) & (deg <= 256))
    rows = np.concatenate([top, empty, rng.choice(light, 400, replace=False),
                           rng.choice(deg.size, n_random, replace=False)])
    return np.unique(rows).astype(np.int32)


def test_rmat22_sampled_rows_and_edges(big, host_inputs):
    import oracle
    wl, g, (Y, dX, dw) = big
    src, dst, w, X, dY = host_inputs
    arr = g.arrays()
    rng = np.random.default_rng(22)
    tol = TOL[torch.bfloat16]
    rows_f = _sample_rows(arr["rowptr_f"].cpu().numpy(), rng)
    ref, bound = oracle.spmm_rows(src, dst, wl.N, w, X, rows_f, by_source=False, with_bound=True)
    assert_within(Y[torch.from_numpy(rows_f).long().cuda()], ref, bound, tol, "rmat22 fwd rows")
    rows_t = _sample_rows(arr["rowptr_t"].cpu().numpy(), rng)
    ref, bound = oracle.spmm_rows(src, dst, wl.N, w, dY, rows_t, by_source=True, with_bound=True)
    assert_within(dX[torch.from_numpy(rows_t).long().cuda()], ref, bound, tol, "rmat22 dX rows")
    edges = np.unique(rng.integers(0, wl.E, 300_000))
    # and every edge of the heaviest source row (it is cut into many tiles)
    rp = arr["rowptr_t"].cpu().numpy().astype(np.int64)
    hub = int(np.argmax(np.diff(rp)))
    hub_edges = arr["transpose_order"][rp[hub]:rp[hub + 1]].cpu().numpy()
    edges = np.unique(np.concatenate([edges, hub_edges]))
    ref, bound = oracle.dw_edges(src, dst, wl.N, X, dY, edges, with_bound=True)
    assert_within(dw[torch.from_numpy(edges).cuda()], ref, bound, TOL_DW, "rmat22 dw edges")


def test_rmat22_adjoint_identity(big):
    wl, g, (Y, dX, dw) = big
    a = torch.sum(Y.double() * wl.dY.double()).item()
    b = torch.sum(wl.X.double() * dX.double()).item()
    c = torch.sum(wl.w.double() * dw.double()).item()
    scale = (torch.sum(Y.double().abs() * wl.dY.double().abs()).item()
             + torch.sum(wl.X.double().abs() * dX.double().abs()).item())
    # bf16 outputs are rounded once (relative 2^-8); fp32 accumulation adds far less
    assert abs(a - c) <= 1e-2 * scale
    assert abs(b - c) <= 1e-2 * scale
    assert np.isfinite([a, b, c]).all()


def test_rmat22_fused_backward_matches(big):
    from tests.gpu_helpers import check_fused_backward
    wl, g, (Y, dX, dw) = big
    check_fused_backward(g, wl, dX, dw)


def test_rmat22_bitwise_reproducible(big):
    wl, g, outs = big
    again = run_path(g, wl)
    for x, y in zip(outs, again):
        if x.dtype == torch.bfloat16:
            x, y = x.view(torch.int16), y.view(torch.int16)
        assert torch.equal(x, y)
