"""Shared helpers of the GPU parity tests (imported only by test files)."""
from __future__ import annotations

import numpy as np
import torch

# Tolerances of the comparison with the fp64 oracle, per output element:
# |gpu - oracle| <= TOL * sum of |terms| of that element (sum_e |w_e x| for
# the SpMMs, sum_h |x dy| for dw).  fp32 features: 1e-5; bf16 features
# (fp32 accumulation, bf16 output rounded once): 1e-2.
TOL = {torch.float32: 1e-5, torch.bfloat16: 1e-2}
# dw is always an fp32 output; with bf16 inputs its only error is the fp32
# accumulation, so the fp32 tolerance applies to it in both cases.
TOL_DW = 1e-5


def lib():
    from __graft_entry__ import build_library
    build_library()
    import gnn_sparse_aggregation_b200 as agb
    return agb


def host(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        t = t.float()  # exact
    return t.numpy()


def assert_within(gpu: torch.Tensor, ref: np.ndarray, bound: np.ndarray, tol: float, what: str):
    got = gpu.detach().double().cpu().numpy()
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    err = np.abs(got - ref)
    lim = tol * bound
    bad = ~(err <= lim)          # NaN counts as bad
    if bad.any():
        idx = np.argwhere(bad)[:5]
        detail = ", ".join(f"{tuple(i)}: got {got[tuple(i)]!r} want {ref[tuple(i)]!r} bound {bound[tuple(i)]!r}"
                           for i in idx)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} elements outside "
                             f"tol {tol} x bound; {detail}")


def run_path(g, wl, stream=None):
    Y = g.fwd(wl.w, wl.X, stream=stream)
    dX = g.dx(wl.w, wl.dY, stream=stream)
    dw = g.dw(wl.X, wl.dY, stream=stream)
    torch.cuda.synchronize()
    return Y, dX, dw


def bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


def check_fused_backward(g, wl, dX, dw):
    """ag_backward must reproduce ag_spmm_dx and ag_sddmm_dw bit for bit."""
    fdX, fdw = g.backward(wl.w, wl.X, wl.dY)
    torch.cuda.synchronize()
    assert torch.equal(bits(fdX), bits(dX)), "fused dX differs from ag_spmm_dx"
    assert torch.equal(bits(fdw), bits(dw)), "fused dw differs from ag_sddmm_dw"


def oracle_full(wl):
    import oracle
    src, dst = host(wl.src), host(wl.dst)
    w, X, dY = host(wl.w), host(wl.X), host(wl.dY)
    Y, BY = oracle.fwd(src, dst, wl.N, w, X, with_bound=True)
    dX, BX = oracle.dx(src, dst, wl.N, w, dY, with_bound=True)
    dw, Bw = oracle.dw(src, dst, wl.N, X, dY, with_bound=True)
    return (Y, BY), (dX, BX), (dw, Bw)


def check_full(g, wl, what=""):
    """Whole-output comparison of fwd, dX and dw with the fp64 oracle."""
    Y, dX, dw = run_path(g, wl)
    (rY, bY), (rX, bX), (rw, bw) = oracle_full(wl)
    tol = TOL[wl.feature_dtype]
    assert_within(Y, rY, bY, tol, f"{what} fwd")
    assert_within(dX, rX, bX, tol, f"{what} dX")
    assert_within(dw, rw, bw, TOL_DW, f"{what} dw")
    check_fused_backward(g, wl, dX, dw)
    return Y, dX, dw


def check_lowering(g, wl):
    import oracle
    ref = oracle.lower(host(wl.src), host(wl.dst), wl.N)
    arr = g.arrays()
    for k, v in ref.items():
        got = arr[k].cpu().numpy()
        assert np.array_equal(got, v), f"{k} differs at {np.flatnonzero(got != v)[:5]}"
