"""ag_spmm_fwd_static_scratch: the forward aggregation with the library's
built-in scratch array instead of caller scratch.

It serves callers that cannot allocate device memory when they call: code
running while a framework owns the allocator (allocating behind its back can
fail or fragment its pool), latency-critical paths where cudaMalloc and
cudaFree may synchronize the device, and plug-in hooks that are handed only
their input and output buffers.  Its output must match ag_spmm_fwd, the entry
point that takes caller scratch, on two calls in a row (the second call finds
the array holding the first call's contents).
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads
from tests.gpu_helpers import TOL, lib

pytestmark = pytest.mark.gpu


def _static_fwd(agb, g, w, X, Y):
    code = agb.AG_F32 if X.dtype == torch.float32 else agb.AG_BF16
    return agb.lib.ag_spmm_fwd_static_scratch(
        g.handle, ctypes.c_void_p(w.data_ptr()), ctypes.c_void_p(X.data_ptr()),
        ctypes.c_void_p(Y.data_ptr()), X.shape[1], code,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _skewed(N=3000, E=40000, seed=3):
    rng = np.random.default_rng(seed)
    src = np.concatenate([rng.integers(0, N, E), rng.integers(0, N, 3000)]).astype(np.int32)
    dst = np.concatenate([rng.integers(0, N // 2, E), np.full(3000, 7)]).astype(np.int32)
    return N, src, dst


@pytest.mark.parametrize("case", ["rmat16-f32-h128", "skewed-bf16-h64", "skewed-f32-h256"])
def test_matches_caller_scratch_forward_on_two_calls(case):
    agb = lib()
    if case == "rmat16-f32-h128":
        wl = workloads.make("rmat16", seed=2, device="cuda")
    else:
        N, src, dst = _skewed()
        dtype = torch.bfloat16 if "bf16" in case else torch.float32
        H = 64 if "h64" in case else 256
        wl = workloads.custom(N, src, dst, H, seed=9, feature_dtype=dtype, device="cuda")
    g = agb.ag_graph_lower(wl.src, wl.dst, wl.N)
    assert g.scratch_bytes(wl.H) > 0                        # this graph needs scratch
    ref = agb.ag_spmm_fwd(g, wl.w, wl.X)
    # elementwise scale of the tolerance: sum over in-edges of |w_e x|
    bound = agb.ag_spmm_fwd(g, wl.w.abs(), wl.X.abs()).double()
    tol = TOL[wl.feature_dtype]
    for _ in range(2):
        Y = torch.full_like(wl.X, float("nan"))
        assert _static_fwd(agb, g, wl.w, wl.X, Y) == 0, agb.lib.ag_last_error()
        torch.cuda.synchronize()
        err = (Y.double() - ref.double()).abs()
        assert bool(torch.all(err <= tol * bound)), float(err.max())


def test_rejects_a_graph_too_large_for_the_builtin_array():
    agb = lib()
    wl = workloads.make("rmat16", seed=2, device="cuda")
    g = agb.ag_graph_lower(wl.src, wl.dst, wl.N)
    H = 1024
    X = torch.zeros((wl.N, H), device="cuda")
    Y = torch.zeros_like(X)
    assert g.scratch_bytes(H) > agb.lib.ag_spmm_static_scratch_capacity()
    assert _static_fwd(agb, g, wl.w, X, Y) == 7          # AG_ERR_WORKSPACE, nothing launched
    assert b"built-in" in agb.lib.ag_last_error()
