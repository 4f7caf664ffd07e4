"""ag_spmm_fwd_static_scratch: the forward aggregation with the library's
built-in scratch array instead of caller scratch.

It serves callers that cannot allocate device memory when they call: code
running while a framework owns the allocator (allocating behind its back can
fail or fragment its pool), latency-critical paths where cudaMalloc and
cudaFree may synchronize the device, and plug-in hooks that are handed only
their input and output buffers.  On two calls in a row (the second call finds
the array holding the first call's contents) its output must equal, bit for
bit, that of ag_spmm_fwd, the entry point that takes caller scratch (both run
the same kernels in the same order), and must agree with the fp64 oracle
within the tolerance of the other parity tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_helpers import TOL, assert_within, bits, host, lib

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
    assert g.stats["spanning_rows_f"] > 0                   # and uses the partial rows in it
    ref = agb.ag_spmm_fwd(g, wl.w, wl.X)
    # the fp64 oracle and its per-element bound sum over in-edges of |w_e x|
    want, bound = oracle.fwd(host(wl.src), host(wl.dst), wl.N, host(wl.w), host(wl.X), with_bound=True)
    for call in range(2):
        Y = torch.full_like(wl.X, float("nan"))
        torch.cuda.synchronize()
        free0, held0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
        assert _static_fwd(agb, g, wl.w, wl.X, Y) == 0, agb.lib.ag_last_error()
        torch.cuda.synchronize()
        if call == 1:  # the first call may still load the library's kernels; the second allocates nothing
            assert torch.cuda.mem_get_info()[0] == free0 and torch.cuda.memory_allocated() == held0
        assert torch.equal(bits(Y), bits(ref)), f"call {call}: differs from ag_spmm_fwd"
        assert_within(Y, want, bound, TOL[wl.feature_dtype], f"{case} call {call}")


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
