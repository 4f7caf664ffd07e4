"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Element-by-element at every size the oracle finishes in seconds (all of the
uniform, SBM, R-MAT-16 and 2-hop configurations, the page's witness and its
edge cases, ragged widths and tails), bit-exact for the lowering, and within
the stated tolerance for the floating-point outputs.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads
from tests.gpu_helpers import TOL, TOL_DW, assert_within, check_full, check_lowering, host, lib, run_path
from tests.gpu_helpers import oracle_full as oracle_full_of
from tests.golden import load

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def agb():
    return lib()


# ----------------------------------------------------------------------------- witness

def test_witness_through_the_c_abi(agb):
    g0 = load("witness_3edge.txt")
    N = g0["N"]
    src = torch.tensor(g0["src"], dtype=torch.int32, device=DEV)
    dst = torch.tensor(g0["dst"], dtype=torch.int32, device=DEV)
    w = torch.tensor(g0["w"], dtype=torch.float32, device=DEV)
    X = torch.tensor(g0["X"], dtype=torch.float32, device=DEV).reshape(N, 1)
    dY = torch.tensor(g0["dY"], dtype=torch.float32, device=DEV).reshape(N, 1)
    g = agb.ag_graph_lower(src, dst, N)
    arr = g.arrays()
    for k in ("edge_order", "rowptr_f", "col_f", "transpose_order", "rowptr_t", "col_t"):
        assert arr[k].cpu().tolist() == g0[k].astype(int).tolist(), k
    Y = agb.ag_spmm_fwd(g, w, X)
    dX = agb.ag_spmm_dx(g, w, dY)
    dw = agb.ag_sddmm_dw(g, X, dY)
    torch.cuda.synchronize()
    assert Y[:, 0].cpu().tolist() == g0["Y"].tolist()
    assert dX[:, 0].cpu().tolist() == g0["dX"].tolist()
    assert dw.cpu().tolist() == g0["dw"].tolist()
    # the same through bf16 features (all values are exact in bf16)
    Yb = agb.ag_spmm_fwd(g, w, X.bfloat16())
    dXb = agb.ag_spmm_dx(g, w, dY.bfloat16())
    dwb = agb.ag_sddmm_dw(g, X.bfloat16(), dY.bfloat16())
    torch.cuda.synchronize()
    assert Yb[:, 0].float().cpu().tolist() == g0["Y"].tolist()
    assert dXb[:, 0].float().cpu().tolist() == g0["dX"].tolist()
    assert dwb.cpu().tolist() == g0["dw"].tolist()


# ----------------------------------------------------------------------------- configurations

@pytest.fixture(scope="module", params=["uniform", "sbm", "rmat16", "twohop"])
def config(request, agb):
    wl = workloads.make(request.param, seed=1, device=DEV)
    return wl, agb.ag_graph_lower(wl.src, wl.dst, wl.N)


def test_config_lowering_bit_exact(config):
    wl, g = config
    check_lowering(g, wl)


def test_config_full_parity(config):
    wl, g = config
    check_full(g, wl, wl.name)


def test_config_bitwise_reproducible(config):
    wl, g = config
    a = run_path(g, wl)
    sc = g.scratch(wl.H)
    if sc is not None:
        sc.fill_(0x7f)        # stale scratch contents must not leak into the result
    b = run_path(g, wl)
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.uint8) if x.dtype == torch.bfloat16 else x,
                           y.view(torch.uint8) if y.dtype == torch.bfloat16 else y)


def test_config_no_edge_feature_temporary(config):
    """No [E, H] carrier: the per-call scratch holds two fp32 rows per tile for
    rows cut by tile boundaries, two float [E] buffers and one float [N],
    far below E x H (witness section: no buffer larger than the per-node,
    per-edge or row-pointer arrays is allowed)."""
    wl, g = config
    s = g.stats
    spans = s["spanning_rows_f"] + s["spanning_rows_t"]
    rnd = lambda b: (b + 255) // 256 * 256
    assert g.scratch_bytes(wl.H) == (rnd(2 * 4 * wl.H * s["tiles"] if spans else 0) + 2 * rnd(4 * wl.E)
                                     + rnd(4 * wl.N))
    assert g.scratch_bytes(wl.H) < wl.E * wl.H * 4 // 4
    assert g.workspace.numel() < 80 * (wl.N + wl.E) + (1 << 16)


def test_rmat16_has_long_spanning_rows(config):
    wl, g = config
    if wl.name != "rmat16":
        pytest.skip("rows cut into many tiles are exercised by the R-MAT graph")
    s = g.stats
    assert s["long_spanning_rows_f"] > 0 and s["spanning_rows_f"] > s["long_spanning_rows_f"]
    assert s["long_spanning_rows_t"] > 0 and s["max_degree_f"] > 5000


# ----------------------------------------------------------------------------- edge cases

def graph(agb, N, src, dst, H, dtype=torch.float32, seed=5, wdist="normal"):
    wl = workloads.custom(N, src, dst, H, seed=seed, feature_dtype=dtype, wdist=wdist, device=DEV)
    return wl, agb.ag_graph_lower(wl.src, wl.dst, wl.N)


def skewed_edges(N=3000, E=40000, seed=3):
    """Random edges plus a hub with 3,000 in-edges and one with 2,500 out-edges
    (both cut into many tiles), duplicates, self-loops and many empty rows."""
    rng = np.random.default_rng(seed)
    src = rng.integers(0, N // 3, E)
    dst = rng.integers(0, N // 2, E)
    src = np.concatenate([src, rng.integers(0, N, 3000), np.full(2500, 11)])
    dst = np.concatenate([dst, np.full(3000, 7), rng.integers(0, N, 2500)])
    src = np.concatenate([src, [5, 5, 5, 9]])
    dst = np.concatenate([dst, [6, 6, 6, 9]])
    perm = rng.permutation(src.size)
    return N, src[perm].astype(np.int32), dst[perm].astype(np.int32)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("H", [1, 2, 3, 4, 5, 8, 12, 16, 33, 64, 128, 130, 133, 256, 520, 1000, 2056])
def test_widths_and_split_rows(agb, H, dtype):
    N, src, dst = skewed_edges()
    wl, g = graph(agb, N, src, dst, H, dtype)
    assert g.stats["long_spanning_rows_f"] >= 1 and g.stats["long_spanning_rows_t"] >= 1
    check_full(g, wl, f"H={H} {dtype}")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_unaligned_feature_pointers_take_the_narrow_path(agb, dtype):
    N, src, dst = skewed_edges(N=500, E=6000)
    H = 64
    wl, g = graph(agb, N, src, dst, H, dtype)
    elem = 4 if dtype == torch.float32 else 2
    off = 1 if dtype == torch.float32 else 1      # one element: breaks 16-byte alignment
    big = torch.zeros(N * H + off, dtype=dtype, device=DEV)
    Xu = big[off:].view(N, H)
    Xu.copy_(wl.X)
    assert Xu.data_ptr() % 16 == elem * off % 16 != 0
    Y = g.fwd(wl.w, Xu)
    ref = g.fwd(wl.w, wl.X)
    torch.cuda.synchronize()
    # The aligned input takes the shared-memory ring walk of 16-byte vectors,
    # the unaligned one a register walk of narrower vectors.  Any summation
    # order is acceptable within the tolerance (fp32 accumulation against the
    # fp64 oracle), so both are checked there, and each must reproduce itself
    # bit for bit.
    import oracle
    want, bound = oracle.fwd(host(wl.src), host(wl.dst), N, host(wl.w), host(wl.X), with_bound=True)
    assert_within(Y, want, bound, TOL[dtype], "narrow path")
    assert_within(ref, want, bound, TOL[dtype], "wide path")
    Y2 = g.fwd(wl.w, Xu)
    torch.cuda.synchronize()
    assert torch.equal(Y2.float(), Y.float())


def _rows_per_tile_graph(kind, rng):
    N = 6000
    if kind == "unit_rows":      # in-degree 1: a new row at every position
        dst = rng.permutation(N)
    elif kind == "short_rows":   # in-degree 1..3 with empty rows between
        nodes = rng.choice(N, N // 2, replace=False)
        dst = np.repeat(nodes, rng.integers(1, 4, nodes.size))
    else:                        # one row cut by many tiles among rows of in-degree 1 and 9
        dst = np.concatenate([np.full(30000, 17), np.arange(0, N, 3), np.repeat(np.arange(1, N, 7), 9)])
    src = rng.integers(0, N, dst.size)
    perm = rng.permutation(dst.size)
    return N, src[perm].astype(np.int32), dst[perm].astype(np.int32)


@pytest.mark.parametrize("H", [64, 128])
@pytest.mark.parametrize("kind", ["unit_rows", "short_rows", "heavy_and_unit"])
def test_rows_per_tile_extremes(agb, H, kind):
    """bf16 rows of 64 and 128 features (the ring walks) on the extremes of
    rows per tile: every row a single edge (a row switch at every position),
    short rows with empty rows between them, and a row cut by many tiles among
    one-edge rows."""
    rng = np.random.default_rng(H + len(kind))
    N, src, dst = _rows_per_tile_graph(kind, rng)
    wl, g = graph(agb, N, src, dst, H, torch.bfloat16)
    check_full(g, wl, f"{kind} H={H}")


def test_empty_graph_and_one_node(agb):
    # E = 0: outputs are exact zeros, dw is empty
    wl, g = graph(agb, 9, [], [], 6)
    check_lowering(g, wl)
    Y, dX, dw = run_path(g, wl)
    assert torch.count_nonzero(Y) == 0 and torch.count_nonzero(dX) == 0 and dw.numel() == 0
    # N = 1 without and with a self-loop
    wl, g = graph(agb, 1, [], [], 4)
    Y, dX, dw = run_path(g, wl)
    assert torch.count_nonzero(Y) == 0 and dw.numel() == 0
    wl, g = graph(agb, 1, [0], [0], 4)
    check_lowering(g, wl)
    check_full(g, wl, "one node self-loop")


def test_isolated_rows_and_duplicates(agb):
    src = [1, 1, 2, 1, 4, 4]
    dst = [3, 3, 0, 3, 4, 0]
    wl, g = graph(agb, 8, src, dst, 5)
    check_lowering(g, wl)
    Y, dX, dw = check_full(g, wl, "duplicates")
    for r in (1, 2, 5, 6, 7):
        assert torch.count_nonzero(Y[r]) == 0
    for r in (0, 3, 5, 6, 7):
        assert torch.count_nonzero(dX[r]) == 0
    assert dw[0] == dw[1] == dw[3]


def test_all_edges_into_one_node(agb):
    E = 20000
    rng = np.random.default_rng(1)
    wl, g = graph(agb, 50, rng.integers(0, 50, E), np.full(E, 42), 32)
    assert g.stats["max_degree_f"] == E
    check_lowering(g, wl)
    check_full(g, wl, "star")


def test_many_nodes_few_edges(agb):
    wl, g = graph(agb, 200_000, [3, 199_999, 17], [199_998, 0, 17], 8)
    check_lowering(g, wl)
    check_full(g, wl, "sparse")


def test_paired_permutation_keeps_outputs(agb):
    """Permuting src, dst and w together leaves Y and dX unchanged (within the
    tolerance: the CSR rows keep the same edges) and permutes dw exactly."""
    import oracle
    N, src, dst = skewed_edges(N=800, E=9000)
    wl, g = graph(agb, N, src, dst, 16)
    Y, dX, dw = run_path(g, wl)
    perm = torch.randperm(wl.E, generator=torch.Generator().manual_seed(0)).to(DEV)
    g2 = agb.ag_graph_lower(wl.src[perm].contiguous(), wl.dst[perm].contiguous(), N)
    Y2 = g2.fwd(wl.w[perm].contiguous(), wl.X)
    dX2 = g2.dx(wl.w[perm].contiguous(), wl.dY)
    dw2 = g2.dw(wl.X, wl.dY)
    torch.cuda.synchronize()
    s_, d_, w_ = host(wl.src), host(wl.dst), host(wl.w)
    _, bY = oracle.fwd(s_, d_, N, w_, host(wl.X), with_bound=True)
    _, bX = oracle.dx(s_, d_, N, w_, host(wl.dY), with_bound=True)
    assert_within(Y2, Y.double().cpu().numpy(), bY, 2 * TOL[torch.float32], "permuted fwd")
    assert_within(dX2, dX.double().cpu().numpy(), bX, 2 * TOL[torch.float32], "permuted dX")
    assert torch.equal(dw2, dw[perm])       # each edge's dot is computed the same way


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("H", [16, 64, 128, 256])
def test_single_walk_backward_on_source_sorted_coo(agb, H, dtype):
    """A COO list sorted by source makes dw writes sector-local, so ag_backward
    takes the single walk; it must still equal the oracle and the separate
    passes bit for bit (check_full compares both)."""
    N, src, dst = skewed_edges()
    order = np.argsort(src, kind="stable")
    wl, g = graph(agb, N, src[order], dst[order], H, dtype)
    assert g.stats["dw_locality"] >= 0.5
    check_full(g, wl, f"sorted H={H} {dtype}")


def test_single_walk_backward_rmat18_sorted(agb):
    src, dst = workloads.rmat_edges(18, 16, seed=4)
    order = torch.argsort(src.long() * (1 << 18) + dst.long())
    wl, g = graph(agb, 1 << 18, src[order].numpy(), dst[order].numpy(), 128, torch.bfloat16)
    assert g.stats["dw_locality"] >= 0.5
    check_full(g, wl, "rmat18 sorted")


def test_random_order_has_low_locality(config):
    wl, g = config
    if wl.name == "twohop":
        pytest.skip("the sampled block lists edges grouped by sampler")
    assert g.stats["dw_locality"] < 0.5


# ----------------------------------------------------------------------------- API behaviour

def test_non_default_stream(agb):
    N, src, dst = skewed_edges(N=600, E=7000)
    wl, g = graph(agb, N, src, dst, 24)
    ref = run_path(g, wl)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out = (g.fwd(wl.w, wl.X, stream=s), g.dx(wl.w, wl.dY, stream=s), g.dw(wl.X, wl.dY, stream=s))
    s.synchronize()
    for a, b in zip(ref, out):
        assert torch.equal(a, b)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_step_from_host_buffers(agb, dtype):
    N, src, dst = skewed_edges(N=1500, E=20000)
    wl, g = graph(agb, N, src, dst, 40, dtype)
    Y, dX, dw = run_path(g, wl)
    hw, hX, hdY = (t.cpu().pin_memory() for t in (wl.w, wl.X, wl.dY))
    hY = torch.empty_like(hX).pin_memory()
    hdX = torch.empty_like(hX).pin_memory()
    hdw = torch.empty_like(hw).pin_memory()
    staging = torch.empty(agb.ag_step_staging_bytes(g, wl.H, dtype), dtype=torch.uint8, device=DEV)
    agb.ag_step_host(g, hw, hX, hdY, hY, hdX, hdw, staging)
    torch.cuda.synchronize()
    assert torch.equal(hY, Y.cpu()) and torch.equal(hdX, dX.cpu()) and torch.equal(hdw, dw.cpu())


def test_step_from_host_buffers_orders_on_the_callers_stream(agb):
    # three steps back to back on one side stream, sharing one staging
    # buffer; only that stream is synchronized, so every copy (including those
    # on the library's helper streams) must be ordered before it
    N, src, dst = skewed_edges(N=1500, E=20000)
    wl, g = graph(agb, N, src, dst, 32, torch.bfloat16)
    staging = torch.empty(agb.ag_step_staging_bytes(g, wl.H, torch.bfloat16), dtype=torch.uint8, device=DEV)
    ins, outs, refs = [], [], []
    for k in range(3):
        w = wl.w * (k + 1)
        X = (wl.X.float() - k).bfloat16()
        dY = (wl.dY.float() + k).bfloat16()
        refs.append(tuple(t.cpu() for t in (g.fwd(w, X), *g.backward(w, X, dY))))
        ins.append(tuple(t.cpu().pin_memory() for t in (w, X, dY)))
        outs.append((torch.empty_like(ins[-1][1]).pin_memory(), torch.empty_like(ins[-1][1]).pin_memory(),
                     torch.empty_like(ins[-1][0]).pin_memory()))
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    for (hw, hX, hdY), (hY, hdX, hdw) in zip(ins, outs):
        agb.ag_step_host(g, hw, hX, hdY, hY, hdX, hdw, staging, stream=s)
    s.synchronize()
    for (hY, hdX, hdw), (Y, dX, dw) in zip(outs, refs):
        assert torch.equal(hY.view(torch.int16), Y.view(torch.int16))
        assert torch.equal(hdX.view(torch.int16), dX.view(torch.int16))
        assert torch.equal(hdw, dw)


@pytest.mark.parametrize("modes", [(True, True, True, True, True), (True, False, True, True, False)])
def test_pipelined_steps_keep_each_steps_results(agb, modes):
    """Back-to-back pipelined steps (mixed with plain ones) on one staging
    buffer and one side stream: each step's inputs come in while the previous
    step's results go out, and every step must still return exactly its own
    results.  Copies of a few MB each, so that the overlap is real."""
    src, dst = workloads.rmat_edges(17, 16, seed=6)
    N = 1 << 17
    wl, g = graph(agb, N, src.numpy(), dst.numpy(), 64, torch.bfloat16)
    staging = torch.empty(agb.ag_step_staging_bytes(g, wl.H, torch.bfloat16), dtype=torch.uint8, device=DEV)
    ins, outs, refs = [], [], []
    for k in range(len(modes)):
        w = wl.w * (k + 1)
        X = (wl.X.float() * (k + 1) - k).bfloat16()
        dY = (wl.dY.float() + k).bfloat16()
        refs.append(tuple(t.cpu() for t in (g.fwd(w, X), *g.backward(w, X, dY))))
        ins.append(tuple(t.cpu().pin_memory() for t in (w, X, dY)))
        outs.append((torch.empty_like(ins[-1][1]).pin_memory(), torch.empty_like(ins[-1][1]).pin_memory(),
                     torch.empty_like(ins[-1][0]).pin_memory()))
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    for pipelined, (hw, hX, hdY), (hY, hdX, hdw) in zip(modes, ins, outs):
        agb.ag_step_host(g, hw, hX, hdY, hY, hdX, hdw, staging, stream=s, pipelined=pipelined)
    s.synchronize()
    for k, ((hY, hdX, hdw), (Y, dX, dw)) in enumerate(zip(outs, refs)):
        assert torch.equal(hY.view(torch.int16), Y.view(torch.int16)), k
        assert torch.equal(hdX.view(torch.int16), dX.view(torch.int16)), k
        assert torch.equal(hdw, dw), k


def test_pipelined_steps_on_two_staging_buffers_and_two_streams(agb):
    """The bench's end-to-end pattern: pipelined steps alternating between two
    staging buffers, each on its own stream, so that a step's copies in and
    compute can overlap the previous step's compute and copies out.  Every
    step must return exactly its own results (different inputs per step)."""
    src, dst = workloads.rmat_edges(17, 16, seed=8)
    N = 1 << 17
    wl, g = graph(agb, N, src.numpy(), dst.numpy(), 64, torch.bfloat16)
    nbytes = agb.ag_step_staging_bytes(g, wl.H, torch.bfloat16)
    stagings = [torch.empty(nbytes, dtype=torch.uint8, device=DEV) for _ in range(2)]
    streams = [torch.cuda.Stream() for _ in range(2)]
    ins, outs, refs = [], [], []
    for k in range(6):
        w = wl.w * (k + 1)
        X = (wl.X.float() * (k + 1) - k).bfloat16()
        dY = (wl.dY.float() + k).bfloat16()
        refs.append(tuple(t.cpu() for t in (g.fwd(w, X), *g.backward(w, X, dY))))
        ins.append(tuple(t.cpu().pin_memory() for t in (w, X, dY)))
        outs.append((torch.empty_like(ins[-1][1]).pin_memory(), torch.empty_like(ins[-1][1]).pin_memory(),
                     torch.empty_like(ins[-1][0]).pin_memory()))
    torch.cuda.synchronize()
    for k, ((hw, hX, hdY), (hY, hdX, hdw)) in enumerate(zip(ins, outs)):
        agb.ag_step_host_pipelined(g, hw, hX, hdY, hY, hdX, hdw, stagings[k % 2], stream=streams[k % 2])
    for st in streams:
        st.synchronize()
    for k, ((hY, hdX, hdw), (Y, dX, dw)) in enumerate(zip(outs, refs)):
        assert torch.equal(hY.view(torch.int16), Y.view(torch.int16)), k
        assert torch.equal(hdX.view(torch.int16), dX.view(torch.int16)), k
        assert torch.equal(hdw, dw), k


def test_pipelined_steps_with_a_new_layout_on_the_same_buffer(agb):
    """Pipelined steps of different widths (and dtypes) back to back on one
    staging buffer: a step whose layout differs from the previous step's must
    not start its copies in before the previous step's copies out are done
    (its input part overlaps the previous step's output part), so every step
    still returns exactly what ag_step_host returns for it alone."""
    src, dst = workloads.rmat_edges(16, 16, seed=7)
    N = 1 << 16
    shapes = ((128, torch.bfloat16), (32, torch.float32), (64, torch.bfloat16), (128, torch.bfloat16))
    g = agb.ag_graph_lower(torch.from_numpy(src.numpy()).to(DEV), torch.from_numpy(dst.numpy()).to(DEV), N)
    big = max(agb.ag_step_staging_bytes(g, H, dt) for H, dt in shapes)
    staging = torch.empty(big, dtype=torch.uint8, device=DEV)
    ins, outs, refs = [], [], []
    for k, (H, dt) in enumerate(shapes):
        wl = workloads.custom(N, src.numpy(), dst.numpy(), H, seed=20 + k, feature_dtype=dt, device=DEV)
        refs.append(tuple(t.cpu() for t in (g.fwd(wl.w, wl.X), *g.backward(wl.w, wl.X, wl.dY))))
        ins.append(tuple(t.cpu().pin_memory() for t in (wl.w, wl.X, wl.dY)))
        outs.append((torch.empty_like(ins[-1][1]).pin_memory(), torch.empty_like(ins[-1][1]).pin_memory(),
                     torch.empty_like(ins[-1][0]).pin_memory()))
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    for (hw, hX, hdY), (hY, hdX, hdw) in zip(ins, outs):
        agb.ag_step_host(g, hw, hX, hdY, hY, hdX, hdw, staging, stream=s, pipelined=True)
    s.synchronize()
    for k, ((hY, hdX, hdw), (Y, dX, dw)) in enumerate(zip(outs, refs)):
        bits = (lambda t: t.view(torch.int16)) if Y.dtype == torch.bfloat16 else (lambda t: t.view(torch.int32))
        assert torch.equal(bits(hY), bits(Y)), k
        assert torch.equal(bits(hdX), bits(dX)), k
        assert torch.equal(hdw, dw), k


@pytest.mark.parametrize("case", ["uniform", "sbm", "rmat16", "twohop", "narrow-H20", "bf16-H128", "empty"])
def test_step_equals_forward_then_backward(agb, case):
    """ag_step (forward and fused backward in one call, the two overlapped on
    two streams) returns exactly what ag_spmm_fwd followed by ag_backward
    returns, on the shapes of the single backward walk and on the others
    (which take the two calls in order), and twice in a row on one scratch."""
    if case in ("uniform", "sbm", "rmat16", "twohop"):
        wl = workloads.make(case, seed=4, device=DEV)
    elif case == "empty":
        wl = workloads.custom(50, [], [], 32, seed=4, device=DEV)
    else:
        N, src, dst = skewed_edges(N=2000, E=30000)
        H, dt = (20, torch.float32) if case == "narrow-H20" else (128, torch.bfloat16)
        wl = workloads.custom(N, src, dst, H, seed=4, feature_dtype=dt, device=DEV)
    g = agb.ag_graph_lower(wl.src, wl.dst, wl.N)
    ref_Y = g.fwd(wl.w, wl.X)
    ref_dX, ref_dw = g.backward(wl.w, wl.X, wl.dY)
    bits = (lambda t: t.view(torch.int16)) if wl.X.dtype == torch.bfloat16 else (lambda t: t.view(torch.int32))
    for _ in range(2):
        Y, dX, dw = agb.ag_step(g, wl.w, wl.X, wl.dY)
        torch.cuda.synchronize()
        assert torch.equal(bits(Y), bits(ref_Y))
        assert torch.equal(bits(dX), bits(ref_dX))
        assert torch.equal(dw, ref_dw)
    if case == "rmat16":
        (rY, bY), (rX, bX), (rw, bw) = oracle_full_of(wl)
        assert_within(Y, rY, bY, TOL[wl.feature_dtype], "step fwd")
        assert_within(dX, rX, bX, TOL[wl.feature_dtype], "step dX")
        assert_within(dw, rw, bw, TOL_DW, "step dw")


def test_errors_are_reported_not_launched(agb):
    N, src, dst = skewed_edges(N=300, E=2000)
    wl, g = graph(agb, N, src, dst, 8)
    L = agb.lib
    Y = torch.empty_like(wl.X)
    sc = g.scratch(8)
    sp, sn = (ctypes.c_void_p(sc.data_ptr()), sc.numel()) if sc is not None else (None, 0)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    # host memory where device memory is required
    hostX = np.zeros((N, 8), np.float32)
    rc = L.ag_spmm_fwd(g.handle, p(wl.w), hostX.ctypes.data_as(ctypes.c_void_p), p(Y), 8, 0, sp, sn, None)
    assert rc == 4 and b"device" in L.ag_last_error()
    pinned = torch.zeros(N, 8).pin_memory()
    assert L.ag_sddmm_dw(g.handle, p(pinned), p(wl.dY), p(torch.empty(wl.E, device=DEV)), 8, 0, sp, sn, None) == 4
    # unknown dtype code, bad width
    assert L.ag_spmm_fwd(g.handle, p(wl.w), p(wl.X), p(Y), 8, 7, sp, sn, None) == 3
    assert L.ag_spmm_dx(g.handle, p(wl.w), p(wl.dY), p(Y), 0, 0, sp, sn, None) == 2
    # scratch too small for the rows cut by tile boundaries
    N2, s2, d2 = skewed_edges(N=3000, E=1000)
    wl2, g2 = graph(agb, N2, s2, d2, 8)
    need = g2.scratch_bytes(8)
    assert need > 0
    tiny = torch.empty(16, dtype=torch.uint8, device=DEV)
    Y2 = torch.empty_like(wl2.X)
    assert L.ag_spmm_fwd(g2.handle, p(wl2.w), p(wl2.X), p(Y2), 8, 0, p(tiny), 16, None) == 7
    # index outside [0, N) is caught on the device before anything is built
    bad_dst = wl.dst.clone()
    bad_dst[123] = N
    with pytest.raises(agb.AggraphError) as ei:
        agb.ag_graph_lower(wl.src, bad_dst, N)
    assert ei.value.status_name == "AG_ERR_INDEX_RANGE" and "123" in str(ei.value)
    bad_src = wl.src.clone()
    bad_src[7] = -1
    with pytest.raises(agb.AggraphError) as ei:
        agb.ag_graph_lower(bad_src, wl.dst, N)
    assert ei.value.status_name == "AG_ERR_INDEX_RANGE"
    # shape and dtype rejection in the binding
    with pytest.raises(agb.AggraphError):
        g.fwd(wl.w[:-1], wl.X)
    with pytest.raises(agb.AggraphError):
        g.fwd(wl.w, wl.X[:-1])
    with pytest.raises(agb.AggraphError):
        g.fwd(wl.w, wl.X.half())
    with pytest.raises(agb.AggraphError):
        g.dw(wl.X, wl.dY.bfloat16())
    # the context is still healthy after all of the above
    check_full(g, wl, "after errors")
