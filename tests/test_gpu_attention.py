"""Parity of the edge-softmax attention (CUDA path through the C ABI) with
the fp64 oracle.

Tolerances follow the arithmetic of the CUDA path:
  * scores: fp32 dot products, |ds_e| <= 1e-5 * scale * B_e with
    B_e = sum_h |Q[dst_e, h] K[src_e, h]| (the SpMM/SDDMM tolerance);
  * alpha: a shift of every score of row r by at most d_r = 1e-5 * scale *
    max_e B_e moves alpha_e by at most a factor exp(2 d_r); expf, the division
    and the fp32 sum of exponentials (a scan of depth 5 per 32 positions,
    then one combine per 32-position chunk and per tile, all terms positive)
    add at most 1e-6 * (8 + cnt_r / 256) relative.  Together rel_r;
  * Y = A_alpha V: |dY| <= (rel_r + TOL) * sum_e alpha_e |V|;
  * gradients: the same propagation through ds_e = scale alpha_e (dalpha_e
    - c_r), written out in `_grad_bounds`, plus TOL of the final SpMMs
    (which also covers bf16 output rounding).
"""
import numpy as np
import pytest
import torch

import workloads
from tests.gpu_helpers import TOL, assert_within, host, lib

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def agb():
    return lib()


def _qkv(wl, dtype, seed=11, unaligned=False):
    mk = lambda s: workloads.features(wl.N, wl.H, dtype, seed * 1000 + s, DEV)
    out = [mk(1), mk(2), mk(3), mk(4)]   # Q, K, V, upstream gradient G
    if unaligned:
        # the same values one element into a larger buffer: not 16-byte aligned
        moved = []
        for t in out:
            big = torch.zeros(t.numel() + 1, dtype=dtype, device=DEV)
            u = big[1:].view(t.shape)
            u.copy_(t)
            assert u.data_ptr() % 16 != 0
            moved.append(u)
        out = moved
    return out


def _row_rel(src, dst, N, Q, K, scale):
    """rel_r of the module docstring, per destination row."""
    B = np.einsum("eh,eh->e", np.abs(Q[dst].astype(np.float64)), np.abs(K[src].astype(np.float64)))
    Bmax = np.zeros(N)
    np.maximum.at(Bmax, dst, B)
    cnt = np.bincount(dst, minlength=N).astype(np.float64)
    d = 1e-5 * scale * Bmax
    return (np.exp(2 * d) - 1) + 1e-6 * (8 + cnt / 256)


def _grad_bounds(src, dst, N, Q, K, V, G, scale, alpha, rel, tol):
    """Error bounds of dQ, dK, dV (fp64, [N, H] each)."""
    a = alpha
    Bd = np.einsum("eh,eh->e", np.abs(G[dst].astype(np.float64)), np.abs(V[src].astype(np.float64)))
    da = np.einsum("eh,eh->e", G[dst].astype(np.float64), V[src].astype(np.float64))
    C = np.bincount(dst, weights=a * Bd, minlength=N)                  # >= |c_r|
    c = np.bincount(dst, weights=a * da, minlength=N)
    cnt = np.bincount(dst, minlength=N).astype(np.float64)
    relr = rel[dst]
    dC = np.bincount(dst, weights=a * (relr * Bd + 1e-5 * Bd), minlength=N) + 1e-6 * (8 + cnt / 256) * C
    dds = scale * (relr * a * (Bd + C[dst]) + a * (1e-5 * Bd + dC[dst]))
    ds = scale * a * (da - c[dst])
    wq = dds + tol * np.abs(ds)
    H = Q.shape[1]
    bQ = np.zeros((N, H))
    bK = np.zeros((N, H))
    bV = np.zeros((N, H))
    np.add.at(bQ, dst, wq[:, None] * np.abs(K[src].astype(np.float64)))
    np.add.at(bK, src, wq[:, None] * np.abs(Q[dst].astype(np.float64)))
    np.add.at(bV, src, ((relr + tol) * a)[:, None] * np.abs(G[dst].astype(np.float64)))
    return bQ, bK, bV


def _check_attention(agb, wl, dtype, what, unaligned=False):
    import oracle
    g = agb.ag_graph_lower(wl.src, wl.dst, wl.N)
    Q, K, V, G = _qkv(wl, dtype, unaligned=unaligned)
    scale = 1.0 / np.sqrt(wl.H)
    Y, alpha = agb.ag_attn_fwd(g, Q, K, V, scale)
    dQ, dK, dV = agb.ag_attn_backward(g, Q, K, V, scale, alpha, G)
    torch.cuda.synchronize()
    src, dst = host(wl.src), host(wl.dst)
    hQ, hK, hV, hG = host(Q), host(K), host(V), host(G)
    _, ra, rY, bY = oracle.attn_fwd(src, dst, wl.N, hQ, hK, hV, scale, with_bound=True)
    rel = _row_rel(src, dst, wl.N, hQ, hK, scale)
    tol = TOL[dtype]
    assert_within(alpha, ra, ra * rel[dst], 1.0, f"{what} alpha")
    assert_within(Y, rY, bY * (rel[:, None] + tol), 1.0, f"{what} Y")
    rQ, rK, rV, _ = oracle.attn_bwd(src, dst, wl.N, hQ, hK, hV, scale, ra, hG)
    bQ, bK, bV = _grad_bounds(src, dst, wl.N, hQ, hK, hV, hG, scale, ra, rel, tol)
    assert_within(dQ, rQ, bQ, 1.0, f"{what} dQ")
    assert_within(dK, rK, bK, 1.0, f"{what} dK")
    assert_within(dV, rV, bV, 1.0, f"{what} dV")
    # deterministic: a second run gives the same bits
    Y2, alpha2 = agb.ag_attn_fwd(g, Q, K, V, scale)
    dQ2, _, _ = agb.ag_attn_backward(g, Q, K, V, scale, alpha2, G)
    torch.cuda.synchronize()
    assert torch.equal(alpha2, alpha) and torch.equal(Y2, Y) and torch.equal(dQ2, dQ)
    return g, alpha


@pytest.mark.parametrize("name,dtype", [("uniform", torch.float32), ("sbm", torch.float32),
                                        ("rmat16", torch.float32), ("twohop", torch.float32),
                                        ("rmat16", torch.bfloat16), ("sbm", torch.bfloat16)])
def test_attention_matches_oracle(agb, name, dtype):
    wl = workloads.make(name, seed=4, device=DEV)
    g, alpha = _check_attention(agb, wl, dtype, f"{name}/{dtype}")
    # every row with edges is a distribution
    sums = torch.zeros(wl.N, dtype=torch.float64, device=DEV).index_add_(0, wl.dst.long(), alpha.double())
    has = torch.bincount(wl.dst.long(), minlength=wl.N) > 0
    assert torch.allclose(sums[has], torch.ones_like(sums[has]), atol=1e-5)


@pytest.mark.parametrize("H,dtype", [(1, torch.float32), (3, torch.float32), (8, torch.bfloat16),
                                     (33, torch.float32), (40, torch.bfloat16)])
def test_attention_narrow_and_ragged_widths(agb, H, dtype):
    # widths that take the register (non-ring) walks and ragged vector tails
    rng = np.random.default_rng(H)
    N, E = 700, 6000
    src = np.concatenate([rng.integers(0, N, E), rng.integers(0, N, 900)])
    dst = np.concatenate([rng.integers(0, N // 2, E), np.full(900, 5)])
    wl = workloads.custom(N, src, dst, H, seed=H, device=DEV)
    _check_attention(agb, wl, dtype, f"H={H}/{dtype}")


@pytest.mark.parametrize("H,dtype", [(16, torch.float32), (32, torch.float32), (128, torch.float32),
                                     (32, torch.bfloat16), (256, torch.bfloat16)])
def test_attention_ring_widths(agb, H, dtype):
    # every width whose rows are 4 to 32 16-byte vectors (the shared-memory
    # ring walks), with one heavy row cut by tiles
    rng = np.random.default_rng(100 + H)
    N, E = 900, 9000
    src = np.concatenate([rng.integers(0, N, E), rng.integers(0, N, 1500)])
    dst = np.concatenate([rng.integers(0, 2 * N // 3, E), np.full(1500, 11)])
    wl = workloads.custom(N, src, dst, H, seed=H, device=DEV)
    _check_attention(agb, wl, dtype, f"ring H={H}/{dtype}")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_attention_unaligned_inputs_take_the_register_walks(agb, dtype):
    # unaligned Q, K, V and dY take the register walks of narrower vectors
    # instead of the ring walks: the same bounds hold, and the results
    # reproduce themselves
    wl = workloads.make("sbm", seed=4, device=DEV)
    _check_attention(agb, wl, dtype, f"unaligned/{dtype}", unaligned=True)


def test_attention_skewed_rows_cut_by_many_tiles(agb):
    # one destination with 40,000 inputs (cut into many tiles), a few light
    # rows, empty rows and duplicate edges
    rng = np.random.default_rng(21)
    N, H = 5000, 32
    src = np.concatenate([rng.integers(0, N, 40000), rng.integers(0, N, 3000), [7, 7, 7]])
    dst = np.concatenate([np.full(40000, 17), rng.integers(0, 200, 3000), [9, 9, 9]])
    wl = workloads.custom(N, src, dst, H, seed=9, device=DEV)
    g, _ = _check_attention(agb, wl, torch.float32, "skewed")
    assert g.stats["long_spanning_rows_f"] >= 1


def test_attention_single_edge_rows_and_empty_graph(agb):
    N, H = 300, 8
    rng = np.random.default_rng(5)
    src = rng.integers(0, N, N)
    dst = np.arange(N)
    wl = workloads.custom(N, src, dst, H, seed=3, device=DEV)
    g = agb.ag_graph_lower(wl.src, wl.dst, N)
    Q, K, V, _ = _qkv(wl, torch.float32)
    Y, alpha = agb.ag_attn_fwd(g, Q, K, V, 0.5)
    torch.cuda.synchronize()
    assert torch.equal(alpha, torch.ones_like(alpha))
    assert torch.equal(Y, V[wl.src.long()])
    z = torch.zeros(0, dtype=torch.int32, device=DEV)
    g0 = agb.ag_graph_lower(z, z, 4)
    X = torch.randn(4, 8, device=DEV)
    Y0, a0 = agb.ag_attn_fwd(g0, X, X, X, 1.0)
    dQ, dK, dV = agb.ag_attn_backward(g0, X, X, X, 1.0, a0, X)
    torch.cuda.synchronize()
    assert a0.numel() == 0 and not Y0.any() and not dQ.any() and not dK.any() and not dV.any()


def test_attention_rejects_bad_arguments(agb):
    wl = workloads.make("uniform", seed=1, device=DEV)
    g = agb.ag_graph_lower(wl.src, wl.dst, wl.N)
    with pytest.raises(agb.AggraphError):
        agb.ag_attn_fwd(g, wl.X, wl.X, wl.X, float("inf"))
    with pytest.raises(agb.AggraphError):
        agb.ag_attn_fwd(g, wl.X, wl.X.double(), wl.X, 1.0)
