"""Seeded synthetic inputs for weighted GNN aggregation.

This module only draws graphs, weights and features; it holds none of the
aggregation arithmetic, and both the oracle-side tests and the CUDA path take
their inputs from it.  Every draw is seeded.  Topologies that need sampling
without replacement (SBM, 2-hop) are drawn with numpy PCG64 on the host;
R-MAT edges and all dense features are drawn with a seeded ``torch.Generator``
on the requested device, so that the 67M-edge R-MAT graph and its 1 GiB
feature matrices can be made on the GPU in milliseconds.  A given
(config, seed, device) always produces the same tensors.

Workload shapes follow the pages' workloads:
  * "uniform"  -- N=1,024, E=8,192, src/dst iid uniform, H=16 fp32
  * "sbm"      -- 20 blocks of 1,000 nodes, p_in=0.025, p_out=1.7e-4, H=64 fp32
                  (stands in for the reading guide's 566K-edge SBM, "The problem
                  in one sentence"; that graph is not available here)
  * "rmat16"   -- R-MAT scale 16, edge factor 16, (.57,.19,.19,.05), H=128 fp32
  * "rmat22"   -- R-MAT scale 22, edge factor 16, H=128 bf16 features
  * "twohop"   -- 1,024 seeds, [15, 10] distinct-neighbour 2-hop block, H=256 fp32
                  (shaped like the AetherGraph NeighborLoader batch of the
                  "PyTorch Geometric Integration" section: seeds first, then
                  nodes in hop order, edges neighbour -> sampler)
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

CONFIGS = ("uniform", "sbm", "rmat16", "rmat22", "twohop")

RMAT_PROBS = (0.57, 0.19, 0.19, 0.05)


@dataclass
class Workload:
    name: str
    N: int
    E: int
    H: int
    feature_dtype: torch.dtype
    src: torch.Tensor   # [E] int32, COO order
    dst: torch.Tensor   # [E] int32, COO order
    w: torch.Tensor     # [E] fp32, COO order
    X: torch.Tensor     # [N, H] feature dtype
    dY: torch.Tensor    # [N, H] feature dtype

    def to(self, device) -> "Workload":
        return Workload(self.name, self.N, self.E, self.H, self.feature_dtype,
                        self.src.to(device), self.dst.to(device), self.w.to(device),
                        self.X.to(device), self.dY.to(device))


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(int(seed))
    return g


def features(N: int, H: int, dtype: torch.dtype, seed: int, device="cpu") -> torch.Tensor:
    """[N, H] iid N(0, 1), drawn in fp32 and rounded once to `dtype`."""
    g = _gen(device, seed)
    x = torch.randn((N, H), generator=g, device=device, dtype=torch.float32)
    return x if dtype == torch.float32 else x.to(dtype)


def weights(E: int, dist: str, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(device, seed)
    if dist == "normal":
        return torch.randn(E, generator=g, device=device, dtype=torch.float32)
    if dist == "uniform":
        return torch.rand(E, generator=g, device=device, dtype=torch.float32)
    raise ValueError(dist)


# ----------------------------------------------------------------------------- topologies

def uniform_edges(N: int, E: int, seed: int, device="cpu"):
    """src, dst iid uniform on [0, N); duplicates and self-loops kept."""
    g = _gen(device, seed)
    src = torch.randint(0, N, (E,), generator=g, device=device, dtype=torch.int64)
    dst = torch.randint(0, N, (E,), generator=g, device=device, dtype=torch.int64)
    return src.to(torch.int32), dst.to(torch.int32)


def rmat_edges(scale: int, edge_factor: int, seed: int, device="cpu", probs=RMAT_PROBS):
    """R-MAT: every edge picks one quadrant per level with probabilities
    (a, b, c, d); the quadrant's row bit goes to src, its column bit to dst.
    No noise and no id scrambling, so hubs sit at ids with few one-bits.
    Edges come out in generation order (iid), duplicates and self-loops kept."""
    a, b, c, _ = probs
    E = edge_factor << scale
    g = _gen(device, seed)
    src = torch.zeros(E, dtype=torch.int32, device=device)
    dst = torch.zeros(E, dtype=torch.int32, device=device)
    t1, t2, t3 = a, a + b, a + b + c
    for level in range(scale):
        u = torch.rand(E, generator=g, device=device, dtype=torch.float32)
        row_bit = (u >= t2).to(torch.int32)
        col_bit = (((u >= t1) & (u < t2)) | (u >= t3)).to(torch.int32)
        src |= row_bit << level
        dst |= col_bit << level
        del u, row_bit, col_bit
    return src, dst


def sbm_edges(n_blocks: int, block_size: int, p_in: float, p_out: float, seed: int):
    """Directed SBM over ordered pairs i != j: per ordered block pair, a binomial
    edge count and that many distinct positions; edge list shuffled at the end."""
    rng = np.random.Generator(np.random.PCG64(seed))
    srcs, dsts = [], []
    bs = block_size
    for bi in range(n_blocks):
        for bj in range(n_blocks):
            same = bi == bj
            n_pairs = bs * (bs - 1) if same else bs * bs
            k = int(rng.binomial(n_pairs, p_in if same else p_out))
            if k == 0:
                continue
            pos = rng.choice(n_pairs, size=k, replace=False)
            if same:
                i = pos // (bs - 1)
                jj = pos % (bs - 1)
                j = jj + (jj >= i)
            else:
                i = pos // bs
                j = pos % bs
            srcs.append(bi * bs + i)
            dsts.append(bj * bs + j)
    src = np.concatenate(srcs).astype(np.int32)
    dst = np.concatenate(dsts).astype(np.int32)
    perm = rng.permutation(src.shape[0])
    return torch.from_numpy(src[perm].copy()), torch.from_numpy(dst[perm].copy())


def _floyd_rows(rng, n: int, k: int, rows: int) -> np.ndarray:
    """Robert Floyd's algorithm for k distinct values of [0, n), run for `rows`
    independent samples at once: at step j in [n-k, n) draw t in [0, j]; keep
    t unless it was already chosen, in which case keep j."""
    out = np.empty((rows, k), np.int64)
    for s, j in enumerate(range(n - k, n)):
        t = rng.integers(0, j + 1, size=rows)
        dup = (out[:, :s] == t[:, None]).any(axis=1) if s else np.zeros(rows, bool)
        out[:, s] = np.where(dup, j, t)
    return out


def twohop_edges(n_seeds: int, fanouts, n_global: int, seed: int):
    """2-hop sampled block: seeds, then per hop every sampler slot draws
    `fanout` distinct neighbours (Floyd).  Edges run neighbour -> sampler.
    Local ids by first appearance: seeds, then hop 1, then hop 2.
    Returns src, dst (int32 torch, local ids), N and the per-hop counts."""
    rng = np.random.Generator(np.random.PCG64(seed))
    seeds = _floyd_rows(rng, n_global, n_seeds, 1)[0]
    frontier = seeds
    order_ids = [seeds]
    e_src, e_dst = [], []
    for fan in fanouts:
        nb = _floyd_rows(rng, n_global, fan, frontier.shape[0])   # [slots, fan]
        e_dst.append(np.repeat(frontier, fan))
        e_src.append(nb.reshape(-1))
        frontier = nb.reshape(-1)
        order_ids.append(frontier)
    all_ids = np.concatenate(order_ids)
    uniq, first = np.unique(all_ids, return_index=True)
    rank = np.empty(uniq.shape[0], np.int64)
    rank[np.argsort(first, kind="stable")] = np.arange(uniq.shape[0])
    to_local = lambda g: rank[np.searchsorted(uniq, g)]
    src = to_local(np.concatenate(e_src)).astype(np.int32)
    dst = to_local(np.concatenate(e_dst)).astype(np.int32)
    return torch.from_numpy(src), torch.from_numpy(dst), int(uniq.shape[0])


# ----------------------------------------------------------------------------- configs

def make(name: str, seed: int = 1, device="cpu", rmat_scale: int | None = None) -> Workload:
    """One of the five configurations, all tensors on `device`.  rmat_scale
    overrides the R-MAT scale of "rmat16"/"rmat22" (same edge factor, width
    and dtypes) for smaller profiling cases."""
    dev = torch.device(device)
    s = int(seed) * 1000
    if name == "uniform":
        N, E, H, fdt, wdist = 1024, 8192, 16, torch.float32, "normal"
        src, dst = uniform_edges(N, E, s + 1, dev)
    elif name == "sbm":
        H, fdt, wdist = 64, torch.float32, "uniform"
        src, dst = sbm_edges(20, 1000, 0.025, 1.7e-4, s + 1)
        N, E = 20000, int(src.shape[0])
    elif name in ("rmat16", "rmat22"):
        scale = 16 if name == "rmat16" else 22
        if rmat_scale is not None:
            scale = int(rmat_scale)
        H, wdist = 128, "normal"
        fdt = torch.float32 if name == "rmat16" else torch.bfloat16
        src, dst = rmat_edges(scale, 16, s + 1, dev)
        N, E = 1 << scale, 16 << scale
    elif name == "twohop":
        H, fdt, wdist = 256, torch.float32, "uniform"
        src, dst, N = twohop_edges(1024, (15, 10), 1_000_000, s + 1)
        E = int(src.shape[0])
    else:
        raise ValueError(f"unknown workload {name!r}; expected one of {CONFIGS}")
    src, dst = src.to(dev), dst.to(dev)
    w = weights(E, wdist, s + 2, dev)
    X = features(N, H, fdt, s + 3, dev)
    dY = features(N, H, fdt, s + 4, dev)
    return Workload(name, N, E, H, fdt, src, dst, w, X, dY)


def custom(N: int, src, dst, H: int, seed: int = 7, feature_dtype=torch.float32,
           wdist: str = "normal", device="cpu", name: str = "custom") -> Workload:
    """Features and weights for a caller-given topology (edge-case graphs)."""
    dev = torch.device(device)
    src = torch.as_tensor(np.asarray(src, dtype=np.int32)).to(dev)
    dst = torch.as_tensor(np.asarray(dst, dtype=np.int32)).to(dev)
    E = int(src.shape[0])
    return Workload(name, N, E, H, feature_dtype, src, dst,
                    weights(E, wdist, seed * 1000 + 2, dev),
                    features(N, H, feature_dtype, seed * 1000 + 3, dev),
                    features(N, H, feature_dtype, seed * 1000 + 4, dev))
