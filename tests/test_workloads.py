"""Shape, range and determinism checks of the seeded synthetic inputs."""
import numpy as np
import pytest
import torch

import workloads


def test_uniform_shape_and_determinism():
    a = workloads.make("uniform", seed=1)
    b = workloads.make("uniform", seed=1)
    c = workloads.make("uniform", seed=2)
    assert (a.N, a.E, a.H) == (1024, 8192, 16)
    assert a.src.dtype == torch.int32 and a.w.dtype == torch.float32
    assert a.X.shape == (1024, 16) and a.X.dtype == torch.float32
    for k in ("src", "dst", "w", "X", "dY"):
        assert torch.equal(getattr(a, k), getattr(b, k))
    assert not torch.equal(a.src, c.src)
    assert int(a.src.min()) >= 0 and int(a.src.max()) < 1024
    assert int(a.dst.min()) >= 0 and int(a.dst.max()) < 1024


def test_sbm_edge_count_and_blocks():
    wl = workloads.make("sbm", seed=1)
    src, dst = wl.src.numpy(), wl.dst.numpy()
    expected = 20 * 1000 * 999 * 0.025 + 20 * 19 * 1000 * 1000 * 1.7e-4
    assert abs(wl.E - expected) < 5 * np.sqrt(expected)
    assert np.all(src != dst)                                # ordered pairs i != j
    pairs = src.astype(np.int64) * wl.N + dst
    assert np.unique(pairs).size == wl.E                     # distinct positions
    same = (src // 1000) == (dst // 1000)
    assert 0.85 < same.mean() < 0.92                         # ~499.5K in / ~64.6K out
    assert float(wl.w.min()) >= 0.0 and float(wl.w.max()) < 1.0
    assert wl.X.shape == (20000, 64)


def test_rmat_small_scale_skew():
    src, dst = workloads.rmat_edges(16, 16, seed=5)
    E = 16 << 16
    assert src.shape == (E,) and int(src.max()) < (1 << 16) and int(dst.min()) >= 0
    indeg = np.bincount(dst.numpy(), minlength=1 << 16)
    # node 0 draws every column bit 0: expected in-degree E * (a + c)^16
    expect0 = E * (0.57 + 0.19) ** 16
    assert abs(indeg[0] - expect0) < 6 * np.sqrt(expect0)
    assert indeg.argmax() == 0
    outdeg = np.bincount(src.numpy(), minlength=1 << 16)
    assert outdeg.argmax() == 0


def test_rmat16_config():
    wl = workloads.make("rmat16", seed=1)
    assert (wl.N, wl.E, wl.H) == (65536, 1 << 20, 128)
    assert wl.X.dtype == torch.float32


def test_twohop_block_structure():
    wl = workloads.make("twohop", seed=1)
    src, dst = wl.src.numpy(), wl.dst.numpy()
    assert wl.E == 1024 * 15 + 1024 * 15 * 10 == 168960
    assert 150_000 < wl.N < 160_000
    assert wl.X.shape == (wl.N, 256)
    hop1_dst, hop2_dst = dst[:15360], dst[15360:]
    assert np.all(hop1_dst < 1024)                           # seeds are local ids 0..1023
    assert np.array_equal(np.bincount(hop1_dst, minlength=1024), np.full(1024, 15))
    # each hop-1 sampler slot has 10 distinct neighbours
    s2 = src[15360:].reshape(15360, 10)
    assert all(np.unique(row).size == 10 for row in s2[:500])
    s1 = src[:15360].reshape(1024, 15)
    assert all(np.unique(row).size == 15 for row in s1)
    assert int(src.max()) == wl.N - 1 and int(dst.max()) < wl.N


def test_twohop_first_appearance_numbering():
    src, dst, N = workloads.twohop_edges(8, (3, 2), 50, seed=3)
    src, dst = src.numpy(), dst.numpy()
    assert np.array_equal(np.unique(dst[:24]), np.arange(8))   # seeds first
    # new ids appear in increasing order along the hop-ordered id stream
    stream = np.concatenate([np.arange(8), src[:24], src[24:]])
    first = []
    for v in stream:
        if v not in first:
            first.append(v)
    assert first == list(range(N))


def test_floyd_distinct():
    rng = np.random.Generator(np.random.PCG64(0))
    out = workloads._floyd_rows(rng, 20, 20, 50)              # k = n: a permutation
    assert all(sorted(r) == list(range(20)) for r in out)
    out = workloads._floyd_rows(rng, 1000, 15, 400)
    assert all(np.unique(r).size == 15 for r in out)
    assert out.min() >= 0 and out.max() < 1000


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_features_seeded(dtype):
    a = workloads.features(10, 8, dtype, seed=3)
    b = workloads.features(10, 8, dtype, seed=3)
    assert a.dtype == dtype and torch.equal(a, b)
