"""fp64 CPU oracle for weighted GNN aggregation (test infrastructure only).

Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding in ``gnn_sparse_aggregation_b200``) never imports, links or runs
it, and this package imports nothing from the product path.

The arithmetic lives in ``oracle.c`` (plain C, fp64, one thread); this module
only compiles it with gcc and marshals numpy arrays.  Functions follow the
tinymesh "Weighted aggregation experiment" page ("Decision", "Edge order is
explicit") and the COO loop of the PyTorch Geometric reading guide (Step 2,
without the m x d temporary, which Step 3 says the fused path drops).

The further aggregators (mean, GCN-normalised weights, edge-softmax
attention) follow the same reading guide: Step 3 (GCN's normalised adjacency,
the sum and mean reductions of spmm) and Step 4 (SDDMM scores, a softmax per
destination row, then the SpMM).

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
and ``tests/test_oracle_ext_pins.py`` against the hand-derived "Exact
witness" fixture, dense matrix products, library stable sorts and softmax,
closed forms, the adjoint identity and finite differences.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None

_P = ctypes.c_void_p
_I64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so beside it (gcc, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
             "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        lib.oracle_lower.argtypes = [_I64, _I64, _P, _P, _P, _P, _P, _P, _P, _P]
        for name in ("oracle_fwd", "oracle_dx", "oracle_dw"):
            getattr(lib, name).argtypes = [_I64, _I64, _I64, _P, _P, _P, _P, _P, _P]
        lib.oracle_spmm_rows.argtypes = [_I64, _I64, _I64, _P, _P, _P, _P, ctypes.c_int,
                                         _I64, _P, _P, _P]
        lib.oracle_dw_edges.argtypes = [_I64, _I64, _I64, _P, _P, _P, _P, _I64, _P, _P, _P]
        for name in ("oracle_mean_fwd", "oracle_mean_dx", "oracle_mean_dw"):
            getattr(lib, name).argtypes = [_I64, _I64, _I64, _P, _P, _P, _P, _P, _P]
        lib.oracle_gcn_norm.argtypes = [_I64, _I64, _P, _P, _P, _P]
        lib.oracle_attn_fwd.argtypes = [_I64, _I64, _I64, _P, _P, _P, _P, _P, ctypes.c_double,
                                        _P, _P, _P, _P]
        lib.oracle_attn_bwd.argtypes = [_I64, _I64, _I64, _P, _P, _P, _P, _P, ctypes.c_double,
                                        _P, _P, _P, _P, _P, _P]
        lib.oracle_attn_sampled.argtypes = [_I64, _I64, _I64, _P, _P, _P, _P, _P, ctypes.c_double, _P,
                                            _I64, _P, _I64, _P, _P, _P, _P, _P, _P, _P, _P, _P]
        for name in ("oracle_attn_sampled", "oracle_lower", "oracle_fwd", "oracle_dx", "oracle_dw",
                     "oracle_spmm_rows", "oracle_dw_edges", "oracle_mean_fwd", "oracle_mean_dx",
                     "oracle_mean_dw", "oracle_gcn_norm", "oracle_attn_fwd", "oracle_attn_bwd"):
            getattr(lib, name).restype = ctypes.c_int
        _lib = lib
    return _lib


class OracleError(ValueError):
    pass


_CODES = {1: "bad size", 2: "index out of range", 3: "out of memory"}


def _check(rc: int) -> None:
    if rc != 0:
        raise OracleError(_CODES.get(rc, f"oracle error {rc}"))


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _f32(a) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype != np.float32:
        # fp64 inputs would be rounded here; the oracle is defined on fp32/bf16 values
        a = a.astype(np.float32)
    return np.ascontiguousarray(a)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def lower(src, dst, N: int) -> dict:
    """Forward CSR (destination-owned) and transpose CSR (source-owned)."""
    src, dst = _i32(src), _i32(dst)
    E = src.shape[0]
    assert dst.shape[0] == E
    out = {
        "rowptr_f": np.zeros(N + 1, np.int32), "col_f": np.zeros(E, np.int32),
        "edge_order": np.zeros(E, np.int32),
        "rowptr_t": np.zeros(N + 1, np.int32), "col_t": np.zeros(E, np.int32),
        "transpose_order": np.zeros(E, np.int32),
    }
    _check(_load().oracle_lower(N, E, _ptr(src), _ptr(dst),
                                _ptr(out["rowptr_f"]), _ptr(out["col_f"]), _ptr(out["edge_order"]),
                                _ptr(out["rowptr_t"]), _ptr(out["col_t"]),
                                _ptr(out["transpose_order"])))
    return out


def _spmm_like(fn_name, src, dst, N, a, b, out_rows, with_bound):
    src, dst = _i32(src), _i32(dst)
    a, b = _f32(a), _f32(b)
    E = src.shape[0]
    H = b.shape[1] if b.ndim == 2 else a.shape[1]
    out = np.zeros((out_rows, H) if fn_name != "oracle_dw" else (E,), np.float64)
    bound = np.zeros_like(out) if with_bound else None
    _check(getattr(_load(), fn_name)(N, E, H, _ptr(src), _ptr(dst), _ptr(a), _ptr(b),
                                     _ptr(out), _ptr(bound) if with_bound else None))
    return (out, bound) if with_bound else out


def fwd(src, dst, N: int, w, X, with_bound: bool = False):
    """Y = A_w X with A_w[dst_e, src_e] = w_e; fp64 [N, H]."""
    return _spmm_like("oracle_fwd", src, dst, N, w, X, N, with_bound)


def dx(src, dst, N: int, w, dY, with_bound: bool = False):
    """dX = A_w^T dY; fp64 [N, H]."""
    return _spmm_like("oracle_dx", src, dst, N, w, dY, N, with_bound)


def dw(src, dst, N: int, X, dY, with_bound: bool = False):
    """dw_e = dot(X[src_e], dY[dst_e]); fp64 [E], COO order."""
    src, dst = _i32(src), _i32(dst)
    X, dY = _f32(X), _f32(dY)
    E = src.shape[0]
    H = X.shape[1]
    out = np.zeros(E, np.float64)
    bound = np.zeros(E, np.float64) if with_bound else None
    _check(_load().oracle_dw(N, E, H, _ptr(src), _ptr(dst), _ptr(X), _ptr(dY), _ptr(out),
                             _ptr(bound) if with_bound else None))
    return (out, bound) if with_bound else out


def spmm_rows(src, dst, N: int, w, feat, rows, by_source: bool, with_bound: bool = False):
    """Rows `rows` of fwd (by_source=False) or of dx (by_source=True)."""
    src, dst = _i32(src), _i32(dst)
    w, feat = _f32(w), _f32(feat)
    rows = _i32(rows)
    E = src.shape[0]
    H = feat.shape[1]
    out = np.zeros((rows.shape[0], H), np.float64)
    bound = np.zeros_like(out) if with_bound else None
    _check(_load().oracle_spmm_rows(N, E, H, _ptr(src), _ptr(dst), _ptr(w), _ptr(feat),
                                    1 if by_source else 0, rows.shape[0], _ptr(rows),
                                    _ptr(out), _ptr(bound) if with_bound else None))
    return (out, bound) if with_bound else out


def dw_edges(src, dst, N: int, X, dY, edges, with_bound: bool = False):
    """dw for the listed COO ordinals."""
    src, dst = _i32(src), _i32(dst)
    X, dY = _f32(X), _f32(dY)
    edges = np.ascontiguousarray(np.asarray(edges, dtype=np.int64))
    E = src.shape[0]
    H = X.shape[1]
    out = np.zeros(edges.shape[0], np.float64)
    bound = np.zeros_like(out) if with_bound else None
    _check(_load().oracle_dw_edges(N, E, H, _ptr(src), _ptr(dst), _ptr(X), _ptr(dY),
                                   edges.shape[0], _ptr(edges), _ptr(out),
                                   _ptr(bound) if with_bound else None))
    return (out, bound) if with_bound else out


# ----------------------------------------------------------------------------- further aggregators

def mean_fwd(src, dst, N: int, w, X, with_bound: bool = False):
    """Y[r] = sum over edges into r of w_e X[src_e], divided by the number of
    edges into r (0 for rows without edges); fp64 [N, H]."""
    return _spmm_like("oracle_mean_fwd", src, dst, N, w, X, N, with_bound)


def mean_dx(src, dst, N: int, w, dY, with_bound: bool = False):
    """dX[s] = sum over edges out of s of (w_e / cnt(dst_e)) dY[dst_e]."""
    return _spmm_like("oracle_mean_dx", src, dst, N, w, dY, N, with_bound)


def mean_dw(src, dst, N: int, X, dY, with_bound: bool = False):
    """dw_e = dot(X[src_e], dY[dst_e]) / cnt(dst_e), COO order."""
    src, dst = _i32(src), _i32(dst)
    X, dY = _f32(X), _f32(dY)
    E = src.shape[0]
    out = np.zeros(E, np.float64)
    bound = np.zeros(E, np.float64) if with_bound else None
    _check(_load().oracle_mean_dw(N, E, X.shape[1], _ptr(src), _ptr(dst), _ptr(X), _ptr(dY),
                                  _ptr(out), _ptr(bound) if with_bound else None))
    return (out, bound) if with_bound else out


def gcn_norm(src, dst, N: int, w=None) -> np.ndarray:
    """D^-1/2 A_w D^-1/2 as edge weights (COO order), D = weighted in-degree;
    w=None means unit weights; deg <= 0 contributes a factor 0."""
    src, dst = _i32(src), _i32(dst)
    E = src.shape[0]
    wf = None if w is None else _f32(w)
    out = np.zeros(E, np.float64)
    _check(_load().oracle_gcn_norm(N, E, _ptr(src), _ptr(dst), None if wf is None else _ptr(wf),
                                   _ptr(out)))
    return out


def attn_fwd(src, dst, N: int, Q, K, V, scale: float, with_bound: bool = False):
    """Edge-softmax attention: returns (s, alpha, Y[, bound]) with s and alpha
    in COO order (fp64) and Y [N, H] (fp64)."""
    src, dst = _i32(src), _i32(dst)
    Q, K, V = _f32(Q), _f32(K), _f32(V)
    E = src.shape[0]
    H = Q.shape[1]
    s = np.zeros(E, np.float64)
    alpha = np.zeros(E, np.float64)
    Y = np.zeros((N, H), np.float64)
    bound = np.zeros_like(Y) if with_bound else None
    _check(_load().oracle_attn_fwd(N, E, H, _ptr(src), _ptr(dst), _ptr(Q), _ptr(K), _ptr(V),
                                   float(scale), _ptr(s), _ptr(alpha), _ptr(Y),
                                   _ptr(bound) if with_bound else None))
    return (s, alpha, Y, bound) if with_bound else (s, alpha, Y)


def attn_bwd(src, dst, N: int, Q, K, V, scale: float, alpha, dY):
    """Gradients (dQ, dK, dV, ds) of the attention for upstream gradient dY;
    alpha is the fp64 alpha of attn_fwd."""
    src, dst = _i32(src), _i32(dst)
    Q, K, V, dY = _f32(Q), _f32(K), _f32(V), _f32(dY)
    alpha = np.ascontiguousarray(np.asarray(alpha, np.float64))
    E = src.shape[0]
    H = Q.shape[1]
    dQ = np.zeros((N, H), np.float64)
    dK = np.zeros((N, H), np.float64)
    dV = np.zeros((N, H), np.float64)
    ds = np.zeros(E, np.float64)
    _check(_load().oracle_attn_bwd(N, E, H, _ptr(src), _ptr(dst), _ptr(Q), _ptr(K), _ptr(V),
                                   float(scale), _ptr(alpha), _ptr(dY), _ptr(dQ), _ptr(dK),
                                   _ptr(dV), _ptr(ds)))
    return dQ, dK, dV, ds


def attn_sampled(src, dst, N: int, Q, K, V, scale: float, dY, rows_r, rows_s):
    """Y, dQ on destination rows rows_r and dK, dV on source rows rows_s of
    the attention and its gradients, with their tolerance scales: returns a
    dict with Y, dQ, dK, dV and absY, absdQ, absdK, absdV."""
    src, dst = _i32(src), _i32(dst)
    Q, K, V, dY = _f32(Q), _f32(K), _f32(V), _f32(dY)
    rows_r, rows_s = _i32(rows_r), _i32(rows_s)
    E = src.shape[0]
    H = Q.shape[1]
    r = {k: np.zeros((rows_r.shape[0], H), np.float64) for k in ("Y", "dQ", "absY", "absdQ")}
    s = {k: np.zeros((rows_s.shape[0], H), np.float64) for k in ("dK", "dV", "absdK", "absdV")}
    _check(_load().oracle_attn_sampled(N, E, H, _ptr(src), _ptr(dst), _ptr(Q), _ptr(K), _ptr(V), float(scale),
                                       _ptr(dY), rows_r.shape[0], _ptr(rows_r), rows_s.shape[0], _ptr(rows_s),
                                       _ptr(r["Y"]), _ptr(r["dQ"]), _ptr(s["dK"]), _ptr(s["dV"]),
                                       _ptr(r["absY"]), _ptr(r["absdQ"]), _ptr(s["absdK"]), _ptr(s["absdV"])))
    return {**r, **s}
