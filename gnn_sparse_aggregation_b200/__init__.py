"""Fused weighted GNN aggregation on B200 (sm_100a): Python binding.

This module only marshals torch tensors into the C ABI of ``libaggraph.so``
(declared in ``include/aggraph.h``); every step of the computation runs in the
library's CUDA kernels.  There is no CPU fallback: importing this package fails
if the library has not been built, and every call fails on tensors that are
not on a CUDA device.

Operations (tinymesh "Weighted aggregation experiment", sections "Decision"
and "Edge order is explicit"), with A_w[dst_e, src_e] = w_e:

    ag_graph_lower(src, dst, N)  -> Graph   forward CSR + transpose CSR + order maps
    ag_spmm_fwd(g, w, X)         -> Y  = A_w X
    ag_spmm_dx(g, w, dY)         -> dX = A_w^T dY
    ag_sddmm_dw(g, X, dY)        -> dw_e = dot(X[src_e], dY[dst_e])   (COO order)
    ag_backward(g, w, X, dY)     -> (dX, dw) in one pass over the transpose CSR
    ag_step(g, w, X, dY)         -> (Y, dX, dw): forward and fused backward in one call, overlapped
    ag_step_host(g, w, X, dY, ...)  the three from host buffers, copies included
    ag_step_host_pipelined(...)     the same for back-to-back steps (copies overlap across steps)
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

__all__ = ["AggraphError", "Graph", "ag_graph_lower", "ag_spmm_fwd", "ag_spmm_dx", "ag_sddmm_dw", "ag_backward",
           "ag_mean_fwd", "ag_mean_backward", "ag_gcn_norm", "ag_attn_fwd", "ag_attn_backward", "ag_step",
           "ag_step_host", "ag_step_host_pipelined", "ag_step_staging_bytes", "ag_graph_workspace_bytes", "lib", "LIB_PATH",
           "declared_symbols", "AG_F32", "AG_BF16"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libaggraph.so")
HEADER_PATH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                           "include", "aggraph.h")

AG_F32, AG_BF16 = 0, 1
_STATUS = {0: "AG_OK", 1: "AG_ERR_INVALID_ARG", 2: "AG_ERR_SHAPE", 3: "AG_ERR_DTYPE",
           4: "AG_ERR_DEVICE", 5: "AG_ERR_INDEX_RANGE", 6: "AG_ERR_CUDA", 7: "AG_ERR_WORKSPACE"}

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python gnn_sparse_aggregation_b200/_build.py` "
        "(or __graft_entry__.build()); there is no fallback implementation")


class AggraphError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_STATUS.get(status, status)}: {message}")
        self.status = status
        self.status_name = _STATUS.get(status, str(status))


class Stats(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("E", ctypes.c_int64), ("device", ctypes.c_int32),
                ("tile_edges", ctypes.c_int32), ("tiles", ctypes.c_int64),
                ("max_degree_f", ctypes.c_int64), ("max_degree_t", ctypes.c_int64),
                ("nonempty_rows_f", ctypes.c_int64), ("spanning_rows_f", ctypes.c_int64),
                ("long_spanning_rows_f", ctypes.c_int64), ("nonempty_rows_t", ctypes.c_int64),
                ("spanning_rows_t", ctypes.c_int64), ("long_spanning_rows_t", ctypes.c_int64),
                ("workspace_bytes_used", ctypes.c_size_t), ("dw_locality", ctypes.c_double)]

    def as_dict(self) -> dict:
        return {name: getattr(self, name) for name, _ in self._fields_}


_P, _I64, _SZ, _I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
_PP = ctypes.POINTER(ctypes.c_void_p)

def _bind(handle: ctypes.CDLL) -> ctypes.CDLL:
    """Declares the C signatures of libaggraph on a loaded library handle."""
    handle.ag_graph_workspace_bytes.argtypes = [_I64, _I64]
    handle.ag_graph_workspace_bytes.restype = _SZ
    handle.ag_graph_lower.argtypes = [_P, _P, _I64, _I64, _P, _SZ, _P, _PP]
    handle.ag_graph_arrays.argtypes = [_P] + [_PP] * 6
    handle.ag_graph_get_stats.argtypes = [_P, ctypes.POINTER(Stats)]
    handle.ag_spmm_scratch_bytes.argtypes = [_P, _I64]
    handle.ag_spmm_scratch_bytes.restype = _SZ
    handle.ag_spmm_fwd.argtypes = [_P, _P, _P, _P, _I64, _I, _P, _SZ, _P]
    handle.ag_spmm_dx.argtypes = [_P, _P, _P, _P, _I64, _I, _P, _SZ, _P]
    handle.ag_sddmm_dw.argtypes = [_P, _P, _P, _P, _I64, _I, _P, _SZ, _P]
    handle.ag_backward.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _I, _P, _SZ, _P]
    handle.ag_mean_fwd.argtypes = [_P, _P, _P, _P, _I64, _I, _P, _SZ, _P]
    handle.ag_mean_backward.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _I, _P, _SZ, _P]
    handle.ag_gcn_norm_scratch_bytes.argtypes = [_P]
    handle.ag_gcn_norm_scratch_bytes.restype = _SZ
    handle.ag_gcn_norm.argtypes = [_P, _P, _P, _P, _SZ, _P]
    handle.ag_attn_scratch_bytes.argtypes = [_P, _I64]
    handle.ag_attn_scratch_bytes.restype = _SZ
    handle.ag_attn_fwd.argtypes = [_P, _P, _P, _P, ctypes.c_float, _P, _P, _I64, _I, _P, _SZ, _P]
    handle.ag_attn_backward.argtypes = [_P, _P, _P, _P, ctypes.c_float, _P, _P, _P, _P, _P, _I64, _I, _P,
                                        _SZ, _P]
    handle.ag_spmm_fwd_static_scratch.argtypes = [_P, _P, _P, _P, _I64, _I, _P]
    handle.ag_spmm_static_scratch_capacity.argtypes = []
    handle.ag_spmm_static_scratch_capacity.restype = _SZ
    handle.ag_step_staging_bytes.argtypes = [_P, _I64, _I]
    handle.ag_step_staging_bytes.restype = _SZ
    handle.ag_step_host.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I64, _I, _P, _SZ, _P]
    handle.ag_step_host_pipelined.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I64, _I, _P, _SZ, _P]
    handle.ag_step_scratch_bytes.argtypes = [_P, _I64]
    handle.ag_step_scratch_bytes.restype = _SZ
    handle.ag_step.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I64, _I, _P, _SZ, _P]
    handle.ag_graph_free.argtypes = [_P]
    handle.ag_graph_free.restype = None
    handle.ag_last_error.restype = ctypes.c_char_p
    handle.ag_status_string.argtypes = [_I]
    handle.ag_status_string.restype = ctypes.c_char_p
    for name in ("ag_graph_lower", "ag_graph_arrays", "ag_graph_get_stats", "ag_spmm_fwd", "ag_spmm_dx",
                 "ag_sddmm_dw", "ag_backward", "ag_step", "ag_spmm_fwd_static_scratch", "ag_step_host",
                 "ag_step_host_pipelined", "ag_abi_version",
                 "ag_mean_fwd", "ag_mean_backward", "ag_gcn_norm", "ag_attn_fwd", "ag_attn_backward"):
        getattr(handle, name).restype = _I
    return handle


lib = _bind(ctypes.CDLL(LIB_PATH))


def declared_symbols(header: str = HEADER_PATH) -> list[str]:
    """Names of the functions include/aggraph.h declares."""
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ag_[a-z0-9_]+)\s*\(", text)))


def _check(rc: int) -> None:
    if rc != 0:
        raise AggraphError(rc, lib.ag_last_error().decode(errors="replace"))


def _stream(device: torch.device, stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream if hasattr(s, "cuda_stream") else int(s))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return AG_F32
    if t.dtype == torch.bfloat16:
        return AG_BF16
    raise AggraphError(3, f"feature dtype {t.dtype} is not supported (float32 or bfloat16)")


def _ptr(t: torch.Tensor | None):
    return None if t is None or t.numel() == 0 else ctypes.c_void_p(t.data_ptr())


def _need_cuda(name: str, t: torch.Tensor) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise AggraphError(4, f"{name} must be a CUDA tensor (got device {t.device})")
    if not t.is_contiguous():
        raise AggraphError(2, f"{name} must be contiguous")


def ag_graph_workspace_bytes(N: int, E: int) -> int:
    return int(lib.ag_graph_workspace_bytes(N, E))


class Graph:
    """A lowered fixed topology (owns its device workspace tensor)."""

    def __init__(self, src: torch.Tensor, dst: torch.Tensor, num_nodes: int, stream=None):
        for name, t in (("src", src), ("dst", dst)):
            _need_cuda(name, t)
            if t.dtype != torch.int32 or t.dim() != 1:
                raise AggraphError(3 if t.dtype != torch.int32 else 2, f"{name} must be a 1-D int32 tensor")
        if src.shape != dst.shape:
            raise AggraphError(2, "src and dst must have the same length")
        self.device = src.device
        self.N, self.E = int(num_nodes), int(src.shape[0])
        nbytes = ag_graph_workspace_bytes(self.N, self.E)
        if nbytes == 0:
            raise AggraphError(2, f"unsupported sizes N={self.N}, E={self.E}")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        handle = ctypes.c_void_p()
        self._h = None
        _check(lib.ag_graph_lower(_ptr(src), _ptr(dst), self.N, self.E,
                                  ctypes.c_void_p(self.workspace.data_ptr()), nbytes,
                                  _stream(self.device, stream), ctypes.byref(handle)))
        self._h = handle
        st = Stats()
        _check(lib.ag_graph_get_stats(self._h, ctypes.byref(st)))
        self.stats = st.as_dict()
        self._scratch: dict = {}
        self._step_scratch: dict = {}

    @property
    def handle(self) -> ctypes.c_void_p:
        if self._h is None:
            raise AggraphError(1, "graph is closed")
        return self._h

    def scratch_bytes(self, H: int) -> int:
        return int(lib.ag_spmm_scratch_bytes(self.handle, H))

    def scratch(self, H: int) -> torch.Tensor | None:
        """Device scratch of the per-call functions at width H (allocated once per H)."""
        n = self.scratch_bytes(H)
        if n == 0:
            return None
        t = self._scratch.get(H)
        if t is None:
            t = torch.empty(n, dtype=torch.uint8, device=self.device)
            self._scratch[H] = t
        return t

    def arrays(self) -> dict:
        """Device int32 views of rowptr_f, col_f, edge_order, rowptr_t, col_t, transpose_order."""
        ptrs = [ctypes.c_void_p() for _ in range(6)]
        _check(lib.ag_graph_arrays(self.handle, *[ctypes.byref(p) for p in ptrs]))
        base = self.workspace.data_ptr()
        names = ("rowptr_f", "col_f", "edge_order", "rowptr_t", "col_t", "transpose_order")
        sizes = (self.N + 1, self.E, self.E, self.N + 1, self.E, self.E)
        out = {}
        for name, p, n in zip(names, ptrs, sizes):
            off = (p.value or base) - base
            out[name] = self.workspace[off:off + 4 * n].view(torch.int32)
        return out

    def close(self) -> None:
        if self._h is not None:
            lib.ag_graph_free(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # convenience methods
    def fwd(self, w, X, out=None, stream=None):
        return ag_spmm_fwd(self, w, X, out, stream)

    def dx(self, w, dY, out=None, stream=None):
        return ag_spmm_dx(self, w, dY, out, stream)

    def dw(self, X, dY, out=None, stream=None):
        return ag_sddmm_dw(self, X, dY, out, stream)

    def backward(self, w, X, dY, dX=None, dw=None, stream=None):
        return ag_backward(self, w, X, dY, dX, dw, stream)


def ag_graph_lower(src: torch.Tensor, dst: torch.Tensor, N: int, stream=None) -> Graph:
    return Graph(src, dst, N, stream)


def _check_feat(g: Graph, name: str, t: torch.Tensor) -> int:
    _need_cuda(name, t)
    if t.dim() != 2 or t.shape[0] != g.N:
        raise AggraphError(2, f"{name} must be [N={g.N}, H], got {tuple(t.shape)}")
    return _dtype_code(t)


def _check_edge_vec(g: Graph, name: str, t: torch.Tensor) -> None:
    _need_cuda(name, t)
    if t.dtype != torch.float32:
        raise AggraphError(3, f"{name} must be float32")
    if t.dim() != 1 or t.shape[0] != g.E:
        raise AggraphError(2, f"{name} must be [E={g.E}], got {tuple(t.shape)}")


def _spmm(fn, g: Graph, w, F, out, stream, names, w_optional=False):
    if w is not None or not w_optional:
        _check_edge_vec(g, "w", w)
    code = _check_feat(g, names[0], F)
    H = F.shape[1]
    if out is None:
        out = torch.empty_like(F)
    elif out.shape != F.shape or out.dtype != F.dtype:
        raise AggraphError(2, f"{names[1]} must match {names[0]} in shape and dtype")
    else:
        _need_cuda(names[1], out)
    scr = g.scratch(H)
    _check(fn(g.handle, _ptr(w), _ptr(F), _ptr(out), H, code, _ptr(scr),
              0 if scr is None else scr.numel(), _stream(g.device, stream)))
    return out


def ag_spmm_fwd(g: Graph, w: torch.Tensor, X: torch.Tensor, out=None, stream=None) -> torch.Tensor:
    """Y = A_w X (destination-owned forward CSR)."""
    return _spmm(lib.ag_spmm_fwd, g, w, X, out, stream, ("X", "Y"))


def ag_spmm_dx(g: Graph, w: torch.Tensor, dY: torch.Tensor, out=None, stream=None) -> torch.Tensor:
    """dX = A_w^T dY (source-owned transpose CSR)."""
    return _spmm(lib.ag_spmm_dx, g, w, dY, out, stream, ("dY", "dX"))


def ag_sddmm_dw(g: Graph, X: torch.Tensor, dY: torch.Tensor, out=None, stream=None) -> torch.Tensor:
    """dw_e = dot(X[src_e], dY[dst_e]) in COO order (float32 [E])."""
    code = _check_feat(g, "X", X)
    if _check_feat(g, "dY", dY) != code or dY.shape != X.shape:
        raise AggraphError(2, "X and dY must have the same shape and dtype")
    if out is None:
        out = torch.empty(g.E, dtype=torch.float32, device=g.device)
    else:
        _check_edge_vec(g, "dw", out)
    scr = g.scratch(X.shape[1])
    _check(lib.ag_sddmm_dw(g.handle, _ptr(X), _ptr(dY), _ptr(out), X.shape[1], code, _ptr(scr),
                           0 if scr is None else scr.numel(), _stream(g.device, stream)))
    return out


def ag_backward(g: Graph, w: torch.Tensor, X: torch.Tensor, dY: torch.Tensor, dX=None, dw=None,
                stream=None):
    """(dX, dw) = (A_w^T dY, dot(X[src_e], dY[dst_e])) in one pass over the transpose CSR."""
    _check_edge_vec(g, "w", w)
    code = _check_feat(g, "X", X)
    if _check_feat(g, "dY", dY) != code or dY.shape != X.shape:
        raise AggraphError(2, "X and dY must have the same shape and dtype")
    if dX is None:
        dX = torch.empty_like(dY)
    elif dX.shape != dY.shape or dX.dtype != dY.dtype:
        raise AggraphError(2, "dX must match dY in shape and dtype")
    else:
        _need_cuda("dX", dX)
    if dw is None:
        dw = torch.empty(g.E, dtype=torch.float32, device=g.device)
    else:
        _check_edge_vec(g, "dw", dw)
    H = X.shape[1]
    scr = g.scratch(H)
    _check(lib.ag_backward(g.handle, _ptr(w), _ptr(X), _ptr(dY), _ptr(dX), _ptr(dw), H, code, _ptr(scr),
                           0 if scr is None else scr.numel(), _stream(g.device, stream)))
    return dX, dw


def ag_step(g: Graph, w: torch.Tensor, X: torch.Tensor, dY: torch.Tensor, Y=None, dX=None, dw=None,
            stream=None):
    """(Y, dX, dw) = (A_w X, A_w^T dY, dot(X[src_e], dY[dst_e])) in one call: the forward
    pass and the fused backward pass, overlapped (bitwise equal to ag_spmm_fwd + ag_backward)."""
    _check_edge_vec(g, "w", w)
    code = _check_feat(g, "X", X)
    if _check_feat(g, "dY", dY) != code or dY.shape != X.shape:
        raise AggraphError(2, "X and dY must have the same shape and dtype")
    outs = []
    for name, t in (("Y", Y), ("dX", dX)):
        if t is None:
            t = torch.empty_like(X)
        elif t.shape != X.shape or t.dtype != X.dtype:
            raise AggraphError(2, f"{name} must match X in shape and dtype")
        else:
            _need_cuda(name, t)
        outs.append(t)
    if dw is None:
        dw = torch.empty(g.E, dtype=torch.float32, device=g.device)
    else:
        _check_edge_vec(g, "dw", dw)
    H = X.shape[1]
    n = int(lib.ag_step_scratch_bytes(g.handle, H))
    scr = g._step_scratch.get(H)
    if scr is None or scr.numel() < n:
        scr = torch.empty(max(n, 1), dtype=torch.uint8, device=g.device)
        g._step_scratch[H] = scr
    _check(lib.ag_step(g.handle, _ptr(w), _ptr(X), _ptr(dY), _ptr(outs[0]), _ptr(outs[1]), _ptr(dw), H, code,
                       _ptr(scr), n, _stream(g.device, stream)))
    return outs[0], outs[1], dw


def ag_mean_fwd(g: Graph, w, X: torch.Tensor, out=None, stream=None) -> torch.Tensor:
    """Y[r] = mean over the edges into r of w_e X[src_e] (w=None: unit weights)."""
    return _spmm(lib.ag_mean_fwd, g, w, X, out, stream, ("X", "Y"), w_optional=True)


def ag_mean_backward(g: Graph, w, X: torch.Tensor, dY: torch.Tensor, dX=None, dw=None, want_dw=True,
                     stream=None):
    """Gradients of ag_mean_fwd: (dX, dw) with dw = None when want_dw is False."""
    if w is not None:
        _check_edge_vec(g, "w", w)
    code = _check_feat(g, "X", X)
    if _check_feat(g, "dY", dY) != code or dY.shape != X.shape:
        raise AggraphError(2, "X and dY must have the same shape and dtype")
    if dX is None:
        dX = torch.empty_like(dY)
    elif dX.shape != dY.shape or dX.dtype != dY.dtype:
        raise AggraphError(2, "dX must match dY in shape and dtype")
    else:
        _need_cuda("dX", dX)
    if want_dw:
        if dw is None:
            dw = torch.empty(g.E, dtype=torch.float32, device=g.device)
        else:
            _check_edge_vec(g, "dw", dw)
    else:
        dw = None
    H = X.shape[1]
    scr = g.scratch(H)
    _check(lib.ag_mean_backward(g.handle, _ptr(w), _ptr(X), _ptr(dY), _ptr(dX), _ptr(dw), H, code, _ptr(scr),
                                0 if scr is None else scr.numel(), _stream(g.device, stream)))
    return dX, dw


def ag_gcn_norm(g: Graph, w=None, out=None, stream=None) -> torch.Tensor:
    """GCN-normalised weights D^-1/2 A_w D^-1/2 in COO order (w=None: unit weights)."""
    if w is not None:
        _check_edge_vec(g, "w", w)
    if out is None:
        out = torch.empty(g.E, dtype=torch.float32, device=g.device)
    else:
        _check_edge_vec(g, "w_norm", out)
    n = int(lib.ag_gcn_norm_scratch_bytes(g.handle))
    scr = torch.empty(max(n, 1), dtype=torch.uint8, device=g.device)
    _check(lib.ag_gcn_norm(g.handle, _ptr(w), _ptr(out), _ptr(scr), n, _stream(g.device, stream)))
    return out


def _attn_scratch(g: Graph, H: int) -> torch.Tensor:
    n = int(lib.ag_attn_scratch_bytes(g.handle, H))
    key = ("attn", H)
    t = g._scratch.get(key)
    if t is None or t.numel() < n:
        t = torch.empty(max(n, 1), dtype=torch.uint8, device=g.device)
        g._scratch[key] = t
    return t


def _same_feats(g: Graph, names, ts) -> int:
    code = _check_feat(g, names[0], ts[0])
    for name, t in zip(names[1:], ts[1:]):
        if _check_feat(g, name, t) != code or t.shape != ts[0].shape:
            raise AggraphError(2, f"{name} must match {names[0]} in shape and dtype")
    return code


def ag_attn_fwd(g: Graph, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, scale: float, Y=None, alpha=None,
                stream=None):
    """Edge-softmax attention: (Y, alpha) with alpha in COO order."""
    code = _same_feats(g, ("Q", "K", "V"), (Q, K, V))
    if Y is None:
        Y = torch.empty_like(V)
    else:
        _same_feats(g, ("V", "Y"), (V, Y))
    if alpha is None:
        alpha = torch.empty(g.E, dtype=torch.float32, device=g.device)
    else:
        _check_edge_vec(g, "alpha", alpha)
    H = Q.shape[1]
    scr = _attn_scratch(g, H)
    _check(lib.ag_attn_fwd(g.handle, _ptr(Q), _ptr(K), _ptr(V), float(scale), _ptr(Y), _ptr(alpha), H, code,
                           _ptr(scr), scr.numel(), _stream(g.device, stream)))
    return Y, alpha


def ag_attn_backward(g: Graph, Q, K, V, scale: float, alpha, dY, dQ=None, dK=None, dV=None, stream=None):
    """Gradients (dQ, dK, dV) of ag_attn_fwd for the upstream gradient dY."""
    code = _same_feats(g, ("Q", "K", "V", "dY"), (Q, K, V, dY))
    _check_edge_vec(g, "alpha", alpha)
    outs = []
    for name, t in (("dQ", dQ), ("dK", dK), ("dV", dV)):
        if t is None:
            t = torch.empty_like(Q)
        else:
            _same_feats(g, ("Q", name), (Q, t))
        outs.append(t)
    H = Q.shape[1]
    scr = _attn_scratch(g, H)
    _check(lib.ag_attn_backward(g.handle, _ptr(Q), _ptr(K), _ptr(V), float(scale), _ptr(alpha), _ptr(dY),
                                _ptr(outs[0]), _ptr(outs[1]), _ptr(outs[2]), H, code, _ptr(scr), scr.numel(),
                                _stream(g.device, stream)))
    return tuple(outs)


def ag_spmm_fwd_static_scratch(g: Graph, w: torch.Tensor, X: torch.Tensor, out=None, stream=None) -> torch.Tensor:
    """Y = A_w X like ag_spmm_fwd, using the library's built-in scratch array
    instead of a scratch tensor, for callers that cannot allocate device
    memory at call time (see include/aggraph.h for the limits)."""
    _check_edge_vec(g, "w", w)
    code = _check_feat(g, "X", X)
    if out is None:
        out = torch.empty_like(X)
    elif out.shape != X.shape or out.dtype != X.dtype:
        raise AggraphError(2, "Y must match X in shape and dtype")
    else:
        _need_cuda("Y", out)
    _check(lib.ag_spmm_fwd_static_scratch(g.handle, _ptr(w), _ptr(X), _ptr(out), X.shape[1], code,
                                          _stream(g.device, stream)))
    return out


def ag_step_staging_bytes(g: Graph, H: int, dtype: torch.dtype) -> int:
    code = AG_F32 if dtype == torch.float32 else AG_BF16
    return int(lib.ag_step_staging_bytes(g.handle, H, code))


def ag_step_host(g: Graph, w: torch.Tensor, X: torch.Tensor, dY: torch.Tensor, Y: torch.Tensor,
                 dX: torch.Tensor, dw: torch.Tensor, staging: torch.Tensor, stream=None, pipelined=False) -> None:
    """Forward, feature gradient and weight gradient from host buffers.

    w, X, dY are host inputs and Y, dX, dw host outputs (page-locked tensors
    make the copies asynchronous); staging is a device uint8 tensor of
    ag_step_staging_bytes(g, H, X.dtype) bytes.  Enqueues on `stream`; the
    outputs are valid after that stream is synchronized.  pipelined=True calls
    ag_step_host_pipelined (the staging tensor then belongs to the steps)."""
    for name, t in (("w", w), ("X", X), ("dY", dY), ("Y", Y), ("dX", dX), ("dw", dw)):
        if t.is_cuda or not t.is_contiguous():
            raise AggraphError(4, f"{name} must be a contiguous host tensor")
    code = _dtype_code(X)
    _need_cuda("staging", staging)
    fn = lib.ag_step_host_pipelined if pipelined else lib.ag_step_host
    _check(fn(g.handle, _ptr(w), _ptr(X), _ptr(dY), _ptr(Y), _ptr(dX), _ptr(dw),
              X.shape[1], code, ctypes.c_void_p(staging.data_ptr()), staging.numel(),
              _stream(g.device, stream)))


def ag_step_host_pipelined(g: Graph, w: torch.Tensor, X: torch.Tensor, dY: torch.Tensor, Y: torch.Tensor,
                           dX: torch.Tensor, dw: torch.Tensor, staging: torch.Tensor, stream=None) -> None:
    """ag_step_host for back-to-back steps: this step's copies in overlap the
    previous step's copies out on the same staging tensor."""
    ag_step_host(g, w, X, dY, Y, dX, dw, staging, stream, pipelined=True)
