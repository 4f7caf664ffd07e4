"""The C-ABI library loads and exports what include/aggraph.h declares, and its
host-side argument checks answer without a GPU (no compute call here)."""
import ctypes
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def agb():
    from __graft_entry__ import build_library
    build_library()
    import gnn_sparse_aggregation_b200 as m
    return m


def test_every_declared_symbol_is_exported(agb):
    names = agb.declared_symbols()
    assert {"ag_graph_lower", "ag_spmm_fwd", "ag_spmm_dx", "ag_sddmm_dw"} <= set(names)
    out = subprocess.run(["nm", "-D", "--defined-only", agb.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in names:
        assert name in exported, name
        assert hasattr(agb.lib, name)
    # nothing else of ours leaks out of the library
    ours = {s for s in exported if s.startswith("ag_")}
    assert ours == set(names)


def test_status_strings_and_version(agb):
    assert agb.lib.ag_abi_version() == 102
    for code, name in agb._STATUS.items():
        assert agb.lib.ag_status_string(code).decode() == name


def test_workspace_bytes_is_linear_and_rejects_bad_sizes(agb):
    f = agb.ag_graph_workspace_bytes
    assert f(0, 10) == 0 and f(-1, 0) == 0 and f(10, -1) == 0
    assert f(1 << 31, 0) == 0 and f(10, 1 << 31) == 0
    assert f(1, 0) > 0
    # at least the two CSRs and two order maps of "Edge order is explicit"
    for N, E in ((1, 0), (3, 3), (1000, 8192), (1 << 22, 1 << 26)):
        assert f(N, E) >= 4 * (2 * E + 2 * (N + 1) + 2 * E)
    # O(N + E): a fixed number of bytes per node and per edge, plus alignment slack
    big = f(1 << 22, 1 << 26)
    assert big <= 64 * (1 << 22) + 64 * (1 << 26)


def test_host_side_rejections_without_gpu(agb):
    lib = agb.lib
    out = ctypes.c_void_p()
    assert lib.ag_graph_lower(None, None, 0, 0, None, 0, None, ctypes.byref(out)) == 2
    assert b"N" in lib.ag_last_error()
    assert lib.ag_graph_lower(None, None, 5, -1, None, 0, None, ctypes.byref(out)) == 2
    assert lib.ag_graph_lower(None, None, 5, 3, ctypes.c_void_p(256), 1 << 20, None,
                              ctypes.byref(out)) == 1                     # null src/dst, E > 0
    assert lib.ag_graph_lower(None, None, 5, 0, None, 0, None, ctypes.byref(out)) == 1
    assert lib.ag_graph_lower(None, None, 5, 0, ctypes.c_void_p(256), 16, None,
                              ctypes.byref(out)) == 7                     # workspace too small
    assert lib.ag_graph_lower(None, None, 5, 0, ctypes.c_void_p(8), 1 << 20, None,
                              ctypes.byref(out)) == 7                     # misaligned
    assert out.value is None
    assert lib.ag_spmm_fwd(None, None, None, None, 4, 0, None, 0, None) == 1
    assert lib.ag_spmm_dx(None, None, None, None, 4, 0, None, 0, None) == 1
    assert lib.ag_sddmm_dw(None, None, None, None, 4, 0, None, 0, None) == 1
    assert lib.ag_mean_fwd(None, None, None, None, 4, 0, None, 0, None) == 1
    assert lib.ag_mean_backward(None, None, None, None, None, None, 4, 0, None, 0, None) == 1
    assert lib.ag_gcn_norm(None, None, None, None, 0, None) == 1
    assert lib.ag_gcn_norm_scratch_bytes(None) == 0
    assert lib.ag_attn_fwd(None, None, None, None, 1.0, None, None, 4, 0, None, 0, None) == 1
    assert lib.ag_attn_backward(None, None, None, None, 1.0, None, None, None, None, None, 4, 0, None, 0,
                                None) == 1
    assert lib.ag_attn_scratch_bytes(None, 4) == 0
    assert lib.ag_graph_get_stats(None, None) == 1
    assert lib.ag_spmm_scratch_bytes(None, 4) == 0
    assert lib.ag_step_staging_bytes(None, 4, 0) == 0
    for step in (lib.ag_step_host, lib.ag_step_host_pipelined):
        assert step(None, None, None, None, None, None, None, 4, 0, None, 0, None) == 1
    lib.ag_graph_free(None)


def test_product_path_does_not_touch_the_oracle():
    code = ("import sys; import gnn_sparse_aggregation_b200 as m; "
            "assert not any(k == 'oracle' or k.startswith('oracle.') for k in sys.modules), "
            "[k for k in sys.modules if 'oracle' in k]")
    subprocess.run([sys.executable, "-c", code], cwd=ROOT, check=True)
    pkg = os.path.join(ROOT, "gnn_sparse_aggregation_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".h", ".cuh", ".cpp")):
                text = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in text and "from oracle" not in text, fn
                assert "liboracle" not in text and "oracle.c" not in text, fn


def test_binding_refuses_cpu_tensors(agb):
    import torch
    src = torch.zeros(3, dtype=torch.int32)
    with pytest.raises(agb.AggraphError) as ei:
        agb.ag_graph_lower(src, src, 3)
    assert ei.value.status_name == "AG_ERR_DEVICE"
