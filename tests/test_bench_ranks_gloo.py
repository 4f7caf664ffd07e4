"""The multi-rank logic of bench.py on CPU: two gloo ranks."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    slowest = bench.max_over_ranks(10.0 + 5.0 * rank, torch.device("cpu"))
    rate = bench.whole_job_rate(world, 1000, 4, slowest)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, slowest, rate))


def test_max_over_ranks_and_whole_job_rate():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, slowest, rate in got:
        assert slowest == 15.0                       # max over ranks, on every rank
        assert rate == pytest.approx(2 * 1000 * 4 / 0.015)


def test_single_rank_is_identity():
    import torch
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--gpus", "2"],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.strip() == ""


def test_reference_arm_prints_the_contract_line():
    # the oracle on a small workload: one JSON line with the base contract's
    # keys, the reference marker and the CPU-baseline / end-to-end objects
    import json
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "uniform",
                          "--steps", "2", "--warmup", "1", "--cpu-seconds", "0.2"],
                         cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 2 and d["warmup"] == 1
    assert d["higher_is_better"] is True and d["vs_baseline"] is None
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert "N=1024, E=8192, H=16" in d["config"]["workload"]


def test_algorithmic_bytes_and_launch_count():
    sys.path.insert(0, ROOT)
    import bench
    N, E, H = 1 << 22, 1 << 26, 128
    a = bench.algorithmic_bytes(N, E, H, 2)
    # CSR + order map + weights + input rows once + output rows once
    assert a["fwd"] == 4 * (N + 1) + 12 * E + 2 * N * H * 2
    assert abs(a["fwd"] / 1e9 - 2.97) < 0.01 and abs(a["backward"] / 1e9 - 4.31) < 0.01
    rows = bench.row_bytes(N, E, H, 2)
    assert rows["mean_fwd"] == a["fwd"] and rows["mean_backward"] == a["backward"]

    class W:
        pass
    wl = W()
    wl.E, wl.N = E, N
    st = {"spanning_rows_f": 5, "spanning_rows_t": 0}
    assert bench.launches_per_step_of(st, wl) == 3 + 3
    wl.E = 0
    assert bench.launches_per_step_of(st, wl) == 2


def test_traffic_record_keys_on_code_not_comments():
    sys.path.insert(0, ROOT)
    import bench
    src = 'int a = 1; // note\n/* block\n comment */ const char *s = "// kept /* too */";\n\n  char c = \'"\';  \n'
    assert bench.code_only(src) == 'int a = 1;\n  const char *s = "// kept /* too */";\n  char c = \'"\';'
    assert bench.code_only("x = 1;\n// only a comment\n") == bench.code_only("x = 1;\n")
    assert bench.code_only("x = 1;") != bench.code_only("x = 2;")


def test_dram_fraction():
    sys.path.insert(0, ROOT)
    import bench
    # 11.42 GB in 3.16 ms against 6551.4 GB/s: about 55 %
    assert abs(bench.dram_frac(11.42e9, 3.16, 6551.4) - 0.5516) < 1e-3
