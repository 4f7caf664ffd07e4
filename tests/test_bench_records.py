"""The committed ncu records that bench.py reports beside its timings (CPU).

bench.py attaches measured DRAM bytes and the walks' L2 hit rates to its JSON
line only while the record was taken on the current kernel sources; these
tests check that gate and the shape of the committed record, without a GPU.
"""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

RECORD = os.path.join(ROOT, "profiles", "dram_traffic.json")


def test_committed_record_covers_the_four_calls():
    with open(RECORD) as f:
        d = json.load(f)
    rec = d["rmat22"]
    for op in ("fwd", "backward", "dx", "dw"):
        r = rec[op]
        assert len(r["source_hash"]) == 16
        assert r["bytes_per_launch"] == sum(r["kernels"].values())
        assert 0.0 < r["l2_hit"]["pct"] < 100.0
        assert r["l2_hit"]["kernel"].startswith(("k_tiles_ring", "k_walk"))
    # the calls' DRAM bytes exceed their algorithmic bytes (2.97 / 4.31 GB)
    algo = bench.algorithmic_bytes(1 << 22, 1 << 26, 128, 2)
    assert rec["fwd"]["bytes_per_launch"] > algo["fwd"]
    assert rec["backward"]["bytes_per_launch"] > algo["backward"]


def test_record_is_reported_only_for_matching_sources(monkeypatch):
    with open(RECORD) as f:
        h = json.load(f)["rmat22"]["backward"]["source_hash"]
    monkeypatch.setattr(bench, "source_hash", lambda: h)
    assert bench.ncu_traffic("rmat22", "backward") > 0
    assert bench.ncu_l2_hit("rmat22", "backward")["pct"] > 0
    monkeypatch.setattr(bench, "source_hash", lambda: "0" * 16)
    assert bench.ncu_traffic("rmat22", "backward") is None
    assert bench.ncu_l2_hit("rmat22", "backward") is None
    # other workloads have no record
    monkeypatch.setattr(bench, "source_hash", lambda: h)
    assert bench.ncu_record("twohop", "backward") is None


@pytest.mark.parametrize("edit", ["comment", "blank"])
def test_source_hash_ignores_comments_and_blank_lines(edit):
    code = "int f() {\n    return 1;  // one\n}\n"
    other = code.replace("// one", "// another") if edit == "comment" else code.replace("{\n", "{\n\n")
    assert bench.code_only(code) == bench.code_only(other)
    assert bench.code_only(code) != bench.code_only(code.replace("return 1", "return 2"))


def test_clock_summary_keeps_the_samples_of_the_timed_region():
    import datetime
    clk = bench.ClockSampler(0)
    base = datetime.datetime(2026, 1, 2, 3, 4, 5)
    lines = []
    for k, mhz in enumerate([345, 345, 1965, 1950, 1965, 345]):   # idle, idle, load x3, idle
        stamp = (base + datetime.timedelta(milliseconds=20 * k)).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        cap = "Active" if k == 3 else "Not Active"
        lines.append(f"{stamp}, 0, {mhz}, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, {cap}")
    clk.out.write("\n".join(lines).encode() + b"\n")
    clk.t0 = base + datetime.timedelta(milliseconds=30)
    clk.t1 = base + datetime.timedelta(milliseconds=90)
    s = clk.summary()
    assert s["samples"] == 3 and s["sm_mhz"] == 1965 and s["window"] == "timed region"
    assert s["reasons"] == ["sw_power_cap"] and s["sm_max_mhz"] == 1965


def test_clock_summary_falls_back_when_the_region_is_shorter_than_a_sample():
    import datetime
    clk = bench.ClockSampler(0)
    base = datetime.datetime(2026, 1, 2, 3, 4, 5)
    stamp = base.strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    clk.out.write(f"{stamp}, 0, 1900, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, Not Active\n".encode())
    clk.t0 = base + datetime.timedelta(milliseconds=5)
    clk.t1 = base + datetime.timedelta(milliseconds=8)
    s = clk.summary()
    assert s["samples"] == 1 and s["window"] == "around the timed region" and s["reasons"] == []
