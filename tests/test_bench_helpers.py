"""CPU checks of bench.py's bookkeeping behind the reported roofline: the kernel
source hash, the stored per-launch DRAM traffic it gates, and the timing summary."""
import json
import os
import re

import numpy as np
import pytest

import bench
from io_aware_exact_24_b200.inputs import DECODE_WORKLOADS, WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_hashed_sources_cover_every_forward_source_the_library_includes():
    # a forward source left out of the hash would let stored traffic outlive a kernel change
    api = open(os.path.join(ROOT, "io_aware_exact_24_b200/csrc/fa_api.cu")).read()
    included = set(re.findall(r'#include "([\w.]+\.cuh)"', api))
    hashed = {os.path.basename(p) for p in bench.KERNEL_SOURCES}
    for f in included:
        if f == "fa_bwd_kernel.cuh":
            continue                      # the backward is not on the forward's roofline line
        assert f in hashed, f
    for p in bench.KERNEL_SOURCES:
        assert os.path.exists(os.path.join(ROOT, p)), p


def test_source_hash_is_stable_and_follows_the_sources(tmp_path, monkeypatch):
    h = bench.kernel_source_hash()
    assert re.fullmatch(r"[0-9a-f]{16}", h) and h == bench.kernel_source_hash()
    a, b = tmp_path / "a.cuh", tmp_path / "b.cu"
    a.write_text("x")
    b.write_text("y")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", ["a.cuh", "b.cu"])
    h1 = bench.kernel_source_hash()
    a.write_text("x ")
    assert bench.kernel_source_hash() != h1


def test_stored_traffic_is_used_only_for_the_sources_it_was_measured_on(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    (tmp_path / "k.cuh").write_text("kernel")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", ["k.cuh"])
    h = bench.kernel_source_hash()
    entry = {"kernel_source_hash": h, "dram_bytes_per_launch": 123, "dram_read_bytes": 100,
             "dram_write_bytes": 23}
    (tmp_path / "profiles" / "dram_traffic.json").write_text(json.dumps({"w": entry}))
    assert bench.load_traffic("w") == 123
    assert bench.load_traffic("other") is None
    (tmp_path / "k.cuh").write_text("kernel, changed")
    assert bench.load_traffic("w") is None


def test_committed_traffic_entries_are_consistent():
    d = json.load(open(os.path.join(ROOT, "profiles", "dram_traffic.json")))
    for name in ("causal_8000_d128", "long_16k_d64"):
        e = d[name]
        assert re.fullmatch(r"[0-9a-f]{16}", e["kernel_source_hash"])
        assert e["dram_bytes_per_launch"] == e["dram_read_bytes"] + e["dram_write_bytes"]
        # reads cover the inputs once (Q, K, V, a few % of K/V re-read across head
        # groups); writes are O and LSE, part of which is still in L2 at the end
        w = WORKLOADS[name]
        qkv = 2 * w.B * w.H * (w.Nq + 2 * w.Nk) * w.d
        out = 2 * w.B * w.H * w.Nq * w.d + 4 * w.B * w.H * w.Nq
        assert 0.98 * qkv <= e["dram_read_bytes"] <= 1.10 * qkv, name
        assert 0.0 <= e["dram_write_bytes"] <= 1.01 * out, name


def test_ms_stats():
    s = bench.ms_stats([1.0, 2.0, 3.0, 4.0, 10.0])
    assert s["mean"] == pytest.approx(4.0) and s["median"] == 3.0 and s["n"] == 5
    assert s["p10"] == pytest.approx(np.percentile([1, 2, 3, 4, 10], 10))
    assert s["p90"] == pytest.approx(np.percentile([1, 2, 3, 4, 10], 90))


def test_kv_larger_than_l2_decides_the_decode_flush():
    assert bench.kv_exceeds_l2(DECODE_WORKLOADS["decode_64k_h8_d128"])    # 268 MB of K and V
    assert bench.kv_exceeds_l2(DECODE_WORKLOADS["decode_16k_d128"])       # 1.07 GB
    assert not bench.kv_exceeds_l2(WORKLOADS["tiny"])
