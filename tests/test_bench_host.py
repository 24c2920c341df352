"""Host-side logic of bench.py: the algorithmic byte counts behind the
roofline, the traffic record's validity check, the mean context lengths and
the L2 statement of the JSON line's config."""
import json
import math
import os
import shutil

import numpy as np

import bench
from workloads.qsa_inputs import WORKLOADS


def test_algorithmic_bytes_256k():
    w = WORKLOADS["b128_256k"]           # T=1, Hq 16, Hkv 2, D 128, bf16, d 128, page 64
    b = bench.algorithmic_bytes(w, 262144, 2)
    n = 65536                            # blocks of a 262,144-token context
    kc = n * (128 + 128 // 4)            # packed keys: low bytes + 2-bit fields
    assert b["index_topk"] == kc + (262144 // 64) * 4 + 128 + 512 * 4
    tokens = 512 * 4
    kv = 2 * tokens * 2 * 128 * 2        # K and V rows of both kv heads
    q = 16 * 128 * 2
    partials = 2 * 16 * (128 + 1) * 4
    assert b["sparse_decode"] == kv + q + 512 * 4 + partials
    # the per-launch figure of the bench line at batch 128
    assert 128 * b["index_topk"] == 1344552960


def test_algorithmic_bytes_fp8_scales_and_mtp_tail():
    w = WORKLOADS["mixed_fp8"]           # e4m3 K/V: 1 byte per element plus scales
    b = bench.algorithmic_bytes(w, 65536, 4)
    tokens = 512 * 4
    assert b["sparse_decode"] >= 2 * tokens * w.Hkv * w.D
    wm = WORKLOADS["mtp_verify"]         # T = 4: the 3 speculative tokens are attended too
    bm = bench.algorithmic_bytes(wm, 65536, 2)
    b1 = bench.algorithmic_bytes(WORKLOADS["b128_256k"], 65536, 2)
    assert bm["sparse_decode"] > b1["sparse_decode"]


def test_traffic_record_checks_the_kernel_source(tmp_path, monkeypatch):
    """The record's traffic is reported only for the kernel source it was
    captured from (checked on a copy of the record pointed at a file of
    known contents)."""
    import hashlib
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "roofline_traffic.json")))
    src = tmp_path / rec["source"]
    os.makedirs(src.parent)
    src.write_text("// kernel source\n")
    rec["source_sha256_prefix"] = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    os.makedirs(tmp_path / "profiles")
    with open(tmp_path / "profiles" / "roofline_traffic.json", "w") as f:
        json.dump(rec, f)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.index_topk_traffic(128) == rec["dram_bytes_per_request"] * 128
    src.write_text("// kernel source\n// changed\n")   # the source moved on: no figure
    assert bench.index_topk_traffic(128) is None


def test_mean_context_of_the_distributions():
    assert bench.mean_context(WORKLOADS["b128_256k"]) == 262144
    assert bench.mean_context(WORKLOADS["mtp_verify"]) == (16384 + 262144) / 2
    rng = np.random.default_rng(0)
    lo, hi = 4096, 1048576
    x = np.exp(rng.uniform(math.log(lo), math.log(hi), size=400_000))
    assert abs(bench.mean_context(WORKLOADS["mixed_fp8"]) / x.mean() - 1) < 0.01


def test_l2_statement():
    big = bench.workload_config(WORKLOADS["b128_256k"], 2, 1)["l2"]
    small = bench.workload_config(WORKLOADS["tiny"], 1, 1)["l2"]
    assert big.startswith("inputs larger than L2") and small.startswith("inputs smaller than L2")


def test_parallel_oracle_timing_counts_every_core():
    res = bench.time_oracle_parallel(WORKLOADS["tiny"], 1, 1, 2)
    assert res["cores"] == 2 and res["queries"] == 2 and res["value"] > 0
