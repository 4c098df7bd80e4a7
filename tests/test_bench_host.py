"""Host-side pieces of bench.py that decide what its JSON line claims: the
committed kernel (1) DRAM traffic is reported only for the workload and the
kernel sources it was captured on, and each workload's line names its own
input recipe."""
import json
import os

import bench
from token_level_sparse_causal_b200 import inputs


def test_recorded_traffic_only_for_its_own_workload_and_sources(tmp_path):
    good = tmp_path / "dram.json"
    good.write_text(json.dumps({"workload": "c3_L131072_h64x8_gmm", "dram_bytes_per_launch": 12345,
                                "kernel_source_sha256_16": bench.kernel_source_hash()}))
    assert bench.recorded_traffic("c3_L131072_h64x8_gmm", str(good)) == 12345.0
    assert bench.recorded_traffic("c4_L262144_h64x8_chains", str(good)) is None
    stale = tmp_path / "stale.json"
    stale.write_text(json.dumps({"workload": "c3_L131072_h64x8_gmm", "dram_bytes_per_launch": 12345,
                                 "kernel_source_sha256_16": "0000000000000000"}))
    assert bench.recorded_traffic("c3_L131072_h64x8_gmm", str(stale)) is None
    assert bench.recorded_traffic("c3_L131072_h64x8_gmm", str(tmp_path / "missing.json")) is None
    bad = tmp_path / "bad.json"
    bad.write_text("not json")
    assert bench.recorded_traffic("c3_L131072_h64x8_gmm", str(bad)) is None


def test_committed_traffic_record_is_well_formed():
    """The committed record names its workload, the reduced-head copy it was
    measured on and the scale to a full launch (whether its hash is current
    depends on the kernel sources)."""
    if not os.path.exists(bench.FA_TRAFFIC_PROFILE):
        return
    rec = json.load(open(bench.FA_TRAFFIC_PROFILE))
    assert rec["workload"] == inputs.WORKLOADS["c3"].name
    measured = rec["measured"]["dram_read_bytes"] + rec["measured"]["dram_write_bytes"]
    assert rec["dram_bytes_per_launch"] == measured * rec["scale_to_full_launch"]


def test_data_recipe_names_each_workloads_inputs():
    r = {k: bench.data_recipe(w) for k, w in inputs.WORKLOADS.items()}
    assert "Gaussian mixture" in r["c3"] and "needle" not in r["c3"]
    assert "16 planted needle keys" in r["c1"]
    assert "256 planted needle keys per KV head" in r["c2"]
    assert "8 multi-hop needle chains of 4 keys" in r["c4"]
    assert "e4m3" in r["c5"] and "1024 planted needle keys per KV head" in r["c5"]
    assert all(v.startswith("synthetic (seeded ") for v in r.values())


def test_both_arms_share_one_config():
    wl = inputs.WORKLOADS["c3"]
    c = bench.arm_config(wl, 1)
    assert c["workload"] == wl.name and c["L"] == 131072 and c["topk"] == 1024 and c["recent"] == 128
    assert "2.1 GB" in c["l2"] and c["parallelism"].endswith("x1")
