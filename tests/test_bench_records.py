"""The ncu traffic records that bench.py reports as `roofline.traffic` (profiles/*.json):
their byte counts add up, their source file exists, and a record is only ever reported for
the exact source and workload it was captured on."""
import importlib.util
import json
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
RECORDS = ["decode_partition_traffic.json", "decode_partition_traffic_chat_prefix_bf16.json", "prefill_tc_traffic.json"]


def load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name", RECORDS)
def test_traffic_record_is_consistent(name):
    with open(os.path.join(ROOT, "profiles", name)) as f:
        rec = json.load(f)
    assert rec["dram_bytes_read"] + rec["dram_bytes_write"] == rec["dram_bytes_per_launch"]
    assert rec["dram_bytes_per_launch"] > 0 and rec["algorithmic_bytes_per_launch"] > 0
    assert os.path.exists(os.path.join(ROOT, rec["source"]))
    assert "--clock-control none" in rec["command"]


@pytest.mark.parametrize("name", RECORDS)
def test_traffic_is_reported_only_for_the_captured_source_and_workload(name, tmp_path):
    bench = load_bench()
    with open(os.path.join(ROOT, "profiles", name)) as f:
        rec = json.load(f)
    changed = tmp_path / "changed.cu"
    changed.write_text("// a kernel that differs from the captured one\n")
    assert bench.kernel_traffic(str(changed), name, rec["workload"]) is None
    assert bench.kernel_traffic(os.path.join(ROOT, rec["source"]), name, rec["workload"] + "_other") is None
    assert bench.kernel_traffic(str(changed), "no_such_record.json", rec["workload"]) is None
