"""Host-side pieces of the benchmark that need no GPU: the kernel-source key of the
committed traffic record, the lookup that scales it to a launch, and the clock
sampler's report when NVML cannot be used."""
import json
import os
import re

import bench


def test_source_hash_is_stable_and_short():
    h = bench.source_hash()
    assert re.fullmatch(r"[0-9a-f]{16}", h)
    assert bench.source_hash() == h


def test_traffic_record_scales_per_layer_bytes_to_the_launch():
    with open(bench.PROFILE_TRAFFIC) as fh:
        records = json.load(fh)
    for key, rec in records.items():
        workload, b = key.rsplit("/B", 1)
        got = bench.profiled_traffic(workload, 32, int(b))
        if rec["source_hash"] == bench.source_hash():
            assert got == int(rec["dram_bytes_per_layer"] * 32)
            # the record is read + write bytes of one captured launch, per layer of its stack
            depth = int(re.search(r"--layers (\d+)", rec["command"]).group(1))
            assert rec["dram_bytes_per_layer"] * depth == rec["dram_bytes_read"] + rec["dram_bytes_write"]
        else:
            assert got is None   # a changed kernel has no traffic figure until re-captured
    assert bench.profiled_traffic("no_such_workload", 32, 1) is None


def test_clock_sampler_without_nvml_reports_it(monkeypatch):
    s = bench.ClockSampler(0)
    s.ok = False
    out = s.summary()
    assert out["sm_mhz"] is None and out["reasons"] == ["nvml unavailable"]
