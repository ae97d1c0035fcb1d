"""Host logic of bench.py that needs no GPU: the DRAM traffic of the attention is reported
only for the profiled workload and only while the attention kernel's sources hash to the
value recorded with the ncu capture; the decode workload's shapes."""
import json
import os

import bench


def test_traffic_reported_only_for_the_profiled_sources():
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "attn_traffic.json")))
    got = bench.attention_traffic(rec["workload"])
    if rec["sources_sha256"] == bench.attention_source_sha():
        assert got == rec["dram_read_bytes"] + rec["dram_write_bytes"]
    else:  # the kernel changed since the capture: no traffic figure
        assert got is None


def test_traffic_withheld_for_other_workloads_and_changed_sources(monkeypatch):
    assert bench.attention_traffic("main_b8_t2048") is None
    monkeypatch.setattr(bench, "attention_source_sha", lambda: "0" * 64)
    assert bench.attention_traffic("long_t16k") is None


def test_decode_workload_is_the_papers_layer():
    class A:
        decode_batch, decode_len, variant = 64, 8192, None
    wl = bench.decode_workload(A)
    assert (wl.dim, wl.N, wl.G, wl.k, wl.d_h, wl.M, wl.T) == (768, 16, 8, 1, 48, 64, 1)
    assert wl.shared and wl.variant == "gqe"
