"""Host logic of bench.py that needs no GPU: the DRAM traffic of the attention and of the
decode cache attention is reported only for the profiled workload and only while the
kernel's sources hash to the value recorded with the ncu capture; the decode workload's
shapes; the reference arm's timing; the clock record read from nvidia-smi's samples."""
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


def test_decode_traffic_reported_only_for_the_profiled_sources(monkeypatch):
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "decode_traffic.json")))
    assert [os.path.basename(p) for p in rec["sources"]] == list(bench.DECODE_SOURCES)
    got = bench.decode_traffic(rec["workload"])
    if rec["sources_sha256"] == bench.decode_source_sha():
        assert got == rec["dram_read_bytes"] + rec["dram_write_bytes"]
    else:
        assert got is None
    assert bench.decode_traffic("decode_b80_l8192") is None
    monkeypatch.setattr(bench, "decode_source_sha", lambda: "0" * 64)
    assert bench.decode_traffic(rec["workload"]) is None


def test_decode_workload_is_the_papers_layer():
    class A:
        decode_batch, decode_len, variant = 64, 8192, None
    wl = bench.decode_workload(A)
    assert (wl.dim, wl.N, wl.G, wl.k, wl.d_h, wl.M, wl.T) == (768, 16, 8, 1, 48, 64, 1)
    assert wl.shared and wl.variant == "gqe"


def test_reference_arm_reports_the_time_it_ran():
    """--impl reference runs the oracle on a bounded sample each step: ms_per_step is the
    time those steps took (the whole command takes at least steps x ms_per_step), the value
    is the extrapolated throughput, and the config dict is the GPU arm's."""
    import subprocess
    import sys
    import time
    t0 = time.perf_counter()
    r = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--impl",
                        "reference", "--workload", "tiny_f32", "--steps", "2", "--warmup", "3",
                        "--cpu-rows", "64"], capture_output=True, text=True, timeout=300)
    wall = time.perf_counter() - t0
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["steps"] == 2
    assert 2 * line["ms_per_step"] / 1e3 <= wall
    assert line["extrapolated_ms_per_full_step"] >= line["ms_per_step"]
    wl = bench.W.WORKLOADS["tiny_f32"]
    assert line["config"] == bench.prefill_config(wl, 1)
    assert line["cpu_baseline"]["value"] == line["value"]


def test_clock_sampler_reads_nvidia_smi_samples(tmp_path):
    """The clock record beside a timed run: the median SM clock over the busy samples (idle
    ones, under half the fastest, left out), the maximum clock, and every throttle reason
    seen active (nvidia-smi's csv,noheader,nounits rows of ClockSampler.FIELDS)."""
    import tempfile

    class Proc:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

    rows = [
        "345, 1965, 120.1, 0x0000000000000001, Not Active, Not Active, Not Active, Not Active",
        "1965, 1965, 850.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "1950, 1965, 990.2, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "1965, 1965, 870.4, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ]
    s = object.__new__(bench.ClockSampler)
    s.proc = Proc()
    s.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False, dir=tmp_path)
    s.file.write("\n".join(rows) + "\n")
    rec = s.stop()
    assert rec["samples"] == 4
    assert rec["sm_mhz"] == 1965.0 and rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["sw_power_cap"]
    # a hardware slowdown is reported by name, so the run can be rejected
    s2 = object.__new__(bench.ClockSampler)
    s2.proc = Proc()
    s2.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False, dir=tmp_path)
    s2.file.write("1500, 1965, 600, 0x8, Active, Not Active, Not Active, Not Active\n")
    assert s2.stop()["reasons"] == ["hw_slowdown"]
    # no nvidia-smi: no clock figures, and the record says why
    s3 = object.__new__(bench.ClockSampler)
    s3.proc = None
    assert s3.stop() == {"sm_mhz": None, "sm_max_mhz": None,
                         "reasons": ["nvidia-smi unavailable"]}
