#!/usr/bin/env python
"""GQE attention prefill benchmark on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one gqe_forward over the workload (router, K/V/shared projection, bucketed
routed Q projection, attention, output construction, W_o, aux loss) with its inputs
already in HBM. Before each timed step the L2 cache is flushed by writing 256 MiB (the
inputs of the default workload are smaller than L2); each step is timed with CUDA events
on the launching stream, and the K step times are summed. Under torchrun every rank runs
its own replica of the workload (the layer has no cross-sequence exchange), the time is
the maximum over ranks and `value` counts the tokens of all ranks.

Rank 0 prints one JSON line. Besides the metric it reports:
  roofline      the attention kernel's achieved TFLOP/s (active FLOPs / its event-timed
                duration) against the measured bf16 dense peak;
  speedup_vs_kE the same kernels with every expert active (k = E), the in-run GQA
                comparator;
  e2e           the same metric through the public API with host buffers: every timed step
                copies its x in from pinned host memory and its y and aux loss out; the
                copies run on their own streams and overlap the neighbouring steps' forwards
                (rotating buffer sets larger than L2 together);
  cpu_baseline  the float64 CPU oracle on a bounded sample of the same workload (rank 0,
                one GPU only).
--impl reference times the CPU oracle alone (the only reference there is: the pages ship
no code), one bounded sample per step.

--mode decode times one gqe_decode step of B sequences over their KV caches, captured once
in a CUDA graph and replayed K times back to back (a step is ~200 us of GPU work in six
launches; replays keep the host's launch speed out of the number), and reports the eager
per-step time beside it. --mode backward times gqe_forward + gqe_backward.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from moe_query_head_b200 import workloads as W  # noqa: E402

METRIC = "GQE prefill tokens/s @1 B200; % bf16 tensor peak (active FLOPs); speedup vs k=E"
DECODE_METRIC = "GQE decode tokens/s @1 B200 (one new token per sequence over its KV cache)"
BACKWARD_METRIC = "GQE training-step tokens/s @1 B200 (layer forward + backward)"
DECODE_BASE = "main_b8_t2048"  # the paper's layer shapes: dim 768, N 16, G 8, k 1, d_h 48
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FLUSH_BYTES = 256 << 20


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long_t16k", choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--variant", default=None, choices=["gqe", "weighted_concat", "hard_concat"],
                    help="output construction (default: the workload's)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--mode", default="prefill", choices=["prefill", "decode", "backward"],
                    help="prefill (default, the headline), one decode step with a KV cache, "
                         "or a training step of the layer (forward + backward)")
    ap.add_argument("--decode-batch", type=int, default=64, help="decode: sequences per step")
    ap.add_argument("--decode-len", type=int, default=8192,
                    help="decode: tokens already cached per sequence")
    ap.add_argument("--parallel", default="replicas", choices=["replicas", "groups"],
                    help="N > 1: independent replicas (default, weak scaling) or one layer "
                         "split by groups over the ranks with an all-reduce of y (strong)")
    ap.add_argument("--cpu-rows", type=int, default=2048,
                    help="query rows in the oracle's bounded sample")
    a = ap.parse_args()
    a.warmup = max(a.warmup, 3)
    return a


ATTENTION_SOURCES = ("tc_attention.cu", "exp2_fma.cuh", "tc_ptx.cuh", "gqe_common.cuh")
DECODE_SOURCES = ("decode.cu", "gqe_common.cuh", "tc_ptx.cuh")


def source_sha(names) -> str:
    """sha256 over a kernel's translation unit and the headers it includes (in csrc/)."""
    import hashlib
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(ROOT, "moe_query_head_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def attention_source_sha() -> str:
    return source_sha(ATTENTION_SOURCES)


def decode_source_sha() -> str:
    return source_sha(DECODE_SOURCES)


def kernel_traffic(record: str, workload: str, sha_fn):
    """DRAM bytes per launch from a committed ncu capture (profiles/<record>), if that
    capture was taken on this workload and on the kernel's current sources; else None."""
    rec_path = os.path.join(ROOT, "profiles", record)
    try:
        with open(rec_path) as f:
            rec = json.load(f)
        sha = sha_fn()
    except OSError:
        return None
    if rec.get("sources_sha256") != sha or rec.get("workload") != workload:
        return None
    return int(rec["dram_read_bytes"]) + int(rec["dram_write_bytes"])


def attention_traffic(workload: str):
    """The attention kernel's DRAM bytes per launch (profiles/attn_traffic.json)."""
    return kernel_traffic("attn_traffic.json", workload, attention_source_sha)


def decode_traffic(workload: str):
    """The decode cache attention's DRAM bytes per launch (profiles/decode_traffic.json)."""
    return kernel_traffic("decode_traffic.json", workload, decode_source_sha)


def reduce_max_over_ranks(values, dist, device):
    """Each value's maximum over all ranks (times of a multi-GPU run are the slowest
    rank's). `dist` is torch.distributed with an initialised process group."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def whole_job_tokens_per_s(tokens_per_rank: int, world: int, total_ms: float, steps: int):
    """Tokens of all ranks per second of the (max-over-ranks) time of one step."""
    return tokens_per_rank * world / (total_ms / steps / 1e3)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------------------
# Clock sampling during the timed region.
# ----------------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.proc = None
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def wait_first(self, timeout: float = 5.0):
        """Returns once nvidia-smi has written its first sample (or after `timeout` s), so
        the samples cover the timed region however slowly the tool starts."""
        t_end = time.time() + timeout
        while self.proc is not None and time.time() < t_end:
            self.file.flush()
            if os.path.getsize(self.file.name) > 0:
                return
            time.sleep(0.05)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.file.read().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.file.name)
        busy = [s for s in sm if s > 0.5 * max(sm)] if sm else []
        return {"sm_mhz": statistics.median(busy) if busy else None,
                "sm_max_mhz": max(mx) if mx else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------------------
# The CPU oracle on a bounded sample (cpu_baseline and --impl reference).
# ----------------------------------------------------------------------------------------

def oracle_sample(inp: W.Inputs, n_rows: int) -> dict:
    """Time the oracle's steps on the whole workload, except that the per-row steps (routed
    and shared queries, attention, output construction, W_o) run on n_rows evenly spaced
    token rows; the full-workload time is the whole-workload steps plus the per-row time
    scaled by M / n_rows."""
    import oracle
    wl = inp.wl
    f = inp.f64
    x = f("x")
    layer = oracle.Layer(dim=wl.dim, N=wl.N, G=wl.G, k=wl.k, d_h=wl.d_h, shared=wl.shared,
                         variant=wl.variant, causal=wl.causal)
    t0 = time.perf_counter()
    rt = oracle.route(x, f("W_r"), wl.G, wl.k)
    oracle.aux_loss(rt.counts, rt.prob_sum, wl.M, wl.G, wl.k)
    K, V = oracle.kv_projection(x, f("W_k"), f("W_v"), wl.G, wl.d_h)
    t1 = time.perf_counter()
    rows = np.linspace(0, wl.M - 1, n_rows).round().astype(np.int64)
    xs = x[rows]
    Q = oracle.routed_queries(xs, f("W_q"), rt.sel[rows], wl.G, wl.E, wl.d_h)
    if wl.shared:
        Q = np.concatenate([Q, oracle.shared_query(xs, f("W_shared"))[None]], axis=0)
    O = np.empty((Q.shape[0], rows.size, wl.d_h))
    for b in range(wl.B):
        m = np.nonzero(rows // wl.T == b)[0]
        if m.size == 0:
            continue
        tk = slice(b * wl.T, (b + 1) * wl.T)
        for s in range(Q.shape[0]):
            h = oracle.stream_kv_head(s, wl.k, wl.G)
            O[s, m] = oracle.attention_rows(Q[s, m], rows[m] % wl.T, K[h, tk], V[h, tk], wl.causal)
    sub = oracle.Routing(rt.logits[rows], rt.p[rows], rt.sel[rows], rt.p_sel[rows],
                         rt.gates[rows], rt.w[rows], rt.counts, rt.prob_sum)
    Z = oracle.combine(O, sub, layer)
    oracle.output_projection(Z, f("W_o"))
    t2 = time.perf_counter()
    est = (t1 - t0) + (t2 - t1) * wl.M / rows.size
    return {"whole_s": t1 - t0, "rows_s": t2 - t1, "rows": int(rows.size), "est_s": est,
            "tokens_per_s": wl.M / est}


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_sample_desc(wl, rows):
    return (f"{wl.name}: routing, aux loss and K/V projection over all {wl.M} tokens; "
            f"queries, attention, output construction and W_o on {rows} evenly spaced token "
            f"rows, scaled by {wl.M}/{rows} (float64 numpy oracle)")


# ----------------------------------------------------------------------------------------
# Our arm.
# ----------------------------------------------------------------------------------------

def _upload(inp, torch):
    out = {}
    for n in ("x", "W_r", "W_q", "W_k", "W_v", "W_shared", "W_o"):
        a = inp.raw(n)
        if a is None:
            out[n] = None
        elif inp.wl.dtype == "bf16":
            out[n] = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
        else:
            out[n] = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return out


def prefill_config(wl, world: int) -> dict:
    """The workload's description in the JSON line (identical for both arms)."""
    return {"workload": wl.name, "dim": wl.dim, "N": wl.N, "G": wl.G, "k": wl.k,
            "d_h": wl.d_h, "B": wl.B, "T": wl.T, "variant": wl.variant,
            "shared": wl.shared, "causal": wl.causal,
            "l2": "flushed before every timed step (256 MiB write)",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


def bench_ours(args, rank, world, dist):
    import torch
    from moe_query_head_b200 import gqe as G

    wl = W.WORKLOADS[args.workload]
    if args.variant:
        wl = wl.with_(variant=args.variant)
    inp = W.generate(wl)
    dev = _upload(inp, torch)
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    code = G.GQE_BF16 if wl.dtype == "bf16" else G.GQE_F32
    variant = W.VARIANT_IDS[wl.variant]
    W_s = dev["W_shared"] if wl.shared else None

    h = G.gqe_create(wl.dim, wl.N, wl.G, wl.k, wl.d_h, code, wl.M)
    out = torch.empty((wl.M, wl.dim), dtype=tdt, device="cuda")
    aux = torch.zeros(1, dtype=torch.float32, device="cuda")
    # the all-active comparator: same inputs, k = E, W_o of the wider concatenation
    kE = wl.all_active()
    hE = G.gqe_create(wl.dim, wl.N, wl.G, kE.k, wl.d_h, code, wl.M)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(wl.seed + 1000)
    W_oE = (torch.randn((wl.dim, kE.D_o), generator=gen, device="cuda") * 0.02).to(tdt)
    outE = torch.empty_like(out)
    # the exact-GQA comparator (the pages' own baseline): every expert active, the routed
    # outputs concatenated as they are, no shared head, so W_o reads the N heads of a dense
    # GQA layer
    hG = G.gqe_create(wl.dim, wl.N, wl.G, kE.k, wl.d_h, code, wl.M)
    W_oG = (torch.randn((wl.dim, wl.N * wl.d_h), generator=gen, device="cuda") * 0.02).to(tdt)
    outG = torch.empty_like(out)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    def fwd(handle, k, W_o, o, shared=W_s, var=variant):
        G.gqe_forward(handle, dev["x"], wl.B, wl.T, dev["W_r"], dev["W_q"], dev["W_k"],
                      dev["W_v"], shared, W_o, wl.N, wl.G, k, wl.d_h, var, int(wl.causal), o,
                      aux)

    def fwd_gqa():
        fwd(hG, kE.k, W_oG, outG, shared=None, var=W.VARIANT_IDS["hard_concat"])

    stage_ev = [torch.cuda.Event(enable_timing=True) for _ in range(G.GQE_NUM_STAGES + 1)]
    for e in stage_ev:
        e.record()
    torch.cuda.synchronize()

    def timed(fn, steps, stages=None):
        s_ev = torch.cuda.Event(enable_timing=True)
        e_ev = torch.cuda.Event(enable_timing=True)
        total = 0.0
        st_tot = np.zeros(G.GQE_NUM_STAGES)
        for _ in range(steps):
            flush.zero_()
            s_ev.record()
            fn()
            e_ev.record()
            torch.cuda.synchronize()
            total += s_ev.elapsed_time(e_ev)
            if stages:
                for i in range(G.GQE_NUM_STAGES):
                    st_tot[i] += stages[i].elapsed_time(stages[i + 1])
        return total, st_tot

    gpu_id = torch.cuda.get_device_properties(0).uuid
    gpu_id = f"GPU-{gpu_id}" if not str(gpu_id).startswith("GPU-") else str(gpu_id)

    # warm-up
    for _ in range(args.warmup):
        fwd(h, wl.k, dev["W_o"], out)
        fwd(hE, kE.k, W_oE, outE)
        fwd_gqa()
    torch.cuda.synchronize()
    st = G.gqe_check_device_status(h)
    if st != G.GQE_OK:
        raise RuntimeError("device status after warm-up: " + G.status_str(st))

    sampler = ClockSampler(gpu_id)
    sampler.wait_first()
    time.sleep(0.1)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    total_ms, _ = timed(lambda: fwd(h, wl.k, dev["W_o"], out), args.steps)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    launches = G.gqe_kernel_launches(h)
    # the per-stage breakdown in a separate pass: events between the kernels keep each
    # kernel from starting while the previous one finishes, so they stay out of the
    # headline timing
    G.gqe_set_stage_events(h, stage_ev)
    _, stage_ms = timed(lambda: fwd(h, wl.k, dev["W_o"], out), args.steps, stage_ev)
    G.gqe_set_stage_events(h, None)
    totalE_ms, _ = timed(lambda: fwd(hE, kE.k, W_oE, outE), args.steps)
    totalG_ms, _ = timed(fwd_gqa, args.steps)

    # end to end through the public API with host buffers, run the way a serving loop runs
    # it: every step copies its input in from pinned host memory and its output and aux
    # loss back out, on streams of their own, so step i's copy-in and step i-1's copy-out
    # overlap step i's forward. Buffer sets rotate; together they exceed L2 (no step finds
    # the previous one's data there), which stands in for the L2 flush of the device timing.
    x_bytes = dev["x"].numel() * dev["x"].element_size()
    y_bytes = out.numel() * out.element_size()
    n_sets = max(2, -(-2 * 128 * 2**20 // (x_bytes + y_bytes)))
    x_src = dev["x"].cpu()
    x_hosts = [torch.empty(dev["x"].shape, dtype=tdt).pin_memory() for _ in range(n_sets)]
    for xh in x_hosts:
        xh.copy_(x_src)
    y_hosts = [torch.empty(out.shape, dtype=tdt).pin_memory() for _ in range(n_sets)]
    aux_hosts = [torch.empty(1, dtype=torch.float32).pin_memory() for _ in range(n_sets)]
    x_devs = [torch.empty_like(dev["x"]) for _ in range(n_sets)]
    y_devs = [torch.empty_like(out) for _ in range(n_sets)]
    aux_devs = [torch.zeros(1, dtype=torch.float32, device="cuda") for _ in range(n_sets)]
    s_comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(n_sets)]
    ev_fwd = [torch.cuda.Event() for _ in range(n_sets)]
    ev_out = [torch.cuda.Event() for _ in range(n_sets)]

    def e2e_steps(steps, start_ev=None):
        if start_ev is not None:
            s_in.wait_event(start_ev)
        for i in range(steps):
            b = i % n_sets
            s_in.wait_event(ev_fwd[b])  # the last forward that read x_devs[b] is done
            with torch.cuda.stream(s_in):
                x_devs[b].copy_(x_hosts[b], non_blocking=True)
            ev_in[b].record(s_in)
            s_comp.wait_event(ev_in[b])
            s_comp.wait_event(ev_out[b])  # y_devs[b] has been copied out
            G.gqe_forward(h, x_devs[b], wl.B, wl.T, dev["W_r"], dev["W_q"], dev["W_k"],
                          dev["W_v"], W_s, dev["W_o"], wl.N, wl.G, wl.k, wl.d_h, variant,
                          int(wl.causal), y_devs[b], aux_devs[b], stream=s_comp)
            ev_fwd[b].record(s_comp)
            s_out.wait_event(ev_fwd[b])
            with torch.cuda.stream(s_out):
                y_hosts[b].copy_(y_devs[b], non_blocking=True)
                aux_hosts[b].copy_(aux_devs[b], non_blocking=True)
            ev_out[b].record(s_out)
        s_comp.wait_stream(s_in)
        s_comp.wait_stream(s_out)  # every output is on the host

    e2e_steps(n_sets)
    torch.cuda.synchronize()
    e2e_s, e2e_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_s.record(s_comp)
    e2e_steps(args.steps, e2e_s)
    e2e_e.record(s_comp)
    torch.cuda.synchronize()
    e2e_ms = e2e_s.elapsed_time(e2e_e)
    clocks = sampler.stop()
    st = G.gqe_check_device_status(h)
    if st != G.GQE_OK:
        raise RuntimeError("device status after timing: " + G.status_str(st))

    att_i = [G.gqe_stage_name(i) for i in range(G.GQE_NUM_STAGES)].index("attention")
    if dist:
        total_ms, totalE_ms, totalG_ms, e2e_ms, att_ms_tot = reduce_max_over_ranks(
            [total_ms, totalE_ms, totalG_ms, e2e_ms, stage_ms[att_i]], dist, "cuda")
    else:
        att_ms_tot = float(stage_ms[att_i])

    peaks, peak_src = load_peaks()
    ms = total_ms / args.steps
    msE = totalE_ms / args.steps
    msG = totalG_ms / args.steps
    tokens = wl.M * world
    value = whole_job_tokens_per_s(wl.M, world, total_ms, args.steps)
    flops = wl.active_flops()
    S = wl.n_streams
    att_flops = (2.0 * wl.B * wl.d_h * wl.T * (wl.T + 1) * S if wl.causal
                 else 4.0 * wl.B * wl.d_h * wl.T * wl.T * S)
    att_ms = att_ms_tot / args.steps
    att_tflops = att_flops / (att_ms / 1e3) / 1e12
    peak = float(peaks["bf16_tflops"])
    res = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if wl.dtype == "bf16" else "f32",
        "data": "synthetic (seeded normal inputs and random-init weights of the layer shapes)",
        "config": prefill_config(wl, world),
        "active_tflops": flops / (ms / 1e3) / 1e12,
        "frac_of_bf16_peak": flops / (ms / 1e3) / 1e12 / peak,
        "speedup_vs_kE": msE / ms,
        "kE_tokens_per_s": tokens / (msE / 1e3),
        "speedup_vs_exact_gqa": msG / ms,
        "exact_gqa_tokens_per_s": tokens / (msG / 1e3),
        "exact_gqa": "the same kernels with k = E, hard_concat and no shared head: a dense "
                     "GQA layer with N query heads",
        "stages_ms": {G.gqe_stage_name(i): float(stage_ms[i] / args.steps)
                      for i in range(G.GQE_NUM_STAGES)},
        "roofline": {"kernel": "attention", "bound": "tensor", "achieved": att_tflops,
                     "peak": peak, "unit": "TFLOP/s", "frac": att_tflops / peak,
                     "peak_source": f"{peak_src} bf16 dense (burst)",
                     "traffic": attention_traffic(wl.name),
                     "traffic_unit": "bytes per launch (ncu dram read + write)"},
        "e2e": {"value": tokens / (e2e_ms / args.steps / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": int(x_bytes),
                "d2h_bytes_per_step": int(y_bytes + 4),
                "pipelined": f"copy-in, forward and copy-out of consecutive steps overlap on "
                             f"three streams; {n_sets} rotating buffer sets, together larger "
                             f"than L2"},
        "gpu_launches": int(launches * args.steps),
        "clocks": clocks,
    }
    G.gqe_destroy(h)
    G.gqe_destroy(hE)
    G.gqe_destroy(hG)
    return res, inp


# ----------------------------------------------------------------------------------------
# Decode mode: one gqe_decode step (one new token per sequence over its KV cache).
# ----------------------------------------------------------------------------------------

def decode_workload(args):
    wl = W.WORKLOADS[DECODE_BASE].with_(B=args.decode_batch, T=1)
    if args.variant:
        wl = wl.with_(variant=args.variant)
    return wl


def oracle_decode_sample(wl, L: int, n_seq: int) -> dict:
    """The float64 oracle's decode step on n_seq sequences with L cached tokens each (the
    same layer and cache length as the GPU run; seeded host inputs)."""
    from oracle import gqe_oracle as go
    sub = wl.with_(B=n_seq)
    d = W.generate_decode(sub, [L] * n_seq, L + 1)
    inp = d.inp
    layer = go.Layer(wl.dim, wl.N, wl.G, wl.k, wl.d_h, shared=wl.shared, variant=wl.variant)
    args64 = [inp.f64(n) for n in ("W_r", "W_q", "W_k", "W_v", "W_shared", "W_o")]
    kc, vc, x = d.k_cache.astype(np.float64), d.v_cache.astype(np.float64), inp.f64("x")
    t0 = time.perf_counter()
    go.decode(layer, x, kc, vc, d.lengths, *args64)
    dt = time.perf_counter() - t0
    return {"seconds": dt, "tokens_per_s": n_seq / dt,
            "sample": f"{n_seq} sequences of the decode workload ({L} cached tokens each), "
                      f"float64 numpy oracle; tokens/s of that sample"}


def bench_decode(args, rank, world, dist):
    import torch
    from moe_query_head_b200 import gqe as G

    wl = decode_workload(args)
    B, L = args.decode_batch, args.decode_len
    L_max = L + 64
    inp = W.generate(wl)  # the B new tokens and the layer's weights
    dev = _upload(inp, torch)
    variant = W.VARIANT_IDS[wl.variant]
    W_s = dev["W_shared"] if wl.shared else None
    # caches: seeded normal values with the spread of a projected K/V element (bf16, on the
    # device; together larger than L2, so no flush is needed between steps)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(wl.seed + 2000)
    sd = (wl.w_std if wl.w_std is not None else (1.0 / wl.dim) ** 0.5) * wl.dim ** 0.5
    shape = (wl.G, B, L_max, wl.d_h)
    kc = torch.randn(shape, generator=gen, device="cuda", dtype=torch.bfloat16).mul_(sd)
    vc = torch.randn(shape, generator=gen, device="cuda", dtype=torch.bfloat16).mul_(sd)
    lengths = torch.full((B,), L, dtype=torch.int32, device="cuda")
    h = G.gqe_create(wl.dim, wl.N, wl.G, wl.k, wl.d_h, G.GQE_BF16, B)
    out = torch.empty((B, wl.dim), dtype=torch.bfloat16, device="cuda")
    aux = torch.zeros(1, dtype=torch.float32, device="cuda")
    kE = wl.all_active()
    hE = G.gqe_create(wl.dim, wl.N, wl.G, kE.k, wl.d_h, G.GQE_BF16, B)
    W_oE = (torch.randn((wl.dim, kE.D_o), generator=gen, device="cuda") * 0.02).to(torch.bfloat16)
    outE = torch.empty_like(out)

    def step(handle, k, W_o, o, x=None, stream=None):
        G.gqe_decode(handle, dev["x"] if x is None else x, B, kc, vc, L_max, lengths,
                     dev["W_r"], dev["W_q"], dev["W_k"], dev["W_v"], W_s, W_o, wl.N, wl.G, k,
                     wl.d_h, variant, o, aux, stream=stream)

    stage_ev = [torch.cuda.Event(enable_timing=True) for _ in range(G.GQE_NUM_STAGES + 1)]
    for e in stage_ev:
        e.record()
    torch.cuda.synchronize()

    def timed(fn, steps, stages=None):
        s_ev = torch.cuda.Event(enable_timing=True)
        e_ev = torch.cuda.Event(enable_timing=True)
        total = 0.0
        st_tot = np.zeros(G.GQE_NUM_STAGES)
        for _ in range(steps):
            s_ev.record()
            fn()
            e_ev.record()
            torch.cuda.synchronize()
            total += s_ev.elapsed_time(e_ev)
            if stages:
                for i in range(G.GQE_NUM_STAGES):
                    st_tot[i] += stages[i].elapsed_time(stages[i + 1])
        return total, st_tot

    gpu_id = torch.cuda.get_device_properties(0).uuid
    gpu_id = f"GPU-{gpu_id}" if not str(gpu_id).startswith("GPU-") else str(gpu_id)
    for _ in range(args.warmup):
        step(h, wl.k, dev["W_o"], out)
        step(hE, kE.k, W_oE, outE)
    torch.cuda.synchronize()
    st = G.gqe_check_device_status(h)
    if st != G.GQE_OK:
        raise RuntimeError("device status after warm-up: " + G.status_str(st))
    # A serving loop replays a captured step: each step is then one graph launch, so the
    # timing does not depend on how fast the host issues a step's six kernel launches
    # (about 200 us of GPU work). The eager per-step time is reported beside it.
    def capture(fn):
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            fn()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            fn()
        return graph

    g_step = capture(lambda: step(h, wl.k, dev["W_o"], out))
    g_stepE = capture(lambda: step(hE, kE.k, W_oE, outE))
    launches = G.gqe_kernel_launches(h)

    def replayed(graph, steps):
        s_ev = torch.cuda.Event(enable_timing=True)
        e_ev = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        s_ev.record()
        for _ in range(steps):
            graph.replay()
        e_ev.record()
        torch.cuda.synchronize()
        return s_ev.elapsed_time(e_ev)

    for _ in range(args.warmup):
        g_step.replay()
        g_stepE.replay()
    torch.cuda.synchronize()
    sampler = ClockSampler(gpu_id)
    sampler.wait_first()
    time.sleep(0.1)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    total_ms = replayed(g_step, args.steps)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    totalE_ms = replayed(g_stepE, args.steps)
    eager_ms, _ = timed(lambda: step(h, wl.k, dev["W_o"], out), args.steps)
    G.gqe_set_stage_events(h, stage_ev)
    _, stage_ms = timed(lambda: step(h, wl.k, dev["W_o"], out), args.steps, stage_ev)
    G.gqe_set_stage_events(h, None)
    # end to end through the API: each step copies its tokens in from pinned host memory
    # and its output and aux loss back out, on the same stream
    x_host = dev["x"].cpu().pin_memory()
    y_host = torch.empty(out.shape, dtype=torch.bfloat16).pin_memory()
    aux_host = torch.empty(1, dtype=torch.float32).pin_memory()
    x_dev = torch.empty_like(dev["x"])

    def e2e_step():
        x_dev.copy_(x_host, non_blocking=True)
        step(h, wl.k, dev["W_o"], out, x=x_dev)
        y_host.copy_(out, non_blocking=True)
        aux_host.copy_(aux, non_blocking=True)

    e2e_ms, _ = timed(e2e_step, args.steps)
    clocks = sampler.stop()
    st = G.gqe_check_device_status(h)
    if st != G.GQE_OK:
        raise RuntimeError("device status after timing: " + G.status_str(st))
    att_i = [G.gqe_stage_name(i) for i in range(G.GQE_NUM_STAGES)].index("attention")
    att_tot = float(stage_ms[att_i])
    if dist:
        total_ms, totalE_ms, e2e_ms, att_tot, eager_ms = reduce_max_over_ranks(
            [total_ms, totalE_ms, e2e_ms, att_tot, eager_ms], dist, "cuda")
    peaks, peak_src = load_peaks()
    ms = total_ms / args.steps
    # algorithmic bytes of the cache attention: every cached K and V row read once, the new
    # rows read from the workspace and written into the caches
    kv_bytes = B * wl.G * (L + 1) * wl.d_h * 2 * 2 + B * wl.G * wl.d_h * 2 * 2
    att_ms = att_tot / args.steps
    gbs = kv_bytes / (att_ms / 1e3) / 1e9
    hbm = float(peaks["hbm_gbs"])
    res = {
        "metric": DECODE_METRIC, "value": B * world / (ms / 1e3), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded normal tokens, caches and random-init weights of the layer "
                "shapes)",
        "config": {"workload": f"decode_b{B}_l{L}", "dim": wl.dim, "N": wl.N, "G": wl.G,
                   "k": wl.k, "d_h": wl.d_h, "B": B, "cache_len": L, "L_max": L_max,
                   "variant": wl.variant, "shared": wl.shared,
                   "l2": f"caches ({2 * kc.numel() * 2 / 2**30:.2f} GiB) larger than L2; "
                         f"no flush",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "timing": "CUDA-graph replays of one captured gqe_decode step, back to back (the "
                  "same-kernels k = E comparator likewise)",
        "eager_ms_per_step": eager_ms / args.steps,
        "speedup_vs_kE": (totalE_ms / args.steps) / ms,
        "kE_tokens_per_s": B * world / (totalE_ms / args.steps / 1e3),
        "stages_ms": {G.gqe_stage_name(i): float(stage_ms[i] / args.steps)
                      for i in range(G.GQE_NUM_STAGES)},
        "roofline": {"kernel": "decode attention (cache read, merge)", "bound": "hbm",
                     "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                     "peak_source": f"{peak_src} HBM copy",
                     "traffic": decode_traffic(f"decode_b{B}_l{L}"),
                     "algorithmic_bytes": kv_bytes},
        "e2e": {"value": B * world / (e2e_ms / args.steps / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": int(x_host.numel() * 2),
                "d2h_bytes_per_step": int(y_host.numel() * 2 + 4)},
        "gpu_launches": int(launches * args.steps),
        "clocks": clocks,
    }
    del g_step, g_stepE
    G.gqe_destroy(h)
    G.gqe_destroy(hE)
    return res, wl


# ----------------------------------------------------------------------------------------
# Backward mode: one training step of the layer (gqe_forward + gqe_backward).
# ----------------------------------------------------------------------------------------

def backward_flops(wl) -> dict:
    """Algorithmic FLOPs (2 per multiply-add) of the backward pass: attention 2.5 times the
    forward's (dV = P^T dO, dP = dO V^T, dQ = dS K, dK = dS^T Q against the forward's two
    products), and every projection's two gradient GEMMs (weights and input) at its active
    size."""
    M, d, h = wl.M, wl.dim, wl.d_h
    S = wl.n_streams
    att_fwd = (2.0 * wl.B * h * wl.T * (wl.T + 1) * S if wl.causal
               else 4.0 * wl.B * h * wl.T * wl.T * S)
    proj = 2.0 * (2.0 * M * d * (wl.N + (2 * wl.G + (1 if wl.shared else 0)) * h
                                 + h * wl.G * wl.k) + 2.0 * M * wl.D_o * d)
    return {"attention": 2.5 * att_fwd, "projections": proj, "total": 2.5 * att_fwd + proj}


def bench_backward(args, rank, world, dist):
    import torch
    from moe_query_head_b200 import gqe as G

    wl = W.WORKLOADS[args.workload]
    if args.variant:
        wl = wl.with_(variant=args.variant)
    inp = W.generate(wl)
    dev = _upload(inp, torch)
    variant = W.VARIANT_IDS[wl.variant]
    W_s = dev["W_shared"] if wl.shared else None
    h = G.gqe_create(wl.dim, wl.N, wl.G, wl.k, wl.d_h, G.GQE_BF16, wl.M)
    G.gqe_enable_backward(h)
    out = torch.empty((wl.M, wl.dim), dtype=torch.bfloat16, device="cuda")
    aux = torch.zeros(1, dtype=torch.float32, device="cuda")
    dy = torch.from_numpy(W.f32_to_bf16_bits(W.grad_output(wl)).view(np.int16)).view(
        torch.bfloat16).cuda()
    f32 = lambda *s: torch.empty(s, dtype=torch.float32, device="cuda")  # noqa: E731
    g = [f32(wl.M, wl.dim), f32(wl.N, wl.dim), f32(wl.N * wl.d_h, wl.dim),
         f32(wl.G * wl.d_h, wl.dim), f32(wl.G * wl.d_h, wl.dim),
         f32(wl.d_h, wl.dim) if wl.shared else None, f32(wl.dim, wl.D_o)]
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    def fwd():
        G.gqe_forward(h, dev["x"], wl.B, wl.T, dev["W_r"], dev["W_q"], dev["W_k"], dev["W_v"],
                      W_s, dev["W_o"], wl.N, wl.G, wl.k, wl.d_h, variant, int(wl.causal), out,
                      aux)

    def bwd():
        G.gqe_backward(h, dev["x"], wl.B, wl.T, dev["W_r"], dev["W_q"], dev["W_k"], dev["W_v"],
                       W_s, dev["W_o"], wl.N, wl.G, wl.k, wl.d_h, variant, int(wl.causal), dy,
                       0.01, *g)

    gpu_id = torch.cuda.get_device_properties(0).uuid
    gpu_id = f"GPU-{gpu_id}" if not str(gpu_id).startswith("GPU-") else str(gpu_id)
    for _ in range(args.warmup):
        fwd()
        bwd()
    torch.cuda.synchronize()
    if G.gqe_check_device_status(h) != G.GQE_OK:
        raise RuntimeError("device status after warm-up")
    sampler = ClockSampler(gpu_id)
    sampler.wait_first()
    time.sleep(0.1)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    tot, tf, tb = 0.0, 0.0, 0.0
    for _ in range(args.steps):
        flush.zero_()
        ev[0].record()
        fwd()
        ev[1].record()
        bwd()
        ev[2].record()
        torch.cuda.synchronize()
        tf += ev[0].elapsed_time(ev[1])
        tb += ev[1].elapsed_time(ev[2])
        tot += ev[0].elapsed_time(ev[2])
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks = sampler.stop()
    if G.gqe_check_device_status(h) != G.GQE_OK:
        raise RuntimeError("device status after timing")
    launches = G.gqe_kernel_launches(h) + G.gqe_backward_launches(h)
    if dist:
        tot, tf, tb = reduce_max_over_ranks([tot, tf, tb], dist, "cuda")
    peaks, peak_src = load_peaks()
    ms, msf, msb = tot / args.steps, tf / args.steps, tb / args.steps
    bf = backward_flops(wl)
    fflops = wl.active_flops()
    peak = float(peaks["bf16_tflops"])
    res = {
        "metric": BACKWARD_METRIC, "value": wl.M * world / (ms / 1e3), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded normal inputs, upstream gradient and random-init weights "
                "of the layer shapes)",
        "config": dict(prefill_config(wl, world), aux_grad=0.01),
        "forward_ms": msf, "backward_ms": msb,
        "active_tflops": (fflops + bf["total"]) / (ms / 1e3) / 1e12,
        "frac_of_bf16_peak": (fflops + bf["total"]) / (ms / 1e3) / 1e12 / peak,
        "backward_active_tflops": bf["total"] / (msb / 1e3) / 1e12,
        "backward_flops": bf,
        "roofline": {"kernel": "backward pass (all kernels)", "bound": "tensor",
                     "achieved": bf["total"] / (msb / 1e3) / 1e12, "peak": peak,
                     "unit": "TFLOP/s", "frac": bf["total"] / (msb / 1e3) / 1e12 / peak,
                     "peak_source": f"{peak_src} bf16 dense (burst)", "traffic": None},
        "e2e": None,
        "gpu_launches": int(launches * args.steps),
        "clocks": clocks,
    }
    G.gqe_destroy(h)
    return res


# ----------------------------------------------------------------------------------------
# Group-parallel prefill: one layer split by groups over the ranks (strong scaling).
# ----------------------------------------------------------------------------------------

def bench_groups(args, rank, world, dist):
    """Rank r computes groups group_ranges(G, world)[r] of the layer (gqe_set_group_range with
    its weight slices) and the ranks' shares of y are summed by one NCCL all-reduce; a step
    is the forward of every rank plus the all-reduce, timed on the device, max over ranks."""
    import torch
    from moe_query_head_b200 import gqe as G
    from moe_query_head_b200 import group_parallel as GP

    wl = W.WORKLOADS[args.workload]
    if args.variant:
        wl = wl.with_(variant=args.variant)
    inp = W.generate(wl)
    dev = _upload(inp, torch)
    g0, g1 = GP.group_ranges(wl.G, world)[rank]
    sh = GP.GroupShard(dim=wl.dim, N=wl.N, G=wl.G, k=wl.k, d_h=wl.d_h, variant=wl.variant,
                       causal=wl.causal, max_tokens=wl.M, g0=g0, g1=g1, W_r=dev["W_r"],
                       W_q=dev["W_q"], W_k=dev["W_k"], W_v=dev["W_v"],
                       W_shared=dev["W_shared"] if wl.shared else None, W_o=dev["W_o"])
    out = torch.empty((wl.M, wl.dim), dtype=torch.bfloat16, device="cuda")
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    def step():
        sh.forward_allreduce(dev["x"], wl.B, wl.T, out, dist)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if G.gqe_check_device_status(sh.h) != G.GQE_OK:
        raise RuntimeError("device status after warm-up")
    gpu_id = torch.cuda.get_device_properties(torch.cuda.current_device()).uuid
    gpu_id = f"GPU-{gpu_id}" if not str(gpu_id).startswith("GPU-") else str(gpu_id)
    sampler = ClockSampler(gpu_id)
    sampler.wait_first()
    time.sleep(0.1)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    s_ev, e_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    total = 0.0
    for _ in range(args.steps):
        flush.zero_()
        s_ev.record()
        step()
        e_ev.record()
        torch.cuda.synchronize()
        total += s_ev.elapsed_time(e_ev)
    if dist:
        dist.barrier()
    clocks = sampler.stop()
    launches = G.gqe_kernel_launches(sh.h)
    if dist:
        (total,) = reduce_max_over_ranks([total], dist, "cuda")
    peaks, peak_src = load_peaks()
    ms = total / args.steps
    peak = float(peaks["bf16_tflops"])
    flops = wl.active_flops()
    res = {
        "metric": METRIC, "value": wl.M / (ms / 1e3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded normal inputs and random-init weights of the layer shapes)",
        "config": dict(prefill_config(wl, world), parallelism=f"groups x{world}"),
        "active_tflops": flops / (ms / 1e3) / 1e12,
        "frac_of_bf16_peak": flops / (ms / 1e3) / 1e12 / peak / world,
        "roofline": None, "e2e": None,
        "gpu_launches": int(launches * args.steps), "clocks": clocks,
    }
    sh.close()
    return res


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference" and args.mode == "decode":
        if rank != 0:
            return 0
        wl = decode_workload(args)
        n_seq = 4
        for _ in range(args.warmup):
            oracle_decode_sample(wl, args.decode_len, n_seq)
        samples = [oracle_decode_sample(wl, args.decode_len, n_seq) for _ in range(args.steps)]
        value = sum(s["tokens_per_s"] for s in samples) / len(samples)
        res = {"impl": "reference", "metric": DECODE_METRIC, "value": value, "unit": "tokens/s",
               "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
               "ms_per_step": args.decode_batch / value * 1e3, "higher_is_better": True,
               "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
               "config": {"workload": f"decode_b{args.decode_batch}_l{args.decode_len}",
                          "dim": wl.dim, "N": wl.N, "G": wl.G, "k": wl.k, "d_h": wl.d_h,
                          "B": args.decode_batch, "cache_len": args.decode_len,
                          "variant": wl.variant},
               "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(),
                                "kind": "oracle", "sample": samples[0]["sample"]},
               "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                       "d2h_bytes_per_step": 0}}
        print(json.dumps(res))
        return 0

    if args.impl == "reference":
        if rank != 0:
            return 0
        wl = W.WORKLOADS[args.workload]
        if args.variant:
            wl = wl.with_(variant=args.variant)
        inp = W.generate(wl)
        rows = max(16, args.cpu_rows)
        for _ in range(args.warmup):
            oracle_sample(inp, rows)
        samples = [oracle_sample(inp, rows) for _ in range(args.steps)]
        # what ran: each step is the bounded sample; the throughput is the whole workload's
        # tokens over the sample's time extrapolated to every row
        ran_s = sum(s["whole_s"] + s["rows_s"] for s in samples) / len(samples)
        est = sum(s["est_s"] for s in samples) / len(samples)
        value = wl.M / est
        res = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
               "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
               "ms_per_step": ran_s * 1e3, "higher_is_better": True, "scaling": "weak",
               "vs_baseline": None, "dtype": "f64", "data": "synthetic",
               "config": prefill_config(wl, 1),
               "extrapolated_ms_per_full_step": est * 1e3,
               "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(),
                                "kind": "oracle", "sample": cpu_sample_desc(wl, rows),
                                "seconds": ran_s},
               "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                       "d2h_bytes_per_step": 0}}
        print(json.dumps(res))
        return 0

    import torch
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as td
        torch.cuda.set_device(local)
        td.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = td
    else:
        torch.cuda.set_device(0)
    if args.parallel == "groups" and world > 1 and args.mode == "prefill":
        res = bench_groups(args, rank, world, dist)
        if rank == 0:
            print(json.dumps(res))
        dist.barrier()
        dist.destroy_process_group()
        return 0
    if args.mode == "backward":
        res = bench_backward(args, rank, world, dist)
        if rank == 0:
            print(json.dumps(res))
        if dist:
            dist.barrier()
            dist.destroy_process_group()
        return 0
    if args.mode == "decode":
        res, wl = bench_decode(args, rank, world, dist)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                s = oracle_decode_sample(wl, args.decode_len, 4)
                res["cpu_baseline"] = {"value": s["tokens_per_s"], "unit": "tokens/s",
                                       "cores": blas_threads(), "kind": "oracle",
                                       "sample": s["sample"], "seconds": s["seconds"]}
            print(json.dumps(res))
        if dist:
            dist.barrier()
            dist.destroy_process_group()
        return 0
    res, inp = bench_ours(args, rank, world, dist)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            s = oracle_sample(inp, args.cpu_rows)
            res["cpu_baseline"] = {"value": s["tokens_per_s"], "unit": "tokens/s",
                                   "cores": blas_threads(), "kind": "oracle",
                                   "sample": cpu_sample_desc(inp.wl, s["rows"]),
                                   "seconds": s["whole_s"] + s["rows_s"]}
        print(json.dumps(res))
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
