"""CUDA-graph capture and replay through the C ABI: gqe_forward, gqe_decode, and a training
step (gqe_forward + gqe_backward) captured as one graph.

A captured call is replayed several times with new inputs copied into its static buffers,
with eager calls on the same handle in between; every replay must give exactly the eager
result for the same input (output, aux loss, routing counts), and the handle's device
status must stay clean. The kernels keep their per-call state (the routing cursors' two
alternating sets and the set flag, the attention's work counter) in device memory, so a
replay that reused a stale cursor set would show up as wrong counts and a status error.
One replay is also checked against the float64 oracle."""
import numpy as np
import pytest
import torch

from moe_query_head_b200 import workloads as W
from tests.gqe_testlib import (GpuRun, check_output, oracle_forward, rel_l2, to_device,
                               to_host_f64)

pytestmark = pytest.mark.gpu

MAIN = W.WORKLOADS["main_b8_t2048"]


def _capture(fn):
    """fn() once on a side stream (warm-up), then captured into a graph."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def _fwd(run: GpuRun):
    wl, d = run.wl, run.dev
    run.G.gqe_forward(run.h, d["x"], wl.B, wl.T, d["W_r"], d["W_q"], d["W_k"], d["W_v"],
                      d["W_shared"] if wl.shared else None, d["W_o"], wl.N, wl.G, wl.k, wl.d_h,
                      W.VARIANT_IDS[wl.variant], int(wl.causal), run.out, run.aux)


@pytest.mark.parametrize("wl", [MAIN.with_(B=2, T=300),
                                MAIN.with_(B=1, T=200, N=12, G=4, k=1),
                                MAIN.with_(B=1, T=333, variant="weighted_concat")],
                         ids=["routing_in_dense_projection", "experts_3_per_group",
                              "weighted_concat"])
def test_forward_graph_replays_match_eager(wl):
    inp = W.generate(wl)
    xs = [to_device(inp, "x"), to_device(W.generate(wl.with_(seed=wl.seed + 11)), "x")]
    eager = GpuRun(inp)
    ref = []
    for x in xs:
        eager.dev["x"] = x
        _fwd(eager)
        assert eager.G.gqe_check_device_status(eager.h) == eager.G.GQE_OK
        ref.append((eager.out.clone(), eager.aux.clone(), eager.routing()[2]))
    eager.close()

    run = GpuRun(inp)
    run.dev["x"] = xs[0].clone()  # the graph's static input
    g = _capture(lambda: _fwd(run))
    for step, i in enumerate([0, 1, 1, 0, 1, 0, 0]):
        run.dev["x"].copy_(xs[i])
        if step == 4:
            _fwd(run)  # an eager call on the same handle between replays
        else:
            g.replay()
        torch.cuda.synchronize()
        assert run.G.gqe_check_device_status(run.h) == run.G.GQE_OK, step
        y, aux, counts = ref[i]
        assert torch.equal(run.out, y), f"replay {step}: y differs from the eager call"
        assert torch.equal(run.aux, aux), f"replay {step}: aux loss differs"
        assert np.array_equal(run.routing()[2], counts), f"replay {step}: counts differ"
    # the last replay (input 0) against the oracle
    check_output(to_host_f64(run.out), oracle_forward(inp).y, "bf16")
    del g
    run.close()


def _dev_bf16(a_f32):
    bits = W.f32_to_bf16_bits(a_f32)
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def test_decode_graph_replays_match_eager():
    """Three generation steps of a captured gqe_decode (lengths advanced between replays on
    the device) against the same steps run eagerly on a copy of the caches: outputs and the
    caches bit-identical. Positions span one-CTA and split-chunk sequences."""
    lengths0 = [5, 700, 1500, 64, 0, 1023]
    d = W.generate_decode(MAIN, lengths0, 2048)
    wl = d.inp.wl
    from moe_query_head_b200 import gqe as G
    dev = {n: (None if d.inp.raw(n) is None else
               torch.from_numpy(d.inp.raw(n).view(np.int16)).view(torch.bfloat16).cuda())
           for n in ("x", "W_r", "W_q", "W_k", "W_v", "W_shared", "W_o")}
    xs = [dev["x"].roll(s, 0).contiguous() for s in range(3)]

    def state():
        return (_dev_bf16(d.k_cache), _dev_bf16(d.v_cache),
                torch.tensor(lengths0, dtype=torch.int32, device="cuda"),
                torch.empty((wl.M, wl.dim), dtype=torch.bfloat16, device="cuda"),
                torch.zeros(1, dtype=torch.float32, device="cuda"))

    def step(h, x, kc, vc, lens, out, aux):
        G.gqe_decode(h, x, wl.M, kc, vc, kc.shape[2], lens, dev["W_r"], dev["W_q"], dev["W_k"],
                     dev["W_v"], dev["W_shared"], dev["W_o"], wl.N, wl.G, wl.k, wl.d_h,
                     W.VARIANT_IDS[wl.variant], out, aux)

    he = G.gqe_create(wl.dim, wl.N, wl.G, wl.k, wl.d_h, G.GQE_BF16, wl.M)
    kc, vc, lens, out, aux = state()
    ref = []
    for x in xs:
        step(he, x, kc, vc, lens, out, aux)
        assert G.gqe_check_device_status(he) == G.GQE_OK
        ref.append((out.clone(), aux.clone()))
        lens += 1
    ref_caches = (kc, vc)

    hg = G.gqe_create(wl.dim, wl.N, wl.G, wl.k, wl.d_h, G.GQE_BF16, wl.M)
    kc, vc, lens, out, aux = state()
    xg = xs[0].clone()
    g = _capture(lambda: step(hg, xg, kc, vc, lens, out, aux))
    for s, x in enumerate(xs):
        xg.copy_(x)
        g.replay()
        torch.cuda.synchronize()
        assert G.gqe_check_device_status(hg) == G.GQE_OK, s
        assert torch.equal(out, ref[s][0]), f"step {s}: y differs from the eager step"
        assert torch.equal(aux, ref[s][1]), f"step {s}: aux loss differs"
        lens += 1
    assert torch.equal(kc, ref_caches[0]) and torch.equal(vc, ref_caches[1])
    del g
    G.gqe_destroy(he)
    G.gqe_destroy(hg)


def test_training_step_graph_replays_match_eager():
    """gqe_forward + gqe_backward captured together (the backward's GEMMs run in cuBLAS with
    the handle's preset workspace) and replayed with new x and dy: y bit-identical to the
    eager step's, every gradient equal to the eager step's within rel-L2 1e-6 (the same
    kernels; a library GEMM may pick another reduction order under capture)."""
    from moe_query_head_b200 import gqe as G
    wl = MAIN.with_(B=1, T=300)
    inp = W.generate(wl)
    xs = [to_device(inp, "x"), to_device(W.generate(wl.with_(seed=wl.seed + 5)), "x")]
    dys = [_dev_bf16(W.grad_output(wl)), _dev_bf16(W.grad_output(wl, seed_offset=1))]
    names = ("x", "W_r", "W_q", "W_k", "W_v", "W_shared", "W_o")
    shapes = dict(x=(wl.M, wl.dim), W_r=(wl.N, wl.dim), W_q=(wl.N * wl.d_h, wl.dim),
                  W_k=(wl.G * wl.d_h, wl.dim), W_v=(wl.G * wl.d_h, wl.dim),
                  W_shared=(wl.d_h, wl.dim), W_o=(wl.dim, wl.D_o))

    def make():
        run = GpuRun(inp)
        G.gqe_enable_backward(run.h)
        run.dy = dys[0].clone()
        run.g = {n: torch.zeros(shapes[n], dtype=torch.float32, device="cuda") for n in names}
        return run

    def train_step(run):
        _fwd(run)
        d, g = run.dev, run.g
        G.gqe_backward(run.h, d["x"], wl.B, wl.T, d["W_r"], d["W_q"], d["W_k"], d["W_v"],
                       d["W_shared"], d["W_o"], wl.N, wl.G, wl.k, wl.d_h,
                       W.VARIANT_IDS[wl.variant], int(wl.causal), run.dy, 0.01, g["x"],
                       g["W_r"], g["W_q"], g["W_k"], g["W_v"], g["W_shared"], g["W_o"])

    eager = make()
    ref = []
    for x, dy in zip(xs, dys):
        eager.dev["x"], eager.dy = x, dy
        train_step(eager)
        assert G.gqe_check_device_status(eager.h) == G.GQE_OK
        ref.append((eager.out.clone(), {n: eager.g[n].clone() for n in names}))
    eager.close()

    run = make()
    run.dev["x"] = xs[0].clone()
    g = _capture(lambda: train_step(run))
    for step, i in enumerate([1, 0, 1]):
        run.dev["x"].copy_(xs[i])
        run.dy.copy_(dys[i])
        g.replay()
        torch.cuda.synchronize()
        assert G.gqe_check_device_status(run.h) == G.GQE_OK, step
        assert torch.equal(run.out, ref[i][0]), f"replay {step}: y differs"
        for n in names:
            err = rel_l2(run.g[n].cpu().numpy(), ref[i][1][n].cpu().numpy())
            assert err <= 1e-6, (step, n, err)
    del g
    run.close()
