"""GPU parity of the backward pass (gqe_backward, through the C ABI) against the float64
oracle's backward on identical seeded inputs: every gradient (x, W_r, W_q, W_k, W_v,
W_shared, W_o) within rel-L2 GRAD_REL_L2 of the oracle's.

The tolerance: the GPU path stores dZ's consumers, dO, dQ, dK, dV and the router logits'
gradient in bf16 (relative rounding 2^-9 each) and recomputes P in fp32 from bf16 Q, K;
every gradient is a sum of such terms, so its rel-L2 error is a small multiple of 2^-9
(about 2e-3), as the forward's bf16 tolerance is. The router weights' gradient is a
difference of products (dl = p (dp - sum p dp), dp_sel = (dw - sum dw w) / P_t), which can
cancel and raise the relative error; it gets the same bound, checked on the gqe variant
whose slot feeds it and on the aux term alone.

Cases: several query and key tiles with a ragged tail, causal and not, the three variants,
every head dim the bf16 path accepts (16 to 64 on the two-CTA-per-SM kernels, 80 to 128 on
the one-CTA-per-SM ones), three experts per group, no shared head, and the aux loss's
gradient alone (dy = 0)."""
import numpy as np
import pytest
import torch

from moe_query_head_b200 import workloads as W
from tests.gqe_testlib import GpuRun, rel_l2, to_host_f64

pytestmark = pytest.mark.gpu

GRAD_REL_L2 = 1e-2


def _bf16(a):
    return torch.from_numpy(W.f32_to_bf16_bits(a).view(np.int16)).view(torch.bfloat16).cuda()


def _oracle_backward(inp, dy, dA):
    import oracle
    wl = inp.wl
    f = inp.f64
    layer = oracle.Layer(dim=wl.dim, N=wl.N, G=wl.G, k=wl.k, d_h=wl.d_h, shared=wl.shared,
                         variant=wl.variant, causal=wl.causal)
    return oracle.backward(layer, f("x"), wl.B, wl.T, f("W_r"), f("W_q"), f("W_k"), f("W_v"),
                           f("W_shared"), f("W_o"), dy.astype(np.float64), dA)


def _gpu_backward(run: GpuRun, dy, dA):
    from moe_query_head_b200 import gqe as G
    wl, d = run.wl, run.dev
    G.gqe_enable_backward(run.h)
    z = lambda *s: torch.full(s, float("nan"), dtype=torch.float32, device="cuda")  # noqa
    g = dict(x=z(wl.M, wl.dim), W_r=z(wl.N, wl.dim), W_q=z(wl.N * wl.d_h, wl.dim),
             W_k=z(wl.G * wl.d_h, wl.dim), W_v=z(wl.G * wl.d_h, wl.dim),
             W_shared=z(wl.d_h, wl.dim) if wl.shared else None, W_o=z(wl.dim, wl.D_o))
    G.gqe_backward(run.h, d["x"], wl.B, wl.T, d["W_r"], d["W_q"], d["W_k"], d["W_v"],
                   d["W_shared"] if wl.shared else None, d["W_o"], wl.N, wl.G, wl.k, wl.d_h,
                   W.VARIANT_IDS[wl.variant], int(wl.causal), _bf16(dy), dA, g["x"], g["W_r"],
                   g["W_q"], g["W_k"], g["W_v"], g["W_shared"], g["W_o"])
    assert G.gqe_check_device_status(run.h) == G.GQE_OK
    return {k: (None if v is None else v.cpu().numpy().astype(np.float64)) for k, v in g.items()}


def _check(wl, dA=0.01, zero_dy=False):
    inp = W.generate(wl)
    dy = np.zeros((wl.M, wl.dim), np.float32) if zero_dy else W.grad_output(wl)
    run = GpuRun(inp).forward()
    got = _gpu_backward(run, dy, dA)
    ref = _oracle_backward(inp, dy, dA)
    errs = {}
    for name in ("x", "W_r", "W_q", "W_k", "W_v", "W_shared", "W_o"):
        r = getattr(ref, name)
        if r is None:
            assert got[name] is None
            continue
        assert np.isfinite(got[name]).all(), name
        if zero_dy and name != "W_r" and name != "x":
            assert np.abs(got[name]).max() == 0.0, name
            continue
        errs[name] = rel_l2(got[name], r)
    run.close()
    bad = {k: v for k, v in errs.items() if not v <= GRAD_REL_L2}
    assert not bad, (errs, bad)
    return errs


MAIN = W.WORKLOADS["main_b8_t2048"]
WIDE = W.WORKLOADS["wide_k2"]
CASES = {
    "main_ragged": MAIN.with_(B=2, T=300),
    "main_noncausal": MAIN.with_(B=1, T=260, causal=False),
    "main_long": MAIN.with_(B=1, T=1030),
    "main_no_shared": MAIN.with_(B=1, T=200, shared=False),
    "wide_gqe": WIDE.with_(B=1, T=300),
    "wide_weighted": WIDE.with_(B=1, T=300, variant="weighted_concat"),
    "wide_hard": WIDE.with_(B=1, T=300, variant="hard_concat"),
    "experts_3_per_group": MAIN.with_(B=1, T=200, N=12, G=4, k=1),
    "dh16": MAIN.with_(B=1, T=200, d_h=16),
    "dh32": MAIN.with_(B=2, T=150, d_h=32),
    "dh80": MAIN.with_(B=1, T=300, d_h=80),
    "dh96_noncausal": MAIN.with_(B=2, T=150, d_h=96, causal=False),
    "dh112_weighted": MAIN.with_(B=1, T=260, d_h=112, variant="weighted_concat"),
    "dh128": MAIN.with_(B=1, T=300, d_h=128),
    "dh128_noncausal_k2": WIDE.with_(dim=768, B=1, T=200, d_h=128, causal=False),
}


@pytest.mark.parametrize("case", list(CASES))
def test_backward_matches_oracle(case):
    _check(CASES[case])


def test_backward_single_key_rows():
    """T = 1: every query attends to its one key, so P = 1, D = <dO, O> = <dO, V> = dP and
    dS = P (dP - D) = 0: the query and key gradients (hence dW_q, dW_k, dW_shared) vanish
    up to rounding, while dV = dO and the other gradients match the oracle."""
    wl = MAIN.with_(B=3, T=1)
    inp = W.generate(wl)
    dy = W.grad_output(wl)
    run = GpuRun(inp).forward()
    got = _gpu_backward(run, dy, 0.01)
    ref = _oracle_backward(inp, dy, 0.01)
    run.close()
    for name in ("x", "W_r", "W_v", "W_o"):
        assert rel_l2(got[name], getattr(ref, name)) <= GRAD_REL_L2, name
    scale = np.abs(got["W_v"]).max()
    for name in ("W_q", "W_k", "W_shared"):
        assert np.abs(got[name]).max() <= 1e-2 * scale, name
        assert np.abs(getattr(ref, name)).max() <= 1e-9 * scale, name


def test_backward_aux_term_alone():
    """dy = 0: only the aux loss's gradient reaches the router (dx and dW_r), every other
    gradient is exactly zero."""
    _check(MAIN.with_(B=1, T=256), dA=0.5, zero_dy=True)


def test_backward_deterministic_and_requires_matching_forward():
    from moe_query_head_b200 import gqe as G
    wl = MAIN.with_(B=1, T=300)
    inp = W.generate(wl)
    dy = W.grad_output(wl)
    run = GpuRun(inp).forward()
    a = _gpu_backward(run, dy, 0.01)
    b = _gpu_backward(run, dy, 0.01)
    for k in a:
        if a[k] is not None:
            assert np.array_equal(a[k], b[k]), k
    d = run.dev
    z = torch.zeros((wl.M, wl.dim), dtype=torch.float32, device="cuda")
    with pytest.raises(G.GQEError) as e:  # T differs from the forward's
        G.gqe_backward(run.h, d["x"], 1, 299, d["W_r"], d["W_q"], d["W_k"], d["W_v"],
                       d["W_shared"], d["W_o"], wl.N, wl.G, wl.k, wl.d_h, 0, 1, _bf16(dy), 0.0,
                       z, z, z, z, z, z, z)
    assert e.value.status == G.GQE_ERR_INVALID_ARG
    run.close()


def test_backward_two_phases_equal_one_call():
    """On a whole layer, gqe_backward_begin with its own <dslot, slot> fed to
    gqe_backward_finish gives exactly the one-call gqe_backward's gradients."""
    from moe_query_head_b200 import gqe as G
    wl = WIDE.with_(B=1, T=300)
    inp = W.generate(wl)
    dy = W.grad_output(wl)
    run = GpuRun(inp).forward()
    a = _gpu_backward(run, dy, 0.01)
    d = run.dev
    f32 = lambda *s: torch.full(s, float("nan"), dtype=torch.float32, device="cuda")  # noqa
    g = dict(x=f32(wl.M, wl.dim), W_r=f32(wl.N, wl.dim), W_q=f32(wl.N * wl.d_h, wl.dim),
             W_k=f32(wl.G * wl.d_h, wl.dim), W_v=f32(wl.G * wl.d_h, wl.dim),
             W_shared=f32(wl.d_h, wl.dim), W_o=f32(wl.dim, wl.D_o))
    sd = f32(wl.M)
    args = (run.h, d["x"], wl.B, wl.T, d["W_r"], d["W_q"], d["W_k"], d["W_v"], d["W_shared"],
            d["W_o"], wl.N, wl.G, wl.k, wl.d_h, W.VARIANT_IDS[wl.variant], int(wl.causal),
            _bf16(dy))
    G.gqe_backward_begin(*args, sd)
    G.gqe_backward_finish(*args, 0.01, sd, g["x"], g["W_r"], g["W_q"], g["W_k"], g["W_v"],
                          g["W_shared"], g["W_o"])
    assert G.gqe_check_device_status(run.h) == G.GQE_OK
    for k_, v in g.items():
        assert np.array_equal(v.cpu().numpy().astype(np.float64), a[k_]), k_
    run.close()


def test_backward_unsupported_shapes():
    """float32 handles (the CUDA-core path) have no backward."""
    from moe_query_head_b200 import gqe as G
    h = G.gqe_create(64, 4, 2, 1, 16, G.GQE_F32, 64)
    with pytest.raises(G.GQEError) as e:
        G.gqe_enable_backward(h)
    assert e.value.status == G.GQE_ERR_UNSUPPORTED
    G.gqe_destroy(h)


@pytest.mark.parametrize("name", ["long_t16k", "main_b8_t2048", "wide_k2", "large_skew"])
def test_backward_full_size_last_rows(name):
    """At the benchmark's full sizes, in its launch configuration: the input gradient of the
    last 256 positions of every sequence against the oracle's row-restricted backward (which
    needs only the queries at those positions), within the bf16 tolerance."""
    import oracle
    wl = W.WORKLOADS[name]
    inp = W.cached(name)
    dy = W.grad_output(wl)
    run = GpuRun(inp).forward()
    got = _gpu_backward(run, dy, 0.01)
    run.close()
    t_min = wl.T - 256
    f = inp.f64
    layer = oracle.Layer(dim=wl.dim, N=wl.N, G=wl.G, k=wl.k, d_h=wl.d_h, shared=wl.shared,
                         variant=wl.variant, causal=wl.causal)
    ref = oracle.backward_x_rows(layer, f("x"), wl.B, wl.T, f("W_r"), f("W_q"), f("W_k"),
                                 f("W_v"), f("W_shared"), f("W_o"), dy.astype(np.float64), 0.01,
                                 t_min)
    rows = np.concatenate([np.arange(b * wl.T + t_min, (b + 1) * wl.T) for b in range(wl.B)])
    assert rel_l2(got["x"][rows], ref) <= GRAD_REL_L2
    for k_, v in got.items():
        if v is not None:
            assert np.isfinite(v).all(), k_
