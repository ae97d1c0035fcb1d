"""GPU parity of group-parallel execution on one GPU: the ranks' shares of the layer (each a
handle restricted to its group range by gqe_set_group_range, with the rank's weight slices)
run one after another, and their sum is checked against the float64 oracle's whole-layer
y at the bf16 tolerances. Every share's routing and aux loss are the whole layer's
(bit-exact routing, aux within 1e-4 relative). The shares run as separate launches with no
waits between ranks, so one GPU can run them in turn; the multi-process sum itself is the
NCCL all-reduce that group_parallel.GroupShard.forward_allreduce issues. The backward on the
split (gqe_backward_begin / gqe_backward_finish with the ranks' <dslot, slot> summed in
between) is checked the same way against the oracle's whole-layer gradients."""
import numpy as np
import pytest
import torch

from moe_query_head_b200 import group_parallel as GP
from moe_query_head_b200 import workloads as W
from tests.gqe_testlib import AUX_REL, check_output, oracle_forward, to_device, to_host_f64

pytestmark = pytest.mark.gpu

CASES = {
    "main_2_ranks": (W.WORKLOADS["main_b8_t2048"].with_(B=2, T=300), 2),
    "main_3_ranks_uneven": (W.WORKLOADS["main_b8_t2048"].with_(B=1, T=257), 3),
    "main_8_ranks": (W.WORKLOADS["main_b8_t2048"].with_(B=1, T=200), 8),
    "wide_2_ranks": (W.WORKLOADS["wide_k2"].with_(B=1, T=300), 2),
    "wide_weighted_4_ranks": (W.WORKLOADS["wide_k2"].with_(B=1, T=200,
                                                        variant="weighted_concat"), 4),
    "main_no_shared_2_ranks": (W.WORKLOADS["main_b8_t2048"].with_(B=1, T=200, shared=False,
                                                              variant="hard_concat"), 2),
}


@pytest.mark.parametrize("case", list(CASES))
def test_group_shards_sum_to_the_layer(case):
    from moe_query_head_b200 import gqe as GQ
    wl, world = CASES[case]
    inp = W.generate(wl)
    d = {n: to_device(inp, n) for n in ("x", "W_r", "W_q", "W_k", "W_v", "W_shared", "W_o")}
    ref = oracle_forward(inp)
    total = torch.zeros((wl.M, wl.dim), dtype=torch.float32, device="cuda")
    for g0, g1 in GP.group_ranges(wl.G, world):
        sh = GP.GroupShard(dim=wl.dim, N=wl.N, G=wl.G, k=wl.k, d_h=wl.d_h, variant=wl.variant,
                           causal=wl.causal, max_tokens=wl.M, g0=g0, g1=g1, W_r=d["W_r"],
                           W_q=d["W_q"], W_k=d["W_k"], W_v=d["W_v"],
                           W_shared=d["W_shared"] if wl.shared else None, W_o=d["W_o"])
        out = torch.full((wl.M, wl.dim), float("nan"), dtype=torch.bfloat16, device="cuda")
        sh.forward(d["x"], wl.B, wl.T, out)
        assert GQ.gqe_check_device_status(sh.h) == GQ.GQE_OK
        total += out.float()
        sel = torch.empty((wl.M, wl.G, wl.k), dtype=torch.int32, device="cuda")
        counts = torch.empty((wl.N,), dtype=torch.int32, device="cuda")
        GQ.gqe_get_routing(sh.h, sel=sel, counts=counts)
        torch.cuda.synchronize()
        assert np.array_equal(sel.cpu().numpy(), ref.routing.sel.astype(np.int32))
        assert np.array_equal(counts.cpu().numpy(), ref.routing.counts.astype(np.int32))
        aux = float(sh.aux.cpu()[0])
        assert abs(aux - ref.aux) <= AUX_REL * abs(ref.aux), (aux, ref.aux)
        sh.close()
    check_output(total.cpu().numpy().astype(np.float64), ref.y, "bf16")


def test_group_range_errors():
    from moe_query_head_b200 import gqe as GQ
    h = GQ.gqe_create(768, 16, 8, 1, 48, GQ.GQE_BF16, 64)
    for g0, g1 in ((0, 0), (3, 2), (-1, 4), (0, 9)):
        with pytest.raises(GQ.GQEError) as e:
            GQ.gqe_set_group_range(h, g0, g1)
        assert e.value.status == GQ.GQE_ERR_INVALID_ARG
    GQ.gqe_destroy(h)
    # routing outside the dense projection (N not a power of two): whole layers only
    h = GQ.gqe_create(768, 12, 4, 1, 48, GQ.GQE_BF16, 64)
    with pytest.raises(GQ.GQEError) as e:
        GQ.gqe_set_group_range(h, 0, 2)
    assert e.value.status == GQ.GQE_ERR_UNSUPPORTED
    GQ.gqe_destroy(h)


def test_group_shards_full_size_sampled():
    """The long-context workload split over 2 ranks, at full size, on sampled rows of the
    summed output against the oracle's rows (routing bit-exact on every rank)."""
    from moe_query_head_b200 import gqe as GQ
    from tests.gqe_testlib import oracle_rows, sample_rows
    wl = W.WORKLOADS["long_t16k"]
    inp = W.cached("long_t16k")
    d = {n: to_device(inp, n) for n in ("x", "W_r", "W_q", "W_k", "W_v", "W_shared", "W_o")}
    rows = sample_rows(wl)
    ref = oracle_rows(inp, rows)
    total = torch.zeros((wl.M, wl.dim), dtype=torch.float32, device="cuda")
    for g0, g1 in GP.group_ranges(wl.G, 2):
        sh = GP.GroupShard(dim=wl.dim, N=wl.N, G=wl.G, k=wl.k, d_h=wl.d_h, variant=wl.variant,
                           causal=wl.causal, max_tokens=wl.M, g0=g0, g1=g1, W_r=d["W_r"],
                           W_q=d["W_q"], W_k=d["W_k"], W_v=d["W_v"], W_shared=d["W_shared"],
                           W_o=d["W_o"])
        out = torch.empty((wl.M, wl.dim), dtype=torch.bfloat16, device="cuda")
        sh.forward(d["x"], wl.B, wl.T, out)
        assert GQ.gqe_check_device_status(sh.h) == GQ.GQE_OK
        total += out.float()
        counts = torch.empty((wl.N,), dtype=torch.int32, device="cuda")
        GQ.gqe_get_routing(sh.h, counts=counts)
        torch.cuda.synchronize()
        assert np.array_equal(counts.cpu().numpy(), ref["routing"].counts.astype(np.int32))
        sh.close()
    check_output(total.cpu().numpy().astype(np.float64)[rows], ref["y"], "bf16")


MAIN = W.WORKLOADS["main_b8_t2048"]
WIDE = W.WORKLOADS["wide_k2"]
BWD_CASES = {
    "main_2_ranks": (MAIN.with_(B=1, T=300), 2),
    "main_3_ranks_uneven": (MAIN.with_(B=2, T=150), 3),
    "main_8_ranks_noncausal": (MAIN.with_(B=1, T=200, causal=False), 8),
    "wide_gqe_2_ranks": (WIDE.with_(B=1, T=260), 2),
    "wide_weighted_4_ranks": (WIDE.with_(B=1, T=200, variant="weighted_concat"), 4),
    "main_hard_no_shared_2_ranks": (MAIN.with_(B=1, T=200, shared=False,
                                               variant="hard_concat"), 2),
    "dh128_2_ranks": (MAIN.with_(B=1, T=200, d_h=128), 2),
}
GRAD_REL_L2 = 1e-2  # as the whole-layer backward tests: bf16 dO, dQ, dK, dV and dl


@pytest.mark.parametrize("case", list(BWD_CASES))
def test_group_shards_backward_sums_to_the_layer(case):
    """Training on the split: every rank's forward, then phase 1 on every rank, the ranks'
    <dslot, slot> summed (what the all-reduce of GroupShard.backward_allreduce does), phase
    2 on every rank; the ranks' gradient shares placed in the layer's shapes and summed give
    the float64 oracle's gradients of <dy, y> + 0.01 aux for x and every weight."""
    import oracle
    from moe_query_head_b200 import gqe as GQ
    from tests.gqe_testlib import rel_l2
    wl, world = BWD_CASES[case]
    inp = W.generate(wl)
    d = {n: to_device(inp, n) for n in ("x", "W_r", "W_q", "W_k", "W_v", "W_shared", "W_o")}
    dy_h = W.grad_output(wl)
    dy = torch.from_numpy(W.f32_to_bf16_bits(dy_h).view(np.int16)).view(torch.bfloat16).cuda()
    f = inp.f64
    layer = oracle.Layer(dim=wl.dim, N=wl.N, G=wl.G, k=wl.k, d_h=wl.d_h, shared=wl.shared,
                         variant=wl.variant, causal=wl.causal)
    ref = oracle.backward(layer, f("x"), wl.B, wl.T, f("W_r"), f("W_q"), f("W_k"), f("W_v"),
                          f("W_shared"), f("W_o"), dy_h.astype(np.float64), 0.01)
    shards = []
    for g0, g1 in GP.group_ranges(wl.G, world):
        sh = GP.GroupShard(dim=wl.dim, N=wl.N, G=wl.G, k=wl.k, d_h=wl.d_h, variant=wl.variant,
                           causal=wl.causal, max_tokens=wl.M, g0=g0, g1=g1, W_r=d["W_r"],
                           W_q=d["W_q"], W_k=d["W_k"], W_v=d["W_v"],
                           W_shared=d["W_shared"] if wl.shared else None, W_o=d["W_o"])
        sh.enable_backward()
        out = torch.empty((wl.M, wl.dim), dtype=torch.bfloat16, device="cuda")
        sh.forward(d["x"], wl.B, wl.T, out)
        shards.append(sh)
    slot_dot = torch.zeros(wl.M, dtype=torch.float32, device="cuda")
    for sh in shards:
        part = torch.full((wl.M,), float("nan"), dtype=torch.float32, device="cuda")
        sh.backward_begin(d["x"], wl.B, wl.T, dy, part)
        slot_dot += part
    total = None
    for sh in shards:
        g = sh.backward_finish(d["x"], wl.B, wl.T, dy, 0.01, slot_dot)
        assert GQ.gqe_check_device_status(sh.h) == GQ.GQE_OK
        full = GP.full_gradients(g, N=wl.N, G=wl.G, k=wl.k, d_h=wl.d_h, variant=wl.variant,
                                 shared=wl.shared, D_o=wl.D_o, g0=sh.g0, g1=sh.g1)
        total = full if total is None else {n: (None if v is None else v + full[n])
                                            for n, v in total.items()}
    for sh in shards:
        sh.close()
    errs = {}
    for name in ("x", "W_r", "W_q", "W_k", "W_v", "W_shared", "W_o"):
        r = getattr(ref, name)
        if r is None:
            assert total[name] is None
            continue
        got = total[name].cpu().numpy().astype(np.float64)
        assert np.isfinite(got).all(), name
        errs[name] = rel_l2(got, r)
    bad = {n: e for n, e in errs.items() if not e <= GRAD_REL_L2}
    assert not bad, (errs, bad)


def test_backward_phases_need_a_begin():
    """finish without a successful begin after the last forward is refused, as is the
    one-call backward on a group range."""
    from moe_query_head_b200 import gqe as GQ
    wl = MAIN.with_(B=1, T=130)
    inp = W.generate(wl)
    d = {n: to_device(inp, n) for n in ("x", "W_r", "W_q", "W_k", "W_v", "W_shared", "W_o")}
    dy = torch.zeros((wl.M, wl.dim), dtype=torch.bfloat16, device="cuda")
    sh = GP.GroupShard(dim=wl.dim, N=wl.N, G=wl.G, k=wl.k, d_h=wl.d_h, variant=wl.variant,
                       causal=wl.causal, max_tokens=wl.M, g0=0, g1=4, W_r=d["W_r"],
                       W_q=d["W_q"], W_k=d["W_k"], W_v=d["W_v"], W_shared=d["W_shared"],
                       W_o=d["W_o"])
    sh.enable_backward()
    out = torch.empty((wl.M, wl.dim), dtype=torch.bfloat16, device="cuda")
    sh.forward(d["x"], wl.B, wl.T, out)
    sd = torch.zeros(wl.M, dtype=torch.float32, device="cuda")
    with pytest.raises(GQ.GQEError) as e:
        sh.backward_finish(d["x"], wl.B, wl.T, dy, 0.01, sd)
    assert e.value.status == GQ.GQE_ERR_INVALID_ARG
    w = sh.w
    z = lambda *s: torch.zeros(s, dtype=torch.float32, device="cuda")  # noqa: E731
    with pytest.raises(GQ.GQEError) as e:
        GQ.gqe_backward(sh.h, d["x"], wl.B, wl.T, d["W_r"], w["W_q"], w["W_k"], w["W_v"],
                        w["W_shared"], w["W_o"], wl.N, wl.G, wl.k, wl.d_h, 0, 1, dy, 0.01,
                        z(wl.M, wl.dim), z(wl.N, wl.dim), z(*w["W_q"].shape),
                        z(*w["W_k"].shape), z(*w["W_v"].shape), z(wl.d_h, wl.dim),
                        z(*w["W_o"].shape))
    assert e.value.status == GQ.GQE_ERR_UNSUPPORTED
    # begin then finish works; a second finish is refused
    sh.backward_begin(d["x"], wl.B, wl.T, dy, sd)
    sh.backward_finish(d["x"], wl.B, wl.T, dy, 0.01, sd)
    with pytest.raises(GQ.GQEError) as e:
        sh.backward_finish(d["x"], wl.B, wl.T, dy, 0.01, sd)
    assert e.value.status == GQ.GQE_ERR_INVALID_ARG
    sh.close()


DEC_CASES = {
    "main_2_ranks": (MAIN, [0, 5, 63, 64, 200, 511], 512, 2),
    "main_3_ranks_uneven": (MAIN, [3, 130, 300], 320, 3),
    "wide_weighted_4_ranks": (WIDE.with_(variant="weighted_concat"), [10, 257, 70], 260, 4),
    "main_hard_no_shared_8_ranks": (MAIN.with_(shared=False, variant="hard_concat"),
                                    [1, 100], 128, 8),
}


@pytest.mark.parametrize("case", list(DEC_CASES))
def test_group_shards_decode_sums_to_the_layer(case):
    """A decode step on the split: every rank holds its heads' caches and computes its share;
    the shares sum to the float64 oracle's step (y at the bf16 tolerances, routing bit-exact
    on every rank), and each rank writes its heads' new K / V at the new positions and no
    other cache row."""
    from moe_query_head_b200 import gqe as GQ
    from tests.test_decode_gpu import _dev_bf16, oracle_decode
    wl, lengths, L_max, world = DEC_CASES[case]
    d = W.generate_decode(wl, lengths, L_max)
    ref = oracle_decode(d)
    inp = d.inp
    dev = {n: to_device(inp, n) for n in ("x", "W_r", "W_q", "W_k", "W_v", "W_shared", "W_o")}
    kc, vc = _dev_bf16(d.k_cache), _dev_bf16(d.v_cache)
    lens = torch.from_numpy(d.lengths.astype(np.int32)).cuda()
    B = len(lengths)
    total = torch.zeros((B, inp.wl.dim), dtype=torch.float32, device="cuda")
    for g0, g1 in GP.group_ranges(inp.wl.G, world):
        sh = GP.GroupShard(dim=inp.wl.dim, N=inp.wl.N, G=inp.wl.G, k=inp.wl.k, d_h=inp.wl.d_h,
                           variant=inp.wl.variant, causal=True, max_tokens=B, g0=g0, g1=g1,
                           W_r=dev["W_r"], W_q=dev["W_q"], W_k=dev["W_k"], W_v=dev["W_v"],
                           W_shared=dev["W_shared"] if inp.wl.shared else None, W_o=dev["W_o"])
        kr, vr = GP.rank_caches(kc, vc, g0, g1)
        k0, v0 = kr.clone(), vr.clone()
        out = torch.full((B, inp.wl.dim), float("nan"), dtype=torch.bfloat16, device="cuda")
        sh.decode(dev["x"], B, kr, vr, L_max, lens, out)
        assert GQ.gqe_check_device_status(sh.h) == GQ.GQE_OK
        total += out.float()
        sel = torch.empty((B, inp.wl.G, inp.wl.k), dtype=torch.int32, device="cuda")
        GQ.gqe_get_routing(sh.h, sel=sel)
        torch.cuda.synchronize()
        assert np.array_equal(sel.cpu().numpy(), ref.routing.sel.astype(np.int32))
        keep = torch.ones(kr.shape[:3], dtype=torch.bool, device="cuda")
        for b, L in enumerate(d.lengths.tolist()):
            keep[:, b, L] = False
        assert torch.equal(kr[keep], k0[keep]) and torch.equal(vr[keep], v0[keep])
        rows = torch.stack([kr[:, b, L] for b, L in enumerate(d.lengths.tolist())], dim=1)
        np.testing.assert_allclose(to_host_f64(rows), ref.K_new[g0:g1], rtol=1e-2, atol=1e-2)
        sh.close()
    check_output(total.cpu().numpy().astype(np.float64), ref.y, "bf16")
