"""GPU parity of group-parallel execution on one GPU: the ranks' shares of the layer (each a
handle restricted to its group range by gqe_set_group_range, with the rank's weight slices)
run one after another, and their sum is checked against the float64 oracle's whole-layer
y at the bf16 tolerances. Every share's routing and aux loss are the whole layer's
(bit-exact routing, aux within 1e-4 relative). The shares run as separate launches with no
waits between ranks, so one GPU can run them in turn; the multi-process sum itself is the
NCCL all-reduce that group_parallel.GroupShard.forward_allreduce issues."""
import numpy as np
import pytest
import torch

from moe_query_head_b200 import group_parallel as GP
from moe_query_head_b200 import workloads as W
from tests.gqe_testlib import AUX_REL, check_output, oracle_forward, to_device

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
