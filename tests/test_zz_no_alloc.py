"""gqe_route_static: routing from precomputed logits without any device allocation.

Some callers cannot call cudaMalloc (their device memory belongs to another allocator or a
fixed budget, they are plug-in code handed only their input and output buffers, or they
cannot accept cudaMalloc's device-wide synchronisation). gqe_route_static serves them by
keeping its scratch in a file-scope device array. This test calls it through the C ABI
twice in a row, on two different layer shapes (so the second call runs over the first
call's leftover scratch), and checks each result against the routing gqe_forward
produced for the same logits. This file is named to be collected last.
"""
import numpy as np
import pytest
import torch

from moe_query_head_b200 import workloads as W
from tests.gqe_testlib import AUX_REL, GpuRun

pytestmark = pytest.mark.gpu

CASES = [
    W.WORKLOADS["main_b8_t2048"].with_(B=2, T=300),
    W.WORKLOADS["wide_k2"].with_(B=1, T=1000),
]


def _forward_reference(wl):
    run = GpuRun(W.generate(wl)).forward()
    logits = run.tensor("LOGITS", (wl.M, wl.N), torch.float32)
    sel, gates, counts, mean_prob = run.routing()
    aux = float(run.aux.cpu()[0])
    run.close()
    return logits, sel, gates, counts, mean_prob, aux


def test_route_static_matches_forward_twice_in_a_row():
    from moe_query_head_b200 import gqe as G
    refs = [(wl, _forward_reference(wl)) for wl in CASES]
    for wl, (logits, sel_r, gates_r, counts_r, mp_r, aux_r) in refs:
        sel = torch.full((wl.M, wl.G, wl.k), -1, dtype=torch.int32, device="cuda")
        gates = torch.full((wl.M, wl.G, wl.k), float("nan"), device="cuda")
        counts = torch.full((wl.N,), -1, dtype=torch.int32, device="cuda")
        mp = torch.full((wl.N,), float("nan"), device="cuda")
        aux = torch.full((1,), float("nan"), device="cuda")
        G.gqe_route_static(logits, wl.M, wl.N, wl.G, wl.k, sel, gates, counts, mp, aux)
        torch.cuda.synchronize()
        assert np.array_equal(sel.cpu().numpy(), sel_r)
        assert np.array_equal(counts.cpu().numpy(), counts_r)
        np.testing.assert_allclose(gates.cpu().numpy(), gates_r, rtol=0, atol=2e-6)
        np.testing.assert_allclose(mp.cpu().numpy(), mp_r, rtol=1e-6, atol=0)
        a = float(aux.cpu()[0])
        assert abs(a - aux_r) <= AUX_REL * abs(aux_r), (a, aux_r)


def test_route_static_rejects_sizes_beyond_its_scratch():
    from moe_query_head_b200 import gqe as G
    z = torch.zeros(16, device="cuda")
    with pytest.raises(G.GQEError) as e:
        G.gqe_route_static(z, 1 << 18, 16, 8, 1, z, z, z, z)
    assert e.value.status == G.GQE_ERR_WORKSPACE
    with pytest.raises(G.GQEError) as e:
        G.gqe_route_static(z, 40000, 16, 8, 1, z, z, z, z)  # M*G*k > 262144
    assert e.value.status == G.GQE_ERR_WORKSPACE
