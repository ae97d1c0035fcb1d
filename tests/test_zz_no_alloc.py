"""gqe_route_static: routing from precomputed logits without any device allocation.

Some callers cannot call cudaMalloc (their device memory belongs to another allocator or a
fixed budget, they are plug-in code handed only their input and output buffers, or they
cannot accept cudaMalloc's device-wide synchronisation). gqe_route_static serves them by
keeping its scratch in a file-scope device array.

The first test checks it against the float64 oracle on seeded logits drawn on the host,
several calls in a row on different shapes (each call runs over the previous call's
leftover scratch), including the header's limits: N = 64 with k = 8, and M = 131072 tokens
with M * G * k = 262144 entries (1024 router blocks, 32 per lane of the scan). The second
checks it against the routing that gqe_forward produced for the same logits. This file is
named to be collected last.
"""
import numpy as np
import pytest
import torch

from moe_query_head_b200 import workloads as W
from tests.gqe_testlib import AUX_REL, GpuRun

pytestmark = pytest.mark.gpu

# (M, N, G, k): ragged block counts; the largest expert count and top-k; both size limits
ORACLE_CASES = [
    (600, 16, 8, 1),
    (300, 64, 8, 8),
    (517, 64, 8, 3),
    (131072, 4, 2, 1),
    (131072, 64, 1, 2),
    (1000, 32, 8, 2),
]


def _oracle_routing(logits32: np.ndarray, G: int, k: int):
    """The oracle's routing of given logits: oracle.route on x = logits and W_r = I, so
    that its logits x W_r^T are the given values exactly."""
    import oracle
    M, N = logits32.shape
    lg = logits32.astype(np.float64)
    rt = oracle.route(lg, np.eye(N), G, k)
    aux = oracle.aux_loss(rt.counts, rt.prob_sum, M, G, k)
    return rt, aux


def _call(logits: np.ndarray, G: int, k: int):
    from moe_query_head_b200 import gqe as GQ
    M, N = logits.shape
    lg = torch.from_numpy(logits).cuda()
    sel = torch.full((M, G, k), -1, dtype=torch.int32, device="cuda")
    gates = torch.full((M, G, k), float("nan"), device="cuda")
    counts = torch.full((N,), -1, dtype=torch.int32, device="cuda")
    mp = torch.full((N,), float("nan"), device="cuda")
    aux = torch.full((1,), float("nan"), device="cuda")
    GQ.gqe_route_static(lg, M, N, G, k, sel, gates, counts, mp, aux)
    torch.cuda.synchronize()
    return (sel.cpu().numpy(), gates.cpu().numpy(), counts.cpu().numpy(), mp.cpu().numpy(),
            float(aux.cpu()[0]))


def test_route_static_matches_oracle_calls_in_a_row():
    for i, (M, N, G, k) in enumerate(ORACLE_CASES):
        logits = W.router_logits_input(M, N, G, k, seed=10 + i)
        sel, gates, counts, mp, aux = _call(logits, G, k)
        rt, aux_ref = _oracle_routing(logits, G, k)
        assert np.array_equal(sel, rt.sel.astype(np.int32)), (M, N, G, k)
        assert np.array_equal(counts, rt.counts.astype(np.int32)), (M, N, G, k)
        np.testing.assert_allclose(gates, rt.gates, rtol=0, atol=2e-6)
        np.testing.assert_allclose(mp, rt.prob_sum / M, rtol=1e-5, atol=1e-7)
        assert abs(aux - aux_ref) <= AUX_REL * abs(aux_ref), (aux, aux_ref)


FORWARD_CASES = [
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
    refs = [(wl, _forward_reference(wl)) for wl in FORWARD_CASES]
    for wl, (logits, sel_r, gates_r, counts_r, mp_r, aux_r) in refs:
        sel, gates, counts, mp, aux = _call(logits.cpu().numpy(), wl.G, wl.k)
        assert np.array_equal(sel, sel_r)
        assert np.array_equal(counts, counts_r)
        np.testing.assert_allclose(gates, gates_r, rtol=0, atol=2e-6)
        np.testing.assert_allclose(mp, mp_r, rtol=1e-6, atol=0)
        assert abs(aux - aux_r) <= AUX_REL * abs(aux_r), (aux, aux_r)


def test_route_static_rejects_sizes_beyond_its_scratch():
    from moe_query_head_b200 import gqe as G
    z = torch.zeros(16, device="cuda")
    with pytest.raises(G.GQEError) as e:
        G.gqe_route_static(z, 1 << 18, 16, 8, 1, z, z, z, z)
    assert e.value.status == G.GQE_ERR_WORKSPACE
    with pytest.raises(G.GQEError) as e:
        G.gqe_route_static(z, 40000, 16, 8, 1, z, z, z, z)  # M*G*k > 262144
    assert e.value.status == G.GQE_ERR_WORKSPACE
    with pytest.raises(G.GQEError) as e:
        G.gqe_route_static(z, 100, 128, 8, 1, z, z, z, z)  # N above 64
    assert e.value.status == G.GQE_ERR_UNSUPPORTED
