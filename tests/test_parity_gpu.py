"""GPU parity: the CUDA path through the C ABI against the float64 oracle, on identical
seeded inputs. Routing indices and expert counts bit-exact; y within rel-L2 1e-2 and
max-abs 3e-2 (bf16) or rel-L2 1e-5 (fp32); aux loss within 1e-4 relative."""
import numpy as np
import pytest
import torch

from moe_query_head_b200 import workloads as W
from tests.gqe_testlib import (AUX_REL, GpuRun, check_output, oracle_forward, oracle_rows,
                               rel_l2, sample_rows, to_host_f64)

pytestmark = pytest.mark.gpu


def _check_routing(run, sel_ref, counts_ref, gates_ref=None):
    sel, gates, counts, _ = run.routing()
    assert np.array_equal(sel, sel_ref.astype(np.int32)), "routing indices differ"
    assert np.array_equal(counts, counts_ref.astype(np.int32)), "expert counts differ"
    if gates_ref is not None:
        np.testing.assert_allclose(gates, gates_ref, rtol=0, atol=2e-6)


def _check_aux(run, aux_ref):
    aux = float(run.aux.cpu()[0])
    assert abs(aux - aux_ref) <= AUX_REL * abs(aux_ref), (aux, aux_ref)


def _full_check(inp):
    wl = inp.wl
    run = GpuRun(inp).forward()
    ref = oracle_forward(inp)
    _check_routing(run, ref.routing.sel, ref.routing.counts, ref.routing.gates)
    _check_aux(run, ref.aux)
    y = to_host_f64(run.out)
    r, mx = check_output(y, ref.y, wl.dtype)
    return run, ref, r, mx


def test_tiny_f32_full_and_intermediates():
    inp = W.cached("tiny_f32")
    wl = inp.wl
    run, ref, r, _ = _full_check(inp)
    tdt = torch.float32
    K = to_host_f64(run.tensor("K", (wl.G, wl.M, wl.d_h), tdt))
    V = to_host_f64(run.tensor("V", (wl.G, wl.M, wl.d_h), tdt))
    Q = to_host_f64(run.tensor("Q", (wl.n_streams, wl.M, wl.d_h), tdt))
    Z = to_host_f64(run.tensor("Z", (wl.M, wl.D_o), tdt))
    assert rel_l2(K, ref.K) <= 1e-6
    assert rel_l2(V, ref.V) <= 1e-6
    assert rel_l2(Q, ref.Q) <= 1e-6
    assert rel_l2(Z, ref.Z) <= 1e-5
    run.close()


SMALL = {
    "main_ragged": dict(base="main_b8_t2048", B=2, T=300),
    "main_noncausal": dict(base="main_b8_t2048", B=2, T=130, causal=False),
    "main_all_active": dict(base="main_b8_t2048", B=1, T=257, k=2),
    "main_no_shared_hard": dict(base="main_b8_t2048", B=1, T=200, shared=False,
                                variant="hard_concat"),
    "wide_gqe": dict(base="wide_k2", B=1, T=200),
    "wide_weighted": dict(base="wide_k2", B=1, T=200, variant="weighted_concat"),
    "wide_hard": dict(base="wide_k2", B=1, T=200, variant="hard_concat"),
    "large_small": dict(base="large_skew", B=1, T=260, skew=None),
    "tiny_f32_batch": dict(base="tiny_f32", B=3, T=77),
    "one_token": dict(base="main_b8_t2048", B=3, T=1),
    # routing shapes: experts per group not a power of two (the separate routing kernel),
    # one group of 32 (k = 2 of 32 in one warp-wide group), one expert per group
    "experts_3_per_group": dict(base="main_b8_t2048", B=1, T=200, N=12, G=4, k=1),
    "one_group_of_32": dict(base="main_b8_t2048", B=1, T=200, N=32, G=1, k=2),
    "one_expert_per_group": dict(base="main_b8_t2048", B=1, T=200, N=8, G=8, k=1),
    # the largest routing shapes the ABI accepts: 64 experts, top-8 of 8 (every expert
    # active), top-3 of 8, and one group of 64 with top-2
    "n64_g8_k8": dict(base="main_b8_t2048", B=1, T=200, N=64, G=8, k=8),
    "n64_g8_k3": dict(base="main_b8_t2048", B=1, T=230, N=64, G=8, k=3),
    "n64_g1_k2": dict(base="main_b8_t2048", B=1, T=200, N=64, G=1, k=2),
    # fp32 handles at other head dims
    "f32_dh48_noncausal": dict(base="tiny_f32", B=2, T=150, d_h=48, causal=False),
    "f32_dh128": dict(base="tiny_f32", B=1, T=200, d_h=128),
}
# every bf16 head dim the ABI accepts, causal over three query tiles with a ragged tail
# and non-causal over two
for _dh in (16, 32, 48, 64, 80, 96, 112, 128):
    SMALL[f"dh{_dh}_causal"] = dict(base="main_b8_t2048", B=2, T=300, d_h=_dh)
    SMALL[f"dh{_dh}_noncausal"] = dict(base="main_b8_t2048", B=1, T=200, d_h=_dh,
                                       causal=False)
# head dims above 64 (one CTA per SM, 512 TMEM columns): more query tiles, a ragged last
# tile, weighted_concat
SMALL["dh128_long"] = dict(base="main_b8_t2048", B=2, T=1000, d_h=128)
SMALL["dh96_long_weighted"] = dict(base="main_b8_t2048", B=1, T=700, d_h=96,
                                   variant="weighted_concat")


@pytest.mark.parametrize("case", sorted(SMALL))
def test_small_full_oracle(case):
    spec = dict(SMALL[case])
    base = spec.pop("base")
    inp = W.generate(W.WORKLOADS[base].with_(**spec))
    run, *_ = _full_check(inp)
    run.close()


FULL = {
    "main_b8_t2048": {},
    "long_t16k": {},
    "wide_k2": {},
    "wide_k2_weighted": dict(variant="weighted_concat"),
    "wide_k2_hard": dict(variant="hard_concat"),
    "large_skew": {},
    "long_t64k": {},
    "long_t1m": {},
}
# host memory the oracle's float64 rows need at 1M tokens (x, K and V over every token)
HOST_BYTES = {"long_t1m": 40 << 30}


@pytest.mark.parametrize("case", list(FULL))
def test_full_size_sampled(case):
    if case in HOST_BYTES:
        import psutil
        if psutil.virtual_memory().available < HOST_BYTES[case]:
            pytest.skip("not enough host memory for the oracle's float64 rows")
    name = case if case in W.WORKLOADS else "wide_k2"
    inp = W.cached(name, **FULL[case]) if FULL[case] else W.cached(name)
    wl = inp.wl
    run = GpuRun(inp).forward()
    rows = sample_rows(wl)
    ref = oracle_rows(inp, rows)
    rt = ref["routing"]
    _check_routing(run, rt.sel, rt.counts)
    _check_aux(run, ref["aux"])
    y = to_host_f64(run.out)[rows]
    check_output(y, ref["y"], wl.dtype)
    # every output finite
    assert torch.isfinite(run.out.float()).all().item()
    if wl.skew is not None:
        share = rt.counts.reshape(wl.G, wl.E)[:, 0].sum() / (wl.M * wl.G)
        assert abs(share - wl.skew) <= 0.01
    run.close()


def test_deterministic_and_kv_independent_of_routing():
    import dataclasses
    base = W.WORKLOADS["wide_k2"].with_(B=1, T=333)
    inp = W.generate(base)
    a = GpuRun(inp).forward()
    y1 = a.out.clone()
    a.forward()
    assert torch.equal(y1, a.out), "two runs differ"
    K1 = a.tensor("K", (8, 333, 64), torch.bfloat16)
    V1 = a.tensor("V", (8, 333, 64), torch.bfloat16)
    for kw in (dict(variant="hard_concat"), dict(k=4)):
        # identical x and weights; only W_o takes the width of the other concatenation
        wl2 = base.with_(**kw)
        W_o = W.generate(wl2).W_o
        b = GpuRun(dataclasses.replace(inp, wl=wl2, W_o=W_o)).forward()
        assert torch.equal(K1, b.tensor("K", (8, 333, 64), torch.bfloat16))
        assert torch.equal(V1, b.tensor("V", (8, 333, 64), torch.bfloat16))
        b.close()
    a.close()


def test_error_paths_on_device():
    from moe_query_head_b200 import gqe as G
    inp = W.generate(W.WORKLOADS["main_b8_t2048"].with_(B=1, T=64))
    run = GpuRun(inp, max_tokens=64)
    d, wl = run.dev, inp.wl
    args = [d["x"], 2, 64, d["W_r"], d["W_q"], d["W_k"], d["W_v"], d["W_shared"], d["W_o"],
            wl.N, wl.G, wl.k, wl.d_h, 0, 1, run.out, run.aux]
    with pytest.raises(G.GQEError) as e:
        G.gqe_forward(run.h, *args)  # B*T = 128 > max_tokens
    assert e.value.status == G.GQE_ERR_WORKSPACE
    bad = list(args)
    bad[9] = 8  # N differs from the handle
    with pytest.raises(G.GQEError) as e:
        G.gqe_forward(run.h, *bad[:1], 1, *bad[2:])
    assert e.value.status == G.GQE_ERR_INVALID_ARG
    mis = torch.empty(64 * 768 + 1, dtype=torch.bfloat16, device="cuda")[1:]
    bad = list(args)
    bad[0], bad[1] = mis, 1
    with pytest.raises(G.GQEError) as e:
        G.gqe_forward(run.h, *bad)
    assert e.value.status == G.GQE_ERR_INVALID_ARG
    run.close()
