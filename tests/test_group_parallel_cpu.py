"""Host side of group-parallel execution (no GPU): the group ranges, the weight rows and Z /
W_o columns each rank takes, and that the ranks' shares of y, summed by an all-reduce over
world-size-2 gloo ranks, give the whole layer's y. Each rank's share is formed from the
float64 oracle's Z and W_o restricted to the rank's columns (what a rank's kernels compute
for its groups), so the test checks the partition, not the kernels."""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from moe_query_head_b200 import group_parallel as GP
from moe_query_head_b200 import workloads as W


@pytest.mark.parametrize("G,world", [(8, 1), (8, 2), (8, 3), (8, 8), (4, 3), (1, 1)])
def test_group_ranges_cover_every_group_once(G, world):
    r = GP.group_ranges(G, world)
    assert len(r) == world and r[0][0] == 0 and r[-1][1] == G
    sizes = [b - a for a, b in r]
    assert all(r[i][1] == r[i + 1][0] for i in range(world - 1))
    assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1


@pytest.mark.parametrize("variant", ["gqe", "weighted_concat", "hard_concat"])
@pytest.mark.parametrize("shared", [True, False])
def test_z_columns_partition(variant, shared):
    G, k, d_h = 8, 2, 4
    D_o = (G * k + (variant == "gqe") + shared) * d_h
    for world in (1, 2, 3, 8):
        cols = [GP.z_columns(G, k, d_h, variant, shared, a, b)
                for a, b in GP.group_ranges(G, world)]
        allc = np.concatenate(cols)
        slot = np.arange(G * k * d_h, (G * k + 1) * d_h) if variant == "gqe" else []
        # every column once, except the slot, which every rank holds
        u, n = np.unique(allc, return_counts=True)
        assert np.array_equal(u, np.arange(D_o))
        for c, m in zip(u, n):
            assert m == (world if c in set(np.asarray(slot).tolist()) else 1)


def _rank_share(rank, world, wl_name, ret):
    import oracle
    wl = W.WORKLOADS[wl_name].with_(B=1, T=64)
    inp = W.generate(wl)
    f = inp.f64
    layer = oracle.Layer(dim=wl.dim, N=wl.N, G=wl.G, k=wl.k, d_h=wl.d_h, shared=wl.shared,
                         variant=wl.variant, causal=wl.causal)
    res = oracle.forward(layer, f("x"), wl.B, wl.T, f("W_r"), f("W_q"), f("W_k"), f("W_v"),
                         f("W_shared"), f("W_o"))
    g0, g1 = GP.group_ranges(wl.G, world)[rank]
    cols = GP.z_columns(wl.G, wl.k, wl.d_h, wl.variant, wl.shared, g0, g1)
    w = GP.rank_weights(f("W_q"), f("W_k"), f("W_v"), f("W_shared"), f("W_o"), N=wl.N,
                        G=wl.G, k=wl.k, d_h=wl.d_h, variant=wl.variant, g0=g0, g1=g1)
    # the rank's slot share: its streams' part of sum w O (the weights are the layer's)
    Zr = res.Z[:, cols].copy()
    if wl.variant == "gqe":
        nr = (g1 - g0) * wl.k
        slot = np.zeros((wl.M, wl.d_h))
        for s in range(g0 * wl.k, g1 * wl.k):
            g, r = divmod(s, wl.k)
            slot += res.routing.w[:, g, r][:, None] * res.O[s]
        Zr[:, nr * wl.d_h:(nr + 1) * wl.d_h] = slot
    share = torch.from_numpy(Zr @ w["W_o"].T)
    dist.all_reduce(share)
    ret[rank] = float(np.abs(share.numpy() - res.y).max() / np.abs(res.y).max())


def _worker(rank, world, port, wl_name, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ret = {}
    _rank_share(rank, world, wl_name, ret)
    dist.destroy_process_group()
    q.put(ret[rank])


@pytest.mark.parametrize("wl_name", ["main_b8_t2048", "wide_k2"])
def test_shares_sum_to_the_layer_over_gloo(wl_name):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, world, port, wl_name, q)) for r in range(world)]
    for p in procs:
        p.start()
    errs = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert max(errs) < 1e-12, errs


@pytest.mark.parametrize("variant", ["gqe", "weighted_concat", "hard_concat"])
@pytest.mark.parametrize("shared", [True, False])
@pytest.mark.parametrize("world", [1, 2, 3])
def test_full_gradients_place_the_shares(variant, shared, world):
    """A rank's gradient shares come in the shapes of its weight slices; full_gradients puts
    them back at the rows and columns rank_weights took them from, zero elsewhere, so the
    sum over the ranks of the slices of a full array rebuilds it (W_o's slot columns once per
    rank: every rank holds a share of the slot's gradient)."""
    N, G, k, d_h, dim = 16, 8, 2, 4, 6
    E = N // G
    D_o = (G * k + (variant == "gqe") + shared) * d_h
    rng = np.random.default_rng(1)
    A = {"W_q": rng.standard_normal((N * d_h, dim)), "W_k": rng.standard_normal((G * d_h, dim)),
         "W_v": rng.standard_normal((G * d_h, dim)),
         "W_shared": rng.standard_normal((d_h, dim)) if shared else None,
         "W_o": rng.standard_normal((dim, D_o))}
    x = rng.standard_normal((5, dim))
    total = None
    for g0, g1 in GP.group_ranges(G, world):
        s = GP.rank_weights(A["W_q"], A["W_k"], A["W_v"], A["W_shared"], A["W_o"], N=N, G=G,
                            k=k, d_h=d_h, variant=variant, g0=g0, g1=g1)
        assert s["W_q"].shape == ((g1 - g0) * E * d_h, dim)
        s = dict(s, x=x, W_r=np.zeros((N, dim)))
        f = GP.full_gradients(s, N=N, G=G, k=k, d_h=d_h, variant=variant, shared=shared,
                              D_o=D_o, g0=g0, g1=g1)
        # zero outside the rank's rows
        mask = np.ones(N * d_h, bool)
        mask[g0 * E * d_h:g1 * E * d_h] = False
        assert not f["W_q"][mask].any()
        total = f if total is None else {n: (None if v is None else v + f[n])
                                         for n, v in total.items()}
    for n in ("W_q", "W_k", "W_v"):
        assert np.array_equal(total[n], A[n]), n
    if shared:
        assert np.array_equal(total["W_shared"], A["W_shared"])
    times = np.ones(D_o)
    if variant == "gqe":
        times[G * k * d_h:(G * k + 1) * d_h] = world
    assert np.allclose(total["W_o"], A["W_o"] * times[None, :])
    assert np.array_equal(total["x"], world * x)


def test_module_constructor_follows_the_readme():
    """GQEAttention's constructor (no GPU needed until the first call): head_dim defaults to
    dim // num_query_experts, the experts must split evenly over the KV heads, the weights
    have nn.Linear's [out, in] shapes."""
    from moe_query_head_b200.module import GQEAttention
    m = GQEAttention(768)
    assert (m.N, m.G, m.k, m.d_h, m.variant) == (16, 8, 1, 48, "gqe")
    assert tuple(m.W_q.shape) == (16 * 48, 768) and tuple(m.W_o.shape) == (768, 10 * 48)
    assert GQEAttention(768, variant="hard_concat", shared=False).W_o.shape[1] == 8 * 48
    with pytest.raises(ValueError):
        GQEAttention(768, num_query_experts=12, num_kv_heads=8)
    with pytest.raises(ValueError):
        GQEAttention(768, variant="sum")
