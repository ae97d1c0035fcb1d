"""The collectives of the group-parallel runner (moe_query_head_b200.group_parallel.GroupShard)
over world-size-2 gloo ranks on the CPU, with the library binding replaced by a stand-in
that fills each output with a value naming its rank and records what it was given.

Checked: forward_allreduce and decode_allreduce return the sum of the ranks' shares;
backward_allreduce runs phase 1 (gqe_backward_begin), all-reduces <dslot, slot> so that
phase 2 (gqe_backward_finish) of every rank sees the sum over the ranks, passes the aux
coefficient through, and returns gradients in the layer's shapes where every weight row or
W_o column holds the sum of the shares of the ranks that own it (the slot columns of W_o:
every rank; the shared head: the rank with group 0). The kernels are not involved: their
shares are checked against the oracle by the GPU tests."""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from moe_query_head_b200 import group_parallel as GP

DIM, N, G, K, D_H = 16, 4, 2, 1, 4
E = N // G
D_O = (G * K + 1 + 1) * D_H  # routed blocks, the gqe slot, the shared head
B, T = 1, 6


class FakeLib:
    """The calls GroupShard makes, on CPU tensors."""

    def __init__(self, rank):
        self.rank = rank
        self.calls = []

    def gqe_forward(self, h, x, B, T, W_r, W_q, W_k, W_v, W_s, W_o, N, G, k, d_h, variant,
                    causal, out, aux, stream=None):
        self.calls.append("forward")
        out.fill_(float(self.rank + 1))

    def gqe_decode(self, h, x, B, kc, vc, L_max, lengths, W_r, W_q, W_k, W_v, W_s, W_o, N, G,
                   k, d_h, variant, out, aux, stream=None):
        self.calls.append("decode")
        out.fill_(10.0 * (self.rank + 1))

    def gqe_backward_begin(self, h, x, B, T, W_r, W_q, W_k, W_v, W_s, W_o, N, G, k, d_h,
                           variant, causal, dy, slot_dot, stream=None):
        self.calls.append("begin")
        slot_dot.copy_(torch.arange(B * T, dtype=torch.float32) * (self.rank + 1))

    def gqe_backward_finish(self, h, x, B, T, W_r, W_q, W_k, W_v, W_s, W_o, N, G, k, d_h,
                            variant, causal, dy, aux_grad, slot_dot, dx, dW_r, dW_q, dW_k,
                            dW_v, dW_s, dW_o, stream=None):
        self.calls.append("finish")
        self.seen_slot_dot = slot_dot.clone()
        self.seen_aux = aux_grad
        for t in (dx, dW_r, dW_q, dW_k, dW_v, dW_s, dW_o):
            if t is not None:
                t.fill_(float(self.rank + 1))


def _shard(rank, world, weights):
    g0, g1 = GP.group_ranges(G, world)[rank]
    sh = object.__new__(GP.GroupShard)  # no handle: the stand-in needs none
    sh.GQ = FakeLib(rank)
    sh.dim, sh.N, sh.G, sh.k, sh.d_h = DIM, N, G, K, D_H
    sh.variant, sh.causal = "gqe", True
    sh.h = None
    sh.g0, sh.g1 = g0, g1
    sh.W_r = weights["W_r"]
    sh.w = GP.rank_weights(weights["W_q"], weights["W_k"], weights["W_v"], weights["W_shared"],
                           weights["W_o"], N=N, G=G, k=K, d_h=D_H, variant="gqe", g0=g0, g1=g1)
    sh.aux = torch.zeros(1)
    return sh


def _expected_gradients(world):
    """Each weight row or W_o column: the sum of (rank + 1) over the ranks that own it."""
    exp = {"x": np.zeros((B * T, DIM)), "W_r": np.zeros((N, DIM)),
           "W_q": np.zeros((N * D_H, DIM)), "W_k": np.zeros((G * D_H, DIM)),
           "W_v": np.zeros((G * D_H, DIM)), "W_shared": np.zeros((D_H, DIM)),
           "W_o": np.zeros((DIM, D_O))}
    for r, (g0, g1) in enumerate(GP.group_ranges(G, world)):
        v = r + 1.0
        exp["x"] += v
        exp["W_r"] += v
        exp["W_q"][g0 * E * D_H:g1 * E * D_H] += v
        exp["W_k"][g0 * D_H:g1 * D_H] += v
        exp["W_v"][g0 * D_H:g1 * D_H] += v
        if g0 == 0:
            exp["W_shared"] += v
        exp["W_o"][:, GP.z_columns(G, K, D_H, "gqe", True, g0, g1)] += v
    return exp


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        gen = torch.Generator().manual_seed(7)
        weights = {"W_r": torch.randn(N, DIM, generator=gen),
                   "W_q": torch.randn(N * D_H, DIM, generator=gen),
                   "W_k": torch.randn(G * D_H, DIM, generator=gen),
                   "W_v": torch.randn(G * D_H, DIM, generator=gen),
                   "W_shared": torch.randn(D_H, DIM, generator=gen),
                   "W_o": torch.randn(DIM, D_O, generator=gen)}
        sh = _shard(rank, world, weights)
        x = torch.zeros(B * T, DIM)
        out = torch.empty(B * T, DIM)
        sh.forward_allreduce(x, B, T, out, dist)
        fwd = out.clone()
        sh.decode_allreduce(x[:B], B, None, None, 8, None, out[:B], dist)
        dec = out[:B].clone()
        g = sh.backward_allreduce(x, B, T, torch.zeros(B * T, DIM), 0.01, dist, D_o=D_O,
                                  shared=True)
        res = {"fwd": fwd.numpy(), "dec": dec.numpy(), "calls": list(sh.GQ.calls),
               "slot_dot": sh.GQ.seen_slot_dot.numpy(), "aux": sh.GQ.seen_aux,
               "grads": {k: (None if v is None else v.numpy()) for k, v in g.items()}}
        q.put((rank, res))
    finally:
        dist.destroy_process_group()


def test_group_shard_collectives_over_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29600 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=240) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    total = float(sum(r + 1 for r in range(world)))
    exp = _expected_gradients(world)
    for rank in range(world):
        res = got[rank]
        assert res["calls"] == ["forward", "decode", "begin", "finish"]
        assert np.all(res["fwd"] == total)
        assert np.all(res["dec"] == 10.0 * total)
        # phase 2 sees <dslot, slot> summed over the ranks, and the aux coefficient
        np.testing.assert_array_equal(res["slot_dot"], np.arange(B * T) * total)
        assert res["aux"] == pytest.approx(0.01)
        for name, e in exp.items():
            np.testing.assert_array_equal(res["grads"][name], e, err_msg=name)
