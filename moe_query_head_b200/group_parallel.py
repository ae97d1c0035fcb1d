"""Group-parallel execution of one GQE layer over several GPUs (one process per GPU).

Routing is per group ("GQE: Grouped Query Experts" README, Algorithm Overview: a softmax
over the experts of each group, then top-k), and each group has its own dense KV head, so
the layer splits by groups: rank r computes groups [g0, g1) (its KV heads, its experts'
query heads, their attention and their share of the output projection) and the layer's
output is the sum of the ranks' shares: one all-reduce (or reduce-scatter) of y. Every rank
routes every group (the router is N x dim, tiny), so the renormalised slot weights, which
divide by the selected probabilities of all groups, and the load-balancing loss are the
whole layer's on every rank with no exchange. The shared head reads KV head 0 and runs on
the rank that holds group 0.

Training splits the same way. Each rank's backward is local to its groups except for one
number per token: the gqe slot weights divide by the selected probabilities of all groups
(gist.science summary, Output Construction), so the router gradient needs <dslot, slot>
summed over every routed stream. gqe_backward_begin writes the rank's share of it, the
ranks all-reduce those B*T floats, and gqe_backward_finish forms the rank's gradient shares;
the layer's gradients are their sums (full_gradients places a rank's shares in the layer's
shapes).

This module holds the host-side plan (which groups, which weight rows and columns each rank
takes) and a runner that calls the C ABI's gqe_set_group_range / gqe_forward /
gqe_backward_begin / gqe_backward_finish and sums with torch.distributed (NCCL on GPUs).
"""
from __future__ import annotations

import numpy as np


def group_ranges(G: int, world: int) -> list[tuple[int, int]]:
    """Contiguous group ranges, one per rank, sizes differing by at most one (the first
    G % world ranks take one more). Needs 1 <= world <= G."""
    if not 1 <= world <= G:
        raise ValueError("need 1 <= world <= G")
    base, extra = divmod(G, world)
    out, g = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((g, g + n))
        g += n
    return out


def z_columns(G: int, k: int, d_h: int, variant: str, shared: bool, g0: int, g1: int) -> np.ndarray:
    """Columns of the layer's Z (and of W_o) that the range [g0, g1) produces, in the order
    of its own Z: its routed streams (g*k + r for g in the range), the slot (variant gqe:
    every rank adds its streams' share of the one slot), the shared block (the rank with
    g0 == 0)."""
    blocks = list(range(g0 * k, g1 * k))
    nxt = G * k
    if variant == "gqe":
        blocks.append(nxt)
        nxt += 1
    if shared and g0 == 0:
        blocks.append(nxt)
    return np.concatenate([np.arange(b * d_h, (b + 1) * d_h) for b in blocks])


def rank_weights(W_q, W_k, W_v, W_shared, W_o, *, N: int, G: int, k: int, d_h: int,
                 variant: str, g0: int, g1: int) -> dict:
    """The weights a rank passes to gqe_forward after gqe_set_group_range(g0, g1): W_q rows
    of its experts, W_k / W_v rows of its heads, W_shared on the rank with group 0 only, the
    W_o columns of its Z blocks. Works on numpy arrays and torch tensors (contiguous copies)."""
    E = N // G
    cols = z_columns(G, k, d_h, variant, W_shared is not None, g0, g1)

    def rows(a, lo, hi):
        r = a[lo:hi]
        return r.contiguous() if hasattr(r, "contiguous") else np.ascontiguousarray(r)

    if hasattr(W_o, "index_select"):
        import torch
        Wo = W_o.index_select(1, torch.as_tensor(cols, device=W_o.device)).contiguous()
    else:
        Wo = np.ascontiguousarray(W_o[:, cols])
    return {
        "W_q": rows(W_q, g0 * E * d_h, g1 * E * d_h),
        "W_k": rows(W_k, g0 * d_h, g1 * d_h),
        "W_v": rows(W_v, g0 * d_h, g1 * d_h),
        "W_shared": W_shared if g0 == 0 else None,
        "W_o": Wo,
    }


def rank_caches(k_cache, v_cache, g0: int, g1: int):
    """The KV caches [G, B, L_max, d_h] of groups g0 .. g1-1: a rank's own caches for the
    decode step (contiguous copies; the rank keeps them and its steps append to them)."""
    def part(c):
        r = c[g0:g1]
        return r.contiguous() if hasattr(r, "contiguous") else np.ascontiguousarray(r)
    return part(k_cache), part(v_cache)


def full_gradients(shares: dict, *, N: int, G: int, k: int, d_h: int, variant: str,
                   shared: bool, D_o: int, g0: int, g1: int) -> dict:
    """A rank's gradient shares (the shapes of its weight slices, as rank_weights gives them)
    placed in the layer's shapes, zero outside the rank's rows and columns: the layer's
    gradients are the sums of these over the ranks. dx and dW_r are already full-size
    (dW_r is zero outside the rank's experts); W_o's slot columns hold the rank's share of
    the slot's gradient. Works on numpy arrays and torch tensors."""
    E = N // G
    dq, dk, dv, do = shares["W_q"], shares["W_k"], shares["W_v"], shares["W_o"]
    dim = dq.shape[1]
    is_torch = hasattr(dq, "new_zeros")

    def zeros(*shape):
        return dq.new_zeros(shape) if is_torch else np.zeros(shape, dtype=dq.dtype)

    out = {"x": shares["x"], "W_r": shares["W_r"]}
    out["W_q"] = zeros(N * d_h, dim)
    out["W_q"][g0 * E * d_h:g1 * E * d_h] = dq
    out["W_k"] = zeros(G * d_h, dim)
    out["W_k"][g0 * d_h:g1 * d_h] = dk
    out["W_v"] = zeros(G * d_h, dim)
    out["W_v"][g0 * d_h:g1 * d_h] = dv
    out["W_shared"] = None
    if shared:
        out["W_shared"] = shares["W_shared"] if g0 == 0 else zeros(d_h, dim)
    cols = z_columns(G, k, d_h, variant, shared, g0, g1)
    out["W_o"] = zeros(do.shape[0], D_o)
    if is_torch:
        import torch
        out["W_o"][:, torch.as_tensor(cols, device=do.device)] = do
    else:
        out["W_o"][:, cols] = do
    return out


class GroupShard:
    """One rank's share of a GQE layer on the current CUDA device: a handle restricted to
    groups [g0, g1) and the rank's weight slices. forward() returns the rank's share of y;
    forward_allreduce() sums the shares over the process group."""

    def __init__(self, *, dim, N, G, k, d_h, variant, causal, max_tokens, g0, g1, W_r, W_q,
                 W_k, W_v, W_shared, W_o):
        import torch
        from . import gqe as GQ
        self.GQ = GQ
        self.dim, self.N, self.G, self.k, self.d_h = dim, N, G, k, d_h
        self.variant, self.causal = variant, causal
        self.h = GQ.gqe_create(dim, N, G, k, d_h, GQ.GQE_BF16, max_tokens)
        GQ.gqe_set_group_range(self.h, g0, g1)
        self.g0, self.g1 = g0, g1
        self.W_r = W_r
        self.w = rank_weights(W_q, W_k, W_v, W_shared, W_o, N=N, G=G, k=k, d_h=d_h,
                              variant=variant, g0=g0, g1=g1)
        self.aux = torch.zeros(1, dtype=torch.float32, device="cuda")

    def forward(self, x, B, T, out, stream=None):
        from .workloads import VARIANT_IDS
        w = self.w
        self.GQ.gqe_forward(self.h, x, B, T, self.W_r, w["W_q"], w["W_k"], w["W_v"],
                            w["W_shared"], w["W_o"], self.N, self.G, self.k, self.d_h,
                            VARIANT_IDS[self.variant], int(self.causal), out, self.aux, stream)
        return out

    def forward_allreduce(self, x, B, T, out, dist, group=None):
        self.forward(x, B, T, out)
        dist.all_reduce(out, group=group)
        return out

    def decode(self, x, B, k_cache, v_cache, L_max, lengths, out, stream=None):
        """One decode step on this rank's groups: k_cache / v_cache hold its heads only,
        [(g1-g0), B, L_max, d_h] (rank_caches of the layer's caches); `out` receives the
        rank's share of the new tokens' y, and the new K / V are written into its caches."""
        from .workloads import VARIANT_IDS
        w = self.w
        self.GQ.gqe_decode(self.h, x, B, k_cache, v_cache, L_max, lengths, self.W_r, w["W_q"],
                           w["W_k"], w["W_v"], w["W_shared"], w["W_o"], self.N, self.G, self.k,
                           self.d_h, VARIANT_IDS[self.variant], out, self.aux, stream)
        return out

    def decode_allreduce(self, x, B, k_cache, v_cache, L_max, lengths, out, dist, group=None):
        self.decode(x, B, k_cache, v_cache, L_max, lengths, out)
        dist.all_reduce(out, group=group)
        return out

    def enable_backward(self):
        self.GQ.gqe_enable_backward(self.h)

    def backward_begin(self, x, B, T, dy, slot_dot, stream=None):
        """Phase 1 of this rank's backward of its last forward: writes the rank's share of
        <dslot, slot> per token into slot_dot (float32 [B*T], device)."""
        from .workloads import VARIANT_IDS
        w = self.w
        self.GQ.gqe_backward_begin(self.h, x, B, T, self.W_r, w["W_q"], w["W_k"], w["W_v"],
                                   w["W_shared"], w["W_o"], self.N, self.G, self.k, self.d_h,
                                   VARIANT_IDS[self.variant], int(self.causal), dy, slot_dot,
                                   stream)

    def backward_finish(self, x, B, T, dy, aux_grad, slot_dot, stream=None) -> dict:
        """Phase 2, given <dslot, slot> summed over the ranks: this rank's gradient shares
        (float32 device tensors in the shapes of its weight slices)."""
        import torch
        from .workloads import VARIANT_IDS
        w = self.w
        f32 = lambda *s: torch.empty(s, dtype=torch.float32, device=x.device)  # noqa: E731
        g = {"x": f32(B * T, self.dim), "W_r": f32(self.N, self.dim),
             "W_q": f32(*w["W_q"].shape), "W_k": f32(*w["W_k"].shape),
             "W_v": f32(*w["W_v"].shape),
             "W_shared": None if w["W_shared"] is None else f32(*w["W_shared"].shape),
             "W_o": f32(*w["W_o"].shape)}
        self.GQ.gqe_backward_finish(self.h, x, B, T, self.W_r, w["W_q"], w["W_k"], w["W_v"],
                                    w["W_shared"], w["W_o"], self.N, self.G, self.k, self.d_h,
                                    VARIANT_IDS[self.variant], int(self.causal), dy, aux_grad,
                                    slot_dot, g["x"], g["W_r"], g["W_q"], g["W_k"], g["W_v"],
                                    g["W_shared"], g["W_o"], stream)
        return g

    def backward_allreduce(self, x, B, T, dy, aux_grad, dist, *, D_o, shared, group=None):
        """The layer's gradients on every rank: begin, an all-reduce of <dslot, slot>,
        finish, then an all-reduce of each gradient placed in the layer's shapes."""
        import torch
        slot_dot = torch.empty(B * T, dtype=torch.float32, device=x.device)
        self.backward_begin(x, B, T, dy, slot_dot)
        dist.all_reduce(slot_dot, group=group)
        g = full_gradients(self.backward_finish(x, B, T, dy, aux_grad, slot_dot), N=self.N,
                           G=self.G, k=self.k, d_h=self.d_h, variant=self.variant,
                           shared=shared, D_o=D_o, g0=self.g0, g1=self.g1)
        for t in g.values():
            if t is not None:
                dist.all_reduce(t, group=group)
        return g

    def close(self):
        if self.h:
            self.GQ.gqe_destroy(self.h)
            self.h = None
