"""A PyTorch module over the C ABI with the interface of the "GQE: Grouped Query Experts"
README (Usage, Parameters): ``GQEAttention(dim, num_query_experts=16, num_kv_heads=8,
top_k=1, head_dim=None, variant="gqe")``, ``y = attn(x)`` and ``collect_aux_loss(model)``, the
layer trained with ``loss.backward()`` after adding 0.01 times the aux loss to the task loss.

The module owns its weights as float32 parameters in nn.Linear layout ([out, in], no
biases): W_r [N, dim], W_q [N d_h, dim], W_k, W_v [G d_h, dim], W_shared [d_h, dim] and W_o
[dim, D_o]. Each call casts them and the input to bf16 and runs gqe_forward; the backward
runs gqe_backward (the whole layer's gradients in float32). This file only marshals
arguments: every step of the layer runs in the library's kernels.

The library keeps one layer's forward state per handle. A backward whose forward is no longer
the handle's last (another call of the same module in between) runs that forward again
before gqe_backward. Reading the aux loss's gradient coefficient synchronises the stream.
"""
from __future__ import annotations

import math

import torch
from torch import nn

from . import gqe as G


class _GQEFunction(torch.autograd.Function):
    """y, aux = the layer of `mod` on x; backward through gqe_backward."""

    @staticmethod
    def forward(ctx, x, W_r, W_q, W_k, W_v, W_shared, W_o, mod):
        B, T, dim = x.shape
        bf = torch.bfloat16
        xb = x.reshape(B * T, dim).to(bf).contiguous()
        w = [W.detach().to(bf).contiguous() for W in (W_r, W_q, W_k, W_v)]
        ws = W_shared.detach().to(bf).contiguous() if W_shared is not None else None
        wo = W_o.detach().to(bf).contiguous()
        h = mod._handle_for(B * T)
        out = torch.empty((B * T, dim), dtype=bf, device=x.device)
        aux = torch.zeros(1, dtype=torch.float32, device=x.device)
        mod._forward_call(h, xb, B, T, w, ws, wo, out, aux)
        ctx.mod, ctx.B, ctx.T, ctx.call = mod, B, T, mod._calls
        ctx.has_shared = ws is not None
        ctx.x_dtype = x.dtype
        ctx.save_for_backward(xb, *w, wo, *([ws] if ws is not None else []))
        return out.view(B, T, dim), aux[0]

    @staticmethod
    def backward(ctx, dy, daux):
        mod, B, T = ctx.mod, ctx.B, ctx.T
        saved = ctx.saved_tensors
        xb, W_r, W_q, W_k, W_v, W_o = saved[:6]
        W_s = saved[6] if ctx.has_shared else None
        h = mod._h
        if mod._calls != ctx.call:
            # another forward ran on the handle since: restore this call's state
            out = torch.empty((B * T, mod.dim), dtype=torch.bfloat16, device=xb.device)
            aux = torch.zeros(1, dtype=torch.float32, device=xb.device)
            mod._forward_call(h, xb, B, T, [W_r, W_q, W_k, W_v], W_s, W_o, out, aux)
            ctx.call = mod._calls
        G.gqe_enable_backward(h)
        aux_grad = 0.0 if daux is None else float(daux)
        if dy is None:
            dy = torch.zeros((B, T, mod.dim), dtype=torch.bfloat16, device=xb.device)
        dyb = dy.reshape(B * T, mod.dim).to(torch.bfloat16).contiguous()
        f32 = lambda *s: torch.empty(s, dtype=torch.float32, device=xb.device)  # noqa: E731
        g = [f32(B * T, mod.dim), f32(*W_r.shape), f32(*W_q.shape), f32(*W_k.shape),
             f32(*W_v.shape), f32(*W_s.shape) if W_s is not None else None, f32(*W_o.shape)]
        G.gqe_backward(h, xb, B, T, W_r, W_q, W_k, W_v, W_s, W_o, mod.N, mod.G, mod.k, mod.d_h,
                       G.VARIANTS[mod.variant], int(mod.causal), dyb, aux_grad, *g)
        dx = g[0].view(B, T, mod.dim).to(ctx.x_dtype)
        return dx, g[1], g[2], g[3], g[4], g[5], g[6], None


class GQEAttention(nn.Module):
    """GQE attention ("GQE: Grouped Query Experts" README, Parameters): N query-head experts in
    G groups (num_kv_heads, one dense KV head each), the top k of each group per token plus
    the always-on shared head, output construction `variant` ("gqe", "weighted_concat",
    "hard_concat"); head_dim defaults to dim // num_query_experts. Input [B, T, dim], output
    [B, T, dim] in bf16; causal unless causal=False."""

    def __init__(self, dim: int, num_query_experts: int = 16, num_kv_heads: int = 8,
                 top_k: int = 1, head_dim: int | None = None, variant: str = "gqe",
                 shared: bool = True, causal: bool = True):
        super().__init__()
        if num_query_experts % num_kv_heads != 0:
            raise ValueError("num_query_experts must be divisible by num_kv_heads")
        if variant not in G.VARIANTS:
            raise ValueError(f"variant must be one of {sorted(G.VARIANTS)}")
        self.dim, self.N, self.G, self.k = dim, num_query_experts, num_kv_heads, top_k
        self.d_h = head_dim if head_dim is not None else dim // num_query_experts
        self.variant, self.shared, self.causal = variant, shared, causal
        d, dh = dim, self.d_h
        self.W_r = nn.Parameter(torch.empty(self.N, d))
        self.W_q = nn.Parameter(torch.empty(self.N * dh, d))
        self.W_k = nn.Parameter(torch.empty(self.G * dh, d))
        self.W_v = nn.Parameter(torch.empty(self.G * dh, d))
        self.W_shared = nn.Parameter(torch.empty(dh, d)) if shared else None
        self.W_o = nn.Parameter(torch.empty(d, self.D_o))
        for p in self.parameters():  # nn.Linear's default: U(-1/sqrt(in), 1/sqrt(in))
            bound = 1.0 / math.sqrt(p.shape[1])
            nn.init.uniform_(p, -bound, bound)
        self._h = None
        self._max_tokens = 0
        self._device = None
        self._calls = 0
        self._aux = None

    @property
    def D_o(self) -> int:
        return (self.G * self.k + (self.variant == "gqe") + self.shared) * self.d_h

    def _handle_for(self, M: int):
        dev = torch.cuda.current_device()
        if self._h is None or M > self._max_tokens or dev != self._device:
            self._release()
            self._h = G.gqe_create(self.dim, self.N, self.G, self.k, self.d_h, G.GQE_BF16, M)
            self._max_tokens, self._device = M, dev
        return self._h

    def _forward_call(self, h, xb, B, T, w, ws, wo, out, aux):
        G.gqe_forward(h, xb, B, T, w[0], w[1], w[2], w[3], ws, wo, self.N, self.G, self.k,
                      self.d_h, G.VARIANTS[self.variant], int(self.causal), out, aux)
        self._calls += 1

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        if x.dim() != 3 or x.shape[2] != self.dim:
            raise ValueError(f"expected input [B, T, {self.dim}]")
        y, aux = _GQEFunction.apply(x, self.W_r, self.W_q, self.W_k, self.W_v, self.W_shared,
                                    self.W_o, self)
        self._aux = aux
        return y

    def allocate_cache(self, B: int, L_max: int, device=None):
        """Empty KV caches for generation: k_cache, v_cache [G, B, L_max, d_h] in bf16."""
        shape = (self.G, B, L_max, self.d_h)
        dev = device if device is not None else self.W_r.device
        return (torch.zeros(shape, dtype=torch.bfloat16, device=dev),
                torch.zeros(shape, dtype=torch.bfloat16, device=dev))

    @torch.no_grad()
    def decode_step(self, x_new: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                    lengths: torch.Tensor) -> torch.Tensor:
        """One generation step (gqe_decode): x_new [B, dim], one new token per sequence at
        position lengths[b] (int32, on the device); its K / V are written into the caches at
        that row and y_new [B, dim] (bf16) is returned. The caller advances `lengths`."""
        B = x_new.shape[0]
        bf = torch.bfloat16
        h = self._handle_for(B)
        w = [W.to(bf).contiguous() for W in (self.W_r, self.W_q, self.W_k, self.W_v)]
        ws = self.W_shared.to(bf).contiguous() if self.W_shared is not None else None
        out = torch.empty((B, self.dim), dtype=bf, device=x_new.device)
        aux = torch.zeros(1, dtype=torch.float32, device=x_new.device)
        G.gqe_decode(h, x_new.to(bf).contiguous(), B, k_cache, v_cache, k_cache.shape[2],
                     lengths, w[0], w[1], w[2], w[3], ws, self.W_o.to(bf).contiguous(), self.N,
                     self.G, self.k, self.d_h, G.VARIANTS[self.variant], out, aux)
        self._calls += 1  # the handle's saved state is no longer a forward's
        return out

    def aux_loss(self) -> torch.Tensor | None:
        """The Switch load-balancing loss of the last call (a differentiable scalar)."""
        return self._aux

    def _release(self):
        if self._h is not None:
            G.gqe_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self._release()
        except Exception:
            pass


def collect_aux_loss(model: nn.Module) -> torch.Tensor:
    """The sum of the aux losses of the last calls of every GQEAttention in `model` (the
    README's collect_aux_loss; the caller applies its coefficient, 0.01 in the README)."""
    total = None
    for m in model.modules():
        if isinstance(m, GQEAttention) and m._aux is not None:
            total = m._aux if total is None else total + m._aux
    if total is None:
        p = next(model.parameters(), None)
        return torch.zeros((), device=p.device if p is not None else None)
    return total
