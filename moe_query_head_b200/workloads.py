"""Seeded synthetic workloads for the GQE attention forward pass.

This module only draws inputs; it computes none of the layer's outputs. Both the CUDA
path's tests/bench and the CPU oracle's tests take their inputs from here, as the exact
same bits (bf16 workloads are rounded once, here, and the oracle receives the rounded
values upcast to float64).

Three input-conditioning steps look at router logits (plain dot products x . W_r[e]):
  * the margin filter redraws token rows whose gap between the k-th and (k+1)-th logit
    of some group is below the margin, so that the top-k decision is the same in any
    precision;
  * the balance check redraws W_r until every expert's load is near uniform;
  * the skew calibration picks the router weight that sends a target share of tokens
    to expert 0 of each group.
They only shape the input distribution. An error in them could make routing ties more
likely or the skew inexact; it cannot make a wrong kernel agree with the oracle.

The paper's workloads (FineWeb-Edu text through a trained 250M-parameter model) are not
available; these tensors take only the layer shapes of the paper's main setting
("GQE: Grouped Query Experts" README, Parameters) and the sizes of the benchmark configs.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from functools import lru_cache

import numpy as np

VARIANT_IDS = {"gqe": 0, "weighted_concat": 1, "hard_concat": 2}


@dataclass(frozen=True)
class Workload:
    name: str
    dim: int
    N: int
    G: int
    k: int
    d_h: int
    B: int
    T: int
    dtype: str = "bf16"          # "bf16" or "f32"
    shared: bool = True
    variant: str = "gqe"
    causal: bool = True
    seed: int = 0
    w_std: float | None = 0.02   # None: N(0, 1/dim) for W_r, W_q, W_k, W_v, W_shared
    margin: float | None = 1e-3  # top-k logit gap enforced by redrawing rows of x
    balance: float | None = None  # max relative deviation of expert loads from uniform
    skew: float | None = None    # target share of tokens routed to expert 0 of each group

    @property
    def E(self) -> int:
        return self.N // self.G

    @property
    def M(self) -> int:
        return self.B * self.T

    @property
    def n_streams(self) -> int:
        return self.G * self.k + (1 if self.shared else 0)

    @property
    def D_o(self) -> int:
        return (self.G * self.k + (1 if self.variant == "gqe" else 0)
                + (1 if self.shared else 0)) * self.d_h

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    def all_active(self) -> "Workload":
        """The same layer with every expert active (k = E): the in-run GQA comparator."""
        return replace(self, k=self.E, name=self.name + "_kE")

    def active_flops(self) -> float:
        """FLOPs (2 per multiply-add) the method must compute, not the work it skips:
        router, K/V (+shared) projection, routed Q projection, attention, W_o."""
        M, d, h = self.M, self.dim, self.d_h
        S = self.n_streams
        f = 2.0 * M * d * self.N
        f += 2.0 * M * d * (2 * self.G + (1 if self.shared else 0)) * h
        f += 2.0 * M * d * h * self.G * self.k
        if self.causal:
            f += 2.0 * self.B * h * self.T * (self.T + 1) * S
        else:
            f += 4.0 * self.B * h * self.T * self.T * S
        f += 2.0 * M * self.D_o * d
        return f


WORKLOADS = {
    # Tiny fp32 check. W_o ~ N(0, 1/(heads * d_h)) with heads = D_o / d_h = 4.
    "tiny_f32": Workload("tiny_f32", dim=64, N=4, G=2, k=1, d_h=16, B=1, T=128,
                         dtype="f32", seed=0, w_std=None),
    # The paper's main layer setting (N=16, G=8, k=1, d_h = 768/16).
    "main_b8_t2048": Workload("main_b8_t2048", dim=768, N=16, G=8, k=1, d_h=48, B=8,
                              T=2048, seed=2),
    # Long-context prefill, near-uniform expert loads.
    "long_t16k": Workload("long_t16k", dim=768, N=16, G=8, k=1, d_h=48, B=1, T=16384,
                          seed=3, balance=0.10),
    # Wider groups: E = 4 per group, k = 2.
    "wide_k2": Workload("wide_k2", dim=2048, N=32, G=8, k=2, d_h=64, B=2, T=8192, seed=4),
    # Contexts beyond 32K: the long-context layer at 64K and 128K tokens (the pages quote the
    # prefill speedup from 4K up to 1024K tokens).
    "long_t64k": Workload("long_t64k", dim=768, N=16, G=8, k=1, d_h=48, B=1, T=65536, seed=6),
    "long_t128k": Workload("long_t128k", dim=768, N=16, G=8, k=1, d_h=48, B=1, T=131072,
                           seed=7),
    "long_t1m": Workload("long_t1m", dim=768, N=16, G=8, k=1, d_h=48, B=1, T=1048576,
                         seed=8),
    # Large and skewed: 70% of tokens to expert 0 of each group.
    "large_skew": Workload("large_skew", dim=4096, N=32, G=8, k=1, d_h=128, B=1, T=32768,
                           seed=5, skew=0.70),
}


# ----------------------------------------------------------------------------------------
# bf16 rounding (round to nearest even), done once on the host.
# ----------------------------------------------------------------------------------------

def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even. No NaNs expected."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def quantize(a: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values to the workload dtype; returns float32 values exactly
    representable in that dtype (bf16 values are held in float32 containers)."""
    a32 = np.asarray(a, dtype=np.float32)
    if dtype == "f32":
        return a32
    return bf16_bits_to_f32(f32_to_bf16_bits(a32))


# ----------------------------------------------------------------------------------------
# Input conditioning (see module docstring).
# ----------------------------------------------------------------------------------------

def _topk_gaps(x: np.ndarray, W_r: np.ndarray, G: int, k: int) -> np.ndarray:
    """Per row, the smallest over groups of (k-th largest - (k+1)-th largest) logit."""
    M = x.shape[0]
    E = W_r.shape[0] // G
    if k >= E:
        return np.full(M, np.inf)
    lg = (x.astype(np.float64) @ W_r.astype(np.float64).T).reshape(M, G, E)
    s = -np.sort(-lg, axis=2)
    return (s[:, :, k - 1] - s[:, :, k]).min(axis=1)


def _expert0_share(x: np.ndarray, W_r: np.ndarray, G: int) -> float:
    M = x.shape[0]
    E = W_r.shape[0] // G
    lg = (x.astype(np.float64) @ W_r.astype(np.float64).T).reshape(M, G, E)
    return float((np.argmax(lg, axis=2) == 0).mean())


def _loads(x: np.ndarray, W_r: np.ndarray, G: int, k: int) -> np.ndarray:
    """Tokens per expert under top-k of the logits (lowest index first on ties)."""
    M = x.shape[0]
    E = W_r.shape[0] // G
    lg = (x.astype(np.float64) @ W_r.astype(np.float64).T).reshape(M, G, E)
    order = np.argsort(-lg, axis=2, kind="stable")[:, :, :k]
    return np.stack([np.bincount(order[:, g].ravel(), minlength=E) for g in range(G)]).ravel()


@dataclass
class Inputs:
    """One workload's tensors. Float32 containers hold values exact in `wl.dtype`."""

    wl: Workload
    x: np.ndarray
    W_r: np.ndarray
    W_q: np.ndarray
    W_k: np.ndarray
    W_v: np.ndarray
    W_shared: np.ndarray | None
    W_o: np.ndarray
    report: dict

    def f64(self, name: str) -> np.ndarray | None:
        a = getattr(self, name)
        return None if a is None else a.astype(np.float64)

    def raw(self, name: str) -> np.ndarray | None:
        """The tensor as the device receives it: uint16 bf16 bits or float32."""
        a = getattr(self, name)
        if a is None:
            return None
        return f32_to_bf16_bits(a) if self.wl.dtype == "bf16" else a


def generate(wl: Workload) -> Inputs:
    """Draw the workload's tensors from PCG64(seed): x, W_r, W_q, W_k, W_v, W_shared,
    W_o in that order (W_o last, so every other tensor is the same across variants and
    across k)."""
    rng = np.random.Generator(np.random.PCG64(wl.seed))
    M, d, N, G, k, h = wl.M, wl.dim, wl.N, wl.G, wl.k, wl.d_h
    std = wl.w_std if wl.w_std is not None else (1.0 / d) ** 0.5
    q = lambda a: quantize(a, wl.dtype)  # noqa: E731
    x = q(rng.standard_normal((M, d)))
    W_r = q(rng.standard_normal((N, d)) * std)
    W_q = q(rng.standard_normal((N * h, d)) * std)
    W_k = q(rng.standard_normal((G * h, d)) * std)
    W_v = q(rng.standard_normal((G * h, d)) * std)
    W_s = q(rng.standard_normal((h, d)) * std)
    ostd = wl.w_std if wl.w_std is not None else (1.0 / wl.D_o) ** 0.5
    W_o = q(rng.standard_normal((d, wl.D_o)) * ostd)
    report: dict = {}

    if wl.skew is not None:
        # Constant last feature and a router weight beta on it for expert 0 of each group.
        x[:, d - 1] = 1.0
        base = W_r.copy()
        base[np.arange(G) * wl.E, d - 1] = 0.0
        lo, hi = 0.0, 32.0
        for _ in range(40):
            mid = 0.5 * (lo + hi)
            Wt = base.copy()
            Wt[np.arange(G) * wl.E, d - 1] = q(np.array([mid]))[0]
            if _expert0_share(x, Wt, G) < wl.skew:
                lo = mid
            else:
                hi = mid
        beta = float(q(np.array([0.5 * (lo + hi)]))[0])
        W_r = base
        W_r[np.arange(G) * wl.E, d - 1] = beta
        report["beta"] = beta

    if wl.balance is not None:
        for i in range(1, 50):
            loads = _loads(x, W_r, G, k)
            target = M * k / wl.E
            if np.abs(loads / target - 1).max() <= wl.balance:
                break
            r2 = np.random.Generator(np.random.PCG64(wl.seed + 100 * i))
            W_r = q(r2.standard_normal((N, d)) * std)
            report["router_redraws"] = i

    if wl.margin is not None:
        r2 = np.random.Generator(np.random.PCG64([wl.seed, 1]))
        redrawn = 0
        for _ in range(100):
            bad = np.nonzero(_topk_gaps(x, W_r, G, k) < wl.margin)[0]
            if bad.size == 0:
                break
            redrawn += bad.size
            x[bad] = q(r2.standard_normal((bad.size, d)))
            if wl.skew is not None:
                x[bad, d - 1] = 1.0
        else:
            raise RuntimeError("margin filter did not converge")
        report["rows_redrawn"] = redrawn

    if wl.skew is not None:
        report["expert0_share"] = _expert0_share(x, W_r, G)
    return Inputs(wl, x, W_r, W_q, W_k, W_v, W_s if wl.shared else None, W_o, report)


def router_logits_input(M: int, N: int, G: int, k: int, seed: int,
                        margin: float = 1e-3) -> np.ndarray:
    """Router logits [M, N] as float32, N(0, 1) from PCG64([seed, 3]), for the entry point
    that routes precomputed logits. Rows whose gap between the k-th and (k+1)-th largest
    logit of some group is below `margin` are redrawn, as the margin filter above does for
    x, so that the top-k decision is the same in any precision."""
    rng = np.random.Generator(np.random.PCG64([seed, 3]))
    lg = rng.standard_normal((M, N)).astype(np.float32)
    E = N // G
    if k >= E:
        return lg
    for _ in range(100):
        s = -np.sort(-lg.astype(np.float64).reshape(M, G, E), axis=2)
        bad = np.nonzero((s[:, :, k - 1] - s[:, :, k]).min(axis=1) < margin)[0]
        if bad.size == 0:
            return lg
        lg[bad] = rng.standard_normal((bad.size, N)).astype(np.float32)
    raise RuntimeError("margin filter did not converge")


def grad_output(wl: Workload, seed_offset: int = 0) -> np.ndarray:
    """An upstream gradient dy [M, dim] for the backward pass: N(0, 1) from
    PCG64([seed, 4 + seed_offset]), rounded to the workload's dtype."""
    rng = np.random.Generator(np.random.PCG64([wl.seed, 4 + seed_offset]))
    return quantize(rng.standard_normal((wl.M, wl.dim)), wl.dtype)


@dataclass
class DecodeInputs:
    """One decode step's inputs: `inp` holds the B new tokens (x [B, dim], one per
    sequence, margin filter applied) and the layer's weights; the caches hold values exact
    in bf16 (float32 containers)."""

    inp: Inputs
    k_cache: np.ndarray    # [G, B, L_max, d_h]
    v_cache: np.ndarray
    lengths: np.ndarray    # [B] int32: the new tokens' positions

    def raw_cache(self, name: str) -> np.ndarray:
        return f32_to_bf16_bits(getattr(self, name))


def generate_decode(wl: Workload, lengths, L_max: int) -> DecodeInputs:
    """A decode step on the workload's layer: B = len(lengths) sequences, each with one new
    token (drawn as generate(wl with B, T = 1) draws its x and weights) at position
    lengths[b] < L_max. Cache entries are N(0, s^2) with s the standard deviation of a
    projected K/V element under the workload's weights (sqrt(dim) * weight std, x ~ N(0, 1)),
    from PCG64([seed, 2]); rows at and after each position are drawn too (the step must not
    read them)."""
    lengths = np.asarray(lengths, dtype=np.int32)
    B = lengths.size
    if lengths.min() < 0 or lengths.max() >= L_max:
        raise ValueError("every position must lie inside the cache")
    inp = generate(wl.with_(B=B, T=1))
    std = wl.w_std if wl.w_std is not None else (1.0 / wl.dim) ** 0.5
    s = std * wl.dim ** 0.5
    rng = np.random.Generator(np.random.PCG64([wl.seed, 2]))
    shape = (wl.G, B, L_max, wl.d_h)
    k_cache = quantize(rng.standard_normal(shape, dtype=np.float32) * s, "bf16")
    v_cache = quantize(rng.standard_normal(shape, dtype=np.float32) * s, "bf16")
    return DecodeInputs(inp, k_cache, v_cache, lengths)


@lru_cache(maxsize=4)
def cached(name: str, **overrides) -> Inputs:
    wl = WORKLOADS[name]
    if overrides:
        wl = replace(wl, **overrides)
    return generate(wl)
