"""Helpers shared by the GPU parity tests: upload a workload, run the CUDA path through
the C ABI, run the oracle on the same inputs, compare."""
from __future__ import annotations

import numpy as np
import torch

from moe_query_head_b200 import workloads as W

BF16_REL_L2 = 1e-2
BF16_MAX_ABS = 3e-2
F32_REL_L2 = 1e-5
AUX_REL = 1e-4


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def to_device(inp: W.Inputs, name: str):
    a = inp.raw(name)
    if a is None:
        return None
    if inp.wl.dtype == "bf16":
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def to_host_f64(t) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


class GpuRun:
    """Runs gqe_forward on one workload and keeps the handle for inspection."""

    def __init__(self, inp: W.Inputs, max_tokens: int | None = None):
        from moe_query_head_b200 import gqe as G
        self.G = G
        wl = inp.wl
        self.wl = wl
        self.inp = inp
        dt = G.GQE_BF16 if wl.dtype == "bf16" else G.GQE_F32
        self.h = G.gqe_create(wl.dim, wl.N, wl.G, wl.k, wl.d_h, dt, max_tokens or wl.M)
        self.dev = {n: to_device(inp, n) for n in ("x", "W_r", "W_q", "W_k", "W_v", "W_shared", "W_o")}
        tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
        self.out = torch.full((wl.M, wl.dim), float("nan"), dtype=tdt, device="cuda")
        self.aux = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")

    def forward(self):
        wl, d = self.wl, self.dev
        self.G.gqe_forward(self.h, d["x"], wl.B, wl.T, d["W_r"], d["W_q"], d["W_k"], d["W_v"],
                           d["W_shared"] if wl.shared else None, d["W_o"], wl.N, wl.G, wl.k,
                           wl.d_h, W.VARIANT_IDS[wl.variant], int(wl.causal), self.out, self.aux)
        st = self.G.gqe_check_device_status(self.h)
        assert st == self.G.GQE_OK, self.G.status_str(st)
        return self

    def routing(self):
        wl = self.wl
        sel = torch.empty((wl.M, wl.G, wl.k), dtype=torch.int32, device="cuda")
        gates = torch.empty((wl.M, wl.G, wl.k), dtype=torch.float32, device="cuda")
        counts = torch.empty((wl.N,), dtype=torch.int32, device="cuda")
        mp = torch.empty((wl.N,), dtype=torch.float32, device="cuda")
        self.G.gqe_get_routing(self.h, sel, gates, counts, mp)
        torch.cuda.synchronize()
        return sel.cpu().numpy(), gates.cpu().numpy(), counts.cpu().numpy(), mp.cpu().numpy()

    def tensor(self, which: str, shape, dtype):
        t = torch.empty(shape, dtype=dtype, device="cuda")
        self.G.gqe_get_tensor(self.h, which, t)
        torch.cuda.synchronize()
        return t

    def close(self):
        self.G.gqe_destroy(self.h)


def oracle_layer(wl: W.Workload):
    import oracle
    return oracle.Layer(dim=wl.dim, N=wl.N, G=wl.G, k=wl.k, d_h=wl.d_h, shared=wl.shared,
                        variant=wl.variant, causal=wl.causal)


def oracle_forward(inp: W.Inputs):
    import oracle
    f = inp.f64
    return oracle.forward(oracle_layer(inp.wl), f("x"), inp.wl.B, inp.wl.T, f("W_r"), f("W_q"),
                          f("W_k"), f("W_v"), f("W_shared"), f("W_o"))


def oracle_rows(inp: W.Inputs, rows):
    import oracle
    f = inp.f64
    return oracle.forward_rows(oracle_layer(inp.wl), f("x"), inp.wl.B, inp.wl.T, f("W_r"),
                               f("W_q"), f("W_k"), f("W_v"), f("W_shared"), f("W_o"), rows)


def sample_rows(wl: W.Workload, n: int = 48, seed: int = 0) -> np.ndarray:
    """Rows spread over every sequence: the first and last positions, tile edges (multiples
    of 128 and their neighbours) and random positions."""
    rng = np.random.default_rng(seed)
    pos = {0, 1, wl.T - 1, min(127, wl.T - 1), min(128, wl.T - 1), min(255, wl.T - 1)}
    pos |= set(rng.integers(0, wl.T, size=n).tolist())
    rows = []
    for b in range(wl.B):
        for t in sorted(pos):
            rows.append(b * wl.T + t)
    rows = np.array(sorted(set(rows)))
    if rows.size > 4 * n:
        rows = np.sort(rng.choice(rows, 4 * n, replace=False))
    return rows


def check_output(y_gpu: np.ndarray, y_ref: np.ndarray, dtype: str):
    r = rel_l2(y_gpu, y_ref)
    mx = float(np.abs(y_gpu - y_ref).max()) if y_ref.size else 0.0
    assert np.isfinite(y_gpu).all(), "non-finite output"
    if dtype == "bf16":
        assert r <= BF16_REL_L2 and mx <= BF16_MAX_ABS, (r, mx)
    else:
        assert r <= F32_REL_L2, r
    return r, mx
