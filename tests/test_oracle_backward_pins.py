"""Pins of the oracle's backward pass (CPU only).

The explicit gradient formulas of oracle.backward are checked against two computations that
share none of them: torch's float64 autograd through a forward written here with torch
operations (the selected sets held constant, as the definition states), and central finite
differences of the oracle's forward pass (itself pinned in test_oracle_pins.py). Two facts
fixed by the definition are checked exactly: hard_concat gives the router no gradient from y,
and without any routed output the aux-loss gradient has a closed form. Planted mistakes in
the attention backward and in the router's derivatives (a detached slot denominator, a
dropped aux term, a softmax Jacobian without its off-diagonal part) must be caught.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import gqe_oracle as go


def rand_case(rng, layer, B, T, router_scale=4.0):
    d, N, G, h = layer.dim, layer.N, layer.G, layer.d_h
    M = B * T
    x = rng.standard_normal((M, d))
    W_r = rng.standard_normal((N, d)) * router_scale / math.sqrt(d)
    W_q = rng.standard_normal((N * h, d)) / math.sqrt(d)
    W_k = rng.standard_normal((G * h, d)) / math.sqrt(d)
    W_v = rng.standard_normal((G * h, d)) / math.sqrt(d)
    W_s = rng.standard_normal((h, d)) / math.sqrt(d) if layer.shared else None
    W_o = rng.standard_normal((d, layer.D_o)) / math.sqrt(layer.D_o)
    dy = rng.standard_normal((M, d))
    return x, W_r, W_q, W_k, W_v, W_s, W_o, dy


def torch_objective(layer, B, T, sel, counts, dA, x, W_r, W_q, W_k, W_v, W_s, W_o, dy):
    """<dy, y> + dA * L of the GQE layer, written with torch operations; sel and counts (the
    forward's selection) are constants."""
    M, d = x.shape
    G, k, E, h, N = layer.G, layer.k, layer.E, layer.d_h, layer.N
    p = torch.softmax((x @ W_r.T).view(M, G, E), dim=2)
    sel_t = torch.as_tensor(sel, dtype=torch.int64)
    p_sel = torch.gather(p, 2, sel_t)
    w = p_sel / p_sel.sum(dim=(1, 2), keepdim=True)
    K = (x @ W_k.T).view(B, T, G, h).permute(0, 2, 1, 3)        # [B, G, T, h]
    V = (x @ W_v.T).view(B, T, G, h).permute(0, 2, 1, 3)
    Wq3 = W_q.view(N, h, d)
    outs = []
    for g in range(G):
        for r in range(k):
            We = Wq3[g * E + sel_t[:, g, r]]                        # [M, h, d]
            q = torch.einsum("md,mhd->mh", x, We).view(B, T, h)
            outs.append(F.scaled_dot_product_attention(q, K[:, g], V[:, g],
                                                       is_causal=layer.causal).reshape(M, h))
    blocks = []
    for g in range(G):
        for r in range(k):
            o = outs[g * k + r]
            if layer.variant == "weighted_concat":
                o = o * p_sel[:, g, r][:, None]
            blocks.append(o)
    if layer.variant == "gqe":
        blocks.append(sum(w[:, g, r][:, None] * outs[g * k + r]
                          for g in range(G) for r in range(k)))
    if layer.shared:
        qs = (x @ W_s.T).view(B, T, h)
        blocks.append(F.scaled_dot_product_attention(qs, K[:, 0], V[:, 0],
                                                     is_causal=layer.causal).reshape(M, h))
    y = torch.cat(blocks, dim=1) @ W_o.T
    f = torch.as_tensor(counts, dtype=torch.float64).view(G, E) / (M * k)
    L = (E * (f * p.mean(dim=0)).sum(dim=1)).mean()
    return (dy * y).sum() + dA * L


CASES = [
    dict(k=1, variant="gqe", shared=True, causal=True),
    dict(k=2, variant="gqe", shared=True, causal=True),
    dict(k=2, variant="weighted_concat", shared=True, causal=False),
    dict(k=1, variant="hard_concat", shared=False, causal=True),
    dict(k=3, variant="gqe", shared=False, causal=False),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_backward_matches_torch_autograd(case):
    c = CASES[case]
    layer = go.Layer(dim=16, N=12, G=3, k=c["k"], d_h=4, shared=c["shared"],
                     variant=c["variant"], causal=c["causal"])
    rng = np.random.default_rng(20 + case)
    B, T = 2, 7
    x, W_r, W_q, W_k, W_v, W_s, W_o, dy = rand_case(rng, layer, B, T)
    dA = 0.37
    g = go.backward(layer, x, B, T, W_r, W_q, W_k, W_v, W_s, W_o, dy, dA)
    rt = go.route(x, W_r, layer.G, layer.k)
    names = ["x", "W_r", "W_q", "W_k", "W_v", "W_s", "W_o"]
    vals = [x, W_r, W_q, W_k, W_v, W_s, W_o]
    ts = [None if v is None else torch.tensor(v, dtype=torch.float64, requires_grad=True)
          for v in vals]
    obj = torch_objective(layer, B, T, rt.sel, rt.counts, dA, *ts,
                          torch.tensor(dy, dtype=torch.float64))
    obj.backward()
    mine = [g.x, g.W_r, g.W_q, g.W_k, g.W_v, g.W_shared, g.W_o]
    for name, t, m in zip(names, ts, mine):
        if t is None:
            assert m is None
            continue
        ref = t.grad.numpy()
        np.testing.assert_allclose(m, ref, rtol=1e-9, atol=1e-11 * max(1.0, np.abs(ref).max()),
                                   err_msg=name)


def objective(layer, B, T, vals, dy, dA):
    fw = go.forward(layer, vals[0], B, T, *vals[1:])
    return float((dy * fw.y).sum() + dA * fw.aux), fw.routing.sel


def test_backward_matches_finite_differences():
    layer = go.Layer(dim=12, N=8, G=2, k=2, d_h=4, shared=True, variant="gqe", causal=True)
    rng = np.random.default_rng(31)
    B, T = 2, 5
    x, W_r, W_q, W_k, W_v, W_s, W_o, dy = rand_case(rng, layer, B, T)
    dA = 1.3
    vals = [x, W_r, W_q, W_k, W_v, W_s, W_o]
    g = go.backward(layer, x, B, T, W_r, W_q, W_k, W_v, W_s, W_o, dy, dA)
    grads = [g.x, g.W_r, g.W_q, g.W_k, g.W_v, g.W_shared, g.W_o]
    _, sel0 = objective(layer, B, T, vals, dy, dA)
    eps = 1e-6
    for i in range(len(vals)):
        for trial in range(2):
            v = rng.standard_normal(vals[i].shape)
            plus = [a.copy() for a in vals]
            minus = [a.copy() for a in vals]
            plus[i] += eps * v
            minus[i] -= eps * v
            fp, sp = objective(layer, B, T, plus, dy, dA)
            fm, sm = objective(layer, B, T, minus, dy, dA)
            assert np.array_equal(sp, sel0) and np.array_equal(sm, sel0)  # selection held
            fd = (fp - fm) / (2 * eps)
            an = float((grads[i] * v).sum())
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (i, fd, an)


def test_hard_concat_router_gets_no_output_gradient():
    layer = go.Layer(dim=16, N=8, G=2, k=1, d_h=4, shared=True, variant="hard_concat")
    rng = np.random.default_rng(40)
    B, T = 1, 9
    x, W_r, W_q, W_k, W_v, W_s, W_o, dy = rand_case(rng, layer, B, T)
    g0 = go.backward(layer, x, B, T, W_r, W_q, W_k, W_v, W_s, W_o, dy, 0.0)
    assert np.array_equal(g0.W_r, np.zeros_like(W_r))
    g1 = go.backward(layer, x, B, T, W_r, W_q, W_k, W_v, W_s, W_o, dy, 1.0)
    assert np.abs(g1.W_r).max() > 0


def test_aux_only_gradient_closed_form():
    """With dy = 0 only the aux loss remains: dL/dlogit[t, g, j] =
    (E / (G M)) p[t,g,j] (f[g,j] - sum_j' p[t,g,j'] f[g,j'])."""
    layer = go.Layer(dim=16, N=8, G=2, k=1, d_h=4, shared=True, variant="gqe")
    rng = np.random.default_rng(41)
    B, T = 2, 6
    x, W_r, W_q, W_k, W_v, W_s, W_o, _ = rand_case(rng, layer, B, T)
    M, G, E = B * T, layer.G, layer.E
    g = go.backward(layer, x, B, T, W_r, W_q, W_k, W_v, W_s, W_o, np.zeros((M, 16)), 1.0)
    rt = go.route(x, W_r, G, layer.k)
    f = rt.counts.reshape(G, E) / (M * layer.k)
    p = rt.p
    dl = (E / (G * M)) * p * (f[None] - (p * f[None]).sum(axis=2, keepdims=True))
    np.testing.assert_allclose(g.W_r, dl.reshape(M, -1).T @ x, rtol=1e-12, atol=1e-15)
    for a in (g.W_q, g.W_k, g.W_v, g.W_shared, g.W_o):
        assert np.array_equal(a, np.zeros_like(a))


def test_planted_mistake_in_attention_backward_is_caught(monkeypatch):
    """Dropping the rowsum(dO * O) term of dS must break the autograd pin."""
    real = go.attention_rows_backward

    def wrong(q, t_pos, K, V, dO, causal):
        d_h = q.shape[1]
        scale = 1.0 / math.sqrt(d_h)
        s = (q @ K.T) * scale
        if causal:
            s = np.where(np.arange(K.shape[0])[None, :] <= t_pos[:, None], s, -np.inf)
        e = np.exp(s - s.max(axis=1, keepdims=True))
        P = e / e.sum(axis=1, keepdims=True)
        dS = P * (dO @ V.T)
        return (dS @ K) * scale, (dS.T @ q) * scale, P.T @ dO

    monkeypatch.setattr(go, "attention_rows_backward", wrong)
    with pytest.raises(AssertionError):
        test_backward_matches_torch_autograd(0)
    monkeypatch.setattr(go, "attention_rows_backward", real)


def _slot_denominator_detached(dw, w, p_sel):
    return dw / p_sel.sum(axis=(1, 2), keepdims=True)


def _aux_gradient_dropped(counts, M, G, k):
    return np.zeros((G, counts.shape[0] // G))


def _softmax_jacobian_diagonal_only(p, dp):
    return p * dp


@pytest.mark.parametrize("name,mistake", [
    ("slot_weights_backward", _slot_denominator_detached),
    ("aux_loss_grad_p", _aux_gradient_dropped),
    ("group_softmax_backward", _softmax_jacobian_diagonal_only),
])
def test_planted_router_backward_mistake_is_caught(name, mistake, monkeypatch):
    """Plausible mistakes in the router's derivatives (a detached slot denominator, a
    forgotten aux term, the softmax Jacobian without its off-diagonal part) break the autograd
    pin of the gqe variant with the aux loss."""
    monkeypatch.setattr(go, name, mistake)
    with pytest.raises(AssertionError):
        test_backward_matches_torch_autograd(0)


@pytest.mark.parametrize("variant,N,G,k", [("gqe", 6, 3, 1), ("weighted_concat", 6, 3, 1),
                                           ("hard_concat", 6, 3, 1), ("gqe", 8, 2, 2)])
def test_backward_x_rows_equals_the_full_backward(variant, N, G, k):
    """The row-restricted input gradient (queries at positions >= t_min only) equals those
    rows of the full backward's dx: causally, nothing earlier reaches them."""
    layer = go.Layer(dim=12, N=N, G=G, k=k, d_h=4, shared=True, variant=variant)
    rng = np.random.default_rng(31)
    B, T, t_min = 2, 23, 15
    x, W_r, W_q, W_k, W_v, W_s, W_o, dy = rand_case(rng, layer, B, T)
    full = go.backward(layer, x, B, T, W_r, W_q, W_k, W_v, W_s, W_o, dy, 0.3)
    part = go.backward_x_rows(layer, x, B, T, W_r, W_q, W_k, W_v, W_s, W_o, dy, 0.3, t_min)
    rows = np.concatenate([np.arange(b * T + t_min, (b + 1) * T) for b in range(B)])
    np.testing.assert_allclose(part, full.x[rows], rtol=1e-10, atol=1e-12)
