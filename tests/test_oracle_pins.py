"""Pins of the CPU oracle to facts fixed outside itself (CPU only).

Each test checks the oracle against something other than its own formulas: brute-force
enumeration, closed forms, a library routine (torch's float64 scaled_dot_product_attention),
an independently written dense GQA layer, and the facts the pages state in words.
The mutation tests at the end plant plausible mistakes in the oracle and check that one
of these pins catches each.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import gqe_oracle as go

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_layer_inputs(rng, layer, M, scale=1.0):
    d, N, G, h = layer.dim, layer.N, layer.G, layer.d_h
    x = rng.standard_normal((M, d))
    W_r = rng.standard_normal((N, d)) * scale / math.sqrt(d)
    W_q = rng.standard_normal((N * h, d)) / math.sqrt(d)
    W_k = rng.standard_normal((G * h, d)) / math.sqrt(d)
    W_v = rng.standard_normal((G * h, d)) / math.sqrt(d)
    W_s = rng.standard_normal((h, d)) / math.sqrt(d) if layer.shared else None
    W_o = rng.standard_normal((d, layer.D_o)) / math.sqrt(layer.D_o)
    return x, W_r, W_q, W_k, W_v, W_s, W_o


# ---------------------------------------------------------------------------------------
# Routing
# ---------------------------------------------------------------------------------------

def brute_force_topk(logits_row_group, k):
    """All C(E,k) subsets; the best has the largest logit sum; among equal sums the
    lexicographically smallest index tuple (lower index wins ties)."""
    E = len(logits_row_group)
    best, best_sum = None, -math.inf
    for sub in itertools.combinations(range(E), k):  # lexicographic order
        s = sum(logits_row_group[j] for j in sub)
        if s > best_sum:
            best, best_sum = sub, s
    return best


@pytest.mark.parametrize("N,G,k", [(8, 2, 1), (8, 2, 2), (8, 2, 3), (12, 3, 4), (4, 2, 2)])
def test_routing_matches_brute_force_with_ties(N, G, k):
    rng = np.random.default_rng(10 + N + k)
    M, d = 60, 6
    # Small integers: logits are exact integers in any precision, with many ties.
    x = rng.integers(-2, 3, size=(M, d)).astype(np.float64)
    W_r = rng.integers(-1, 2, size=(N, d)).astype(np.float64)
    W_r[1] = W_r[0]  # identical experts force exact ties
    rt = go.route(x, W_r, G, k)
    E = N // G
    logits = x @ W_r.T
    for t in range(M):
        for g in range(G):
            want = brute_force_topk(list(logits[t, g * E:(g + 1) * E]), k)
            assert tuple(rt.sel[t, g]) == want, (t, g, logits[t, g * E:(g + 1) * E])


def test_routing_zero_router_picks_lowest_indices():
    rng = np.random.default_rng(1)
    M, d, N, G, k = 40, 8, 12, 3, 2
    x = rng.standard_normal((M, d))
    rt = go.route(x, np.zeros((N, d)), G, k)
    assert (rt.sel == np.arange(k)[None, None, :]).all()
    np.testing.assert_allclose(rt.p, 1.0 / (N // G), rtol=0, atol=1e-15)
    np.testing.assert_allclose(rt.gates, 1.0 / k, rtol=0, atol=1e-15)
    np.testing.assert_allclose(rt.w, 1.0 / (G * k), rtol=0, atol=1e-15)


@pytest.mark.parametrize("k", [1, 2, 3, 4])
def test_routing_invariants(k):
    """k distinct experts per group, counts sum to M*k, gates sum to 1 per group, slot
    weights sum to 1 per token ("GQE" README Algorithm Overview; the MoE invariants of
    the CSE Roadmap tutorial, Mixture of experts)."""
    rng = np.random.default_rng(2 + k)
    M, d, N, G = 200, 16, 16, 4
    x = rng.standard_normal((M, d))
    W_r = rng.standard_normal((N, d))
    rt = go.route(x, W_r, G, k)
    for t in range(M):
        for g in range(G):
            assert len(set(rt.sel[t, g])) == k
            assert list(rt.sel[t, g]) == sorted(rt.sel[t, g])
    assert rt.counts.reshape(G, -1).sum(axis=1).tolist() == [M * k] * G
    np.testing.assert_allclose(rt.gates.sum(axis=2), 1.0, atol=1e-12)
    np.testing.assert_allclose(rt.w.sum(axis=(1, 2)), 1.0, atol=1e-12)
    np.testing.assert_allclose(rt.p.sum(axis=2), 1.0, atol=1e-12)
    # p is the softmax of the group's logits: its log differences are the logit differences.
    lg = (x @ W_r.T).reshape(M, G, -1)
    np.testing.assert_allclose(np.log(rt.p[:, :, 1:]) - np.log(rt.p[:, :, :1]),
                               lg[:, :, 1:] - lg[:, :, :1], atol=1e-10)
    if k == N // G:  # all active: gates are the full softmax
        np.testing.assert_allclose(rt.gates, rt.p, atol=1e-15)
    # prob_sum is the column sum of p; counts match the selections one by one.
    np.testing.assert_allclose(rt.prob_sum, rt.p.reshape(M, N).sum(axis=0), atol=1e-12)
    E = N // G
    c = np.zeros(N, dtype=int)
    for t in range(M):
        for g in range(G):
            for j in rt.sel[t, g]:
                c[g * E + j] += 1
    assert (c == rt.counts).all()


# ---------------------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("T,d_h", [(1, 8), (7, 16), (64, 48), (130, 32)])
def test_attention_matches_torch_sdpa_f64(causal, T, d_h):
    rng = np.random.default_rng(T * 7 + d_h)
    q = rng.standard_normal((T, d_h))
    K = rng.standard_normal((T, d_h))
    V = rng.standard_normal((T, d_h))
    got = go.attention_rows(q, np.arange(T), K, V, causal, chunk=17)
    want = F.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(K)[None, None],
        torch.from_numpy(V)[None, None], is_causal=causal)[0, 0].numpy()
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_attention_closed_forms():
    rng = np.random.default_rng(5)
    T, d_h = 50, 12
    V = rng.standard_normal((T, d_h))
    q = rng.standard_normal((T, d_h))
    # K = 0: uniform weights, causal output is the running mean of V.
    got = go.attention_rows(q, np.arange(T), np.zeros((T, d_h)), V, True)
    want = np.cumsum(V, axis=0) / np.arange(1, T + 1)[:, None]
    np.testing.assert_allclose(got, want, atol=1e-13)
    # The first position attends only to itself.
    K = rng.standard_normal((T, d_h))
    got = go.attention_rows(q[:1], np.array([0]), K, V, True)
    np.testing.assert_allclose(got[0], V[0], atol=1e-15)


# ---------------------------------------------------------------------------------------
# Whole layer
# ---------------------------------------------------------------------------------------

def dense_gqa_layer(x, B, T, W_q, W_k, W_v, W_o, N, G, d_h, causal):
    """An all-active GQA attention layer written independently of the oracle, with
    torch's float64 SDPA: N query heads, head h reads KV head h // (N/G)."""
    M, d = x.shape
    xt = torch.from_numpy(x).reshape(B, T, d)
    q = (xt @ torch.from_numpy(W_q).T).reshape(B, T, N, d_h).transpose(1, 2)
    k = (xt @ torch.from_numpy(W_k).T).reshape(B, T, G, d_h).transpose(1, 2)
    v = (xt @ torch.from_numpy(W_v).T).reshape(B, T, G, d_h).transpose(1, 2)
    rep = N // G
    k = k.repeat_interleave(rep, dim=1)
    v = v.repeat_interleave(rep, dim=1)
    o = F.scaled_dot_product_attention(q, k, v, is_causal=causal)
    z = o.transpose(1, 2).reshape(M, N * d_h)
    return (z @ torch.from_numpy(W_o).T).numpy()


@pytest.mark.parametrize("N,G,causal", [(4, 2, True), (8, 2, True), (6, 3, False)])
def test_all_active_equals_dense_gqa(N, G, causal):
    """k = E, hard_concat, no shared head: the layer is the all-active GQA layer."""
    E = N // G
    layer = go.Layer(dim=24, N=N, G=G, k=E, d_h=8, shared=False, variant="hard_concat",
                     causal=causal)
    rng = np.random.default_rng(N * 10 + G)
    B, T = 2, 19
    x, W_r, W_q, W_k, W_v, _, W_o = rand_layer_inputs(rng, layer, B * T)
    res = go.forward(layer, x, B, T, W_r, W_q, W_k, W_v, None, W_o)
    want = dense_gqa_layer(x, B, T, W_q, W_k, W_v, W_o, N, G, layer.d_h, causal)
    np.testing.assert_allclose(res.y, want, rtol=1e-10, atol=1e-12)


def test_routed_stream_equals_dense_head_output():
    """For any k, routed stream (g, r) at token t equals dense head g*E + sel[t,g,r]."""
    layer = go.Layer(dim=32, N=8, G=2, k=2, d_h=8, shared=True, variant="gqe")
    rng = np.random.default_rng(9)
    B, T = 1, 33
    x, W_r, W_q, W_k, W_v, W_s, W_o = rand_layer_inputs(rng, layer, B * T)
    res = go.forward(layer, x, B, T, W_r, W_q, W_k, W_v, W_s, W_o)
    xt = torch.from_numpy(x).reshape(B, T, -1)
    E = layer.E
    for g in range(layer.G):
        kk = (xt @ torch.from_numpy(W_k[g * 8:(g + 1) * 8]).T)[:, None]
        vv = (xt @ torch.from_numpy(W_v[g * 8:(g + 1) * 8]).T)[:, None]
        for j in range(E):
            h = g * E + j
            qq = (xt @ torch.from_numpy(W_q[h * 8:(h + 1) * 8]).T)[:, None]
            o = F.scaled_dot_product_attention(qq, kk, vv, is_causal=True)[0, 0].numpy()
            for r in range(layer.k):
                rows = np.nonzero(res.routing.sel[:, g, r] == j)[0]
                np.testing.assert_allclose(res.O[g * layer.k + r, rows], o[rows], atol=1e-12)
    # Shared stream: W_shared over KV head 0 (the stated reading).
    qq = (xt @ torch.from_numpy(W_s).T)[:, None]
    kk = (xt @ torch.from_numpy(W_k[:8]).T)[:, None]
    vv = (xt @ torch.from_numpy(W_v[:8]).T)[:, None]
    o = F.scaled_dot_product_attention(qq, kk, vv, is_causal=True)[0, 0].numpy()
    np.testing.assert_allclose(res.O[layer.G * layer.k], o, atol=1e-12)


def test_active_head_count_matches_pages():
    with open(os.path.join(GOLDEN, "active_heads.json")) as f:
        gold = json.load(f)
    layer = go.Layer(dim=768, N=gold["N"], G=gold["G"], k=gold["k"], d_h=48,
                     shared=gold["shared"])
    assert layer.n_streams == gold["active_query_heads"]
    assert round(100 * layer.n_streams / gold["all_active_heads"]) == gold[
        "active_fraction_rounded_percent"]
    assert go.default_head_dim(768, 16) == 48
    # D_o: 8 routed + slot + shared blocks of 48
    assert layer.D_o == 10 * 48
    assert go.Layer(768, 16, 8, 1, 48, variant="hard_concat").D_o == 9 * 48
    assert go.Layer(2048, 32, 8, 2, 64, variant="gqe").D_o == 18 * 64
    with pytest.raises(ValueError):
        go.Layer(768, 15, 8, 1, 48)
    with pytest.raises(ValueError):
        go.Layer(768, 16, 8, 3, 48)


@pytest.mark.parametrize("variant", ["hard_concat", "gqe", "weighted_concat"])
def test_identical_experts_collapse(variant):
    """Identical experts make the router irrelevant (the MoE check of the CSE Roadmap
    tutorial, Mixture of experts): with all query experts of a group equal, hard_concat
    does not depend on W_r. If, in addition, every group has the same experts and the
    same KV head, the gqe slot equals the common head output (slot weights sum to 1), and
    weighted_concat scales it by p."""
    layer = go.Layer(dim=16, N=6, G=2, k=1, d_h=8, shared=True, variant=variant)
    rng = np.random.default_rng(3)
    B, T = 2, 21
    x, W_r, W_q, W_k, W_v, W_s, W_o = rand_layer_inputs(rng, layer, B * T)
    h = layer.d_h
    one = W_q[:h].copy()
    W_q = np.concatenate([one] * layer.N)
    W_k = np.concatenate([W_k[:h]] * layer.G)
    W_v = np.concatenate([W_v[:h]] * layer.G)
    ys = []
    for seed in (11, 12):
        W_r2 = np.random.default_rng(seed).standard_normal(W_r.shape)
        res = go.forward(layer, x, B, T, W_r2, W_q, W_k, W_v, W_s, W_o)
        ys.append(res)
    if variant in ("hard_concat", "gqe"):
        np.testing.assert_allclose(ys[0].y, ys[1].y, atol=1e-12)
    o_common = ys[0].O[0]
    if variant == "gqe":
        np.testing.assert_allclose(ys[0].Z[:, 2 * h:3 * h], o_common, atol=1e-12)
    if variant == "weighted_concat":
        p = ys[0].routing.p_sel[:, 0, 0]
        np.testing.assert_allclose(ys[0].Z[:, :h], p[:, None] * o_common, atol=1e-12)


def test_weighted_concat_uniform_router():
    """W_r = 0: every p = 1/E, so weighted_concat's routed blocks are O / E."""
    layer = go.Layer(dim=16, N=8, G=2, k=2, d_h=4, shared=True, variant="weighted_concat")
    rng = np.random.default_rng(4)
    x, _, W_q, W_k, W_v, W_s, W_o = rand_layer_inputs(rng, layer, 30)
    res = go.forward(layer, x, 1, 30, np.zeros((8, 16)), W_q, W_k, W_v, W_s, W_o)
    S_r = layer.G * layer.k
    for s in range(S_r):
        np.testing.assert_allclose(res.Z[:, s * 4:(s + 1) * 4], res.O[s] / layer.E, atol=1e-14)
    np.testing.assert_allclose(res.Z[:, S_r * 4:], res.O[S_r], atol=0)


def test_gqe_slot_uniform_router_is_mean():
    """W_r = 0: slot weights are 1/(G k), so the slot is the mean of the routed outputs."""
    layer = go.Layer(dim=16, N=8, G=2, k=2, d_h=4, shared=False, variant="gqe")
    rng = np.random.default_rng(6)
    x, _, W_q, W_k, W_v, _, W_o = rand_layer_inputs(rng, layer, 25)
    res = go.forward(layer, x, 1, 25, np.zeros((8, 16)), W_q, W_k, W_v, None, W_o)
    np.testing.assert_allclose(res.Z[:, 16:20], res.O.mean(axis=0), atol=1e-14)
    np.testing.assert_allclose(res.y, res.Z @ W_o.T, atol=1e-14)


def test_gqe_slot_hand_computed_non_uniform_router():
    """The gqe slot with a non-uniform router, against values worked out by hand.

    G = 2 groups of E = 2 experts, k = 1, d_h = 2, no shared head; two sequences of one
    token each, so every stream's attention output is its head's single value row
    (O = V_0). Token 0 = e_0 has group logits (ln 3, 0) and (ln 2, 0): it takes expert 0
    in both groups with p = 3/4 and 2/3. Token 1 = e_1 has (0, ln 4) and (0, ln 1.5): it
    takes expert 1 in both with p = 4/5 and 3/5. The value heads are V_0 = (1, 0) and
    V_1 = (0, 1) for both tokens. The slot renormalises the selected p over all G k
    selections of the token (gist.science summary, Output Construction: a weighted sum of
    the selected expert outputs using router probabilities), so token 0's slot is
    (3/4, 2/3) / (3/4 + 2/3) = (9/17, 8/17) and token 1's is (4/5, 3/5) / (7/5) =
    (4/7, 3/7). Per-group gates (1 each at k = 1) or gates / G (1/2 each) give other
    values."""
    layer = go.Layer(dim=4, N=4, G=2, k=1, d_h=2, shared=False, variant="gqe")
    x = np.array([[1.0, 0, 0, 0], [0, 1.0, 0, 0]])
    W_r = np.zeros((4, 4))
    W_r[:, 0] = [math.log(3.0), 0.0, math.log(2.0), 0.0]
    W_r[:, 1] = [0.0, math.log(4.0), 0.0, math.log(1.5)]
    W_v = np.zeros((4, 4))
    W_v[0, :2] = 1.0  # head 0, column 0
    W_v[3, :2] = 1.0  # head 1, column 1
    rng = np.random.default_rng(11)
    W_q = rng.standard_normal((8, 4))
    W_k = rng.standard_normal((4, 4))
    W_o = rng.standard_normal((4, layer.D_o))
    res = go.forward(layer, x, 2, 1, W_r, W_q, W_k, W_v, None, W_o)
    assert res.routing.sel[:, :, 0].tolist() == [[0, 0], [1, 1]]
    np.testing.assert_allclose(res.routing.p_sel[:, :, 0], [[0.75, 2 / 3], [0.8, 0.6]],
                               atol=1e-15)
    slot = res.Z[:, 4:6]
    np.testing.assert_allclose(slot, [[9 / 17, 8 / 17], [4 / 7, 3 / 7]], atol=1e-15)
    # the hard-concat blocks are the heads' value rows
    np.testing.assert_allclose(res.Z[:, 0:4], [[1, 0, 0, 1], [1, 0, 0, 1]], atol=1e-15)


# ---------------------------------------------------------------------------------------
# Load-balancing loss
# ---------------------------------------------------------------------------------------

def test_aux_loss_closed_forms():
    rng = np.random.default_rng(7)
    M, d, N, G, k = 64, 10, 8, 2, 1
    E = N // G
    x = rng.standard_normal((M, d))
    # Uniform router: Pbar = 1/E exactly, so L = 1 whatever the counts.
    rt = go.route(x, np.zeros((N, d)), G, k)
    assert go.aux_loss(rt.counts, rt.prob_sum, M, G, k) == pytest.approx(1.0, abs=1e-14)
    # Exactly balanced counts: f = 1/E, so L = 1 whatever the probabilities.
    counts = np.full(N, M * k // E)
    prob_sum = rng.random((G, E))
    prob_sum = (prob_sum / prob_sum.sum(axis=1, keepdims=True) * M).ravel()
    assert go.aux_loss(counts, prob_sum, M, G, k) == pytest.approx(1.0, abs=1e-13)
    # Full collapse on expert 0 with p -> 1: L -> E.
    W_r = np.zeros((N, d))
    x1 = np.concatenate([x[:, :-1], np.ones((M, 1))], axis=1)
    W_r[np.arange(G) * E, -1] = 60.0
    rt = go.route(x1, W_r, G, k)
    assert (rt.sel == 0).all()
    assert go.aux_loss(rt.counts, rt.prob_sum, M, G, k) == pytest.approx(E, rel=1e-12)
    # A hand-computed case: G=1, E=2, k=1, two tokens both routed to expert 0 with
    # p = (0.75, 0.25): f = (1, 0), Pbar = (0.75, 0.25), L = 2 * 0.75 = 1.5.
    l = math.log(3.0)
    rt = go.route(np.array([[l], [l]]), np.array([[1.0], [0.0]]), 1, 1)
    np.testing.assert_allclose(rt.p[:, 0], [[0.75, 0.25]] * 2, atol=1e-15)
    assert go.aux_loss(rt.counts, rt.prob_sum, 2, 1, 1) == pytest.approx(1.5, abs=1e-14)


def test_forward_rows_matches_forward():
    layer = go.Layer(dim=20, N=8, G=4, k=1, d_h=4, shared=True, variant="gqe")
    rng = np.random.default_rng(8)
    B, T = 3, 17
    x, W_r, W_q, W_k, W_v, W_s, W_o = rand_layer_inputs(rng, layer, B * T)
    full = go.forward(layer, x, B, T, W_r, W_q, W_k, W_v, W_s, W_o)
    rows = np.array([0, 5, 16, 17, 30, 50])
    part = go.forward_rows(layer, x, B, T, W_r, W_q, W_k, W_v, W_s, W_o, rows)
    np.testing.assert_allclose(part["y"], full.y[rows], atol=1e-13)
    assert part["aux"] == pytest.approx(full.aux, abs=1e-15)


# ---------------------------------------------------------------------------------------
# Planted mistakes: each must make at least one pin above fail.
# ---------------------------------------------------------------------------------------

def _topk_high_index_on_ties(logits, G, k):
    M, N = logits.shape
    E = N // G
    l32 = logits.astype(np.float32).reshape(M, G, E)
    order = np.argsort(-l32[:, :, ::-1], axis=2, kind="stable")[:, :, :k]
    return np.sort(E - 1 - order, axis=2).astype(np.int32)


def _attention_wrong_scale(q, t_pos, K, V, causal, chunk=1024):
    return _orig_attention_rows(q * math.sqrt(q.shape[1]) ** -1, t_pos, K, V, causal, chunk)


def _attention_mask_dropped(q, t_pos, K, V, causal, chunk=1024):
    return _orig_attention_rows(q, t_pos, K, V, False, chunk)


_orig_attention_rows = go.attention_rows


def _route_slot_per_group(x, W_r, G, k):
    rt = _orig_route(x, W_r, G, k)
    rt.w = rt.gates.copy()
    return rt


_orig_route = go.route


def _route_slot_gates_over_G(x, W_r, G, k):
    # sums to 1 per token like the true slot weights, but ignores how the groups' selected
    # probabilities compare
    rt = _orig_route(x, W_r, G, k)
    rt.w = rt.gates / G
    return rt


def _kv_transposed(x, W_k, W_v, G, d_h):
    K, V = _orig_kv(x, W_k, W_v, G, d_h)
    return V, K


_orig_kv = go.kv_projection


def _shared_reads_last_head(s, k, G):
    return s // k if s < G * k else G - 1


def _aux_without_E(counts, prob_sum, M, G, k):
    return _orig_aux(counts, prob_sum, M, G, k) / (counts.shape[0] // G)


_orig_aux = go.aux_loss


MUTANTS = {
    "topk_ties_high_index": ("top_k_per_group", _topk_high_index_on_ties,
                             [lambda: test_routing_matches_brute_force_with_ties(8, 2, 1)]),
    "attention_scale": ("attention_rows", _attention_wrong_scale,
                        [lambda: test_attention_matches_torch_sdpa_f64(True, 64, 48)]),
    "attention_mask_dropped": ("attention_rows", _attention_mask_dropped,
                                  [lambda: test_attention_closed_forms(),
                                   lambda: test_all_active_equals_dense_gqa(4, 2, True)]),
    "slot_per_group": ("route", _route_slot_per_group,
                       [lambda: test_routing_invariants(1),
                        lambda: test_gqe_slot_hand_computed_non_uniform_router()]),
    "slot_gates_over_G": ("route", _route_slot_gates_over_G,
                          [lambda: test_gqe_slot_hand_computed_non_uniform_router()]),
    "kv_swapped": ("kv_projection", _kv_transposed,
                   [lambda: test_all_active_equals_dense_gqa(4, 2, True)]),
    "shared_head_kv": ("stream_kv_head", _shared_reads_last_head,
                       [lambda: test_routed_stream_equals_dense_head_output()]),
    "aux_missing_E": ("aux_loss", _aux_without_E, [lambda: test_aux_loss_closed_forms()]),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn, pins = MUTANTS[name]
    monkeypatch.setattr(go, attr, fn)
    failed = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed >= 1, f"planted mistake {name} was not caught"
