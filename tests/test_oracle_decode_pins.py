"""Pins of the oracle's decode step (CPU only).

The decode step is defined as row L_b of the prefill forward over the sequence whose first
L_b tokens filled the cache. The pins check it against the prefill oracle (itself pinned in
test_oracle_pins.py), against the closed form of attention over a single key (an empty
cache: O = V of the new token), against an independently written all-active GQA decode step
(k = E, hard_concat, no shared head), and against two invariances: cache rows at or beyond
the new position do not matter, and the sequences of a batch do not interact. Planted
mistakes must be caught.
"""
import math

import numpy as np
import pytest

from oracle import gqe_oracle as go


def rand_weights(rng, layer):
    d, N, G, h = layer.dim, layer.N, layer.G, layer.d_h
    W_r = rng.standard_normal((N, d)) / math.sqrt(d)
    W_q = rng.standard_normal((N * h, d)) / math.sqrt(d)
    W_k = rng.standard_normal((G * h, d)) / math.sqrt(d)
    W_v = rng.standard_normal((G * h, d)) / math.sqrt(d)
    W_s = rng.standard_normal((h, d)) / math.sqrt(d) if layer.shared else None
    W_o = rng.standard_normal((d, layer.D_o)) / math.sqrt(layer.D_o)
    return W_r, W_q, W_k, W_v, W_s, W_o


def build(layer, rng, lengths, L_max):
    """Sequences x_b of length lengths[b] + 1, caches holding the prefill K/V of their first
    lengths[b] tokens and random values everywhere else."""
    B = len(lengths)
    W = rand_weights(rng, layer)
    seqs = [rng.standard_normal((L + 1, layer.dim)) for L in lengths]
    Kc = rng.standard_normal((layer.G, B, L_max, layer.d_h)) * 7.0
    Vc = rng.standard_normal((layer.G, B, L_max, layer.d_h)) * 7.0
    for b, L in enumerate(lengths):
        if L:
            K, V = go.kv_projection(seqs[b][:L], W[2], W[3], layer.G, layer.d_h)
            Kc[:, b, :L] = K
            Vc[:, b, :L] = V
    x = np.stack([s[-1] for s in seqs])
    return W, seqs, x, Kc, Vc


@pytest.mark.parametrize("k,variant,shared", [(1, "gqe", True), (2, "gqe", True),
                                              (2, "weighted_concat", True),
                                              (1, "hard_concat", False)])
def test_decode_equals_prefill_row(k, variant, shared):
    layer = go.Layer(dim=24, N=8, G=4, k=k, d_h=4, shared=shared, variant=variant)
    rng = np.random.default_rng(11 + k)
    lengths = [0, 5, 11, 3]
    W, seqs, x, Kc, Vc = build(layer, rng, lengths, L_max=16)
    dec = go.decode(layer, x, Kc, Vc, lengths, *W)
    for b, L in enumerate(lengths):
        full = go.forward(layer, seqs[b], 1, L + 1, *W)
        np.testing.assert_allclose(dec.y[b], full.y[L], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dec.Z[b], full.Z[L], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dec.O[:, b], full.O[:, L], rtol=0, atol=1e-12)
        assert np.array_equal(dec.routing.sel[b], full.routing.sel[L])
        # the new row holds the new token's K/V; every other row is untouched
        np.testing.assert_allclose(dec.K_cache[:, b, L], full.K[:, L], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dec.V_cache[:, b, L], full.V[:, L], rtol=0, atol=1e-12)
        keep = np.ones(16, bool)
        keep[L] = False
        assert np.array_equal(dec.K_cache[:, b, keep], Kc[:, b, keep])
        assert np.array_equal(dec.V_cache[:, b, keep], Vc[:, b, keep])
    # the inputs were not modified
    assert not np.shares_memory(dec.K_cache, Kc)


def test_decode_empty_cache_is_the_new_value():
    """Attention over one key returns that key's value: with every length 0, each stream's
    output is V of the new token at the stream's KV head."""
    layer = go.Layer(dim=16, N=6, G=3, k=1, d_h=4, shared=True, variant="gqe")
    rng = np.random.default_rng(5)
    W = rand_weights(rng, layer)
    x = rng.standard_normal((5, 16))
    Kc = rng.standard_normal((3, 5, 8, 4))
    Vc = rng.standard_normal((3, 5, 8, 4))
    dec = go.decode(layer, x, Kc, Vc, [0] * 5, *W)
    V_new = (x @ W[3].T).reshape(5, 3, 4)
    for s in range(layer.n_streams):
        h = go.stream_kv_head(s, layer.k, layer.G)
        np.testing.assert_allclose(dec.O[s], V_new[:, h], rtol=0, atol=1e-13)


def test_decode_reads_only_positions_up_to_the_new_one():
    layer = go.Layer(dim=16, N=8, G=2, k=2, d_h=8, shared=True, variant="gqe")
    rng = np.random.default_rng(6)
    lengths = [4, 9]
    W, _, x, Kc, Vc = build(layer, rng, lengths, L_max=12)
    a = go.decode(layer, x, Kc, Vc, lengths, *W)
    Kb, Vb = Kc.copy(), Vc.copy()
    for b, L in enumerate(lengths):  # rows at and after the new position
        Kb[:, b, L:] = rng.standard_normal(Kb[:, b, L:].shape) * 100
        Vb[:, b, L:] = rng.standard_normal(Vb[:, b, L:].shape) * 100
    b_ = go.decode(layer, x, Kb, Vb, lengths, *W)
    np.testing.assert_array_equal(a.y, b_.y)
    Kc2 = Kc.copy()
    Kc2[:, 1, 0] += 1.0  # a cached row before the new position does matter
    c = go.decode(layer, x, Kc2, Vc, lengths, *W)
    assert np.abs(c.y[1] - a.y[1]).max() > 1e-6
    np.testing.assert_array_equal(c.y[0], a.y[0])


def test_decode_batch_is_permutation_equivariant():
    layer = go.Layer(dim=16, N=8, G=4, k=1, d_h=4, shared=True, variant="weighted_concat")
    rng = np.random.default_rng(9)
    lengths = [2, 7, 0, 5]
    W, _, x, Kc, Vc = build(layer, rng, lengths, L_max=8)
    a = go.decode(layer, x, Kc, Vc, lengths, *W)
    perm = np.array([2, 0, 3, 1])
    b = go.decode(layer, x[perm], Kc[:, perm], Vc[:, perm], np.array(lengths)[perm], *W)
    np.testing.assert_allclose(b.y, a.y[perm], rtol=0, atol=1e-13)


def test_decode_rejects_positions_outside_the_cache():
    layer = go.Layer(dim=16, N=4, G=2, k=1, d_h=4)
    rng = np.random.default_rng(1)
    W = rand_weights(rng, layer)
    x = rng.standard_normal((2, 16))
    Kc = np.zeros((2, 2, 4, 4))
    with pytest.raises(ValueError):
        go.decode(layer, x, Kc, Kc, [0, 4], *W)
    with pytest.raises(ValueError):
        go.decode(go.Layer(dim=16, N=4, G=2, k=1, d_h=4, causal=False), x, Kc, Kc, [0, 1], *W)


# ---------------------------------------------------------------------------------------
# Planted mistakes: each must make one of the pins above fail.
# ---------------------------------------------------------------------------------------

def _decode_attending_one_key_short(layer, x, K_cache, V_cache, lengths, *W):
    """The new token left out of its own attention (keys 0 .. L-1 only)."""
    real_rows = go.attention_rows

    def short(q, t_pos, K, V, causal, chunk=1024):
        n = K.shape[0]
        if n == 1:  # nothing else to attend to: repeat the only key so the call stays valid
            return real_rows(q, t_pos, K, V, causal, chunk)
        return real_rows(q, t_pos - 1, K[:n - 1], V[:n - 1], causal, chunk)

    go.attention_rows = short
    try:
        return _REAL_DECODE(layer, x, K_cache, V_cache, lengths, *W)
    finally:
        go.attention_rows = real_rows


def _decode_writing_one_row_late(layer, x, K_cache, V_cache, lengths, *W):
    """The new token's K/V written at position L + 1 (attended there)."""
    lengths = np.asarray(lengths)
    K2, V2 = K_cache.copy(), V_cache.copy()
    r = _REAL_DECODE(layer, x, K2, V2, lengths, *W)
    for b, L in enumerate(lengths):
        r.K_cache[:, b, L + 1] = r.K_cache[:, b, L]
        r.K_cache[:, b, L] = K_cache[:, b, L]
    return r


_REAL_DECODE = go.decode


@pytest.mark.parametrize("mistake", [_decode_attending_one_key_short,
                                     _decode_writing_one_row_late])
def test_planted_decode_mistake_is_caught(mistake, monkeypatch):
    monkeypatch.setattr(go, "decode", mistake)
    with pytest.raises(AssertionError):
        test_decode_equals_prefill_row(1, "gqe", True)


def dense_gqa_decode(x, K_cache, V_cache, lengths, W_q, W_k, W_v, W_o, N, G, d_h):
    """An all-active GQA decode step written independently: every query head h of every new
    token attends over its sequence's cached keys of head h // (N / G) plus the new key."""
    B = x.shape[0]
    E = N // G
    out_heads = np.zeros((B, N * d_h))
    for b in range(B):
        L = int(lengths[b])
        for h in range(N):
            g = h // E
            q = W_q[h * d_h:(h + 1) * d_h] @ x[b]
            keys = np.vstack([K_cache[g, b, :L], W_k[g * d_h:(g + 1) * d_h] @ x[b]])
            vals = np.vstack([V_cache[g, b, :L], W_v[g * d_h:(g + 1) * d_h] @ x[b]])
            sc = keys @ q / math.sqrt(d_h)
            wts = np.exp(sc - sc.max())
            out_heads[b, h * d_h:(h + 1) * d_h] = (wts / wts.sum()) @ vals
    return out_heads @ W_o.T


@pytest.mark.parametrize("N,G", [(8, 4), (6, 2), (4, 4)])
def test_all_active_decode_equals_dense_gqa_decode(N, G):
    layer = go.Layer(dim=16, N=N, G=G, k=N // G, d_h=4, shared=False, variant="hard_concat")
    rng = np.random.default_rng(60 + N + G)
    lengths = [0, 3, 9]
    W, _, x, Kc, Vc = build(layer, rng, lengths, L_max=12)
    dec = go.decode(layer, x, Kc, Vc, lengths, *W)
    want = dense_gqa_decode(x, Kc, Vc, lengths, W[1], W[2], W[3], W[5], N, G, layer.d_h)
    np.testing.assert_allclose(dec.y, want, rtol=1e-10, atol=1e-12)
