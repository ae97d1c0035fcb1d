"""CPU oracle for Grouped Query Experts (GQE) attention: the forward (prefill) pass, the
decode step with a KV cache, and the backward pass.

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this module.
The product path (the CUDA library and its Python binding) never calls it and shares
no code with it; this module imports nothing from the product package.

Everything is float64 numpy. Each step is the plain definition, written in the order
the sources give it; numpy's matmul and exp are the only library primitives used.
There is no blocking or fusion, except that attention rows are processed in chunks of
query rows to bound memory, which does not change any row's arithmetic.

Sources (by page title and section):
  [README]   "GQE: Grouped Query Experts" (FrontiersMindAI/GQE README):
             Algorithm Overview, Usage, Parameters, Ablations.
  [Summary]  "Grouped Query Experts: Mixture-of-Experts on GQA Self-Attention",
             gist.science technical summary: Methodology (Architecture and Routing,
             Output Construction), Training and Loss.
  [Tutorial] "Grouped-query attention and mixture of experts" (CSE Roadmap):
             Mixture of experts (MoE).

Pins (tests/test_oracle_pins.py): brute-force routing on tiny inputs, closed forms of
the gates and of the aux loss, torch's float64 scaled_dot_product_attention, the
reduction to an independently written dense GQA layer at k = E, and the
identical-experts collapse. The decode step (tests/test_oracle_decode_pins.py) is pinned to
the forward's row at the new position and to the single-key closed form; the backward pass
(tests/test_oracle_backward_pins.py) to torch autograd through an independently written
forward and to finite differences of the forward. Every function below is pinned; none is
"parity unpinned".
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

VARIANTS = ("gqe", "weighted_concat", "hard_concat")


@dataclass
class Layer:
    """Shapes of one GQE layer ([README] Parameters)."""

    dim: int
    N: int
    G: int
    k: int
    d_h: int
    shared: bool = True
    variant: str = "gqe"
    causal: bool = True

    def __post_init__(self):
        if self.N % self.G != 0:  # [README] Parameters: N must be divisible by G
            raise ValueError("num_query_experts must be divisible by num_kv_heads")
        if not 1 <= self.k <= self.N // self.G:
            raise ValueError("top_k must be in [1, N/G]")
        if self.variant not in VARIANTS:
            raise ValueError(f"unknown variant {self.variant!r}")

    @property
    def E(self) -> int:
        return self.N // self.G

    @property
    def n_streams(self) -> int:
        """Query streams computed per token: G*k routed plus the shared head."""
        return self.G * self.k + (1 if self.shared else 0)

    @property
    def D_o(self) -> int:
        """Width of the concatenated output Z (input width of W_o)."""
        blocks = self.G * self.k + (1 if self.variant == "gqe" else 0) + (1 if self.shared else 0)
        return blocks * self.d_h


def default_head_dim(dim: int, N: int) -> int:
    """[README] Parameters: head_dim defaults to dim // num_query_experts."""
    return dim // N


# ----------------------------------------------------------------------------------------
# Step 1-3: router ([README] Algorithm Overview: softmax over the experts of each group,
# then top-k; [Tutorial] Mixture of experts: mixing weights renormalised to sum to 1).
# ----------------------------------------------------------------------------------------

@dataclass
class Routing:
    logits: np.ndarray   # [M, N] float64
    p: np.ndarray        # [M, G, E] per-group softmax, float64
    sel: np.ndarray      # [M, G, k] int32, selected j in ascending order
    p_sel: np.ndarray    # [M, G, k] p of the selected experts
    gates: np.ndarray    # [M, G, k] p_sel renormalised within the group
    w: np.ndarray        # [M, G, k] p_sel renormalised over all G*k selections (slot weights)
    counts: np.ndarray   # [N] int64 tokens per expert
    prob_sum: np.ndarray  # [N] float64 sum over tokens of p


def router_logits(x: np.ndarray, W_r: np.ndarray) -> np.ndarray:
    """l[t, e] = <x_t, W_r[e]> (no bias)."""
    return x @ W_r.T


def group_softmax(logits: np.ndarray, G: int) -> np.ndarray:
    """Softmax over the E experts inside each of the G groups, with max subtraction."""
    M, N = logits.shape
    E = N // G
    lg = logits.reshape(M, G, E)
    z = np.exp(lg - lg.max(axis=2, keepdims=True))
    return z / z.sum(axis=2, keepdims=True)


def top_k_per_group(logits: np.ndarray, G: int, k: int) -> np.ndarray:
    """The k largest experts of each group, listed in ascending expert index.

    Ranking p equals ranking the logits (softmax is strictly increasing). The decision
    is taken on the logits rounded to fp32, the GPU's precision; ties go to the lower
    index. Returns int32 [M, G, k].
    """
    M, N = logits.shape
    E = N // G
    l32 = logits.astype(np.float32).reshape(M, G, E).astype(np.float64)
    # Take the k experts one at a time: each time the largest logit not yet taken,
    # the lowest index among equal maxima (argmax returns the first maximum).
    taken = np.zeros((M, G, E), dtype=bool)
    mi, gi = np.arange(M)[:, None], np.arange(G)[None, :]
    for _ in range(k):
        j = np.argmax(np.where(taken, -np.inf, l32), axis=2)
        taken[mi, gi, j] = True
    # List each selected set in ascending expert index.
    chosen = np.zeros((M, G, k), dtype=np.int32)
    for g in range(G):
        chosen[:, g, :] = np.nonzero(taken[:, g, :])[1].reshape(M, k)
    return chosen


def route(x: np.ndarray, W_r: np.ndarray, G: int, k: int) -> Routing:
    """Router, gates, slot weights and the statistics the load-balancing loss needs."""
    M = x.shape[0]
    N = W_r.shape[0]
    E = N // G
    logits = router_logits(x, W_r)
    p = group_softmax(logits, G)
    sel = top_k_per_group(logits, G, k)
    p_sel = np.take_along_axis(p, sel.astype(np.int64), axis=2)
    gates = p_sel / p_sel.sum(axis=2, keepdims=True)
    w = p_sel / p_sel.sum(axis=(1, 2), keepdims=True)
    counts = np.zeros(N, dtype=np.int64)
    for g in range(G):
        for r in range(k):
            counts[g * E: (g + 1) * E] += np.bincount(sel[:, g, r], minlength=E)
    prob_sum = p.reshape(M, N).sum(axis=0)
    return Routing(logits, p, sel, p_sel, gates, w, counts, prob_sum)


# ----------------------------------------------------------------------------------------
# Step 4: projections ([README] Algorithm Overview: KV heads dense and unchanged, only the
# selected query heads are computed; an always-on shared query head).
# ----------------------------------------------------------------------------------------

def kv_projection(x: np.ndarray, W_k: np.ndarray, W_v: np.ndarray, G: int, d_h: int):
    """K[g], V[g] = x W_k[g]^T, x W_v[g]^T for every token. Returns [G, M, d_h] each."""
    M = x.shape[0]
    K = (x @ W_k.T).reshape(M, G, d_h).transpose(1, 0, 2).copy()
    V = (x @ W_v.T).reshape(M, G, d_h).transpose(1, 0, 2).copy()
    return K, V


def routed_queries(x: np.ndarray, W_q: np.ndarray, sel: np.ndarray, G: int, E: int,
                   d_h: int) -> np.ndarray:
    """Q[s = g*k + r, t] = x_t W_q[g*E + sel[t,g,r]]^T, only for the selected pairs.

    Returns [G*k, M, d_h]. Each expert's projection is applied only to the tokens that
    selected it.
    """
    M = x.shape[0]
    k = sel.shape[2]
    Q = np.zeros((G * k, M, d_h))
    for g in range(G):
        for j in range(E):
            Wqe = W_q[(g * E + j) * d_h:(g * E + j + 1) * d_h]
            for r in range(k):
                rows = np.nonzero(sel[:, g, r] == j)[0]
                if rows.size:
                    Q[g * k + r, rows] = x[rows] @ Wqe.T
    return Q


def shared_query(x: np.ndarray, W_shared: np.ndarray) -> np.ndarray:
    """The always-on shared head's query for every token: [M, d_h]."""
    return x @ W_shared.T


def stream_kv_head(s: int, k: int, G: int) -> int:
    """KV head read by query stream s: its group for routed streams, head 0 for the
    shared stream (a stated reading: one extra head, and head 0 is the plainest)."""
    return s // k if s < G * k else 0


# ----------------------------------------------------------------------------------------
# Step 5: softmax attention over the unchanged dense K/V.
# ----------------------------------------------------------------------------------------

def attention_rows(q: np.ndarray, t_pos: np.ndarray, K: np.ndarray, V: np.ndarray,
                   causal: bool, chunk: int = 1024) -> np.ndarray:
    """Softmax attention of query rows q [R, d_h] at positions t_pos [R] over one
    sequence's keys K, V [T, d_h]: O = softmax(q K^T / sqrt(d_h)) V, keys u <= t only
    when causal. Rows are independent; they are processed in chunks to bound memory."""
    R, d_h = q.shape
    T = K.shape[0]
    out = np.empty((R, V.shape[1]))
    scale = 1.0 / math.sqrt(d_h)
    for a in range(0, R, chunk):
        b = min(R, a + chunk)
        s = (q[a:b] @ K.T) * scale
        if causal:
            u = np.arange(T)[None, :]
            s = np.where(u <= t_pos[a:b, None], s, -np.inf)
        s = s - s.max(axis=1, keepdims=True)
        e = np.exp(s)
        out[a:b] = (e @ V) / e.sum(axis=1, keepdims=True)
    return out


def attention(Q: np.ndarray, K: np.ndarray, V: np.ndarray, B: int, T: int, k: int, G: int,
              causal: bool) -> np.ndarray:
    """All streams. Q [S, M, d_h], K/V [G, M, d_h]; returns O [S, M, d_h]."""
    S, M, d_h = Q.shape
    O = np.empty_like(Q)
    pos = np.arange(T)
    for s in range(S):
        h = stream_kv_head(s, k, G)
        for b in range(B):
            rows = slice(b * T, (b + 1) * T)
            O[s, rows] = attention_rows(Q[s, rows], pos, K[h, rows], V[h, rows], causal)
    return O


# ----------------------------------------------------------------------------------------
# Step 6-7: output construction by variant ([Summary] Output Construction; [README]
# Ablations) and the output projection.
# ----------------------------------------------------------------------------------------

def combine(O: np.ndarray, routing: Routing, layer: Layer) -> np.ndarray:
    """Build Z [M, D_o] from the stream outputs O [S, M, d_h].

    Column blocks: routed streams g-major then r; then the renormalised slot (variant
    gqe only); then the shared stream (unweighted, whenever the shared head exists).
      hard_concat:     routed outputs as they are.
      weighted_concat: routed output (g, r) times the raw per-group softmax p of its expert.
      gqe:             routed outputs as they are, plus slot = sum_{g,r} w * O.
    """
    G, k, d_h = layer.G, layer.k, layer.d_h
    M = O.shape[1]
    blocks = []
    for g in range(G):
        for r in range(k):
            o = O[g * k + r]
            if layer.variant == "weighted_concat":
                o = o * routing.p_sel[:, g, r][:, None]
            blocks.append(o)
    if layer.variant == "gqe":
        slot = np.zeros((M, d_h))
        for g in range(G):
            for r in range(k):
                slot += routing.w[:, g, r][:, None] * O[g * k + r]
        blocks.append(slot)
    if layer.shared:
        blocks.append(O[G * k])
    return np.concatenate(blocks, axis=1)


def output_projection(Z: np.ndarray, W_o: np.ndarray) -> np.ndarray:
    """y = Z W_o^T."""
    return Z @ W_o.T


# ----------------------------------------------------------------------------------------
# Step 8: Switch-style load-balancing loss ([README] Algorithm Overview; [Summary]
# Training and Loss). The caller's 0.01 coefficient ([README] Usage) is not applied.
# ----------------------------------------------------------------------------------------

def aux_loss(counts: np.ndarray, prob_sum: np.ndarray, M: int, G: int, k: int) -> float:
    """L = (1/G) sum_g E sum_j f_{g,j} Pbar_{g,j}, f = counts / (M k), Pbar = prob_sum / M."""
    N = counts.shape[0]
    E = N // G
    f = counts.astype(np.float64).reshape(G, E) / (M * k)
    P = prob_sum.reshape(G, E) / M
    return float((E * (f * P).sum(axis=1)).mean())


# ----------------------------------------------------------------------------------------
# Whole layer.
# ----------------------------------------------------------------------------------------

@dataclass
class Result:
    routing: Routing
    K: np.ndarray
    V: np.ndarray
    Q: np.ndarray          # [S, M, d_h]: routed streams then the shared stream
    O: np.ndarray          # [S, M, d_h]
    Z: np.ndarray          # [M, D_o]
    y: np.ndarray          # [M, d]
    aux: float
    extra: dict = field(default_factory=dict)


def forward(layer: Layer, x: np.ndarray, B: int, T: int, W_r, W_q, W_k, W_v, W_shared,
            W_o) -> Result:
    """The full GQE attention forward pass on x [B*T, dim] (float64 arrays)."""
    M = x.shape[0]
    assert M == B * T
    rt = route(x, W_r, layer.G, layer.k)
    K, V = kv_projection(x, W_k, W_v, layer.G, layer.d_h)
    Q = routed_queries(x, W_q, rt.sel, layer.G, layer.E, layer.d_h)
    if layer.shared:
        Q = np.concatenate([Q, shared_query(x, W_shared)[None]], axis=0)
    O = attention(Q, K, V, B, T, layer.k, layer.G, layer.causal)
    Z = combine(O, rt, layer)
    y = output_projection(Z, W_o)
    aux = aux_loss(rt.counts, rt.prob_sum, M, layer.G, layer.k)
    return Result(rt, K, V, Q, O, Z, y, aux)


def forward_rows(layer: Layer, x: np.ndarray, B: int, T: int, W_r, W_q, W_k, W_v, W_shared,
                 W_o, rows: np.ndarray) -> dict:
    """y for a subset of token rows only (the same steps restricted to those rows).

    Routing and the aux loss use every token (the loss is a mean over all of them). K/V
    are projected for each sequence's prefix that the sampled rows attend to. Returns a
    dict with y [R, d], Z [R, D_o], sel/gates/w for the rows, counts, prob_sum and aux.
    """
    rows = np.asarray(rows, dtype=np.int64)
    M = x.shape[0]
    rt = route(x, W_r, layer.G, layer.k)
    aux = aux_loss(rt.counts, rt.prob_sum, M, layer.G, layer.k)
    xs = x[rows]
    sel = rt.sel[rows]
    Q = routed_queries(xs, W_q, sel, layer.G, layer.E, layer.d_h)
    if layer.shared:
        Q = np.concatenate([Q, shared_query(xs, W_shared)[None]], axis=0)
    S = Q.shape[0]
    O = np.empty((S, rows.size, layer.d_h))
    b_of = rows // T
    t_of = rows % T
    for b in np.unique(b_of):
        m = np.nonzero(b_of == b)[0]
        last = T if not layer.causal else int(t_of[m].max()) + 1
        xb = x[b * T: b * T + last]
        K, V = kv_projection(xb, W_k, W_v, layer.G, layer.d_h)
        for s in range(S):
            h = stream_kv_head(s, layer.k, layer.G)
            O[s, m] = attention_rows(Q[s, m], t_of[m], K[h], V[h], layer.causal)
    sub = Routing(rt.logits[rows], rt.p[rows], sel, rt.p_sel[rows], rt.gates[rows],
                  rt.w[rows], rt.counts, rt.prob_sum)
    Z = combine(O, sub, layer)
    y = output_projection(Z, W_o)
    return dict(y=y, Z=Z, O=O, sel=sel, gates=rt.gates[rows], w=rt.w[rows],
                p_sel=rt.p_sel[rows], counts=rt.counts, prob_sum=rt.prob_sum, aux=aux,
                routing=rt)


# ----------------------------------------------------------------------------------------
# Decode step with a KV cache ([README] Algorithm Overview: the KV heads stay dense and
# unchanged, so the cache is GQA's; routing and the sparse query heads apply to each new
# token).
# ----------------------------------------------------------------------------------------

@dataclass
class DecodeResult:
    routing: Routing
    K_new: np.ndarray      # [G, B, d_h]: the new tokens' keys (written into the cache)
    V_new: np.ndarray      # [G, B, d_h]
    K_cache: np.ndarray    # [G, B, L_max, d_h] after the step
    V_cache: np.ndarray
    Q: np.ndarray          # [S, B, d_h]
    O: np.ndarray          # [S, B, d_h]
    Z: np.ndarray          # [B, D_o]
    y: np.ndarray          # [B, d]
    aux: float


def decode(layer: Layer, x: np.ndarray, K_cache: np.ndarray, V_cache: np.ndarray, lengths,
           W_r, W_q, W_k, W_v, W_shared, W_o) -> DecodeResult:
    """One generation step for B sequences (float64 arrays).

    x [B, dim] holds each sequence's next token, at position lengths[b]; K_cache / V_cache
    [G, B, L_max, d_h] hold the keys and values of positions 0 .. lengths[b]-1. The new
    token's K and V are written at position lengths[b] of copies of the caches (the inputs
    are not modified), and its output is the causal attention over positions
    0 .. lengths[b], i.e. row lengths[b] of the prefill forward over the whole sequence.
    """
    if not layer.causal:
        raise ValueError("a decode step is causal")
    B = x.shape[0]
    G, k, d_h = layer.G, layer.k, layer.d_h
    L_max = K_cache.shape[2]
    lengths = np.asarray(lengths, dtype=np.int64)
    if lengths.shape != (B,) or np.any(lengths < 0) or np.any(lengths >= L_max):
        raise ValueError("every position must lie inside the cache")
    rt = route(x, W_r, G, k)
    K_new, V_new = kv_projection(x, W_k, W_v, G, d_h)
    Kc = K_cache.copy()
    Vc = V_cache.copy()
    for b in range(B):
        Kc[:, b, lengths[b]] = K_new[:, b]
        Vc[:, b, lengths[b]] = V_new[:, b]
    Q = routed_queries(x, W_q, rt.sel, G, layer.E, d_h)
    if layer.shared:
        Q = np.concatenate([Q, shared_query(x, W_shared)[None]], axis=0)
    S = Q.shape[0]
    O = np.empty((S, B, d_h))
    for s in range(S):
        h = stream_kv_head(s, k, G)
        for b in range(B):
            n = lengths[b] + 1  # the cached positions and the new one
            O[s, b] = attention_rows(Q[s, b][None], np.array([lengths[b]]), Kc[h, b, :n],
                                     Vc[h, b, :n], True)[0]
    Z = combine(O, rt, layer)
    y = output_projection(Z, W_o)
    aux = aux_loss(rt.counts, rt.prob_sum, B, G, k)
    return DecodeResult(rt, K_new, V_new, Kc, Vc, Q, O, Z, y, aux)


# ----------------------------------------------------------------------------------------
# Backward pass: gradients of F = <dy, y> + dA * L, the top-k selection held constant
# ([README] Usage: the aux loss joins the task loss; [Summary] Output Construction: the
# renormalised slot is the router's differentiable path). Each step is the derivative of the
# forward step of the same name, taken in reverse order.
# ----------------------------------------------------------------------------------------

@dataclass
class Grads:
    x: np.ndarray
    W_r: np.ndarray
    W_q: np.ndarray
    W_k: np.ndarray
    W_v: np.ndarray
    W_shared: np.ndarray | None
    W_o: np.ndarray


def attention_rows_backward(q: np.ndarray, t_pos: np.ndarray, K: np.ndarray, V: np.ndarray,
                            dO: np.ndarray, causal: bool):
    """Gradients of O = softmax(q K^T / sqrt(d_h)) V (rows at positions t_pos; keys u <= t
    when causal) with respect to q, K and V, given dO. With P the probabilities:
    dV = P^T dO, dP = dO V^T, dS = P * (dP - rowsum(dO * O)), dq = dS K / sqrt(d_h),
    dK = dS^T q / sqrt(d_h)."""
    d_h = q.shape[1]
    T = K.shape[0]
    scale = 1.0 / math.sqrt(d_h)
    s = (q @ K.T) * scale
    if causal:
        u = np.arange(T)[None, :]
        s = np.where(u <= t_pos[:, None], s, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    e = np.exp(s)
    P = e / e.sum(axis=1, keepdims=True)
    O = P @ V
    dV = P.T @ dO
    dP = dO @ V.T
    dS = P * (dP - (dO * O).sum(axis=1, keepdims=True))
    return (dS @ K) * scale, (dS.T @ q) * scale, dV


def slot_weights_backward(dw: np.ndarray, w: np.ndarray, p_sel: np.ndarray) -> np.ndarray:
    """Gradient reaching the selected p through the slot weights w = p_sel / P_t (P_t the
    token's sum of selected p; numerator and denominator both differentiated):
    dp_sel = (dw - sum(dw * w)) / P_t, per token."""
    P_t = p_sel.sum(axis=(1, 2), keepdims=True)
    return (dw - (dw * w).sum(axis=(1, 2), keepdims=True)) / P_t


def aux_loss_grad_p(counts: np.ndarray, M: int, G: int, k: int) -> np.ndarray:
    """dL / dp[t, g, j] = (1/G) E f[g, j] / M (the counts, hence f, are constant); [G, E]."""
    E = counts.shape[0] // G
    f = counts.reshape(G, E).astype(np.float64) / (M * k)
    return (E / G) * f / M


def group_softmax_backward(p: np.ndarray, dp: np.ndarray) -> np.ndarray:
    """Logit gradient of the per-group softmax: dl = p * (dp - sum_j p dp); [M, G, E]."""
    return p * (dp - (p * dp).sum(axis=2, keepdims=True))


def backward(layer: Layer, x: np.ndarray, B: int, T: int, W_r, W_q, W_k, W_v, W_shared, W_o,
             dy: np.ndarray, dA: float = 0.0) -> Grads:
    """Gradients of <dy, y> + dA * L (y, L: the forward's output and aux loss) with respect to
    x and every weight. The selected sets are the forward's; see the definition's section on
    the backward pass for what is differentiated."""
    M = x.shape[0]
    G, k, E, d_h, N = layer.G, layer.k, layer.E, layer.d_h, layer.N
    fw = forward(layer, x, B, T, W_r, W_q, W_k, W_v, W_shared, W_o)
    rt = fw.routing
    # y = Z W_o^T
    dW_o = dy.T @ fw.Z
    dZ = dy @ W_o
    # output construction (column blocks: routed g-major then r, slot, shared)
    dO = np.zeros_like(fw.O)
    dp_sel = np.zeros((M, G, k))
    col = 0
    for g in range(G):
        for r in range(k):
            s = g * k + r
            blk = dZ[:, col:col + d_h]
            col += d_h
            if layer.variant == "weighted_concat":
                dO[s] += rt.p_sel[:, g, r][:, None] * blk
                dp_sel[:, g, r] += (blk * fw.O[s]).sum(axis=1)
            else:
                dO[s] += blk
    if layer.variant == "gqe":
        dslot = dZ[:, col:col + d_h]
        col += d_h
        dw = np.zeros((M, G, k))
        for g in range(G):
            for r in range(k):
                s = g * k + r
                dO[s] += rt.w[:, g, r][:, None] * dslot
                dw[:, g, r] = (dslot * fw.O[s]).sum(axis=1)
        dp_sel += slot_weights_backward(dw, rt.w, rt.p_sel)
    if layer.shared:
        dO[G * k] += dZ[:, col:col + d_h]
    # router: p of the selected experts, the aux loss's mean p, the per-group softmax
    dp = np.zeros((M, G, E))
    mi = np.arange(M)
    for g in range(G):
        for r in range(k):
            dp[mi, g, rt.sel[:, g, r]] += dp_sel[:, g, r]
    if dA:
        dp += dA * aux_loss_grad_p(rt.counts, M, G, k)[None]
    dl = group_softmax_backward(rt.p, dp).reshape(M, N)
    dW_r = dl.T @ x
    dx = dl @ W_r
    # attention, per stream and sequence; K / V gradients add up over the streams of a head
    dQ = np.zeros_like(fw.Q)
    dK = np.zeros_like(fw.K)
    dV = np.zeros_like(fw.V)
    pos = np.arange(T)
    for s in range(fw.Q.shape[0]):
        h = stream_kv_head(s, k, G)
        for b in range(B):
            rows = slice(b * T, (b + 1) * T)
            dq, dk, dv = attention_rows_backward(fw.Q[s, rows], pos, fw.K[h, rows],
                                                 fw.V[h, rows], dO[s, rows], layer.causal)
            dQ[s, rows] = dq
            dK[h, rows] += dk
            dV[h, rows] += dv
    # projections
    dW_k = np.zeros_like(W_k)
    dW_v = np.zeros_like(W_v)
    for g in range(G):
        rg = slice(g * d_h, (g + 1) * d_h)
        dW_k[rg] = dK[g].T @ x
        dW_v[rg] = dV[g].T @ x
        dx += dK[g] @ W_k[rg] + dV[g] @ W_v[rg]
    dW_q = np.zeros_like(W_q)
    for g in range(G):
        for r in range(k):
            s = g * k + r
            for j in range(E):
                rows = np.nonzero(rt.sel[:, g, r] == j)[0]
                if rows.size == 0:
                    continue
                re = slice((g * E + j) * d_h, (g * E + j + 1) * d_h)
                dW_q[re] += dQ[s, rows].T @ x[rows]
                dx[rows] += dQ[s, rows] @ W_q[re]
    dW_s = None
    if layer.shared:
        dW_s = dQ[G * k].T @ x
        dx += dQ[G * k] @ W_shared
    return Grads(dx, dW_r, dW_q, dW_k, dW_v, dW_s, dW_o)


def backward_x_rows(layer: Layer, x: np.ndarray, B: int, T: int, W_r, W_q, W_k, W_v,
                    W_shared, W_o, dy: np.ndarray, dA: float, t_min: int) -> np.ndarray:
    """Rows of dx (the input gradient of backward) for the positions t >= t_min of every
    sequence, causal layers only, without the work of the earlier rows.

    Causally, key t is read only by queries at positions >= t, so dK and dV of the rows at
    t >= t_min, like dQ and the router gradient of those rows, depend only on the queries at
    positions >= t_min (each attending over its whole prefix). The steps are backward's,
    restricted to those query rows. Returns dx [B * (T - t_min), dim], sequence by sequence.
    """
    if not layer.causal:
        raise ValueError("the row restriction needs a causal layer")
    G, k, E, d_h, N = layer.G, layer.k, layer.E, layer.d_h, layer.N
    M = x.shape[0]
    rt = route(x, W_r, G, k)
    K, V = kv_projection(x, W_k, W_v, G, d_h)
    rows = np.concatenate([np.arange(b * T + t_min, (b + 1) * T) for b in range(B)])
    xs = x[rows]
    R = rows.size
    sel = rt.sel[rows]
    Q = routed_queries(xs, W_q, sel, G, E, d_h)
    if layer.shared:
        Q = np.concatenate([Q, shared_query(xs, W_shared)[None]], axis=0)
    S = Q.shape[0]
    pos = np.arange(t_min, T)
    nr = T - t_min
    O = np.empty((S, R, d_h))
    for s in range(S):
        h = stream_kv_head(s, k, G)
        for b in range(B):
            m = slice(b * nr, (b + 1) * nr)
            seq = slice(b * T, (b + 1) * T)
            O[s, m] = attention_rows(Q[s, m], pos, K[h, seq], V[h, seq], True)
    sub = Routing(rt.logits[rows], rt.p[rows], sel, rt.p_sel[rows], rt.gates[rows], rt.w[rows],
                  rt.counts, rt.prob_sum)
    # output construction and router, as in backward, for these rows
    dZ = dy[rows] @ W_o
    dO = np.zeros_like(O)
    dp_sel = np.zeros((R, G, k))
    col = 0
    for g in range(G):
        for r in range(k):
            s = g * k + r
            blk = dZ[:, col:col + d_h]
            col += d_h
            if layer.variant == "weighted_concat":
                dO[s] += sub.p_sel[:, g, r][:, None] * blk
                dp_sel[:, g, r] += (blk * O[s]).sum(axis=1)
            else:
                dO[s] += blk
    if layer.variant == "gqe":
        dslot = dZ[:, col:col + d_h]
        col += d_h
        dw = np.zeros((R, G, k))
        for g in range(G):
            for r in range(k):
                s = g * k + r
                dO[s] += sub.w[:, g, r][:, None] * dslot
                dw[:, g, r] = (dslot * O[s]).sum(axis=1)
        dp_sel += slot_weights_backward(dw, sub.w, sub.p_sel)
    if layer.shared:
        dO[G * k] += dZ[:, col:col + d_h]
    dp = np.zeros((R, G, E))
    ri = np.arange(R)
    for g in range(G):
        for r in range(k):
            dp[ri, g, sel[:, g, r]] += dp_sel[:, g, r]
    if dA:
        dp += dA * aux_loss_grad_p(rt.counts, M, G, k)[None]
    dl = group_softmax_backward(sub.p, dp).reshape(R, N)
    dx = dl @ W_r
    # attention: the queries at t >= t_min give dQ of their rows and all of dK, dV at
    # t >= t_min
    for s in range(S):
        h = stream_kv_head(s, k, G)
        for b in range(B):
            m = slice(b * nr, (b + 1) * nr)
            seq = slice(b * T, (b + 1) * T)
            dq, dk, dv = attention_rows_backward(Q[s, m], pos, K[h, seq], V[h, seq], dO[s, m],
                                                 True)
            rg = slice(h * d_h, (h + 1) * d_h)
            dx[m] += dk[t_min:] @ W_k[rg] + dv[t_min:] @ W_v[rg]
            if s < G * k:
                g, r = divmod(s, k)
                for j in range(E):
                    sel_rows = np.nonzero(sel[m, g, r] == j)[0]
                    if sel_rows.size:
                        re = slice((g * E + j) * d_h, (g * E + j + 1) * d_h)
                        dx[m][sel_rows] += dq[sel_rows] @ W_q[re]
            else:
                dx[m] += dq @ W_shared
    return dx
