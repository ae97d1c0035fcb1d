"""GPU parity of the decode step (gqe_decode, through the C ABI) against the float64 oracle
on identical seeded inputs: routing indices and counts bit-exact; y within the bf16
tolerances (rel-L2 1e-2, max-abs 3e-2); aux loss within 1e-4 relative; the new token's K/V
written at its position (equal to the step's own projection, and to the oracle's within bf16
rounding) and every other cache row left bit-identical.

Cases cover both ways the attention runs: one CTA per (sequence, group) writing Z directly
(a single 64-key tile, or at least sixteen such pairs per SM of a B200), and split key
chunks combined by the per-sequence finish kernel, which also forms the gqe slot (with one
chunk it forms only the slot; weighted_concat and hard_concat with one chunk launch no
finish kernel). Also: ragged positions (0, tile edges, long), the three variants, every
head dim the ABI accepts,
one to three queries per warp (k up to 8), a layer without the shared head, and the
consistency of a decode step with the GPU prefill row at the same position."""
import numpy as np
import pytest
import torch

from moe_query_head_b200 import workloads as W
from oracle import gqe_oracle as go
from tests.gqe_testlib import AUX_REL, check_output, to_host_f64

pytestmark = pytest.mark.gpu


def _dev_bf16(a_f32):
    bits = W.f32_to_bf16_bits(a_f32)
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


class DecodeRun:
    def __init__(self, d: W.DecodeInputs, max_tokens=None):
        from moe_query_head_b200 import gqe as G
        self.G, self.d, wl = G, d, d.inp.wl
        self.wl = wl
        self.h = G.gqe_create(wl.dim, wl.N, wl.G, wl.k, wl.d_h, G.GQE_BF16, max_tokens or wl.M)
        inp = d.inp
        self.dev = {n: (None if inp.raw(n) is None else
                        torch.from_numpy(inp.raw(n).view(np.int16)).view(torch.bfloat16).cuda())
                    for n in ("x", "W_r", "W_q", "W_k", "W_v", "W_shared", "W_o")}
        self.kc = _dev_bf16(d.k_cache)
        self.vc = _dev_bf16(d.v_cache)
        self.kc0 = self.kc.clone()
        self.vc0 = self.vc.clone()
        self.lengths = torch.from_numpy(d.lengths.astype(np.int32)).cuda()
        self.out = torch.full((wl.M, wl.dim), float("nan"), dtype=torch.bfloat16, device="cuda")
        self.aux = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")

    def step(self, lengths=None):
        wl, dv = self.wl, self.dev
        self.G.gqe_decode(self.h, dv["x"], wl.M, self.kc, self.vc, self.kc.shape[2],
                          self.lengths if lengths is None else lengths, dv["W_r"], dv["W_q"],
                          dv["W_k"], dv["W_v"], dv["W_shared"] if wl.shared else None, dv["W_o"],
                          wl.N, wl.G, wl.k, wl.d_h, W.VARIANT_IDS[wl.variant], self.out,
                          self.aux)
        return self.G.gqe_check_device_status(self.h)

    def routing(self):
        wl = self.wl
        sel = torch.empty((wl.M, wl.G, wl.k), dtype=torch.int32, device="cuda")
        counts = torch.empty((wl.N,), dtype=torch.int32, device="cuda")
        self.G.gqe_get_routing(self.h, sel=sel, counts=counts)
        torch.cuda.synchronize()
        return sel.cpu().numpy(), counts.cpu().numpy()

    def tensor(self, name, shape):
        t = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
        self.G.gqe_get_tensor(self.h, name, t)
        torch.cuda.synchronize()
        return t

    def close(self):
        self.G.gqe_destroy(self.h)


def oracle_decode(d: W.DecodeInputs) -> go.DecodeResult:
    wl, inp = d.inp.wl, d.inp
    layer = go.Layer(wl.dim, wl.N, wl.G, wl.k, wl.d_h, shared=wl.shared, variant=wl.variant,
                     causal=True)
    return go.decode(layer, inp.f64("x"), d.k_cache.astype(np.float64),
                     d.v_cache.astype(np.float64), d.lengths, inp.f64("W_r"), inp.f64("W_q"),
                     inp.f64("W_k"), inp.f64("W_v"), inp.f64("W_shared"), inp.f64("W_o"))


def _check(d: W.DecodeInputs):
    wl = d.inp.wl
    run = DecodeRun(d)
    assert run.step() == run.G.GQE_OK
    ref = oracle_decode(d)
    sel, counts = run.routing()
    assert np.array_equal(sel, ref.routing.sel.astype(np.int32)), "routing indices differ"
    assert np.array_equal(counts, ref.routing.counts.astype(np.int32)), "expert counts differ"
    aux = float(run.aux.cpu()[0])
    assert abs(aux - ref.aux) <= AUX_REL * abs(ref.aux), (aux, ref.aux)
    check_output(to_host_f64(run.out), ref.y, "bf16")
    # the cache: row L_b holds the step's own K/V (bit-exact) and the oracle's within bf16
    # rounding; every other row is untouched
    Kn = run.tensor("K", (wl.G, wl.M, wl.d_h))
    Vn = run.tensor("V", (wl.G, wl.M, wl.d_h))
    keep = torch.ones(run.kc.shape[:3], dtype=torch.bool, device="cuda")
    for b, L in enumerate(d.lengths.tolist()):
        assert torch.equal(run.kc[:, b, L], Kn[:, b])
        assert torch.equal(run.vc[:, b, L], Vn[:, b])
        keep[:, b, L] = False
    assert torch.equal(run.kc[keep], run.kc0[keep])
    assert torch.equal(run.vc[keep], run.vc0[keep])
    np.testing.assert_allclose(to_host_f64(Kn), ref.K_new, rtol=1e-2, atol=1e-2)
    np.testing.assert_allclose(to_host_f64(Vn), ref.V_new, rtol=1e-2, atol=1e-2)
    run.close()


MAIN = W.WORKLOADS["main_b8_t2048"]
WIDE = W.WORKLOADS["wide_k2"]
LARGE = W.WORKLOADS["large_skew"].with_(skew=None)

CASES = {
    # B * G = 56, far fewer than four per SM: many key chunks per pair, merged
    "main_split_ragged": (MAIN, [0, 1, 63, 64, 65, 700, 1023], 1024),
    # B * G = 640: four key chunks per (sequence, group) on a B200
    "main_split4_batch80": (MAIN, list(np.random.default_rng(3).integers(0, 300, 80)), 320),
    # one 64-key tile per sequence: one CTA per (sequence, group) writes Z; the finish
    # kernel forms only the slot
    "main_direct_short": (MAIN, [0, 5, 31, 63, 17], 64),
    # B * G = 2560, at least sixteen CTAs per SM of a B200 without splitting
    "main_direct_batch320": (MAIN, list(np.random.default_rng(7).integers(0, 200, 320)), 256),
    # one chunk and no slot: no finish kernel
    "wide_weighted_direct": (WIDE.with_(variant="weighted_concat"), [0, 40, 63], 64),
    # B * G = 320: two key chunks per (sequence, group), merged
    "main_split_batch40": (MAIN, list(np.random.default_rng(5).integers(0, 300, 40)), 320),
    "main_no_shared_hard": (MAIN.with_(shared=False, variant="hard_concat"), [9, 129, 257], 384),
    "main_all_active": (MAIN.with_(k=2), [0, 77, 500], 512),
    "wide_gqe": (WIDE, [5, 200, 511], 512),
    "wide_weighted": (WIDE.with_(variant="weighted_concat"), [1, 64, 300], 320),
    "wide_hard": (WIDE.with_(variant="hard_concat"), [130, 0, 257], 320),
    "large_d128": (LARGE, [100, 1000], 1024),
    # two and three queries per warp: k = 4 of 4 (five queries in group 0) and k = 8 of 8
    # with 64 experts (nine queries in group 0)
    "wide_k4_qpw2": (WIDE.with_(k=4), [3, 200, 511], 512),
    "n64_k8_qpw3": (MAIN.with_(N=64, G=8, k=8), [0, 65, 300], 320),
    # d_h = 80 with four key chunks per (sequence, group)
    "dh80_split4_batch80": (MAIN.with_(d_h=80),
                            list(np.random.default_rng(6).integers(0, 200, 80)), 256),
}
# every head dim the ABI accepts, split key chunks with ragged positions
for _dh in (16, 32, 80, 96, 112):
    CASES[f"dh{_dh}_split"] = (MAIN.with_(d_h=_dh), [0, 100, 600], 640)


@pytest.mark.parametrize("case", list(CASES))
def test_decode_matches_oracle(case):
    wl, lengths, L_max = CASES[case]
    _check(W.generate_decode(wl, lengths, L_max))


def test_decode_long_caches():
    """Long caches: one sequence (split into many chunks) and 64 sequences (two chunks each)."""
    _check(W.generate_decode(MAIN, [8191], 8192))
    rng = np.random.default_rng(4)
    _check(W.generate_decode(MAIN, list(rng.integers(2000, 4096, 64)), 4096))


def test_decode_equals_gpu_prefill_row():
    """A decode step after a GPU prefill: caches filled with the prefill's own K/V of the
    first T-1 tokens, the last token decoded at position T-1; its output and routing match
    the prefill's last row."""
    from tests.gqe_testlib import GpuRun
    T, B = 300, 2
    wl = MAIN.with_(B=B, T=T)
    inp = W.generate(wl)
    pre = GpuRun(inp).forward()
    K = pre.tensor("K", (wl.G, wl.M, wl.d_h), torch.bfloat16).view(wl.G, B, T, wl.d_h)
    V = pre.tensor("V", (wl.G, wl.M, wl.d_h), torch.bfloat16).view(wl.G, B, T, wl.d_h)
    sel_pre, _, _, _ = pre.routing()
    y_pre = pre.out.view(B, T, wl.dim)[:, T - 1].float().cpu().numpy()
    # decode inputs: the last token of each sequence, caches = prefill K/V (rows >= T-1 are
    # overwritten / unread)
    from moe_query_head_b200 import gqe as G
    h = G.gqe_create(wl.dim, wl.N, wl.G, wl.k, wl.d_h, G.GQE_BF16, B)
    x_last = pre.dev["x"].view(B, T, wl.dim)[:, T - 1].contiguous()
    kc, vc = K.clone(), V.clone()
    lengths = torch.full((B,), T - 1, dtype=torch.int32, device="cuda")
    out = torch.empty((B, wl.dim), dtype=torch.bfloat16, device="cuda")
    d = pre.dev
    G.gqe_decode(h, x_last, B, kc, vc, T, lengths, d["W_r"], d["W_q"], d["W_k"], d["W_v"],
                 d["W_shared"], d["W_o"], wl.N, wl.G, wl.k, wl.d_h, 0, out, None)
    assert G.gqe_check_device_status(h) == G.GQE_OK
    sel = torch.empty((B, wl.G, wl.k), dtype=torch.int32, device="cuda")
    G.gqe_get_routing(h, sel=sel)
    torch.cuda.synchronize()
    assert np.array_equal(sel.cpu().numpy(), sel_pre.reshape(B, T, wl.G, wl.k)[:, T - 1])
    # the new rows equal the prefill's K/V at position T-1 (same projection of the same x)
    assert torch.equal(kc[:, :, T - 1], K[:, :, T - 1])
    assert torch.equal(vc[:, :, T - 1], V[:, :, T - 1])
    y = out.float().cpu().numpy()
    check_output(y.astype(np.float64), y_pre.astype(np.float64), "bf16")
    G.gqe_destroy(h)
    pre.close()


def test_decode_position_outside_cache_is_flagged_and_harmless():
    d = W.generate_decode(MAIN, [3, 10], 16)
    run = DecodeRun(d)
    bad = torch.tensor([3, 16], dtype=torch.int32, device="cuda")  # 16 == L_max
    assert run.step(bad) == run.G.GQE_ERR_INVALID_ARG
    assert torch.equal(run.kc[:, 1], run.kc0[:, 1]) and torch.equal(run.vc[:, 1], run.vc0[:, 1])
    # the status was cleared: a valid step works afterwards
    assert run.step() == run.G.GQE_OK
    run.close()


def test_decode_argument_errors():
    from moe_query_head_b200 import gqe as G
    d = W.generate_decode(MAIN, [3, 10], 16)
    run = DecodeRun(d)
    wl, dv = run.wl, run.dev
    args = [dv["x"], 2, run.kc, run.vc, 16, run.lengths, dv["W_r"], dv["W_q"], dv["W_k"],
            dv["W_v"], dv["W_shared"], dv["W_o"], wl.N, wl.G, wl.k, wl.d_h, 0, run.out, run.aux]
    bad = list(args)
    bad[1] = 3  # B > max_tokens (2)
    with pytest.raises(G.GQEError) as e:
        G.gqe_decode(run.h, *bad)
    assert e.value.status == G.GQE_ERR_WORKSPACE
    bad = list(args)
    bad[2] = None  # no cache
    with pytest.raises(G.GQEError) as e:
        G.gqe_decode(run.h, *bad)
    assert e.value.status == G.GQE_ERR_INVALID_ARG
    run.close()
    h32 = G.gqe_create(wl.dim, wl.N, wl.G, wl.k, wl.d_h, G.GQE_F32, 2)
    with pytest.raises(G.GQEError) as e:
        G.gqe_decode(h32, *args)
    assert e.value.status == G.GQE_ERR_UNSUPPORTED
    G.gqe_destroy(h32)
