"""Seeded input generators (CPU only)."""
import numpy as np
import pytest
import torch

from moe_query_head_b200 import workloads as W


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    a = (rng.standard_normal(100000) * 10.0 ** rng.integers(-8, 8, 100000)).astype(np.float32)
    a[:4] = [0.0, -0.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8]  # ties to even
    ours = W.f32_to_bf16_bits(a)
    theirs = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert (ours == theirs).all()
    back = W.bf16_bits_to_f32(ours)
    assert (back == torch.from_numpy(a).to(torch.bfloat16).float().numpy()).all()


def test_generation_is_deterministic_and_margined():
    wl = W.WORKLOADS["tiny_f32"]
    a, b = W.generate(wl), W.generate(wl)
    for name in ("x", "W_r", "W_q", "W_k", "W_v", "W_shared", "W_o"):
        assert np.array_equal(getattr(a, name), getattr(b, name))
    assert W._topk_gaps(a.x, a.W_r, wl.G, wl.k).min() >= wl.margin
    assert a.W_o.shape == (wl.dim, wl.D_o) == (64, 64)


def test_small_bf16_workload_margin_and_exact_values():
    wl = W.WORKLOADS["main_b8_t2048"].with_(B=1, T=256)
    inp = W.generate(wl)
    assert W._topk_gaps(inp.x, inp.W_r, wl.G, wl.k).min() >= 1e-3
    # bf16 containers hold exact bf16 values
    assert np.array_equal(W.bf16_bits_to_f32(inp.raw("x")), inp.x)
    assert inp.raw("x").dtype == np.uint16


def test_variants_share_every_tensor_but_W_o():
    base = W.WORKLOADS["wide_k2"].with_(B=1, T=64)
    g = W.generate(base)
    h = W.generate(base.with_(variant="hard_concat"))
    for name in ("x", "W_r", "W_q", "W_k", "W_v", "W_shared"):
        assert np.array_equal(getattr(g, name), getattr(h, name))
    assert g.W_o.shape[1] == 18 * 64 and h.W_o.shape[1] == 17 * 64


def test_skew_calibration_small():
    wl = W.WORKLOADS["large_skew"].with_(dim=512, T=4096)
    inp = W.generate(wl)
    assert abs(inp.report["expert0_share"] - 0.70) <= 0.01
    assert (inp.x[:, -1] == 1.0).all()


def test_balance_check_small():
    wl = W.WORKLOADS["long_t16k"].with_(T=4096)
    inp = W.generate(wl)
    loads = W._loads(inp.x, inp.W_r, wl.G, wl.k)
    assert np.abs(loads / (wl.M * wl.k / wl.E) - 1).max() <= 0.10


def test_active_flops_formula():
    # Router + dense + routed Q + attention + W_o at the long-context layer.
    wl = W.WORKLOADS["long_t16k"]
    M, d, h, T = wl.M, 768, 48, 16384
    want = (2 * M * d * 16 + 2 * M * d * 17 * h + 2 * M * d * h * 8
            + 2 * h * T * (T + 1) * 9 + 2 * M * 480 * d)
    assert wl.active_flops() == pytest.approx(want)
    assert wl.active_flops() / 1e9 == pytest.approx(274.6, abs=0.5)
    assert wl.all_active().n_streams == 17


def test_decode_inputs_are_deterministic_exact_and_margined():
    wl = W.WORKLOADS["main_b8_t2048"]
    a = W.generate_decode(wl, [0, 17, 255], 256)
    b = W.generate_decode(wl, [0, 17, 255], 256)
    assert np.array_equal(a.k_cache, b.k_cache) and np.array_equal(a.inp.x, b.inp.x)
    assert a.k_cache.shape == a.v_cache.shape == (wl.G, 3, 256, wl.d_h)
    assert a.lengths.dtype == np.int32 and a.lengths.tolist() == [0, 17, 255]
    # values exact in bf16; the raw bits round-trip
    for name in ("k_cache", "v_cache"):
        c = getattr(a, name)
        assert np.array_equal(W.bf16_bits_to_f32(a.raw_cache(name)), c)
    # the new tokens pass the margin filter; the cache spread is that of a projected K/V
    assert W._topk_gaps(a.inp.x, a.inp.W_r, wl.G, wl.k).min() >= wl.margin
    assert abs(a.k_cache.std() / (wl.w_std * wl.dim ** 0.5) - 1) < 0.02
    # the new tokens and weights are those of generate() with B = 3, T = 1
    g = W.generate(wl.with_(B=3, T=1))
    assert np.array_equal(g.x, a.inp.x) and np.array_equal(g.W_o, a.inp.W_o)


def test_decode_inputs_reject_positions_outside_the_cache():
    with pytest.raises(ValueError):
        W.generate_decode(W.WORKLOADS["main_b8_t2048"], [0, 8], 8)
