"""The FMA-pipe exp2 the attention softmax uses for part of its exponentials.

CPU: the algorithm (round-to-nearest range reduction with the 1.5 * 2^23 add, the degree-2
polynomial in fp32 Horner form, exponent-field scaling) emulated in numpy float32 against
float64 exp2: maximum relative error below 2e-3 on [-125, 9] (the polynomial's minimax error
on [-1/2, 1/2] is 1.89e-3; P is rounded to bf16, 1.95e-3, right after), finite and
non-negative for -inf and very negative inputs.
GPU: the library's own implementation (gqe_exp2_fma) against CUDA's exp2f (torch.exp2).
"""
import numpy as np
import pytest
import torch

COEF = (1.00047162, 0.70411982, 0.23876238)
BOUND = 2e-3


def emulate(x):
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125))
    M = np.float32(12582912.0)
    j = (x + M).astype(np.float32)
    n = (j - M).astype(np.float32)
    f = (x - n).astype(np.float32)
    c = [np.float32(v) for v in COEF]
    p = np.float32(c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = (p * f + c[k]).astype(np.float32)
    bits = (p.view(np.uint32).astype(np.uint64)
            + (j.view(np.uint32).astype(np.uint64) << np.uint64(23))) & np.uint64(0xFFFFFFFF)
    return bits.astype(np.uint32).view(np.float32), f


def test_algorithm_error_bound():
    x = np.linspace(-125, 9, 1_000_001, dtype=np.float32)
    y, f = emulate(x)
    assert np.abs(f).max() <= 0.5
    rel = np.abs(y.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() < BOUND
    # exact powers of two come out within the bound too
    yi, _ = emulate(np.arange(-125, 10, dtype=np.float32))
    assert np.abs(yi / np.exp2(np.arange(-125, 10)) - 1).max() < BOUND


def test_masked_and_tiny_inputs():
    y, _ = emulate(np.array([-np.inf, -1e30, -200.0, -125.0], np.float32))
    assert np.isfinite(y).all() and (y >= 0).all() and (y < 3e-38).all()


@pytest.mark.gpu
def test_library_exp2_matches_cuda_exp2f():
    from moe_query_head_b200 import gqe as G
    x = torch.cat([torch.linspace(-125, 9, 2_000_001, device="cuda"),
                   torch.tensor([-float("inf"), -1e30, 0.0], device="cuda")])
    out = torch.empty_like(x)
    G.gqe_exp2_fma(x, out)
    torch.cuda.synchronize()
    ref = torch.exp2(x[:-3].double())
    rel = (out[:-3].double() / ref - 1).abs().max().item()
    assert rel < BOUND, rel
    tail = out[-3:].cpu()
    assert torch.isfinite(tail).all() and (tail[:2] < 3e-38).all() and tail[2].item() == pytest.approx(1.0, rel=BOUND)
