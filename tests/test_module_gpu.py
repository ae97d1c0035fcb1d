"""The PyTorch module (moe_query_head_b200.module: GQEAttention with the README's
constructor, y = attn(x), collect_aux_loss, loss.backward()) against the float64 oracle: y
at the bf16 tolerances, and through autograd the gradients of <dy, y> + 0.01 aux for x and
every weight within the backward tests' rel-L2 1e-2. Also: a backward whose forward is no
longer the handle's last (the module called again in between) gives the same gradients, and
collect_aux_loss sums the layers of a model."""
import numpy as np
import pytest
import torch

from moe_query_head_b200 import workloads as W
from moe_query_head_b200.module import GQEAttention, collect_aux_loss
from tests.gqe_testlib import check_output, oracle_forward, rel_l2

pytestmark = pytest.mark.gpu

GRAD_REL_L2 = 1e-2
NAMES = ("W_r", "W_q", "W_k", "W_v", "W_shared", "W_o")
MAIN = W.WORKLOADS["main_b8_t2048"]
WIDE = W.WORKLOADS["wide_k2"]


def _module(wl, inp):
    m = GQEAttention(wl.dim, wl.N, wl.G, wl.k, wl.d_h, wl.variant, shared=wl.shared,
                     causal=wl.causal).cuda()
    with torch.no_grad():
        for n in NAMES:
            if getattr(m, n) is not None:
                getattr(m, n).copy_(torch.from_numpy(inp.f64(n)).float())
    return m


def _x(wl, inp):
    return torch.from_numpy(inp.f64("x")).float().view(wl.B, wl.T, wl.dim).cuda()


def _oracle_backward(wl, inp, dy, dA=0.01):
    import oracle
    f = inp.f64
    layer = oracle.Layer(dim=wl.dim, N=wl.N, G=wl.G, k=wl.k, d_h=wl.d_h, shared=wl.shared,
                         variant=wl.variant, causal=wl.causal)
    return oracle.backward(layer, f("x"), wl.B, wl.T, f("W_r"), f("W_q"), f("W_k"), f("W_v"),
                           f("W_shared"), f("W_o"), dy.astype(np.float64), dA)


def _grads(m, x):
    g = {"x": x.grad.reshape(-1, x.shape[-1]).double().cpu().numpy()}
    for n in NAMES:
        p = getattr(m, n)
        g[n] = None if p is None else p.grad.double().cpu().numpy()
    return g


@pytest.mark.parametrize("wl", [MAIN.with_(B=2, T=200), WIDE.with_(B=1, T=260,
                                                                   variant="weighted_concat"),
                                MAIN.with_(B=1, T=150, shared=False, variant="hard_concat")],
                         ids=["main_gqe", "wide_weighted", "main_hard_no_shared"])
def test_module_forward_and_backward_match_the_oracle(wl):
    inp = W.generate(wl)
    m = _module(wl, inp)
    x = _x(wl, inp).requires_grad_()
    y = m(x)
    ref = oracle_forward(inp)
    check_output(y.detach().reshape(wl.M, wl.dim).double().cpu().numpy(), ref.y, "bf16")
    dy_h = W.grad_output(wl)
    dy = torch.from_numpy(dy_h).float().view(wl.B, wl.T, wl.dim).cuda()
    loss = (y.float() * dy).sum() + 0.01 * collect_aux_loss(m)
    loss.backward()
    got = _grads(m, x)
    ref_g = _oracle_backward(wl, inp, dy_h)
    errs = {}
    for n in ("x",) + NAMES:
        r = getattr(ref_g, n)
        if r is None:
            assert got[n] is None
            continue
        assert np.isfinite(got[n]).all(), n
        errs[n] = rel_l2(got[n], r)
    assert all(e <= GRAD_REL_L2 for e in errs.values()), errs


def test_module_backward_after_another_call():
    """Two calls, then the backward of the first: the handle's saved state is the second
    call's, so the first is run again before its backward; its gradients match the oracle."""
    wl = MAIN.with_(B=1, T=200)
    inp = W.generate(wl)
    m = _module(wl, inp)
    x = _x(wl, inp).requires_grad_()
    y1 = m(x)
    m(torch.randn_like(x))  # a second call on the same handle
    dy_h = W.grad_output(wl)
    dy = torch.from_numpy(dy_h).float().view(wl.B, wl.T, wl.dim).cuda()
    (y1.float() * dy).sum().backward()
    got = _grads(m, x)
    ref_g = _oracle_backward(wl, inp, dy_h, dA=0.0)  # the loss has no aux term
    for n in ("x",) + NAMES:
        assert rel_l2(got[n], getattr(ref_g, n)) <= GRAD_REL_L2, n


def test_collect_aux_loss_sums_the_layers():
    wl = MAIN.with_(B=1, T=130)
    inp = W.generate(wl)
    m1, m2 = _module(wl, inp), _module(wl, inp)
    model = torch.nn.Sequential(m1, m2)
    x = _x(wl, inp)
    model(x)
    a = collect_aux_loss(model)
    assert torch.allclose(a, m1.aux_loss() + m2.aux_loss())
    ref_aux = oracle_forward(inp).aux
    assert abs(float(m1.aux_loss().detach()) - ref_aux) <= 1e-4 * ref_aux


def test_module_decode_step_matches_the_oracle():
    """GQEAttention.decode_step over caches filled for a few sequences: y_new at the bf16
    tolerances against the oracle's decode step, the new K / V written at the positions."""
    from tests.test_decode_gpu import _dev_bf16, oracle_decode
    wl = MAIN
    d = W.generate_decode(wl, [0, 37, 200], 256)
    inp = d.inp
    m = _module(inp.wl, inp)
    kc, vc = _dev_bf16(d.k_cache), _dev_bf16(d.v_cache)
    lens = torch.from_numpy(d.lengths.astype(np.int32)).cuda()
    x_new = torch.from_numpy(inp.f64("x")).float().cuda()
    y = m.decode_step(x_new, kc, vc, lens)
    ref = oracle_decode(d)
    check_output(y.double().cpu().numpy(), ref.y, "bf16")
    for b, L in enumerate(d.lengths.tolist()):
        np.testing.assert_allclose(kc[:, b, L].double().cpu().numpy(), ref.K_new[:, b],
                                   rtol=1e-2, atol=1e-2)
