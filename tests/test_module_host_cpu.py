"""Host logic of the PyTorch module (moe_query_head_b200.module) with the library binding
replaced by a CPU stand-in that records its calls: one handle per module, created for the
largest token count seen and re-created only when a call needs more; a backward whose
forward is no longer the handle's last runs that forward again (with the same input)
before gqe_backward; the aux loss's gradient coefficient reaches gqe_backward; a decode
step marks the handle's state as no longer a forward's. The kernels are not involved."""
import pytest
import torch

from moe_query_head_b200 import module as M


class FakeG:
    GQE_BF16 = 0
    VARIANTS = {"gqe": 0, "weighted_concat": 1, "hard_concat": 2}

    def __init__(self):
        self.log = []
        self.next_h = 0

    def gqe_create(self, dim, N, G, k, d_h, dtype, max_tokens):
        self.next_h += 1
        self.log.append(("create", self.next_h, max_tokens))
        return self.next_h

    def gqe_destroy(self, h):
        self.log.append(("destroy", h))

    def gqe_forward(self, h, x, B, T, W_r, W_q, W_k, W_v, W_s, W_o, N, G, k, d_h, variant,
                    causal, out, aux):
        # y = a fixed function of x, so a re-run forward is recognisable by its input
        self.log.append(("forward", h, float(x.float().sum())))
        out.copy_(x.float().mul(2.0).to(out.dtype)[:, : out.shape[1]])
        aux.fill_(0.5)

    def gqe_enable_backward(self, h):
        self.log.append(("enable_backward", h))

    def gqe_backward(self, h, x, B, T, W_r, W_q, W_k, W_v, W_s, W_o, N, G, k, d_h, variant,
                     causal, dy, aux_grad, *grads):
        self.log.append(("backward", h, float(x.float().sum()), aux_grad))
        for g in grads:
            if g is not None:
                g.fill_(1.0)

    def gqe_decode(self, h, x, B, kc, vc, L_max, lengths, W_r, W_q, W_k, W_v, W_s, W_o, N, G,
                   k, d_h, variant, out, aux):
        self.log.append(("decode", h))
        out.zero_()


@pytest.fixture
def fake(monkeypatch):
    f = FakeG()
    monkeypatch.setattr(M, "G", f)
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    return f


@pytest.fixture
def layer(fake):
    """A module factory; every module's stand-in handle is released while the stand-in is
    still installed (a module's __del__ would otherwise pass it to the real library)."""
    made = []

    def make():
        m = M.GQEAttention(dim=16, num_query_experts=4, num_kv_heads=2, top_k=1)
        made.append(m)
        return m

    yield make
    for m in made:
        m._release()


def test_one_handle_grown_only_when_needed(fake, layer):
    m = layer()
    m(torch.randn(1, 8, 16))
    m(torch.randn(2, 3, 16))  # 6 tokens: the 8-token handle serves
    assert [e for e in fake.log if e[0] == "create"] == [("create", 1, 8)]
    m(torch.randn(1, 20, 16))  # 20 tokens: a larger handle replaces it
    assert ("destroy", 1) in fake.log
    assert [e for e in fake.log if e[0] == "create"][-1] == ("create", 2, 20)


def test_backward_reruns_its_forward_when_another_call_intervened(fake, layer):
    m = layer()
    x1 = torch.full((1, 4, 16), 1.0, requires_grad=True)
    x2 = torch.full((1, 4, 16), 3.0)
    y1 = m(x1)
    aux1 = M.collect_aux_loss(m)
    m(x2)  # the handle's state is now x2's forward
    (y1.float().sum() + 0.01 * aux1).backward()
    fwd_x1 = float(x1.detach().to(torch.bfloat16).float().sum())
    tail = fake.log[-3:]
    assert tail[0] == ("forward", 1, fwd_x1)  # x1's forward again, before the backward
    assert tail[1] == ("enable_backward", 1)
    assert tail[2][0] == "backward" and tail[2][2] == fwd_x1
    assert tail[2][3] == pytest.approx(0.01)  # the aux loss's coefficient
    assert x1.grad is not None and torch.all(x1.grad == 1.0)
    assert m.W_q.grad is not None and torch.all(m.W_q.grad == 1.0)


def test_backward_of_the_last_forward_does_not_rerun_it(fake, layer):
    m = layer()
    x = torch.full((1, 4, 16), 1.0, requires_grad=True)
    m(x).float().sum().backward()
    kinds = [e[0] for e in fake.log]
    assert kinds == ["create", "forward", "enable_backward", "backward"]


def test_decode_step_invalidates_the_saved_forward(fake, layer):
    m = layer()
    x = torch.full((1, 4, 16), 1.0, requires_grad=True)
    y = m(x)
    kc, vc = (torch.zeros(2, 1, 8, 4, dtype=torch.bfloat16) for _ in range(2))
    m.decode_step(torch.randn(1, 16), kc, vc, torch.zeros(1, dtype=torch.int32))
    y.float().sum().backward()
    kinds = [e[0] for e in fake.log]
    # the decode step overwrote the handle's state: the forward runs again first
    assert kinds[-4:] == ["decode", "forward", "enable_backward", "backward"]
