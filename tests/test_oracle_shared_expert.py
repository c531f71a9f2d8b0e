"""Pins of the oracle's shared expert ([HP] MoE.forward adds
shared_expert(x_flat), a dense SwiGLU FeedForward, to the routed output).

Independent of the oracle's code: a hand case with a closed form, a
second formulation through torch.nn.functional, and the layer with a zero
routed part."""
import math

import numpy as np
import torch
import torch.nn.functional as F

import oracle as O


def test_shared_expert_hand_case():
    """One token x = 2 with one scalar routed expert (w1 = w3 = w2 = 1,
    weight 1 after renormalisation) and a scalar shared expert (1, 1, 3):
    out = silu(2)*2 + 3*silu(2)*2 = 8 silu(2) = 16 / (1 + e^-2)."""
    one = np.ones((1, 1, 1))
    x = np.array([[2.0]])
    res = O.moe_forward(x, None, one, one, one, 1, True, logits=np.array([[0.0]]),
                        shared=(np.ones((1, 1)), np.ones((1, 1)), np.full((1, 1), 3.0)))
    assert abs(res["out"][0, 0] - 16.0 / (1.0 + math.exp(-2.0))) < 1e-14


def test_shared_expert_matches_torch_feedforward():
    """The shared part alone equals w2(silu(w1 x) * w3 x) written with
    torch.nn.functional.linear (d != hs so a transposed weight fails)."""
    g = torch.Generator().manual_seed(4)
    T, d, hs, E, k = 9, 6, 10, 4, 2
    x = torch.randn(T, d, generator=g, dtype=torch.float64)
    ws1 = torch.randn(hs, d, generator=g, dtype=torch.float64)
    ws3 = torch.randn(hs, d, generator=g, dtype=torch.float64)
    ws2 = torch.randn(d, hs, generator=g, dtype=torch.float64)
    w1 = torch.randn(E, hs, d, generator=g, dtype=torch.float64)
    w3 = torch.randn(E, hs, d, generator=g, dtype=torch.float64)
    w2 = torch.randn(E, d, hs, generator=g, dtype=torch.float64)
    L = torch.randn(T, E, generator=g, dtype=torch.float64).numpy()
    res = O.moe_forward(x.numpy(), None, w1.numpy(), w3.numpy(), w2.numpy(), k, True, logits=L,
                        shared=(ws1.numpy(), ws3.numpy(), ws2.numpy()))
    ref = F.linear(F.silu(F.linear(x, ws1)) * F.linear(x, ws3), ws2).numpy()
    np.testing.assert_allclose(res["shared_out"], ref, rtol=1e-12, atol=1e-12)
    plain = O.moe_forward(x.numpy(), None, w1.numpy(), w3.numpy(), w2.numpy(), k, True, logits=L)
    np.testing.assert_allclose(res["out"] - plain["out"], ref, rtol=1e-11, atol=1e-11)


def test_shared_expert_with_zero_routed_experts():
    """Routed experts with w2 = 0 contribute nothing: the layer output is
    the shared expert's alone."""
    rng = np.random.default_rng(2)
    T, d, h, E, k = 7, 4, 8, 3, 2
    x = rng.normal(size=(T, d))
    w1 = rng.normal(size=(E, h, d))
    w3 = rng.normal(size=(E, h, d))
    w2 = np.zeros((E, d, h))
    ws = (rng.normal(size=(5, d)), rng.normal(size=(5, d)), rng.normal(size=(d, 5)))
    res = O.moe_forward(x, None, w1, w3, w2, k, True, logits=rng.normal(size=(T, E)), shared=ws)
    xt = torch.from_numpy(x)
    ref = F.linear(F.silu(F.linear(xt, torch.from_numpy(ws[0]))) * F.linear(xt, torch.from_numpy(ws[1])),
                   torch.from_numpy(ws[2])).numpy()
    np.testing.assert_allclose(res["out"], ref, rtol=1e-12, atol=1e-12)
