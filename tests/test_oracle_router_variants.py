"""Pins of the oracle's general router (the options of the hyper_parallel
TokenChoiceTopKRouter: sigmoid scores, route_scale, selection-only
expert_bias, node-limited group routing) and of score_before_experts.

Each pin is independent of the oracle's code: hand-worked cases with closed
forms, torch library routines in special cases, a pure-Python restatement of
the router's steps on tiny inputs, and invariants."""
import math

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W


def sig(z):
    return 1.0 / (1.0 + math.exp(-z))


def brute_router(row, k, score, scale, bias, groups, topk_groups, renorm):
    """The router's steps for one token, in plain Python."""
    E = len(row)
    if score == "softmax":
        m = max(row)
        ex = [math.exp(v - m) for v in row]
        s = [v / sum(ex) for v in ex]
    else:
        s = [1.0 / (1.0 + math.exp(-v)) for v in row]
    sc = [v * scale for v in s]
    if groups:
        gs = E // groups
        gmax = [max(sc[g * gs:(g + 1) * gs]) for g in range(groups)]
        keep = sorted(range(groups), key=lambda g: (-gmax[g], g))[:topk_groups]
        sc_m = [sc[e] if e // gs in keep else -math.inf for e in range(E)]
    else:
        sc_m = sc
    keys = [sc_m[e] + (bias[e] if bias is not None else 0.0) for e in range(E)]
    idx = sorted(range(E), key=lambda e: (-keys[e], e))[:k]
    w = [s[e] for e in idx]
    if renorm:
        tot = sum(w)
        w = [v / tot for v in w]
    return idx, [v * scale for v in w]


@pytest.mark.parametrize("seed", range(6))
def test_general_router_brute_force(seed):
    rng = np.random.default_rng(seed)
    T, E = 9, 12
    k = int(rng.integers(1, 5))
    L = rng.integers(-3, 4, size=(T, E)).astype(np.float32) * 0.5   # many ties
    score = ["softmax", "sigmoid"][seed % 2]
    scale = [1.0, 2.5, 0.3][seed % 3]
    bias = rng.normal(size=E) * 0.2 if seed % 3 != 0 else None
    groups, tg = [(0, 0), (3, 2), (4, 2), (6, 3)][seed % 4]
    renorm = bool(seed % 2)
    idx, w, counts, _ = O.router_topk_general(k, logits=L, score=score, renormalize=renorm,
                                              route_scale=scale, expert_bias=bias,
                                              num_groups=groups, topk_groups=tg)
    for t in range(T):
        bi, bw = brute_router(L[t].astype(float).tolist(), k, score, scale,
                              None if bias is None else bias.tolist(), groups, tg, renorm)
        assert idx[t].tolist() == bi
        np.testing.assert_allclose(w[t], bw, rtol=1e-13)
    assert counts.sum() == T * k


def test_general_defaults_equal_the_softmax_router():
    L = W.make_logits(50, 16, 4, seed=3)
    for renorm in (False, True):
        a = O.router_topk(4, renorm, logits=L)
        b = O.router_topk_general(4, logits=L, renormalize=renorm)
        assert np.array_equal(a[0], b[0])
        np.testing.assert_allclose(a[1], b[1], rtol=1e-15)


def test_sigmoid_router_matches_torch():
    L = torch.randn(40, 10, dtype=torch.float64, generator=torch.Generator().manual_seed(1))
    idx, w, _, _ = O.router_topk_general(3, logits=L.numpy(), score="sigmoid")
    s = torch.sigmoid(L)
    tv, ti = torch.topk(s, 3, dim=-1)
    assert np.array_equal(idx, ti.numpy())
    np.testing.assert_allclose(w, tv.numpy(), rtol=1e-14)


def test_expert_bias_selects_but_does_not_weigh():
    """E = 4, k = 1, logits [0, 1, 0, 0]: softmax picks expert 1; a bias of
    0.9 on expert 2 makes it win (0.1749 + 0.9 > 0.4754) while its weight stays
    its probability 1 / (3 + e)."""
    L = np.array([[0.0, 1.0, 0.0, 0.0]])
    idx, w, _, _ = O.router_topk_general(1, logits=L)
    assert idx.tolist() == [[1]]
    idx, w, _, _ = O.router_topk_general(1, logits=L, expert_bias=np.array([0, 0, 0.9, 0]))
    assert idx.tolist() == [[2]]
    np.testing.assert_allclose(w, [[1.0 / (3.0 + math.e)]], rtol=1e-15)


def test_node_limited_routing_hand_case():
    """E = 4 in 2 groups {0,1}, {2,3}; sigmoid scores of [3, -5, 2, 2]:
    group maxima sig(3) > sig(2), so only group 0 is kept and the top-2 are
    experts 0 and 1 although experts 2 and 3 score higher than expert 1."""
    L = np.array([[3.0, -5.0, 2.0, 2.0]])
    idx, w, _, _ = O.router_topk_general(2, logits=L, score="sigmoid", num_groups=2,
                                         topk_groups=1)
    assert idx.tolist() == [[0, 1]]
    np.testing.assert_allclose(w, [[sig(3), sig(-5)]], rtol=1e-15)
    idx, _, _, _ = O.router_topk_general(2, logits=L, score="sigmoid", num_groups=2,
                                         topk_groups=2)
    assert idx.tolist() == [[0, 2]]


def test_route_scale_scales_weights_only():
    L = W.make_logits(30, 8, 2, seed=5)
    a = O.router_topk_general(2, logits=L, score="sigmoid", renormalize=True)
    b = O.router_topk_general(2, logits=L, score="sigmoid", renormalize=True, route_scale=2.5)
    assert np.array_equal(a[0], b[0])
    np.testing.assert_allclose(b[1], 2.5 * a[1], rtol=1e-15)


def test_score_before_experts_hand_case():
    """One token x = 1, two scalar experts (FFN_0(z) = silu(z) z,
    FFN_1(z) = -2 silu(z) z), logits [ln 3, 0], k = 2, renormalised weights
    [0.75, 0.25].  Weights after the experts: 0.75 FFN_0(1) + 0.25 FFN_1(1);
    before them: FFN_0(0.75) + FFN_1(0.25)."""
    w1 = np.array([[[1.0]], [[1.0]]])
    w3 = np.array([[[1.0]], [[-1.0]]])
    w2 = np.array([[[1.0]], [[2.0]]])
    L = np.array([[math.log(3.0), 0.0]])
    x = np.array([[1.0]])
    after = O.moe_forward(x, None, w1, w3, w2, 2, True, logits=L)["out"][0, 0]
    before = O.moe_forward(x, None, w1, w3, w2, 2, True, logits=L,
                           score_before_experts=True)["out"][0, 0]
    silu = lambda z: z * sig(z)  # noqa: E731
    assert abs(after - (0.75 * silu(1) - 0.25 * 2 * silu(1))) < 1e-15
    assert abs(before - (silu(0.75) * 0.75 - 2 * silu(0.25) * 0.25)) < 1e-15
