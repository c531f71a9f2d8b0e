"""Pins of the oracle's load-balance loss (hyper_parallel
_compute_load_balance_loss: E * sum_e f_e P_e).  Closed forms: a perfectly
balanced router gives exactly 1 (the page's own statement of the balanced
value), a router that sends every copy to one expert with weight 1 gives E;
a vectorised restatement with numpy bincount; the empty input gives 0.
The gradient with respect to the routing weights is pinned by central finite
differences of the loss itself (it is linear in the weights) and by the
balanced closed form."""
import numpy as np

import oracle as O
import workloads as W


def test_balanced_router_gives_one():
    # T = 8 tokens, k = 2, E = 4: every expert receives 4 copies, weights 1/2
    idx = np.array([[t % 4, (t + 1) % 4] for t in range(8)])
    w = np.full((8, 2), 0.5)
    assert abs(O.load_balance_loss(w, idx, 4) - 1.0) < 1e-15


def test_collapsed_router_gives_E():
    idx = np.zeros((5, 1), dtype=np.int64)
    w = np.ones((5, 1))
    assert abs(O.load_balance_loss(w, idx, 7) - 7.0) < 1e-15


def test_matches_bincount_formulation():
    L = W.make_logits(300, 16, 4, seed=9)
    idx, w, counts, _ = O.router_topk(4, True, logits=L)
    f = np.bincount(idx.ravel(), minlength=16) / (300 * 4)
    p = np.bincount(idx.ravel(), weights=w.ravel(), minlength=16) / 300
    assert abs(O.load_balance_loss(w, idx, 16) - 16 * np.dot(f, p)) < 1e-12


def test_empty_input():
    assert O.load_balance_loss(np.zeros((0, 2)), np.zeros((0, 2), dtype=np.int64), 4) == 0.0


def test_gradient_matches_finite_differences():
    L = W.make_logits(40, 8, 3, seed=4)
    idx, w, _, _ = O.router_topk(3, True, logits=L)
    g = O.load_balance_loss_grad(idx, 8)
    h = 1e-3
    for t, j in [(0, 0), (5, 2), (17, 1), (39, 0)]:
        wp, wm = w.copy(), w.copy()
        wp[t, j] += h
        wm[t, j] -= h
        fd = (O.load_balance_loss(wp, idx, 8) - O.load_balance_loss(wm, idx, 8)) / (2 * h)
        assert abs(fd - g[t, j]) < 1e-10


def test_gradient_of_the_balanced_router():
    # balanced: f_e = 1/E for every expert, so every entry is 1/T
    idx = np.array([[t % 4, (t + 1) % 4] for t in range(8)])
    g = O.load_balance_loss_grad(idx, 4)
    assert np.allclose(g, 1.0 / 8, rtol=0, atol=1e-15)
