"""Pins of the oracle's capacity drop policy ([PF] PaddleFormers moe_gate.py,
_probs_drop_policy) and of the dispatch and combine of dropped copies.

Pins that do not restate the oracle's sort:
* a rank-by-counting formulation (a copy is kept when fewer than
  `capacity` copies of its expert beat it: a higher score, or the same
  score and a lower token);
* closed forms: capacity >= the largest count keeps everything, capacity 0
  keeps nothing, an expert keeps min(count, capacity) copies;
* a hand case with ties;
* the layer with dropped copies equals the token-by-token definition with
  those copies' weights set to zero.
"""
import numpy as np
import pytest

import oracle as O
import workloads as W


def keep_by_counting(idx, s, capacity):
    T, k = idx.shape
    keep = np.zeros((T, k), dtype=bool)
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            beaten = 0
            for u in range(T):
                for i in range(k):
                    if idx[u, i] == e and (s[u, i] > s[t, j] or (s[u, i] == s[t, j] and u < t)):
                        beaten += 1
            keep[t, j] = beaten < capacity
    return keep


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("capacity", [1, 2, 3, 5])
def test_capacity_matches_rank_by_counting(seed, capacity):
    rng = np.random.default_rng(seed)
    T, E, k = 13, 5, 2
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)])
    s = rng.integers(0, 4, size=(T, k)).astype(np.float64) / 4.0   # many exact ties
    assert np.array_equal(O.capacity_drop(idx, s, capacity), keep_by_counting(idx, s, capacity))


def test_capacity_closed_forms():
    rng = np.random.default_rng(3)
    T, E, k = 40, 6, 3
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)])
    s = rng.random((T, k))
    counts = np.bincount(idx.ravel(), minlength=E)
    assert O.capacity_drop(idx, s, int(counts.max())).all()
    assert not O.capacity_drop(idx, s, 0).any()
    for cap in (1, 4, 9, 17):
        keep = O.capacity_drop(idx, s, cap)
        kept = np.bincount(idx[keep], minlength=E)
        assert np.array_equal(kept, np.minimum(counts, cap))


def test_capacity_hand_case_with_ties():
    # four tokens route to expert 1 with scores .5 .9 .5 .9; capacity 3 keeps
    # the two .9 and the first .5 (token 0), drops token 2's copy
    idx = np.array([[1, 0], [1, 2], [1, 0], [1, 2]])
    s = np.array([[.5, .1], [.9, .2], [.5, .3], [.9, .4]])
    keep = O.capacity_drop(idx, s, 3)
    assert keep[:, 0].tolist() == [True, True, False, True]
    assert keep[:, 1].all()


def test_router_with_capacity_marks_dropped_copies():
    T, E, k = 200, 8, 2
    L = W.make_logits(T, E, k, seed=4)
    L[:, 3] += 2.0                     # expert 3 overloaded
    idx0, w0, c0, _ = O.router_topk_general(k, logits=L, renormalize=True)
    cap = int(c0.max()) - 10
    idx, w, c, _ = O.router_topk_general(k, logits=L, renormalize=True, capacity=cap)
    dropped = idx < 0
    assert dropped.sum() == np.maximum(c0 - cap, 0).sum() > 0
    assert np.array_equal(idx[~dropped], idx0[~dropped])
    assert np.array_equal(w[~dropped], w0[~dropped]) and not w[dropped].any()
    assert np.array_equal(c, np.minimum(c0, cap))


def test_dispatch_and_combine_skip_dropped_copies():
    idx = np.array([[2, -1], [0, 2], [-1, 1], [1, 0]])
    counts, off, src, dst = O.dispatch(idx, 3)
    assert counts.tolist() == [2, 2, 2] and off.tolist() == [0, 2, 4, 6]
    assert src.tolist() == [1, 3, 2, 3, 0, 1]
    assert dst.tolist() == [[4, -1], [0, 5], [-1, 2], [3, 1]]
    y = np.arange(6, dtype=np.float64)[:, None] * np.ones((1, 2))
    out = O.combine(y, dst, np.full((4, 2), 2.0))
    assert out[:, 0].tolist() == [8.0, 10.0, 4.0, 8.0]


def test_layer_with_capacity_equals_zero_weight_definition():
    rng = np.random.default_rng(7)
    T, d, E, k, h = 60, 16, 6, 2, 12
    x = rng.standard_normal((T, d))
    wr = rng.standard_normal((E, d))
    w1 = rng.standard_normal((E, h, d)) / 4
    w3 = rng.standard_normal((E, h, d)) / 4
    w2 = rng.standard_normal((E, d, h)) / 4
    ro = dict(score="softmax", capacity=12)
    res = O.moe_forward(x, wr, w1, w3, w2, k, True, router=ro)
    idx, w = res["topk_idx"], res["topk_w"]
    assert (idx < 0).any()
    ref = O.moe_tokens(x, np.where(idx < 0, 0, idx), np.where(idx < 0, 0.0, w), w1, w3, w2)
    assert np.allclose(res["out"], ref, rtol=1e-12, atol=1e-12)
