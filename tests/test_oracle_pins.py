"""Pins of the fp64 CPU oracle against facts that do not come from the oracle.

Each test checks one oracle function against something independent of its
code: a hand-worked case whose expected values are closed forms, a brute-force
pure-Python restatement on tiny inputs, a different library routine in a
special case, an invariant, or a second formulation printed on the pages
(the dense all-experts branch of ``SpeedupMoeExperts.forward``, QwenLM/Qwen3-Omni
issue #115).  The cases are picked so that a dropped term, a swapped operand,
a wrong sign or an off-by-one index in the oracle fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def sig(z):
    return 1.0 / (1.0 + math.exp(-z))


# ---------------------------------------------------------------- hand cases

def test_hand_case_top1():
    """4 tokens, 2 experts, k = 1 (worked by hand)."""
    L = np.array([[1, 0], [0, 1], [0, 2], [3, 0]], dtype=np.float32)
    idx, w, counts, _ = O.router_topk(1, False, logits=L)
    assert idx.ravel().tolist() == [0, 1, 1, 0]
    assert counts.tolist() == [2, 2]
    np.testing.assert_allclose(w.ravel(), [sig(1), sig(1), sig(2), sig(3)], rtol=1e-15)
    _, w_rn, _, _ = O.router_topk(1, True, logits=L)
    assert np.all(w_rn == 1.0)
    c, off, src, dst = O.dispatch(idx, 2)
    assert off.tolist() == [0, 2, 4]
    assert src.tolist() == [0, 3, 1, 2]
    assert dst.ravel().tolist() == [0, 2, 3, 1]


def test_hand_case_top2_ties_and_layer():
    """4 tokens, 2 experts, k = 2, equal logits; d = h = 1 scalar experts."""
    l3 = math.log(3.0)
    L = np.array([[0, 0], [l3, 0], [0, l3], [0, 0]], dtype=np.float64)
    idx, w, counts, _ = O.router_topk(2, True, logits=L)
    assert idx.tolist() == [[0, 1], [0, 1], [1, 0], [0, 1]]      # tie -> index 0 first
    np.testing.assert_allclose(w, [[.5, .5], [.75, .25], [.75, .25], [.5, .5]], rtol=1e-15)
    c, off, src, dst = O.dispatch(idx, 2)
    assert c.tolist() == [4, 4] and off.tolist() == [0, 4, 8]
    assert src.tolist() == [0, 1, 2, 3, 0, 1, 2, 3]
    assert dst.tolist() == [[0, 4], [1, 5], [6, 2], [3, 7]]
    # expert 0: w1=1, w3=1, w2=1 -> silu(x) x ; expert 1: w1=1, w3=-1, w2=2 -> -2 silu(x) x
    w1 = np.array([[[1.0]], [[1.0]]])
    w3 = np.array([[[1.0]], [[-1.0]]])
    w2 = np.array([[[1.0]], [[2.0]]])
    x = np.array([[1.0], [2.0], [-1.0], [0.0]])
    res = O.moe_forward(x, None, w1, w3, w2, 2, True, logits=L)
    s1, s2, sm1 = 1 * sig(1), 2 * sig(2), -1 * sig(-1)     # silu values
    expect = [0.5 * s1 * 1 - 0.5 * 2 * s1 * 1,
              0.75 * s2 * 2 - 0.25 * 2 * s2 * 2,
              0.75 * (-2 * sm1 * -1) + 0.25 * (sm1 * -1),
              0.0]
    np.testing.assert_allclose(res["out"].ravel(), expect, rtol=1e-14, atol=1e-300)
    np.testing.assert_allclose(res["out"].ravel(),
                               [-0.36552929, 0.88079708, -0.33617678, 0.0], atol=5e-9)


def test_hand_case_regroup():
    """G=1, R=2, L=2, counts_rm [[1,2],[2,1]] (worked by hand)."""
    perm, cem, oem = O.ep_local_regroup(np.array([[[1, 2], [2, 1]]]))
    assert perm.tolist() == [0, 3, 4, 1, 2, 5]
    assert cem.tolist() == [3, 3] and oem.tolist() == [0, 3, 6]


# ---------------------------------------------------------------- brute force

def _brute_topk(row, k):
    return [e for e, _ in sorted(enumerate(row), key=lambda p: (-p[1], p[0]))][:k]


def _brute_dispatch(idx, E, k):
    T = len(idx)
    counts = [0] * E
    for t in range(T):
        for j in range(k):
            counts[idx[t][j]] += 1
    offsets = [0]
    for e in range(E):
        offsets.append(offsets[-1] + counts[e])
    seen = [0] * E
    src = [None] * (T * k)
    dst = [[None] * k for _ in range(T)]
    for t in range(T):              # flat index t*k + j, increasing
        for j in range(k):
            e = idx[t][j]
            s = offsets[e] + seen[e]
            seen[e] += 1
            src[s] = t
            dst[t][j] = s
    return counts, offsets, src, dst


@pytest.mark.parametrize("T,E,k,seed", [(1, 1, 1, 0), (7, 3, 2, 1), (33, 8, 3, 2),
                                        (50, 16, 16, 3), (0, 4, 2, 4)])
def test_router_and_dispatch_brute_force(T, E, k, seed):
    rng = np.random.default_rng(seed)
    # few distinct values -> many ties
    L = rng.integers(-2, 3, size=(T, E)).astype(np.float32)
    idx, w, counts, _ = O.router_topk(k, True, logits=L)
    for t in range(T):
        assert idx[t].tolist() == _brute_topk(L[t].tolist(), k)
    c, off, src, dst = O.dispatch(idx.reshape(T, k), E)
    bc, boff, bsrc, bdst = _brute_dispatch(idx.tolist(), E, k)
    assert c.tolist() == bc and off.tolist() == boff
    assert src.tolist() == bsrc and dst.tolist() == bdst


def test_regroup_brute_force():
    rng = np.random.default_rng(5)
    G, R, L = 3, 4, 5
    c = rng.integers(0, 4, size=(G, R, L))
    perm, cem, oem = O.ep_local_regroup(c)
    # brute: label every input row with its (g, r, l), then sort by (g, l, r, row)
    labels = []
    for g in range(G):
        for r in range(R):
            for l in range(L):
                labels += [(g, l, r)] * int(c[g, r, l])
    order = sorted(range(len(labels)), key=lambda i: (labels[i], i))
    assert perm.tolist() == order
    assert cem.tolist() == [int(c[g, :, l].sum()) for g in range(G) for l in range(L)]


# ------------------------------------------------- second formulation (dense)

def _small_layer(T, d, E, k, h, seed, dtype=torch.float32):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, d, generator=g).to(dtype)
    wr = (torch.randn(E, d, generator=g) * 0.5).to(dtype)
    w1 = (torch.randn(E, h, d, generator=g) / math.sqrt(d)).to(dtype)
    w3 = (torch.randn(E, h, d, generator=g) / math.sqrt(d)).to(dtype)
    w2 = (torch.randn(E, d, h, generator=g) / math.sqrt(h)).to(dtype)
    return x, wr, w1, w3, w2


def test_dense_formulation_matches_loop_cfg0():
    cfg = W.config(0)
    lay = W.make_layer(cfg, "cpu")
    res = O.moe_forward(lay["x"], lay["w_router"], lay["w1"], lay["w3"], lay["w2"],
                        cfg.top_k, cfg.renormalize)
    dense = O.dense_moe(lay["x"], res["topk_idx"], res["topk_w"], lay["w1"], lay["w3"],
                        lay["w2"])
    err = np.linalg.norm(res["out"] - dense) / np.linalg.norm(dense)
    assert err < 1e-12


@pytest.mark.parametrize("ep", [1, 4])
def test_dense_and_token_formulations_bf16(ep):
    x, wr, w1, w3, w2 = _small_layer(40, 32, 8, 3, 48, 7, torch.bfloat16)
    res = O.moe_forward(x, wr, w1, w3, w2, 3, False, ep_ranks=ep)
    dense = O.dense_moe(x, res["topk_idx"], res["topk_w"], w1, w3, w2)
    tok = O.moe_tokens(x, res["topk_idx"], res["topk_w"], w1, w3, w2)
    assert np.linalg.norm(res["out"] - dense) / np.linalg.norm(dense) < 1e-12
    assert np.linalg.norm(tok - dense) / np.linalg.norm(dense) < 1e-12


# ------------------------------------------- special cases = library routines

@pytest.mark.parametrize("d,h", [(16, 24), (20, 20)])
def test_single_expert_is_feedforward(d, h):
    """E = 1, k = 1: the layer is the SwiGLU FeedForward w2(silu(w1 x) * w3 x)
    (hyper_parallel FeedForward.forward); checked with torch.nn.functional in
    float64.  d == h makes a transposed weight fail numerically, not by shape."""
    x, wr, w1, w3, w2 = _small_layer(9, d, 1, 1, h, 11, torch.float64)
    res = O.moe_forward(x, wr, w1, w3, w2, 1, True)
    F = torch.nn.functional
    ref = F.linear(F.silu(F.linear(x, w1[0])) * F.linear(x, w3[0]), w2[0])
    np.testing.assert_allclose(res["out"], ref.numpy(), rtol=1e-12, atol=1e-13)
    assert np.all(res["topk_w"] == 1.0)


def test_router_matches_torch_topk_softmax():
    """Distinct scores: indices equal torch.topk's, weights equal torch.softmax
    gathered (and renormalised like norm_topk_prob)."""
    x, wr, *_ = _small_layer(64, 24, 16, 4, 8, 13, torch.float64)
    idx, w, counts, L = O.router_topk(4, False, x=x, w_router=wr)
    lt = torch.nn.functional.linear(x, wr)
    np.testing.assert_allclose(L, lt.numpy(), rtol=1e-13, atol=1e-13)
    p = torch.softmax(lt, dim=-1)
    tv, ti = torch.topk(p, 4, dim=-1)
    assert (idx == ti.numpy()).all()
    np.testing.assert_allclose(w, tv.numpy(), rtol=1e-13)
    _, wn, _, _ = O.router_topk(4, True, x=x, w_router=wr)
    np.testing.assert_allclose(wn, (tv / tv.sum(-1, keepdim=True)).numpy(), rtol=1e-13)
    assert counts.tolist() == torch.bincount(ti.flatten(), minlength=16).tolist()


def test_k_equals_E_renorm_is_full_softmax():
    L = np.random.default_rng(3).standard_normal((10, 6)).astype(np.float32)
    idx, w, _, _ = O.router_topk(6, True, logits=L)
    full = torch.softmax(torch.from_numpy(L).double(), -1).numpy()
    np.testing.assert_allclose(w, np.take_along_axis(full, idx, 1), rtol=1e-13)


def test_huge_bias_sends_all_tokens_to_one_expert():
    L = np.random.default_rng(4).standard_normal((50, 8)).astype(np.float32)
    L[:, 5] += 1e4
    idx, w, counts, _ = O.router_topk(1, True, logits=L)
    assert (idx[:, 0] == 5).all() and counts[5] == 50


# ---------------------------------------------------------------- invariants

@pytest.mark.parametrize("seed", [0, 1])
def test_dispatch_invariants(seed):
    T, E, k = 300, 12, 4
    L = W.make_logits(T, E, k, seed)
    idx, w, counts, _ = O.router_topk(k, True, logits=L)
    c, off, src, dst = O.dispatch(idx, E)
    assert c.sum() == T * k and off[E] == T * k and np.all(np.diff(off) >= 0)
    assert sorted(dst.ravel().tolist()) == list(range(T * k))      # bijection
    flat = np.empty(T * k, dtype=np.int64)
    flat[dst.ravel()] = np.arange(T * k)                           # slot -> flat
    assert np.array_equal(src, flat // k)
    for e in range(E):
        seg = flat[off[e]:off[e + 1]]
        assert np.all(idx.ravel()[seg] == e) and np.all(np.diff(seg) > 0)
    np.testing.assert_allclose(w.sum(1), 1.0, rtol=0, atol=4 * np.finfo(np.float64).eps)


@pytest.mark.parametrize("k", [1, 2, 4, 8])
def test_combine_after_dispatch_is_identity(k):
    """Identity experts (y = x_perm) with weights 1/k give back x exactly."""
    x = torch.randn(37, 16, generator=torch.Generator().manual_seed(k)).to(torch.bfloat16)
    L = W.make_logits(37, 8, k, k)
    idx, *_ = O.router_topk(k, True, logits=L)
    c, off, src, dst = O.dispatch(idx, 8)
    xp = O.permute_rows(x, src)
    out = O.combine(xp, dst, np.full((37, k), 1.0 / k))
    assert np.array_equal(out, O.as_f64(x))


def test_ep_layout_then_regroup_equals_global_dispatch():
    """Per-source-rank dispatch, rank-major concatenation and the local regroup
    reproduce the single-device expert-major order bit for bit."""
    T, E, k, R = 203, 16, 3, 4
    L = W.make_logits(T, E, k, 9)
    idx, *_ = O.router_topk(k, True, logits=L)
    c, off, src, dst = O.dispatch(idx, E)
    crm, src_rm, dst_rm = O.ep_dispatch_rank_major(idx, E, R)
    assert crm.sum() == T * k
    perm, cem, oem = O.ep_local_regroup(crm)
    assert np.array_equal(src_rm[perm], src)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(len(perm))
    assert np.array_equal(inv[dst_rm], dst)
    assert np.array_equal(cem, c) and np.array_equal(oem, off)


# ---------------------------------------------------------- golden contracts

def test_docstring_shape_contracts():
    g = json.load(open(os.path.join(GOLDEN, "shape_contracts.json")))
    ge = g["grouped_experts"]
    x, _, w1, w3, w2 = _small_layer(10, ge["dim"], ge["num_experts"], 1, ge["hidden_dim"], 1)
    off = np.concatenate([[0], np.cumsum(ge["counts"])])
    assert O.grouped_swiglu(x, off, w1, w3, w2).shape == tuple(ge["out_shape"])
    r = g["router"]
    x, wr, *_ = _small_layer(r["x_shape"][0], r["dim"], r["num_experts"], r["top_k"], 4, 2)
    idx, w, counts, _ = O.router_topk(r["top_k"], False, x=x, w_router=wr)
    assert w.shape == tuple(r["scores_shape"]) and idx.shape == tuple(r["indices_shape"])
    assert counts.shape == tuple(r["counts_shape"])
    m = g["moe"]
    B, S, D = m["x_shape"]
    x, wr, w1, w3, w2 = _small_layer(B * S, D, m["num_experts"], m["top_k"], m["hidden_dim"], 3)
    out = O.moe_forward(x, wr, w1, w3, w2, m["top_k"])["out"].reshape(B, S, D)
    assert out.shape == tuple(m["out_shape"])


def test_zero_tokens_is_empty():
    _, wr, w1, w3, w2 = _small_layer(1, 8, 4, 2, 8, 0)
    res = O.moe_forward(torch.zeros(0, 8), wr, w1, w3, w2, 2)
    assert res["out"].shape == (0, 8) and res["counts"].tolist() == [0, 0, 0, 0]
    assert res["offsets"].tolist() == [0] * 5


# ---------------------------------------------------------- workload recipe

def test_zipf_workload_is_skewed():
    """The skewed workload has empty experts and a max load above 10x mean."""
    cfg = W.config(2)
    lay = W.make_layer(cfg, "cpu", experts=False)
    idx, _, counts, _ = O.router_topk(cfg.top_k, True, x=lay["x"], w_router=lay["w_router"])
    mean = cfg.N / cfg.E
    assert (counts == 0).sum() >= 2 and counts.max() > 10 * mean


def test_make_logits_gap():
    L = W.make_logits(500, 32, 8, 1).astype(np.float64)
    s = -np.sort(-L, axis=1)
    assert np.all(s[:, 7] - s[:, 8] >= 1e-3)
