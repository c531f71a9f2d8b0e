"""Pins of the oracle's backward (the derivative of the layer forward that
[HP] MoE.forward / _run_experts_for_loop and the [QO] training branch
compute, needed by the training path).

None of these re-derives the chain rule the oracle writes out: central
finite differences of the oracle's own (separately pinned) forward, the
same gradients through torch autograd in fp64, the adjoint identity of the
row gather and its scatter-add, and closed forms."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as O
import workloads as W


def _problem(seed=0, N=9, d=5, h=4, E=3, empty=1):
    rng = np.random.default_rng(seed)
    counts = rng.multinomial(N, np.ones(E) / E)
    if empty is not None:
        counts[empty] = 0
        counts[(empty + 1) % E] += N - counts.sum()
    off = np.concatenate([[0], np.cumsum(counts)])
    xp = rng.standard_normal((N, d))
    w1 = rng.standard_normal((E, h, d)) * 0.7
    w3 = rng.standard_normal((E, h, d)) * 0.7
    w2 = rng.standard_normal((E, d, h)) * 0.7
    dy = rng.standard_normal((N, d))
    return xp, off, w1, w3, w2, dy


def _fd(f, a, eps=1e-6):
    """Central differences of the scalar f() in every entry of array a."""
    g = np.zeros_like(a)
    it = np.nditer(a, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = a[i]
        a[i] = old + eps
        fp = f()
        a[i] = old - eps
        fm = f()
        a[i] = old
        g[i] = (fp - fm) / (2 * eps)
    return g


def test_silu_grad_closed_forms():
    """silu'(0) = 1/2, silu'(z) -> 1 for large z and -> 0 for very negative
    z, and agreement with a central difference of silu at a few points."""
    assert O.silu_grad(0.0) == 0.5
    assert abs(O.silu_grad(40.0) - 1.0) < 1e-15
    assert abs(O.silu_grad(-60.0)) < 1e-20
    for z in [-3.0, -0.7, 0.3, 2.5]:
        fd = (O.silu(z + 1e-6) - O.silu(z - 1e-6)) / 2e-6
        assert abs(O.silu_grad(z) - fd) < 1e-9
    # the minimum of silu: silu'(z*) = 0 at z* = -1.27846454276...
    assert abs(O.silu_grad(-1.2784645427610738)) < 1e-12


def test_grouped_swiglu_backward_matches_finite_differences():
    """Every gradient (x_perm, w1, w3, w2) against central differences of
    L = <dy, grouped_swiglu(...)>; one expert is empty (zero gradients)."""
    xp, off, w1, w3, w2, dy = _problem()
    dxp, dw1, dw3, dw2 = O.grouped_swiglu_backward(xp, off, w1, w3, w2, dy)

    def loss():
        return float(np.sum(dy * O.grouped_swiglu(xp, off, w1, w3, w2)))

    for got, a in [(dxp, xp), (dw1, w1), (dw3, w3), (dw2, w2)]:
        ref = _fd(loss, a)
        assert np.max(np.abs(got - ref)) < 1e-6 * (1 + np.max(np.abs(ref))), got.shape
    assert not dw1[1].any() and not dw3[1].any() and not dw2[1].any()


def test_grouped_swiglu_backward_matches_torch_autograd():
    """Same gradients through torch autograd (fp64) on a larger case with
    ragged segments: a second, library route to the derivative."""
    xp, off, w1, w3, w2, dy = _problem(seed=3, N=40, d=16, h=12, E=5, empty=2)
    t = [torch.tensor(a, requires_grad=True) for a in (xp, w1, w3, w2)]
    outs = []
    for e in range(len(off) - 1):
        lo, hi = int(off[e]), int(off[e + 1])
        S = t[0][lo:hi]
        outs.append(F.linear(F.silu(F.linear(S, t[1][e])) * F.linear(S, t[2][e]), t[3][e]))
    torch.sum(torch.cat(outs) * torch.tensor(dy)).backward()
    got = O.grouped_swiglu_backward(xp, off, w1, w3, w2, dy)
    for g, tt in zip(got, t):
        np.testing.assert_allclose(g, tt.grad.numpy(), rtol=1e-11, atol=1e-11)


def test_grouped_preactivations_rebuild_the_forward():
    """silu(G) * U followed by each expert's w2 is the grouped SwiGLU."""
    xp, off, w1, w3, w2, _ = _problem(seed=5, N=20, d=6, h=8, E=4, empty=0)
    G, U = O.grouped_preactivations(xp, off, w1, w3)
    A = O.silu(G) * U
    y = np.zeros((xp.shape[0], w2.shape[1]))
    for e in range(4):
        lo, hi = int(off[e]), int(off[e + 1])
        y[lo:hi] = A[lo:hi] @ w2[e].T
    np.testing.assert_allclose(y, O.grouped_swiglu(xp, off, w1, w3, w2), rtol=1e-12, atol=1e-12)


def test_combine_backward_matches_finite_differences():
    rng = np.random.default_rng(7)
    T, k, d, E = 6, 3, 4, 5
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)])
    _, _, _, dst_pos = O.dispatch(idx, E)
    N = T * k
    y = rng.standard_normal((N, d))
    w = rng.random((T, k))
    dout = rng.standard_normal((T, d))
    dy, dw = O.combine_backward(dout, y, dst_pos, w)

    def loss():
        return float(np.sum(dout * O.combine(y, dst_pos, w)))

    np.testing.assert_allclose(dy, _fd(loss, y), atol=1e-8)
    np.testing.assert_allclose(dw, _fd(loss, w), atol=1e-8)
    dy1, dw1 = O.combine_backward(dout, y, dst_pos, None)
    assert dw1 is None
    np.testing.assert_allclose(dy1[dst_pos[2, 1]], dout[2], rtol=0, atol=0)


def test_dispatch_backward_is_the_adjoint_of_the_gather():
    """<dx_perm, x[src_row]> = <dispatch_backward(dx_perm), x> for all x."""
    rng = np.random.default_rng(11)
    T, k, d, E = 9, 2, 7, 4
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)])
    _, _, src_row, dst_pos = O.dispatch(idx, E)
    x = rng.standard_normal((T, d))
    g = rng.standard_normal((T * k, d))
    lhs = float(np.sum(g * O.permute_rows(x, src_row)))
    rhs = float(np.sum(O.dispatch_backward(g, dst_pos) * x))
    assert abs(lhs - rhs) < 1e-12 * (1 + abs(lhs))


def test_scalar_expert_hand_case():
    """One row s = 1 through one scalar expert (w1 = a, w3 = b, w2 = c):
    y = c b silu(a), so dy/dw2 = b silu(a), dy/dw3 = c silu(a),
    dy/dw1 = c b silu'(a), dy/ds = c (b silu'(a) a + silu(a) b)."""
    a, b, c = 0.8, -1.3, 2.0
    sg = 1 / (1 + math.exp(-a))
    silu, dsilu = a * sg, sg * (1 + a * (1 - sg))
    dxp, dw1, dw3, dw2 = O.grouped_swiglu_backward(
        np.array([[1.0]]), np.array([0, 1]), np.full((1, 1, 1), a), np.full((1, 1, 1), b),
        np.full((1, 1, 1), c), np.array([[1.0]]))
    assert abs(dw2[0, 0, 0] - b * silu) < 1e-15
    assert abs(dw3[0, 0, 0] - c * silu) < 1e-15
    assert abs(dw1[0, 0, 0] - c * b * dsilu) < 1e-15
    assert abs(dxp[0, 0] - (c * b * dsilu * a + c * silu * b)) < 1e-14


@pytest.mark.parametrize("mistake", ["sign_of_dw1", "w1_for_w3", "no_dU_in_dx"])
def test_pins_catch_planted_mistakes(mistake):
    """A plausible slip planted in the oracle's backward (on the CPU) makes
    the finite-difference pin fail: a wrong sign, a wrong weight, a dropped
    term."""
    xp, off, w1, w3, w2, dy = _problem()
    dxp, dw1, dw3, dw2 = O.grouped_swiglu_backward(xp, off, w1, w3, w2, dy)
    if mistake == "sign_of_dw1":
        dw1 = -dw1
    elif mistake == "w1_for_w3":
        dxp, dw1, dw3, dw2 = O.grouped_swiglu_backward(xp, off, w1, w1, w2, dy)
    else:
        # dx_perm without the dU w3 path: the gradient with w3's effect on x removed
        for e in range(len(off) - 1):
            lo, hi = int(off[e]), int(off[e + 1])
            S = xp[lo:hi]
            dA = dy[lo:hi] @ w2[e]
            dxp[lo:hi] -= (dA * O.silu(S @ w1[e].T)) @ w3[e]

    def loss():
        return float(np.sum(dy * O.grouped_swiglu(xp, off, w1, w3, w2)))

    errs = [np.max(np.abs(g - _fd(loss, a))) for g, a in zip((dxp, dw1, dw3, dw2),
                                                             (xp, w1, w3, w2))]
    assert max(errs) > 1e-3


@pytest.mark.parametrize("score,renorm,scale", [("softmax", True, 1.0), ("softmax", False, 2.5),
                                                ("sigmoid", True, 1.0), ("sigmoid", False, 0.7)])
def test_router_backward_matches_finite_differences(score, renorm, scale):
    """d(sum g * w)/d logits by central differences of the general router
    (logits with gaps >= 1e-3 so the selection stays fixed under the
    perturbation), one token at a time."""
    T, E, k = 5, 9, 3
    L = W.make_logits(T, E, k, seed=3)
    rng = np.random.default_rng(4)
    g = rng.standard_normal((T, k))
    idx, w, _, _ = O.router_topk_general(k, logits=L, score=score, renormalize=renorm,
                                         route_scale=scale)
    dz = O.router_backward(L, idx, g, score=score, renormalize=renorm, route_scale=scale)
    Lw = L.astype(np.float64).copy()

    def loss():
        i2, w2, _, _ = O.router_topk_general(k, logits=Lw, score=score, renormalize=renorm,
                                             route_scale=scale)
        assert np.array_equal(i2, idx)
        return float(np.sum(g * w2))

    np.testing.assert_allclose(dz, _fd(loss, Lw), atol=1e-8)


def test_router_backward_gate_gradients_match_torch_autograd():
    """dz, dw_router = dz^T x and dx = dz w_router against autograd of
    softmax -> gather -> renormalise -> scale in fp64."""
    T, E, k, d = 7, 6, 2, 5
    rng = np.random.default_rng(5)
    x = rng.standard_normal((T, d))
    wr = rng.standard_normal((E, d))
    g = rng.standard_normal((T, k))
    idx, _, _, L = O.router_topk_general(k, x=x, w_router=wr, renormalize=True,
                                         route_scale=1.5)
    dz, dwr, dx = O.router_backward(L, idx, g, renormalize=True, route_scale=1.5, x=x,
                                    w_router=wr)
    tx = torch.tensor(x, requires_grad=True)
    tw = torch.tensor(wr, requires_grad=True)
    p = torch.softmax(tx @ tw.T, dim=1).gather(1, torch.tensor(idx))
    (torch.sum(torch.tensor(g) * 1.5 * p / p.sum(1, keepdim=True))).backward()
    np.testing.assert_allclose(dwr, tw.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dx, tx.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_router_backward_closed_forms():
    """k = E with renormalisation: the weights are the softmax itself, whose
    gradient sums to zero per token; top-1 renormalised: w = 1, no gradient."""
    rng = np.random.default_rng(6)
    L = rng.standard_normal((4, 5))
    g = rng.standard_normal((4, 5))
    idx = np.argsort(-L, axis=1)
    dz = O.router_backward(L, idx, g, renormalize=True)
    np.testing.assert_allclose(dz.sum(axis=1), 0.0, atol=1e-14)
    dz1 = O.router_backward(L, idx[:, :1], g[:, :1], renormalize=True)
    np.testing.assert_allclose(dz1, 0.0, atol=1e-15)


def test_whole_layer_gradients_compose_to_finite_differences():
    """The layer's gradients assembled from the oracle's pieces (combine,
    experts, router with its gate, dispatch) equal central differences of
    the whole oracle layer L = <dout, moe_forward(x, w_router, ...)> with
    respect to x and w_router (selection fixed: the gate's logits are well
    separated), and with respect to one expert weight."""
    rng = np.random.default_rng(21)
    T, d, E, k, h = 6, 5, 4, 2, 3
    x = rng.standard_normal((T, d))
    wr = rng.standard_normal((E, d)) * 2.0
    w1 = rng.standard_normal((E, h, d)) * 0.6
    w3 = rng.standard_normal((E, h, d)) * 0.6
    w2 = rng.standard_normal((E, d, h)) * 0.6
    dout = rng.standard_normal((T, d))
    ref = O.moe_forward(x, wr, w1, w3, w2, k, True)
    L = ref["logits"]
    srt = np.sort(L, axis=1)
    assert np.min(srt[:, -k] - srt[:, -k - 1]) > 1e-3   # selection is stable under 1e-6 steps
    dy, dtw = O.combine_backward(dout, ref["y"], ref["dst_pos"], ref["topk_w"])
    dxp, dw1, dw3, dw2 = O.grouped_swiglu_backward(ref["x_perm"], ref["offsets"], w1, w3, w2, dy)
    _, dwr, dxr = O.router_backward(L, ref["topk_idx"], dtw, renormalize=True, x=x, w_router=wr)
    dx = O.dispatch_backward(dxp, ref["dst_pos"]) + dxr

    def loss():
        r = O.moe_forward(x, wr, w1, w3, w2, k, True)
        assert np.array_equal(r["topk_idx"], ref["topk_idx"])
        return float(np.sum(dout * r["out"]))

    np.testing.assert_allclose(dx, _fd(loss, x), atol=2e-7)
    np.testing.assert_allclose(dwr, _fd(loss, wr), atol=2e-7)
    np.testing.assert_allclose(dw2, _fd(loss, w2), atol=2e-7)


def test_scaled_dispatch_backward_matches_finite_differences():
    """score_before_experts: x_perm[p(t, j)] = w[t, j] x[t].  The gradients of
    <G, x_perm> with respect to x and w against central differences."""
    rng = np.random.default_rng(5)
    T, d, E, k = 7, 4, 3, 2
    L = rng.standard_normal((T, E))
    idx, w, _, _ = O.router_topk(k, True, logits=L)
    _, _, src, dst = O.dispatch(idx, E)
    x = rng.standard_normal((T, d))
    G = rng.standard_normal((T * k, d))

    def f():
        xp = np.empty((T * k, d))
        for t in range(T):
            for j in range(k):
                xp[dst[t, j]] = w[t, j] * x[t]
        return float(np.sum(G * xp))

    dx, dw = O.scaled_dispatch_backward(G, dst, w, x)
    np.testing.assert_allclose(dx, _fd(f, x), atol=1e-8)
    np.testing.assert_allclose(dw, _fd(f, w), atol=1e-8)


def test_score_before_experts_layer_gradients_compose_to_finite_differences():
    """The layer with score_before_experts ([HP] MoE.forward: routed rows
    scaled by their weights, unweighted combine): the chain combine (w = 1)
    -> experts -> scaled dispatch -> router equals central differences of
    the oracle layer with respect to x and w_router."""
    rng = np.random.default_rng(22)
    T, d, E, k, h = 6, 5, 4, 2, 3
    x = rng.standard_normal((T, d))
    wr = rng.standard_normal((E, d)) * 2.0
    w1 = rng.standard_normal((E, h, d)) * 0.6
    w3 = rng.standard_normal((E, h, d)) * 0.6
    w2 = rng.standard_normal((E, d, h)) * 0.6
    dout = rng.standard_normal((T, d))
    ref = O.moe_forward(x, wr, w1, w3, w2, k, True, score_before_experts=True)
    srt = np.sort(ref["logits"], axis=1)
    assert np.min(srt[:, -k] - srt[:, -k - 1]) > 1e-3
    dy, _ = O.combine_backward(dout, ref["y"], ref["dst_pos"], None)
    dxp, dw1, dw3, dw2 = O.grouped_swiglu_backward(ref["x_perm"], ref["offsets"], w1, w3, w2, dy)
    dxs, dtw = O.scaled_dispatch_backward(dxp, ref["dst_pos"], ref["topk_w"], x)
    _, dwr, dxr = O.router_backward(ref["logits"], ref["topk_idx"], dtw, renormalize=True, x=x,
                                    w_router=wr)

    def loss():
        r = O.moe_forward(x, wr, w1, w3, w2, k, True, score_before_experts=True)
        assert np.array_equal(r["topk_idx"], ref["topk_idx"])
        return float(np.sum(dout * r["out"]))

    np.testing.assert_allclose(dxs + dxr, _fd(loss, x), atol=2e-7)
    np.testing.assert_allclose(dwr, _fd(loss, wr), atol=2e-7)
    np.testing.assert_allclose(dw1, _fd(loss, w1), atol=2e-7)


def test_shared_expert_gradients_compose_to_finite_differences():
    """A shared expert ([HP] MoE.forward: out = routed + shared_expert(x))
    is a one-segment grouped SwiGLU over every token: its backward with the
    upstream dout gives its share of dx and its weight gradients, against
    central differences of the oracle layer with the shared expert."""
    rng = np.random.default_rng(23)
    T, d, E, k, h, hs = 5, 4, 3, 2, 3, 6
    x = rng.standard_normal((T, d))
    wr = rng.standard_normal((E, d)) * 2.0
    w1 = rng.standard_normal((E, h, d)) * 0.6
    w3 = rng.standard_normal((E, h, d)) * 0.6
    w2 = rng.standard_normal((E, d, h)) * 0.6
    s1 = rng.standard_normal((hs, d)) * 0.6
    s3 = rng.standard_normal((hs, d)) * 0.6
    s2 = rng.standard_normal((d, hs)) * 0.6
    dout = rng.standard_normal((T, d))
    ref = O.moe_forward(x, wr, w1, w3, w2, k, True, shared=(s1, s3, s2))
    srt = np.sort(ref["logits"], axis=1)
    assert np.min(srt[:, -k] - srt[:, -k - 1]) > 1e-3
    dy, dtw = O.combine_backward(dout, ref["y"], ref["dst_pos"], ref["topk_w"])
    dxp, _, _, _ = O.grouped_swiglu_backward(ref["x_perm"], ref["offsets"], w1, w3, w2, dy)
    _, _, dxr = O.router_backward(ref["logits"], ref["topk_idx"], dtw, renormalize=True, x=x,
                                  w_router=wr)
    dxsh, ds1, ds3, ds2 = O.grouped_swiglu_backward(x, np.array([0, T]), s1[None], s3[None],
                                                    s2[None], dout)

    def loss():
        r = O.moe_forward(x, wr, w1, w3, w2, k, True, shared=(s1, s3, s2))
        assert np.array_equal(r["topk_idx"], ref["topk_idx"])
        return float(np.sum(dout * r["out"]))

    dx = O.dispatch_backward(dxp, ref["dst_pos"]) + dxr + dxsh
    np.testing.assert_allclose(dx, _fd(loss, x), atol=2e-7)
    np.testing.assert_allclose(ds1[0], _fd(loss, s1), atol=2e-7)
    np.testing.assert_allclose(ds3[0], _fd(loss, s3), atol=2e-7)
    np.testing.assert_allclose(ds2[0], _fd(loss, s2), atol=2e-7)
