"""GPU parity of the fp32 training path: the training forward of the experts
(G | U and H kept), the backward of the grouped SwiGLU, the router's gate
gradients and the whole layer's gradients composed from the per-step entry
points, all in fp32 on CUDA cores, against the fp64 oracle's derivatives.

Tolerance: the fp32 workload's bar, max|err| <= 1e-5 (1 + |ref|) and
||err||_F <= 1e-5 ||ref||_F.  Every output is a sum of at most a few hundred
fp32 products of O(1) values accumulated in fp32 (a relative error of order
sqrt(K) 2^-24 for K terms of random sign), or a product of two such sums
(the SwiGLU derivative), far inside both bounds at these sizes.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M(cuda_ok):
    from routing_dispatch_grouped_topk_b200 import build
    build.build()
    import routing_dispatch_grouped_topk_b200 as m
    m.lib()
    return m


def close(got, ref, tol=1e-5):
    g = O.as_f64(got)
    ref = np.asarray(ref, dtype=np.float64)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    err = np.abs(g - ref)
    bad = err > tol * (1 + np.abs(ref))
    assert not bad.any(), f"{bad.sum()} elements off, worst {err.max()}"
    den = np.linalg.norm(ref)
    if den > 0:
        assert np.linalg.norm(g - ref) <= tol * den, np.linalg.norm(g - ref) / den


def i32(a):
    return torch.as_tensor(np.asarray(a), dtype=torch.int32, device="cuda")


def expert_problem(counts, d, h, seed):
    g = torch.Generator().manual_seed(seed)
    E, N = len(counts), int(sum(counts))
    xp = torch.randn(N, d, generator=g)
    w1 = torch.randn(E, h, d, generator=g) / math.sqrt(d)
    w3 = torch.randn(E, h, d, generator=g) / math.sqrt(d)
    w2 = torch.randn(E, d, h, generator=g) / math.sqrt(h)
    dy = torch.randn(N, d, generator=g)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    return xp, w1, w3, w2, dy, off


# Empty experts, single rows, segments that end inside and on 32-row tiles,
# d and h that are not multiples of the 32-wide tiles.
CASES = [
    ([5, 0, 33, 1, 70], 36, 20),
    ([64, 0, 1, 129, 40], 96, 52),
    ([130], 64, 64),
    ([0, 0, 17, 0], 128, 256),
]


@pytest.mark.parametrize("counts,d,h", CASES)
def test_f32_train_forward_keeps_g_u_h(M, counts, d, h):
    xp, w1, w3, w2, _, off = expert_problem(counts, d, h, seed=sum(counts) + d)
    c = [t.cuda() for t in (xp, w1, w3, w2)]
    y, h_act, gu, ws = M.grouped_swiglu_train(c[0], i32(off), *c[1:])
    torch.cuda.synchronize()
    assert M.device_status(ws) == 0
    G, U = O.grouped_preactivations(xp, off, w1, w3)
    close(gu[:, :h], G)
    close(gu[:, h:], U)
    close(h_act, O.silu(G) * U)
    close(y, O.grouped_swiglu(xp, off, w1, w3, w2))
    # the inference forward runs the same arithmetic: y is bit-identical
    y_inf, _ = M.grouped_swiglu(c[0], i32(off), *c[1:])
    assert torch.equal(y, y_inf)


@pytest.mark.parametrize("counts,d,h", CASES)
def test_f32_grouped_swiglu_backward_matches_oracle(M, counts, d, h):
    xp, w1, w3, w2, dy, off = expert_problem(counts, d, h, seed=7 * sum(counts) + h)
    c = [t.cuda() for t in (xp, w1, w3, w2)]
    o = i32(off)
    _, h_act, gu, _ = M.grouped_swiglu_train(c[0], o, *c[1:])
    dxp, dw1, dw3, dw2, ws = M.grouped_swiglu_backward(c[0], o, *c[1:], h_act, gu, dy.cuda())
    torch.cuda.synchronize()
    assert M.device_status(ws) == 0
    rdx, rw1, rw3, rw2 = O.grouped_swiglu_backward(xp, off, w1, w3, w2, dy)
    close(dxp, rdx)
    for e, n in enumerate(counts):
        if n == 0:
            assert not dw1[e].any() and not dw3[e].any() and not dw2[e].any()
            continue
        close(dw1[e], rw1[e])
        close(dw3[e], rw3[e])
        close(dw2[e], rw2[e])


def test_f32_backward_rejects_bad_offsets_without_writing(M):
    xp, w1, w3, w2, dy, off = expert_problem([10, 6], 36, 20, seed=2)
    c = [t.cuda() for t in (xp, w1, w3, w2)]
    _, h_act, gu, _ = M.grouped_swiglu_train(c[0], i32(off), *c[1:])
    bad = i32([0, 12, 15])   # ends before N = 16
    N, d = xp.shape
    E, h, _ = w1.shape
    outs = [torch.full((N, d), 3.0, device="cuda")] + [torch.full_like(t, 3.0) for t in c[1:]]
    ws = torch.zeros(M.grouped_swiglu_backward_workspace_size(N, d, h, E, M.MOE_F32),
                     dtype=torch.uint8, device="cuda")
    M.moe_grouped_swiglu_backward(c[0], bad, *c[1:], h_act, gu, dy.cuda(), N, d, h, E,
                                  M.MOE_F32, *outs, ws)
    torch.cuda.synchronize()
    assert M.device_status(ws) & M.MOE_DEV_BAD_OFFSETS
    assert all(bool((t == 3.0).all()) for t in outs)


@pytest.mark.parametrize("score,renorm,scale", [("softmax", True, 1.0), ("sigmoid", False, 0.7)])
@pytest.mark.parametrize("T,E,k,d", [(300, 128, 8, 36), (77, 12, 4, 64), (1000, 8, 2, 128)])
def test_f32_router_backward_matches_oracle(M, score, renorm, scale, T, E, k, d):
    """fp32 x and w_router: dw_router = dz^T x and dx = dz w_router from dz in
    fp32 (no bf16 rounding), with and without the caller's d_logits."""
    L = W.make_logits(T, E, k, seed=T + E)
    idx, w, _, _ = O.router_topk_general(k, logits=L, score=score, renormalize=renorm,
                                         route_scale=scale)
    g = torch.Generator().manual_seed(E)
    gw = torch.randn(T, k, generator=g)
    x = torch.randn(T, d, generator=g)
    wr = torch.randn(E, d, generator=g) * 0.05
    rdz, rdwr, rdx = O.router_backward(L.astype(np.float32), idx, gw, score=score,
                                       renormalize=renorm, route_scale=scale, x=x, w_router=wr)
    for want_dl in (True, False):
        dl, dwr, dx, ws = M.router_backward(torch.from_numpy(L).float().cuda(), i32(idx),
                                            gw.cuda(), x.cuda(), wr.cuda(), want_d_logits=want_dl,
                                            score=score, renormalize=renorm, route_scale=scale)
        torch.cuda.synchronize()
        assert M.device_status(ws) == 0
        assert dwr.dtype == torch.float32 and dx.dtype == torch.float32
        if want_dl:
            err = np.abs(O.as_f64(dl) - rdz)
            rowmax = np.abs(rdz).max(axis=1, keepdims=True)
            # plus the fp32 rounding of the differences of upstream gradients
            # inside the renormalisation's derivative (g_j - sum g w cancels
            # when one weight saturates): 16 ulp of the token's largest g
            gmax = scale * np.abs(gw.double().numpy()).max(axis=1, keepdims=True)
            bound = 2e-5 * (np.abs(rdz) + rowmax) + 16 * 2.0 ** -24 * gmax
            assert np.all(err <= bound), (err / bound).max()
        # dz carries its own fp32 error (2e-5 of the row's largest entry)
        # into sums over T tokens (dw_router) and E experts (dx)
        close(dwr, rdwr, tol=1e-4)
        close(dx, rdx, tol=1e-4)


def test_f32_layer_backward_composed_matches_oracle(M):
    """The fp32 layer's training step through the per-step entry points
    (router with kept logits, dispatch, training forward, combine, then the
    combine, experts, router and dispatch backwards) at the fp32 workload's
    sizes, every gradient against the oracle's chain rule."""
    cfg = W.config(0)
    assert cfg.dtype == "f32"
    T, d, E, k, h = cfg.T, cfg.d, cfg.E, cfg.top_k, cfg.h
    lay = W.make_layer(cfg, device="cpu")
    x, wr, w1, w3, w2 = (lay[n].float() for n in ("x", "w_router", "w1", "w3", "w2"))
    dout = torch.randn(T, d, generator=torch.Generator().manual_seed(9))
    c = [t.cuda() for t in (x, wr, w1, w3, w2)]
    idx, tw, _, logits, _ = M.router_topk(c[0], c[1], k, True, want_logits=True)
    _, off, _, dst, xp, _ = M.dispatch(c[0], idx, E)
    y, h_act, gu, _ = M.grouped_swiglu_train(xp, off, *c[2:])
    out = M.combine(y, dst, tw)
    dy, dtw = M.combine_backward(dout.cuda(), y, dst, tw)
    dxp, dw1, dw3, dw2, _ = M.grouped_swiglu_backward(xp, off, *c[2:], h_act, gu, dy)
    dl, dwr, dxr, _ = M.router_backward(logits, idx, dtw, c[0], c[1], renormalize=True)
    dx = M.dispatch_backward(dxp, dst, dxr)
    torch.cuda.synchronize()

    ref = O.moe_forward(x, wr, w1, w3, w2, k, True)
    assert np.array_equal(idx.cpu().numpy(), ref["topk_idx"])
    close(out, ref["out"])
    rdy, rdtw = O.combine_backward(dout, ref["y"], ref["dst_pos"], ref["topk_w"])
    rdxp, rw1, rw3, rw2 = O.grouped_swiglu_backward(ref["x_perm"], ref["offsets"], w1, w3, w2,
                                                    rdy)
    rdz, rdwr, rdxr = O.router_backward(ref["logits"], ref["topk_idx"], rdtw, renormalize=True,
                                        x=x, w_router=wr)
    rdx = O.dispatch_backward(rdxp, ref["dst_pos"]) + rdxr
    close(dtw, rdtw)
    close(dx, rdx, tol=1e-4)
    for e in range(E):
        close(dw1[e], rw1[e])
        close(dw3[e], rw3[e])
        close(dw2[e], rw2[e])
    close(dwr, rdwr, tol=1e-4)
    err = np.abs(O.as_f64(dl) - rdz)
    gmax = np.abs(rdtw).max(axis=1, keepdims=True)
    assert np.all(err <= 2e-5 * (np.abs(rdz) + np.abs(rdz).max(axis=1, keepdims=True)) +
                  16 * 2.0 ** -24 * gmax)
