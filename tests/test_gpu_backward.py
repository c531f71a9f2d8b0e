"""GPU parity of the training path: the training forward of the experts
(moe_grouped_swiglu_train), the backward of the grouped SwiGLU, of the
combine and of the dispatch, against the fp64 oracle's derivatives.

Tolerances (bf16 operands, fp32 accumulation; the backward reads the
bf16-rounded G, U, H and rounds dG, dU once to bf16 before the next
products, so each output carries at most a few bf16 roundings):

* bf16 outputs: max|err| <= 3e-2 (1 + |ref|) and ||err||_F <= 1e-2 ||ref||_F
* weight gradients (sums over an expert's rows): per expert,
  max|err| <= 6e-2 (|ref| + rms(ref)) and ||err||_F <= 1e-2 ||ref||_F.
  Every term of the sum carries the relative rounding of the saved bf16 G
  and U (about 2^-8, larger near the zero of silu' where it is |G| silu''
  times 2^-9 in absolute terms); the terms have random signs, so the error
  of the sum scales with the size of a typical entry (the RMS), not with
  the entry itself, which can cancel to near zero.  An fp64 emulation of
  exactly these roundings gives max err / (|ref| + rms) = 0.026 on the cases
  below and a Frobenius error of 0.3%.
* fp32 routing-weight gradients (dot products of bf16 rows): |err| <=
  1.01 d 2^-24 sum_i |dout_i y_i| + 1e-30, the worst-case bound of an fp32
  sum of d exact products.

Integer layouts come from the oracle's dispatch; experts with no rows must
get weight gradients that are exactly zero.
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


def f64(t):
    return O.as_f64(t)


def close(got, ref, tol_max=3e-2, tol_fro=1e-2):
    g = f64(got)
    ref = np.asarray(ref, dtype=np.float64)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    err = np.abs(g - ref)
    bad = err > tol_max * (1 + np.abs(ref))
    assert not bad.any(), f"{bad.sum()} elements off, worst {err.max()}"
    den = np.linalg.norm(ref)
    if den > 0:
        assert np.linalg.norm(g - ref) <= tol_fro * den, np.linalg.norm(g - ref) / den


def close_wgrad(got, ref):
    """Weight gradient of one expert: RMS-relative elementwise bound and a
    Frobenius bound (see the module docstring)."""
    g = f64(got)
    ref = np.asarray(ref, dtype=np.float64)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    rms = np.sqrt(np.mean(ref ** 2))
    err = np.abs(g - ref)
    bad = err > 6e-2 * (np.abs(ref) + rms)
    assert not bad.any(), f"{bad.sum()} elements off, worst {(err / (np.abs(ref) + rms)).max()}"
    den = np.linalg.norm(ref)
    if den > 0:
        assert np.linalg.norm(g - ref) <= 1e-2 * den, np.linalg.norm(g - ref) / den


def i32(a):
    return torch.as_tensor(np.asarray(a), dtype=torch.int32, device="cuda")


def expert_problem(counts, d, h, seed):
    """x_perm [N, d], w1/w3 [E, h, d], w2 [E, d, h], dy [N, d] in bf16 with
    the layer's scales (x, dy ~ N(0, 1), weights ~ N(0, 1/fan_in))."""
    g = torch.Generator().manual_seed(seed)
    E, N = len(counts), int(sum(counts))
    bf = torch.bfloat16
    xp = torch.randn(N, d, generator=g).to(bf)
    w1 = (torch.randn(E, h, d, generator=g) / math.sqrt(d)).to(bf)
    w3 = (torch.randn(E, h, d, generator=g) / math.sqrt(d)).to(bf)
    w2 = (torch.randn(E, d, h, generator=g) / math.sqrt(h)).to(bf)
    dy = torch.randn(N, d, generator=g).to(bf)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    return xp, w1, w3, w2, dy, off


# Segment mixes: empty experts, single rows, 64 / 128 boundaries, ragged
# tails, several 128-row tiles; d and h that leave partial 256-column and
# 128-row tiles; the smallest d = h = 64.
CASES = [
    ([64, 0, 1, 129, 300, 17, 128], 256, 192),
    ([5, 250, 0, 77], 320, 128),
    ([130], 64, 64),
    ([0, 0, 63, 65, 0], 128, 320),
]


@pytest.mark.parametrize("counts,d,h", CASES)
def test_train_forward_keeps_g_u_h(M, counts, d, h):
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
    # the same kernels as the inference forward: y is bit-identical
    y_inf, _ = M.grouped_swiglu(c[0], i32(off), *c[1:])
    assert torch.equal(y, y_inf)


@pytest.mark.parametrize("counts,d,h", CASES)
def test_grouped_swiglu_backward_matches_oracle(M, counts, d, h):
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
        close_wgrad(dw1[e], rw1[e])
        close_wgrad(dw3[e], rw3[e])
        close_wgrad(dw2[e], rw2[e])


def test_backward_with_no_rows_zeroes_weight_gradients(M):
    xp, w1, w3, w2, dy, off = expert_problem([0, 0, 0], 128, 64, seed=1)
    c = [t.cuda() for t in (w1, w3, w2)]
    empty = torch.empty(0, 128, dtype=torch.bfloat16, device="cuda")
    dw = [torch.full_like(t, 5.0) for t in c]
    ws = torch.empty(M.grouped_swiglu_backward_workspace_size(0, 128, 64, 3, M.MOE_BF16),
                     dtype=torch.uint8, device="cuda")
    M.moe_grouped_swiglu_backward(empty, i32(off), *c, empty, empty, empty, 0, 128, 64, 3,
                                  M.MOE_BF16, empty, *dw, ws)
    torch.cuda.synchronize()
    assert all(not t.any() for t in dw)


def test_backward_rejects_bad_offsets_without_writing(M):
    xp, w1, w3, w2, dy, off = expert_problem([10, 6], 64, 64, seed=2)
    c = [t.cuda() for t in (xp, w1, w3, w2)]
    _, h_act, gu, _ = M.grouped_swiglu_train(c[0], i32(off), *c[1:])
    dx = torch.full((16, 64), 3.0, dtype=torch.bfloat16, device="cuda")
    dw = [torch.full_like(t, 3.0) for t in c[1:]]
    ws = torch.empty(M.grouped_swiglu_backward_workspace_size(16, 64, 64, 2, M.MOE_BF16),
                     dtype=torch.uint8, device="cuda")
    for bad in ([0, 12, 10], [1, 6, 16], [0, 6, 15]):
        M.moe_grouped_swiglu_backward(c[0], i32(bad), *c[1:], h_act, gu, dy.cuda(), 16, 64, 64,
                                      2, M.MOE_BF16, dx, *dw, ws)
        assert M.device_status(ws) & M.MOE_DEV_BAD_OFFSETS
    assert torch.all(dx == 3.0) and all(torch.all(t == 3.0) for t in dw)


def _routing(T, E, k, seed):
    L = W.make_logits(T, E, k, seed=seed)
    idx, w, _, _ = O.router_topk(k, True, logits=L)
    _, off, src, dst = O.dispatch(idx, E)
    return idx, w, off, src, dst


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("k", [1, 2, 8, 16])
def test_combine_backward_matches_oracle(M, dtype, k):
    T, E, d = 300, 32, 256
    idx, w, off, src, dst = _routing(T, E, k, seed=k)
    g = torch.Generator().manual_seed(k)
    N = T * k
    y = torch.randn(N, d, generator=g).to(dtype)
    dout = torch.randn(T, d, generator=g).to(dtype)
    wt = torch.from_numpy(w).float()
    dy, dw = M.combine_backward(dout.cuda(), y.cuda(), i32(dst), wt.cuda())
    rdy, rdw = O.combine_backward(dout, y, dst, wt)
    if dtype == torch.bfloat16:
        close(dy, rdy)
    else:
        close(dy, rdy, 1e-6, 1e-6)
    # fp32 dot products of d exact products: worst-case recursive-sum bound
    yy, gg = f64(y), f64(dout)
    mag = np.array([[np.abs(gg[t]) @ np.abs(yy[dst[t, j]]) for j in range(k)] for t in range(T)])
    err = np.abs(f64(dw) - rdw)
    assert np.all(err <= 1.01 * d * 2.0 ** -24 * mag + 1e-30), err.max()
    # unweighted, no weight gradient
    dy1, dw1 = M.combine_backward(dout.cuda(), y.cuda(), i32(dst), None, want_dw=False)
    assert dw1 is None
    assert torch.equal(dy1.cpu()[torch.from_numpy(dst[:, 0]).long()], dout)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_dispatch_backward_matches_oracle(M, dtype):
    T, E, k, d = 257, 16, 4, 128
    idx, w, off, src, dst = _routing(T, E, k, seed=5)
    g = torch.Generator().manual_seed(9)
    dxp = torch.randn(T * k, d, generator=g).to(dtype)
    dx = M.dispatch_backward(dxp.cuda(), i32(dst))
    ref = O.dispatch_backward(dxp, dst)
    if dtype == torch.bfloat16:
        close(dx, ref)
    else:
        close(dx, ref, 1e-6, 1e-6)


@pytest.mark.parametrize("cfg_index", [1, 2])
def test_training_chain_full_size_sampled(M, cfg_index):
    """The whole training chain at the Qwen3-30B-A3B layer sizes (T=4096
    near-uniform, T=16384 Zipf-skewed): router and dispatch on the GPU,
    training forward, combine backward of a random dout, experts backward,
    dispatch backward.  The weight gradients of three experts (the first,
    the largest, one in the middle) and the input gradients of 16 sampled
    tokens are checked against the oracle, one expert's rows at a time."""
    cfg = W.config(cfg_index)
    lay = W.make_layer(cfg, device="cuda")
    x, wr, w1, w3, w2 = (lay[n] for n in ("x", "w_router", "w1", "w3", "w2"))
    T, d, E, k, h = cfg.T, cfg.d, cfg.E, cfg.top_k, cfg.h
    idx, tw, counts, _, _ = M.router_topk(x, wr, k, True)
    cnt, off, src, dst, xp, _ = M.dispatch(x, idx, E)
    y, h_act, gu, _ = M.grouped_swiglu_train(xp, off, w1, w3, w2)
    g = torch.Generator(device="cuda").manual_seed(cfg.seed)
    dout = torch.randn(T, d, generator=g, device="cuda").to(torch.bfloat16)
    dy, dtw = M.combine_backward(dout, y, dst, tw)
    dxp, dw1, dw3, dw2, ws = M.grouped_swiglu_backward(xp, off, w1, w3, w2, h_act, gu, dy)
    dx = M.dispatch_backward(dxp, dst)
    torch.cuda.synchronize()
    assert M.device_status(ws) == 0
    offs = off.cpu().numpy().astype(np.int64)
    cnt_h = np.diff(offs)
    # weight gradients of three experts, from their whole segments
    for e in sorted({0, int(np.argmax(cnt_h)), E // 2}):
        lo, hi = int(offs[e]), int(offs[e + 1])
        sub = np.array([0, hi - lo])
        _, rw1, rw3, rw2 = O.grouped_swiglu_backward(
            xp[lo:hi].cpu(), sub, w1[e:e + 1].cpu(), w3[e:e + 1].cpu(), w2[e:e + 1].cpu(),
            dy[lo:hi].cpu())
        close_wgrad(dw1[e], rw1[0])
        close_wgrad(dw3[e], rw3[0])
        close_wgrad(dw2[e], rw2[0])
    # input gradients of sampled tokens: dx_perm rows are row-local, so each
    # expert's sampled rows form their own segment
    rng = np.random.default_rng(cfg.seed)
    toks = rng.choice(T, 16, replace=False)
    dst_h = dst.cpu().numpy()
    idx_h = idx.cpu().numpy()
    rows = {}
    for t in toks:
        for j in range(k):
            rows.setdefault(int(idx_h[t, j]), []).append(int(dst_h[t, j]))
    ref_dxp = {}
    for e, rs in rows.items():
        rs_t = torch.as_tensor(rs, device="cuda").long()
        rdx, _, _, _ = O.grouped_swiglu_backward(
            xp[rs_t].cpu(), np.array([0, len(rs)]), w1[e:e + 1].cpu(), w3[e:e + 1].cpu(),
            w2[e:e + 1].cpu(), dy[rs_t].cpu())
        close(dxp[rs_t], rdx)
        for r, v in zip(rs, rdx):
            ref_dxp[r] = v
    ref_dx = np.stack([sum(ref_dxp[int(dst_h[t, j])] for j in range(k)) for t in toks])
    close(dx[torch.as_tensor(toks, device="cuda").long()], ref_dx)
    # routing-weight gradients of the sampled tokens
    yy = f64(y[torch.as_tensor(dst_h[toks].ravel(), device="cuda").long()]).reshape(16, k, d)
    gg = f64(dout[torch.as_tensor(toks, device="cuda").long()])
    ref_dtw = np.einsum("td,tjd->tj", gg, yy)
    mag = np.einsum("td,tjd->tj", np.abs(gg), np.abs(yy))
    assert np.all(np.abs(f64(dtw[torch.as_tensor(toks, device="cuda").long()]) - ref_dtw)
                  <= 1.01 * d * 2.0 ** -24 * mag + 1e-30)


# ----------------------------------------------------------- router backward
ROUTER_BWD = [("softmax", True, 1.0), ("softmax", False, 2.5), ("sigmoid", True, 1.0),
              ("sigmoid", False, 0.7)]


@pytest.mark.parametrize("score,renorm,scale", ROUTER_BWD)
@pytest.mark.parametrize("T,E,k,d", [(300, 128, 8, 256), (77, 72, 4, 192), (33, 8, 2, 64),
                                     (2100, 64, 8, 256)])
def test_router_backward_matches_oracle(M, score, renorm, scale, T, E, k, d):
    """d_logits (fp32) within 2e-5 of the row's largest entry; dw_router and
    the router's dx (bf16, from dz rounded once to bf16) within the
    RMS-relative bound of sums over mixed-sign terms.  T = 2100 splits
    dw_router over 8 token segments (fp32 partials, a ragged last one)."""
    L = W.make_logits(T, E, k, seed=T + E)
    idx, w, _, _ = O.router_topk_general(k, logits=L, score=score, renormalize=renorm,
                                         route_scale=scale)
    g = torch.Generator().manual_seed(E)
    gw = torch.randn(T, k, generator=g)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16)
    wr = (torch.randn(E, d, generator=g) * 0.05).to(torch.bfloat16)
    dl, dwr, dx, ws = M.router_backward(torch.from_numpy(L).float().cuda(), i32(idx), gw.cuda(),
                                        x.cuda(), wr.cuda(), score=score, renormalize=renorm,
                                        route_scale=scale)
    torch.cuda.synchronize()
    assert M.device_status(ws) == 0
    rdz, rdwr, rdx = O.router_backward(L.astype(np.float32), idx, gw, score=score,
                                       renormalize=renorm, route_scale=scale, x=x, w_router=wr)
    err = np.abs(f64(dl) - rdz)
    rowmax = np.abs(rdz).max(axis=1, keepdims=True)
    assert np.all(err <= 2e-5 * (np.abs(rdz) + rowmax) + 1e-30), err.max()
    close_wgrad(dwr, rdwr)
    close_wgrad(dx, rdx)


@pytest.mark.parametrize("score,renorm", [("softmax", True), ("sigmoid", False)])
def test_router_backward_load_balance_gradient(M, score, renorm):
    """aux_loss_coef: the gradient of coef times the load-balance loss
    ([HP] _compute_load_balance_loss) joins the routing weights' gradient;
    against the oracle's router backward fed d_topk_w + coef * the oracle's
    loss gradient (pinned by finite differences of the loss)."""
    T, E, k, coef = 300, 16, 4, 0.05
    L = W.make_logits(T, E, k, seed=11)
    idx, w, _, _ = O.router_topk_general(k, logits=L, score=score, renormalize=renorm)
    gw = torch.randn(T, k, generator=torch.Generator().manual_seed(3))
    dl, _, _, ws = M.router_backward(torch.from_numpy(L).float().cuda(), i32(idx), gw.cuda(),
                                     score=score, renormalize=renorm, aux_loss_coef=coef)
    dl0, _, _, _ = M.router_backward(torch.from_numpy(L).float().cuda(), i32(idx), gw.cuda(),
                                     score=score, renormalize=renorm)
    torch.cuda.synchronize()
    assert M.device_status(ws) == 0
    g = gw.double().numpy() + coef * O.load_balance_loss_grad(idx, E)
    rdz = O.router_backward(L.astype(np.float32), idx, g, score=score, renormalize=renorm)
    err = np.abs(f64(dl) - rdz)
    rowmax = np.abs(rdz).max(axis=1, keepdims=True)
    assert np.all(err <= 2e-5 * (np.abs(rdz) + rowmax) + 1e-30), err.max()
    assert not torch.equal(dl, dl0)


def test_router_backward_without_gate_gradients(M):
    T, E, k = 50, 16, 2
    L = W.make_logits(T, E, k, seed=1)
    idx, _, _, _ = O.router_topk(k, True, logits=L)
    gw = torch.randn(T, k)
    dl, dwr, dx, ws = M.router_backward(torch.from_numpy(L).float().cuda(), i32(idx), gw.cuda(),
                                        renormalize=True)
    assert dwr is None and dx is None
    rdz = O.router_backward(L.astype(np.float32), idx, gw, renormalize=True)
    assert np.allclose(f64(dl), rdz, atol=2e-6)


def test_layer_backward_full_size_sampled_tokens(M):
    """The whole layer's input gradient at the Qwen3-30B-A3B sizes (T=4096):
    router (logits kept) -> dispatch -> training forward -> combine, then
    combine backward -> experts backward -> router backward -> dispatch
    backward with the router's dx added.  Sampled tokens' dx against the
    oracle (experts' share row by row, router's share from the oracle's
    router backward on the GPU's logits)."""
    cfg = W.config(1)
    lay = W.make_layer(cfg, device="cuda")
    x, wr, w1, w3, w2 = (lay[n] for n in ("x", "w_router", "w1", "w3", "w2"))
    T, d, E, k, h = cfg.T, cfg.d, cfg.E, cfg.top_k, cfg.h
    idx, tw, counts, logits, _ = M.router_topk(x, wr, k, True, want_logits=True)
    cnt, off, src, dst, xp, _ = M.dispatch(x, idx, E)
    y, h_act, gu, _ = M.grouped_swiglu_train(xp, off, w1, w3, w2)
    g = torch.Generator(device="cuda").manual_seed(3)
    dout = torch.randn(T, d, generator=g, device="cuda").to(torch.bfloat16)
    dy, dtw = M.combine_backward(dout, y, dst, tw)
    dxp, _, _, _, ws = M.grouped_swiglu_backward(xp, off, w1, w3, w2, h_act, gu, dy)
    dl, dwr, dxr, rws = M.router_backward(logits, idx, dtw, x, wr, renormalize=True)
    dx = M.dispatch_backward(dxp, dst, dxr)
    torch.cuda.synchronize()
    assert M.device_status(ws) == 0 and M.device_status(rws) == 0
    rng = np.random.default_rng(11)
    toks = np.sort(rng.choice(T, 8, replace=False))
    tt = torch.as_tensor(toks, device="cuda").long()
    # router share for the sampled tokens, from the GPU's logits and dtw
    rdz, _, rdxr = O.router_backward(logits[tt].cpu(), idx[tt].cpu(), dtw[tt].cpu(),
                                     renormalize=True, x=x[tt].cpu(), w_router=wr.cpu())
    # experts' share: dx_perm rows are row-local
    dst_h = dst.cpu().numpy()
    idx_h = idx.cpu().numpy()
    ref = rdxr.copy()
    for a, t in enumerate(toks):
        for j in range(k):
            r = int(dst_h[t, j])
            e = int(idx_h[t, j])
            rr = torch.tensor([r], device="cuda")
            rdx1, _, _, _ = O.grouped_swiglu_backward(
                xp[rr].cpu(), np.array([0, 1]), w1[e:e + 1].cpu(), w3[e:e + 1].cpu(),
                w2[e:e + 1].cpu(), dy[rr].cpu())
            ref[a] += rdx1[0]
    close(dx[tt], ref)


# --------------------------------------------- whole-layer training entry points
def _staged_training(M, x, wr, w1, w3, w2, k, dout, **opts):
    """The layer's training step through the per-step entry points."""
    E = w1.shape[0]
    idx, tw, counts, logits, _ = M.router_topk(x, wr, k, want_logits=True, **opts)
    cnt, off, src, dst, xp, _ = M.dispatch(x, idx, E)
    y, h_act, gu, _ = M.grouped_swiglu_train(xp, off, w1, w3, w2)
    out = M.combine(y, dst, tw)
    dy, dtw = M.combine_backward(dout, y, dst, tw)
    dxp, dw1, dw3, dw2, _ = M.grouped_swiglu_backward(xp, off, w1, w3, w2, h_act, gu, dy)
    ropts = {n: v for n, v in opts.items() if n in ("score", "renormalize", "route_scale")}
    dl, dwr, dxr, _ = M.router_backward(logits, idx, dtw, x, wr, **ropts)
    dx = M.dispatch_backward(dxp, dst, dxr)
    return dict(out=out, dx=dx, dw1=dw1, dw3=dw3, dw2=dw2, dw_router=dwr, d_logits=dl)


@pytest.mark.parametrize("cfg_index", [1, 2])
def test_forward_train_and_backward_equal_the_staged_calls(M, cfg_index):
    """moe_forward_train / moe_backward run the same kernels in the same
    order as the per-step entry points: every output is bit-identical, and
    the forward's output equals moe_forward's."""
    cfg = W.config(cfg_index)
    lay = W.make_layer(cfg, device="cuda")
    x, wr, w1, w3, w2 = (lay[n] for n in ("x", "w_router", "w1", "w3", "w2"))
    g = torch.Generator(device="cuda").manual_seed(5)
    dout = torch.randn(cfg.T, cfg.d, generator=g, device="cuda").to(torch.bfloat16)
    ref = _staged_training(M, x, wr, w1, w3, w2, cfg.top_k, dout, renormalize=True)
    out, state = M.forward_train(x, wr, w1, w3, w2, cfg.top_k, renormalize=True)
    grads = M.backward(state, dout, x, wr, w1, w3, w2, want_d_logits=True)
    torch.cuda.synchronize()
    assert M.device_status(state["state"]) == 0 and M.device_status(grads["ws"]) == 0
    assert torch.equal(out, ref["out"])
    assert torch.equal(out, M.forward(x, wr, w1, w3, w2, cfg.top_k, True))
    for n in ("dx", "dw1", "dw3", "dw2", "dw_router", "d_logits"):
        assert torch.equal(grads[n], ref[n]), n


@pytest.mark.parametrize("opts", [dict(), dict(score="sigmoid", route_scale=2.5),
                                  dict(num_groups=4, topk_groups=2),
                                  dict(aux_loss_coef=0.05)])
def test_layer_backward_matches_oracle(M, opts):
    """Every gradient of the whole layer (x, w_router, w1, w3, w2, logits)
    on a small layer against the oracle's chain rule, with router options."""
    T, d, E, k, h = 200, 256, 16, 4, 192
    g = torch.Generator().manual_seed(len(opts))
    bf = torch.bfloat16
    x = torch.randn(T, d, generator=g).to(bf)
    # logits of std ~8: the fp32 gate and the fp64 oracle select the same experts
    wr = (torch.randn(E, d, generator=g) * 0.5).to(bf)
    w1 = (torch.randn(E, h, d, generator=g) / math.sqrt(d)).to(bf)
    w3 = (torch.randn(E, h, d, generator=g) / math.sqrt(d)).to(bf)
    w2 = (torch.randn(E, d, h, generator=g) / math.sqrt(h)).to(bf)
    dout = torch.randn(T, d, generator=g).to(bf)
    c = [t.cuda() for t in (x, wr, w1, w3, w2)]
    out, state = M.forward_train(*c, k, renormalize=True, **opts)
    grads = M.backward(state, dout.cuda(), *c, want_d_logits=True)
    torch.cuda.synchronize()
    assert M.device_status(state["state"]) == 0 and M.device_status(grads["ws"]) == 0
    # the oracle: forward, then the chain rule step by step
    ro = dict(score=opts.get("score", "softmax"), route_scale=opts.get("route_scale", 1.0),
              num_groups=opts.get("num_groups", 0), topk_groups=opts.get("topk_groups", 0))
    ref = O.moe_forward(x, wr, w1, w3, w2, k, True, router=ro)
    gi = M.router_topk(c[0], c[1], k, True, **opts)[0]
    assert np.array_equal(gi.cpu().numpy(), ref["topk_idx"])
    close(out, ref["out"])
    rdy, rdtw = O.combine_backward(dout, ref["y"], ref["dst_pos"], ref["topk_w"])
    # the load-balance loss's gradient joins the routing weights' gradient
    rdtw = rdtw + opts.get("aux_loss_coef", 0.0) * O.load_balance_loss_grad(ref["topk_idx"], E)
    rdxp, rw1, rw3, rw2 = O.grouped_swiglu_backward(ref["x_perm"], ref["offsets"], w1, w3, w2,
                                                    rdy)
    rdz, rdwr, rdxr = O.router_backward(ref["logits"], ref["topk_idx"], rdtw,
                                        score=ro["score"], renormalize=True,
                                        route_scale=ro["route_scale"], x=x, w_router=wr)
    rdx = O.dispatch_backward(rdxp, ref["dst_pos"]) + rdxr
    close(grads["dx"], rdx)
    for e in range(E):
        if int(ref["counts"][e]) == 0:
            assert not grads["dw1"][e].any()
            continue
        close_wgrad(grads["dw1"][e], rw1[e])
        close_wgrad(grads["dw3"][e], rw3[e])
        close_wgrad(grads["dw2"][e], rw2[e])
    close_wgrad(grads["dw_router"], rdwr)
    # d logits inherit the bf16 rounding of y through d topk_w = <dout, y>.
    # In norm over all tokens:
    gdz = f64(grads["d_logits"])
    assert np.linalg.norm(gdz - rdz) <= 1e-2 * np.linalg.norm(rdz)
    # Element by element on the tokens whose routing weights are not
    # saturated (every selected weight in [1e-3, 1 - 1e-3]; in saturated tokens
    # d logits are differences of nearly equal fp32 terms, and there the
    # router backward is checked on identical inputs at 2e-5 by
    # test_router_backward_matches_oracle).  Bound: the error of each
    # d topk_w[t, j] = <dout[t], y[p(t, j)]> is at most
    # a[t, j] = 2^-8 sum_i |dout_i| (|y_i| + 3 rms(y row)) (one bf16 rounding
    # of y and of the hidden activation before it), carried to the logits by
    # the absolute Jacobian: |err[t, e]| <= sum_j |d w_j / d z_e| a[t, j],
    # plus fp32 slack (and, for sigmoid scores, the fp32 error of s (1 - s)).
    ydst = ref["y"][ref["dst_pos"]]                                  # [T, k, d]
    yrms = np.sqrt(np.mean(ydst ** 2, axis=2, keepdims=True))
    a = 2.0 ** -8 * np.einsum("ti,tji->tj", np.abs(f64(dout)), np.abs(ydst) + 3 * yrms)
    bound = np.zeros_like(rdz)
    for j in range(k):
        onehot = np.zeros((T, k))
        onehot[:, j] = 1.0
        jac_j = O.router_backward(ref["logits"], ref["topk_idx"], onehot, score=ro["score"],
                                  renormalize=True, route_scale=ro["route_scale"])
        bound += np.abs(jac_j) * a[:, j:j + 1]
    bound += 1e-5 * np.abs(rdz).max(axis=1, keepdims=True)
    if ro["score"] == "sigmoid":
        # the kernel's s (1 - s) in fp32: relative error ~2^-23 / (1 - s),
        # large where the sigmoid saturates
        sg = O.sigmoid(ref["logits"])
        bound += np.abs(rdz) * 2.0 ** -20 / np.maximum(1.0 - sg, 2.0 ** -30)
    wsel = np.asarray(ref["topk_w"]) / ro["route_scale"]
    live = np.all((wsel >= 1e-3) & (wsel <= 1 - 1e-3), axis=1)
    print(f"d logits checked element-wise on {live.sum()} of {T} tokens")
    assert live.sum() >= 30     # 93, 200 and 40 of the 200 tokens for the three options
    err = np.abs(gdz - rdz)[live]
    assert np.all(err <= bound[live]), (err / bound[live]).max()


def _small_train_layer(seed, T=200, d=256, E=16, h=192, hs=None):
    g = torch.Generator().manual_seed(seed)
    bf = torch.bfloat16
    x = torch.randn(T, d, generator=g).to(bf)
    wr = (torch.randn(E, d, generator=g) * 0.5).to(bf)
    w1 = (torch.randn(E, h, d, generator=g) / math.sqrt(d)).to(bf)
    w3 = (torch.randn(E, h, d, generator=g) / math.sqrt(d)).to(bf)
    w2 = (torch.randn(E, d, h, generator=g) / math.sqrt(h)).to(bf)
    dout = torch.randn(T, d, generator=g).to(bf)
    sh = None
    if hs:
        sh = ((torch.randn(hs, d, generator=g) / math.sqrt(d)).to(bf),
              (torch.randn(hs, d, generator=g) / math.sqrt(d)).to(bf),
              (torch.randn(d, hs, generator=g) / math.sqrt(hs)).to(bf))
    return x, wr, w1, w3, w2, dout, sh


def test_layer_backward_score_before_experts(M):
    """score_before_experts ([HP] MoE.forward): the routed rows are scaled by
    their weights before the experts and the combine is unweighted.  The
    training forward equals moe_forward with the option bit for bit; every
    gradient against the oracle's chain (unweighted combine -> experts ->
    scaled dispatch -> router), itself pinned by finite differences of the
    oracle layer."""
    T, E, k = 200, 16, 4
    x, wr, w1, w3, w2, dout, _ = _small_train_layer(7, T=T, E=E)
    c = [t.cuda() for t in (x, wr, w1, w3, w2)]
    out, state = M.forward_train(*c, k, renormalize=True, score_before_experts=True)
    grads = M.backward(state, dout.cuda(), *c, want_d_logits=True)
    torch.cuda.synchronize()
    assert M.device_status(state["state"]) == 0 and M.device_status(grads["ws"]) == 0
    assert torch.equal(out, M.forward(*c, k, True, score_before_experts=True))
    ref = O.moe_forward(x, wr, w1, w3, w2, k, True, score_before_experts=True)
    close(out, ref["out"])
    rdy, _ = O.combine_backward(dout, ref["y"], ref["dst_pos"], None)
    rdxp, rw1, rw3, rw2 = O.grouped_swiglu_backward(ref["x_perm"], ref["offsets"], w1, w3, w2,
                                                    rdy)
    rdxs, rdtw = O.scaled_dispatch_backward(rdxp, ref["dst_pos"], ref["topk_w"], x)
    rdz, rdwr, rdxr = O.router_backward(ref["logits"], ref["topk_idx"], rdtw, renormalize=True,
                                        x=x, w_router=wr)
    close(grads["dx"], rdxs + rdxr)
    for e in range(E):
        if int(ref["counts"][e]) == 0:
            continue
        close_wgrad(grads["dw1"][e], rw1[e])
        close_wgrad(grads["dw3"][e], rw3[e])
        close_wgrad(grads["dw2"][e], rw2[e])
    close_wgrad(grads["dw_router"], rdwr)
    gdz = f64(grads["d_logits"])
    assert np.linalg.norm(gdz - rdz) <= 1e-2 * np.linalg.norm(rdz)


@pytest.mark.parametrize("hs", [128, 320])
def test_layer_backward_shared_expert(M, hs):
    """A shared expert ([HP] MoE.forward: out = routed + shared_expert(x)):
    the training forward equals moe_forward_ex with it bit for bit; its
    weight gradients and its share of dx against the oracle (a one-segment
    SwiGLU backward over every token with the upstream dout, pinned with
    the rest of the layer by finite differences of the oracle)."""
    T, E, k = 200, 16, 4
    x, wr, w1, w3, w2, dout, sh = _small_train_layer(8, T=T, E=E, hs=hs)
    c = [t.cuda() for t in (x, wr, w1, w3, w2)]
    shc = tuple(t.cuda() for t in sh)
    out, state = M.forward_train(*c, k, renormalize=True, shared=shc)
    grads = M.backward(state, dout.cuda(), *c, shared=shc)
    torch.cuda.synchronize()
    assert M.device_status(state["state"]) == 0 and M.device_status(grads["ws"]) == 0
    assert torch.equal(out, M.forward(*c, k, True, shared=shc))
    ref = O.moe_forward(x, wr, w1, w3, w2, k, True, shared=sh)
    close(out, ref["out"])
    rdy, rdtw = O.combine_backward(dout, ref["y"], ref["dst_pos"], ref["topk_w"])
    rdxp, _, _, _ = O.grouped_swiglu_backward(ref["x_perm"], ref["offsets"], w1, w3, w2, rdy)
    _, _, rdxr = O.router_backward(ref["logits"], ref["topk_idx"], rdtw, renormalize=True, x=x,
                                   w_router=wr)
    rdxsh, rs1, rs3, rs2 = O.grouped_swiglu_backward(x, np.array([0, T]), sh[0][None],
                                                     sh[1][None], sh[2][None], dout)
    # dx is the sum of three shares that are each rounded to bf16 before the
    # sum (the routed copies', the router's and the shared expert's), so the
    # bf16 bound applies to the magnitude of the shares, not of their sum
    parts = [O.dispatch_backward(rdxp, ref["dst_pos"]), rdxr, rdxsh]
    ref_dx = sum(parts)
    err = np.abs(f64(grads["dx"]) - ref_dx)
    assert np.all(err <= 3e-2 * (1 + sum(np.abs(p) for p in parts))), err.max()
    assert np.linalg.norm(f64(grads["dx"]) - ref_dx) <= 1e-2 * np.linalg.norm(ref_dx)
    close_wgrad(grads["dws1"], rs1[0])
    close_wgrad(grads["dws3"], rs3[0])
    close_wgrad(grads["dws2"], rs2[0])
