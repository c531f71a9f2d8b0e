"""GPU parity of the capacity drop policy ([PF] PaddleFormers moe_gate.py,
_probs_drop_policy) in the router and the layer forward.

The keep decision compares scores across tokens, so it is taken in the
kernel's precision: the oracle's capacity rule is applied to the fp32
scores the router returns (topk_scores), and the routing with the policy
must then equal, bit for bit, the routing without it with the dropped
copies marked (-1, weight 0).  The scores themselves are checked against
the oracle's fp64 scores, and the layer output of a forward with the policy
against the oracle's token-by-token definition over the kept copies.
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


def i32(a):
    return torch.as_tensor(np.asarray(a), dtype=torch.int32, device="cuda")


def routed(M, k, capacity, renorm, score, logits=None, x=None, wr=None):
    T = (logits if logits is not None else x).shape[0]
    sc = torch.empty(T, k, dtype=torch.float32, device="cuda")
    idx, w, counts, _, ws = M.router_topk(x, wr, k, renorm, logits_in=logits, score=score,
                                          capacity=capacity, topk_scores=sc)
    torch.cuda.synchronize()
    assert M.device_status(ws) == 0
    return idx.cpu().numpy(), w.cpu().numpy(), counts.cpu().numpy(), sc.cpu().numpy()


@pytest.mark.parametrize("score,renorm", [("softmax", True), ("sigmoid", False)])
# (6000, 8, 2): the overloaded expert holds more copies than the select
# kernel keeps in shared memory (its passes read the flat copy list)
@pytest.mark.parametrize("T,E,k,frac", [(512, 16, 2, 0.8), (3000, 64, 4, 0.6), (777, 8, 3, 1.1),
                                        (6000, 8, 2, 0.5)])
def test_router_capacity_from_logits(M, score, renorm, T, E, k, frac):
    L = W.make_logits(T, E, k, seed=T + E)
    L[:, 1] += 1.5                          # one expert overloaded
    lg = torch.from_numpy(L).float().cuda()
    idx0, w0, c0, s0 = routed(M, k, 0, renorm, score, logits=lg)
    ridx, rw, _, _ = O.router_topk_general(k, logits=L, score=score, renormalize=renorm)
    assert np.array_equal(idx0, ridx)
    rs = np.take_along_axis(O.softmax(L) if score == "softmax" else O.sigmoid(L), ridx, axis=1)
    assert np.allclose(s0, rs, rtol=2e-6, atol=1e-30)
    cap = max(1, int(frac * T * k / E))
    idx, w, c, s = routed(M, k, cap, renorm, score, logits=lg)
    assert np.array_equal(s, s0)
    keep = O.capacity_drop(idx0, s0, cap)
    assert np.array_equal(idx, np.where(keep, idx0, -1))
    assert np.array_equal(w, np.where(keep, w0, 0.0).astype(np.float32))
    assert np.array_equal(c, np.bincount(idx0[keep], minlength=E))
    assert (~keep).any() and (c <= cap).all()


def test_router_capacity_fused_gate(M):
    """The tcgen05 router (bf16 x, w_router, E <= 256): scores from the fused
    kernel, the capacity applied after it."""
    c = W.config(1)
    lay = W.make_layer(c, "cuda", experts=False)
    x, wr = lay["x"], lay["w_router"]
    idx0, w0, c0, s0 = routed(M, c.top_k, 0, True, "softmax", x=x, wr=wr)
    cap = int(0.9 * c.T * c.top_k / c.E)
    idx, w, cnt, s = routed(M, c.top_k, cap, True, "softmax", x=x, wr=wr)
    keep = O.capacity_drop(idx0, s0, cap)
    assert np.array_equal(idx, np.where(keep, idx0, -1))
    assert np.array_equal(w, np.where(keep, w0, 0.0).astype(np.float32))
    assert np.array_equal(cnt, np.bincount(idx0[keep], minlength=c.E))
    assert (~keep).sum() == np.maximum(c0 - cap, 0).sum() > 0


def test_dispatch_skips_dropped_copies_without_error(M):
    T, E, k = 40, 8, 2
    L = W.make_logits(T, E, k, seed=5)
    idx, *_ = O.router_topk(k, True, logits=L)
    idx[3, 1] = -1
    idx[7, 0] = -1
    x = torch.randn(T, 64).to(torch.bfloat16).cuda()
    gc, goff, gsrc, gdst, gxp, ws = M.dispatch(x, i32(idx), E)
    torch.cuda.synchronize()
    assert M.device_status(ws) == 0
    rc, roff, rsrc, rdst = O.dispatch(idx, E)
    assert np.array_equal(gc.cpu().numpy(), rc)
    assert np.array_equal(goff.cpu().numpy(), roff)
    assert np.array_equal(gdst.cpu().numpy(), rdst)
    n = int(roff[-1])
    assert np.array_equal(gsrc.cpu().numpy()[:n], rsrc)
    assert np.all(gsrc.cpu().numpy()[n:] == -1)


@pytest.mark.parametrize("cfg,frac", [(1, 0.9), (4, 0.8)])
def test_forward_with_capacity(M, cfg, frac):
    """moe_forward_ex with the policy: the routing it returns is the policy
    applied to its own scores, the kept copies run through the experts
    (offsets[E] < T k) and every sampled token's output is the oracle's
    sum over its kept copies."""
    c = W.config(cfg)
    lay = W.make_layer(c, "cuda")
    x, wr, w1, w3, w2 = (lay[n] for n in ("x", "w_router", "w1", "w3", "w2"))
    cap = int(frac * c.T * c.top_k / c.E)
    sc = torch.empty(c.T, c.top_k, dtype=torch.float32, device="cuda")
    res = M.forward(x, wr, w1, w3, w2, c.top_k, c.renormalize, want_router=True, capacity=cap,
                    topk_scores=sc)
    torch.cuda.synchronize()
    assert M.device_status(res["ws"]) == 0
    gi = res["topk_idx"].cpu().numpy()
    gw = res["topk_w"].cpu().numpy()
    dropped = gi < 0
    assert dropped.any()
    assert np.array_equal(res["counts"].cpu().numpy(), np.bincount(gi[~dropped], minlength=c.E))
    # the forward's routing is the router's routing with the policy applied
    i0, w0, _, _, _ = M.router_topk(x, wr, c.top_k, c.renormalize)
    keep = O.capacity_drop(i0.cpu().numpy(), sc.cpu().numpy(), cap)
    assert np.array_equal(gi, np.where(keep, i0.cpu().numpy(), -1))
    toks = np.sort(np.random.default_rng(c.seed).choice(c.T, size=64, replace=False))
    tt = torch.from_numpy(toks)
    ref = O.moe_tokens(x.cpu()[tt], np.where(dropped, 0, gi)[toks],
                       np.where(dropped, 0.0, gw)[toks], w1.cpu(), w3.cpu(), w2.cpu())
    g = O.as_f64(res["out"].cpu()[tt])
    err = np.abs(g - ref)
    assert np.all(err <= 3e-2 * (1 + np.abs(ref))), err.max()
    assert np.linalg.norm(g - ref) <= 1e-2 * np.linalg.norm(ref)
