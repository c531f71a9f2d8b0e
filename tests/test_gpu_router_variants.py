"""GPU parity of the router options -- sigmoid scores, route_scale,
node-limited group routing, selection-only expert_bias, the running
tokens_per_expert histogram -- and of score_before_experts, against the
oracle's general router (hyper_parallel TokenChoiceTopKRouter.forward, in
its order) and MoE.forward.

Selections the kernel makes on the logits themselves (no bias, positive
scale; groups included) are exact and compared bit for bit, order
included.  With a bias or a negative scale the keys c * scale + bias are
computed in fp32 on the GPU (a few roundings: error below 1e-6 times the
largest key of the token), so a token's indices must match exactly where
the oracle's fp64 keys of its top k + 1 experts (and, with groups, the
maxima of its kept and first dropped groups) are separated by more than
MARGIN times that key; elsewhere the GPU's choice must be a top-k within
that margin.  Weights are checked against the oracle's scores
of the experts the GPU chose (fp32 tolerance 1e-5 (1 + |ref|)); layer
outputs with the bf16 / fp32 tolerances of the other parity tests.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W

pytestmark = pytest.mark.gpu

MARGIN = 4e-6


@pytest.fixture(scope="module")
def M(cuda_ok):
    from routing_dispatch_grouped_topk_b200 import build
    build.build()
    import routing_dispatch_grouped_topk_b200 as m
    m.lib()
    return m


def close(got, ref, dtype):
    g = O.as_f64(got)
    ref = np.asarray(ref, dtype=np.float64)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    tol_max, tol_fro = (3e-2, 1e-2) if dtype == torch.bfloat16 else (1e-5, 1e-5)
    err = np.abs(g - ref)
    bad = err > tol_max * (1 + np.abs(ref))
    assert not bad.any(), f"{bad.sum()} elements off, worst {err.max()}"
    den = np.linalg.norm(ref)
    if den > 0:
        assert np.linalg.norm(g - ref) <= tol_fro * den, np.linalg.norm(g - ref) / den


def bias_for(E, seed):
    """A DeepSeek-style load-balancing bias: small, zero-mean, fp32."""
    rng = np.random.default_rng(seed + 500)
    b = rng.normal(size=E) * 0.05
    return (b - b.mean()).astype(np.float32)


def oracle_keys(L64, opts):
    """fp64 scores s and selection keys of the general router, by the
    oracle's own functions (softmax/sigmoid, node_limited_mask)."""
    s = O.softmax(L64) if opts.get("score", "softmax") == "softmax" else O.sigmoid(L64)
    c = s * opts.get("route_scale", 1.0)
    G = opts.get("num_groups", 0)
    if G:
        c = O.node_limited_mask(c, G, opts["topk_groups"])
    b = opts.get("expert_bias")
    keys = c + O.as_f64(b)[None, :] if b is not None else c
    return s, s * opts.get("route_scale", 1.0), keys


def on_logits(opts):
    return opts.get("expert_bias") is None and opts.get("route_scale", 1.0) > 0


def check_router(gi, gw, L, k, renorm, opts, relative=False):
    """GPU (gi, gw) against the oracle on fp32 logits L [T, E].  With
    ``relative`` the margin scales with the k-th and (k+1)-th keys of the
    token instead of its largest one (keys without a bias: each has the
    relative error of its own exponential, and the denominator, common to
    the token's keys, does not change their order)."""
    T, E = L.shape
    L64 = O.as_f64(L)
    idx, w, _, _ = O.router_topk_general(k, logits=L, renormalize=renorm, **opts)
    s, scaled, keys = oracle_keys(L64, opts)
    if on_logits(opts):
        assert np.array_equal(gi, idx)
        sure = np.ones(T, dtype=bool)
    else:
        srt = -np.sort(-keys, axis=1)[:, :k + 1]
        fin = np.where(np.isfinite(srt), np.abs(srt), 0.0)
        if relative:
            margin = MARGIN * fin[:, k - 1:k + 1].max(axis=1)
        else:
            margin = MARGIN * np.maximum(fin.max(axis=1), np.abs(scaled).max(axis=1))
        gaps = srt[:, :-1] - srt[:, 1:]
        sure = (gaps > margin[:, None]).all(axis=1)
        G = opts.get("num_groups", 0)
        if G:
            gmax = -np.sort(-scaled.reshape(T, G, E // G).max(axis=2), axis=1)
            tg = opts["topk_groups"]
            if tg < G:
                sure &= (gmax[:, tg - 1] - gmax[:, tg]) > margin
        assert sure.mean() > 0.8, sure.mean()
        assert np.array_equal(gi[sure], idx[sure])
        # elsewhere: distinct experts whose keys reach the k-th key within the margin
        for t in np.nonzero(~sure)[0]:
            assert len(set(gi[t].tolist())) == k
            if not G:
                assert keys[t, gi[t]].min() >= srt[t, k - 1] - margin[t]
    # weights: the oracle's unbiased scores of the experts the GPU chose
    wr = np.take_along_axis(s, gi.astype(np.int64), axis=1)
    if renorm:
        wr = wr / wr.sum(axis=1, keepdims=True)
    wr = wr * opts.get("route_scale", 1.0)
    close(gw, wr, torch.float32)
    return idx, sure


VARIANTS = [
    dict(score="sigmoid"),
    dict(score="sigmoid", route_scale=2.5),
    dict(score="softmax", route_scale=16.0),
    dict(score="softmax", num_groups=8, topk_groups=3),
    dict(score="sigmoid", num_groups=8, topk_groups=4, route_scale=2.5),
    dict(score="softmax", expert_bias=True),
    dict(score="sigmoid", expert_bias=True, num_groups=8, topk_groups=4, route_scale=2.5),
    dict(score="softmax", route_scale=-0.5),
]


def materialize(opts, E, seed, device="cuda"):
    """Options with the bias drawn; returns (oracle options, GPU options)."""
    o = dict(opts)
    if o.get("expert_bias"):
        o["expert_bias"] = bias_for(E, seed)
    g = dict(o)
    if g.get("expert_bias") is not None:
        g["expert_bias"] = torch.from_numpy(g["expert_bias"]).to(device)
    return o, g


@pytest.mark.parametrize("T,E,k", [(1000, 128, 8), (333, 256, 8), (257, 72, 6)])
@pytest.mark.parametrize("vi", range(len(VARIANTS)))
@pytest.mark.parametrize("renorm", [False, True])
def test_router_options_from_logits(M, T, E, k, vi, renorm):
    opts = dict(VARIANTS[vi])
    if opts.get("num_groups"):
        G = {128: 8, 256: 8, 72: 6}[E]
        opts["num_groups"] = G
        opts["topk_groups"] = min(opts["topk_groups"], G)
        assert k <= opts["topk_groups"] * (E // G)
    o, g = materialize(opts, E, seed=vi)
    L = W.make_logits(T, E, k, seed=vi + 11)
    gi, gw, gc, _, ws = M.router_topk(logits_in=torch.from_numpy(L).cuda(), top_k=k,
                                      renormalize=renorm, **g)
    assert M.device_status(ws) == 0
    gi, gw = gi.cpu().numpy(), gw.cpu()
    check_router(gi, gw, L, k, renorm, o)
    assert np.array_equal(gc.cpu().numpy(), np.bincount(gi.ravel(), minlength=E))


def test_node_limited_hand_case(M):
    """The hand case of the oracle's pins on the GPU: E = 4 in two groups,
    sigmoid scores of [3, -5, 2, 2]; one kept group gives experts {0, 1}."""
    L = torch.tensor([[3.0, -5.0, 2.0, 2.0]], device="cuda")
    gi, gw, _, _, _ = M.router_topk(logits_in=L, top_k=2, renormalize=False, score="sigmoid",
                                    num_groups=2, topk_groups=1)
    assert gi.cpu().tolist() == [[0, 1]]
    s = torch.sigmoid(torch.tensor([3.0, -5.0], dtype=torch.float64)).numpy()
    np.testing.assert_allclose(gw.cpu().numpy()[0], s, rtol=1e-6)
    gi, _, _, _, _ = M.router_topk(logits_in=L, top_k=2, renormalize=False, score="sigmoid",
                                   num_groups=2, topk_groups=2)
    assert gi.cpu().tolist() == [[0, 2]]


def test_expert_bias_hand_case(M):
    """Bias 0.9 on expert 2 of logits [0, 1, 0, 0]: expert 2 is selected and
    weighted by its probability 1 / (3 + e)."""
    L = torch.tensor([[0.0, 1.0, 0.0, 0.0]], device="cuda")
    b = torch.tensor([0.0, 0.0, 0.9, 0.0], device="cuda")
    gi, gw, _, _, _ = M.router_topk(logits_in=L, top_k=1, renormalize=False, expert_bias=b)
    assert gi.cpu().tolist() == [[2]]
    assert abs(gw.item() - 1.0 / (3.0 + np.e)) < 1e-7


def test_tokens_per_expert_accumulates(M):
    """tokens_per_expert += counts on every call ([HP] MoE.forward's running
    histogram); it is never cleared by the library."""
    T, E, k = 777, 64, 4
    L = torch.from_numpy(W.make_logits(T, E, k, seed=5)).cuda()
    tpe = torch.arange(E, dtype=torch.float32, device="cuda")
    for _ in range(2):
        gi, _, gc, _, _ = M.router_topk(logits_in=L, top_k=k, score="sigmoid",
                                        tokens_per_expert=tpe)
    cnt = np.bincount(gi.cpu().numpy().ravel(), minlength=E)
    assert np.array_equal(gc.cpu().numpy(), cnt)
    assert np.array_equal(tpe.cpu().numpy(), np.arange(E) + 2.0 * cnt)


@pytest.mark.parametrize("vi", [0, 4, 6])
def test_router_options_gemm_path(M, vi):
    """Options on top of the tensor-core router GEMM (Qwen3-30B-A3B sizes):
    the oracle routes the GPU's own fp32 logits."""
    c = W.config(1)
    lay = W.make_layer(c, "cuda", experts=False)
    opts = dict(VARIANTS[vi])
    o, g = materialize(opts, c.E, seed=vi)
    gi, gw, gc, logits, ws = M.router_topk(lay["x"], lay["w_router"], c.top_k, True,
                                           want_logits=True, **g)
    assert M.device_status(ws) == 0
    check_router(gi.cpu().numpy(), gw.cpu(), logits.cpu().numpy(), c.top_k, True, o)


def small(T, d, E, h, seed, dtype):
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn(T, d, generator=g).to(dtype)
    w1 = (torch.randn(E, h, d, generator=g) / d ** 0.5).to(dtype)
    w3 = (torch.randn(E, h, d, generator=g) / d ** 0.5).to(dtype)
    w2 = (torch.randn(E, d, h, generator=g) / h ** 0.5).to(dtype)
    return x, w1, w3, w2


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("before", [False, True])
@pytest.mark.parametrize("vi", [0, 4, 5])
def test_forward_options_full_oracle(M, dtype, before, vi):
    T, d, E, k, h = 300, 128, 16, 4, 192
    x, w1, w3, w2 = small(T, d, E, h, seed=vi, dtype=dtype)
    opts = dict(VARIANTS[vi])
    if opts.get("num_groups"):
        opts.update(num_groups=4, topk_groups=2)
    o, g = materialize(opts, E, seed=vi)
    L = W.make_logits(T, E, k, seed=vi + 3)
    res = M.forward(x.cuda(), None, w1.cuda(), w3.cuda(), w2.cuda(), k, True,
                    logits_in=torch.from_numpy(L).cuda(), want_router=True,
                    score_before_experts=before, **g)
    assert M.device_status(res["ws"]) == 0
    ref = O.moe_forward(x, None, w1, w3, w2, k, True, logits=L, router=o,
                        score_before_experts=before)
    gi = res["topk_idx"].cpu().numpy()
    _, sure = check_router(gi, res["topk_w"].cpu(), L, k, True, o)
    assert np.array_equal(res["counts"].cpu().numpy(), np.bincount(gi.ravel(), minlength=E))
    toks = np.nonzero(sure)[0]
    close(res["out"].cpu()[torch.from_numpy(toks)], ref["out"][toks], dtype)


def tokens_before(x_rows, idx_rows, w_rows, w1, w3, w2):
    """out[t] = sum_j FFN_{idx[t, j]}(w[t, j] x[t]) for sampled tokens."""
    x64 = O.as_f64(x_rows)
    w64 = O.as_f64(w_rows)
    out = np.zeros((x64.shape[0], w2.shape[1]))
    for e in np.unique(idx_rows):
        tt, jj = np.nonzero(idx_rows == e)
        ye = O.swiglu_ffn(x64[tt] * w64[tt, jj][:, None], w1[int(e)], w3[int(e)], w2[int(e)])
        np.add.at(out, tt, ye)
    return out


@pytest.mark.parametrize("before", [False, True])
def test_forward_deepseek_style_router_full_size_sampled(M, before):
    """Qwen3-30B-A3B layer sizes with a DeepSeek-V3-style router (sigmoid,
    8 groups keep 4, route_scale 2.5, renormalised), 128 sampled tokens."""
    c = W.config(1)
    lay = W.make_layer(c, "cuda")
    opts = dict(score="sigmoid", num_groups=8, topk_groups=4, route_scale=2.5)
    L = W.make_logits(c.T, c.E, c.top_k, seed=21)
    res = M.forward(lay["x"], lay["w_router"], lay["w1"], lay["w3"], lay["w2"], c.top_k, True,
                    logits_in=torch.from_numpy(L).cuda(), want_router=True,
                    score_before_experts=before, **opts)
    assert M.device_status(res["ws"]) == 0
    gi = res["topk_idx"].cpu().numpy()
    check_router(gi, res["topk_w"].cpu(), L, c.top_k, True, opts)
    idx, w, _, _ = O.router_topk_general(c.top_k, logits=L, renormalize=True, **opts)
    toks = np.sort(np.random.default_rng(1).choice(c.T, size=128, replace=False))
    xs = lay["x"].cpu()[torch.from_numpy(toks)]
    w1, w3, w2 = lay["w1"].cpu(), lay["w3"].cpu(), lay["w2"].cpu()
    if before:
        ref = tokens_before(xs, idx[toks], w[toks], w1, w3, w2)
    else:
        ref = O.moe_tokens(xs, idx[toks], w[toks], w1, w3, w2)
    close(res["out"].cpu()[torch.from_numpy(toks)], ref, torch.bfloat16)


def test_forward_before_experts_ep_equals_single_device_bitwise(M):
    """gpt-oss-120b EP8 sizes: the rank-major dispatch with row scaling,
    regroup, experts and unweighted combine give the single-device result
    bit for bit."""
    c = W.config(4)
    lay = W.make_layer(c, "cuda")
    args = (lay["x"], lay["w_router"], lay["w1"], lay["w3"], lay["w2"], c.top_k, True)
    a = M.forward(*args, ep_ranks=8, score_before_experts=True, score="sigmoid")
    b = M.forward(*args, ep_ranks=1, score_before_experts=True, score="sigmoid")
    assert torch.equal(a, b)


@pytest.mark.parametrize("vi", [0, 5])
def test_load_balance_loss(M, vi):
    """aux_loss = E sum_e f_e P_e of the call ([HP] _compute_load_balance_loss)
    against the oracle on the GPU's own routing (fp32 atomics: 1e-5)."""
    T, E, k = 1000, 128, 8
    o, g = materialize(dict(VARIANTS[vi]), E, seed=vi)
    L = W.make_logits(T, E, k, seed=vi + 31)
    aux = torch.full((1,), -1.0, device="cuda")
    gi, gw, _, _, ws = M.router_topk(logits_in=torch.from_numpy(L).cuda(), top_k=k,
                                     renormalize=True, aux_loss=aux, **g)
    assert M.device_status(ws) == 0
    ref = O.load_balance_loss(gw.cpu().numpy(), gi.cpu().numpy(), E)
    assert abs(aux.item() - ref) <= 1e-5 * abs(ref), (aux.item(), ref)


def test_load_balance_loss_in_forward_and_empty(M):
    c = W.config(1)
    lay = W.make_layer(c, "cuda")
    aux = torch.full((1,), -1.0, device="cuda")
    res = M.forward(lay["x"], lay["w_router"], lay["w1"], lay["w3"], lay["w2"], c.top_k, True,
                    want_router=True, aux_loss=aux)
    assert M.device_status(res["ws"]) == 0
    ref = O.load_balance_loss(res["topk_w"].cpu().numpy(), res["topk_idx"].cpu().numpy(), c.E)
    assert abs(aux.item() - ref) <= 1e-5 * abs(ref), (aux.item(), ref)
    assert 0.9 < ref < 1.1            # a near-uniform router is near the balanced value 1
    aux.fill_(-1.0)
    L0 = torch.zeros(0, 16, device="cuda")
    M.router_topk(logits_in=L0, top_k=2, aux_loss=aux)
    assert aux.item() == 0.0


# Shapes that put the fused tcgen05 router on each cluster size C (= threads
# per token in its scoring): (T, d, E, k) -> C = 8, 4, 2, 1; E not a multiple
# of 4 and k = 1 / 16 included.
FUSED_SHAPES = [(200, 1024, 61, 5), (2500, 512, 130, 16), (3000, 128, 37, 3), (129, 64, 255, 1)]
FUSED_VARIANTS = [dict(), VARIANTS[0], VARIANTS[2], VARIANTS[5], VARIANTS[7]]


@pytest.mark.parametrize("T,d,E,k", FUSED_SHAPES)
@pytest.mark.parametrize("vi", range(len(FUSED_VARIANTS)))
@pytest.mark.parametrize("renorm", [False, True])
def test_fused_router_options(M, T, d, E, k, vi, renorm):
    """The fused router (bf16 gate, no groups) with the options: indices and
    weights against the oracle's general router on the GPU's own fp32
    logits, and the selected experts' unbiased scores (topk_scores)."""
    g = torch.Generator().manual_seed(T + d + E + k)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16).cuda()
    wr = (torch.randn(E, d, generator=g) * (2.0 / d ** 0.5)).to(torch.bfloat16).cuda()
    o, go = materialize(dict(FUSED_VARIANTS[vi]), E, seed=vi)
    sc = torch.empty(T, k, dtype=torch.float32, device="cuda")
    gi, gw, gc, logits, ws = M.router_topk(x, wr, k, renorm, want_logits=True, topk_scores=sc,
                                           **go)
    torch.cuda.synchronize()
    assert M.device_status(ws) == 0
    gi = gi.cpu().numpy()
    L = logits.cpu().numpy()
    # A negative scale selects the smallest scores, far below the token's
    # largest key: their margin is taken relative to the keys at the cut.
    check_router(gi, gw.cpu(), L, k, renorm, o,
                 relative=o.get("expert_bias") is None and o.get("route_scale", 1) < 0)
    assert np.array_equal(gc.cpu().numpy(), np.bincount(gi.ravel(), minlength=E))
    s, _, _ = oracle_keys(O.as_f64(L), o)
    close(sc.cpu(), np.take_along_axis(s, gi.astype(np.int64), axis=1), torch.float32)


# Node-limited groups on the tensor-core router (split-K gate and the
# warp-per-token top-k) over token counts, reductions and expert counts
GROUP_SHAPES = [(200, 1024, 64, 5), (6000, 512, 128, 16), (3000, 128, 32, 3), (129, 64, 256, 1)]


@pytest.mark.parametrize("T,d,E,k", GROUP_SHAPES)
@pytest.mark.parametrize("vi", [3, 4, 6])
@pytest.mark.parametrize("renorm", [False, True])
def test_router_node_limited_groups_gemm(M, T, d, E, k, vi, renorm):
    """Group-limited routing (8 groups; 3 or 4 kept) on the bf16 gate, with
    sigmoid scores, a scale and a selection-only bias: indices and weights
    against the oracle's general router on the GPU's own logits."""
    g = torch.Generator().manual_seed(T + d + E + k + vi)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16).cuda()
    wr = (torch.randn(E, d, generator=g) * (2.0 / d ** 0.5)).to(torch.bfloat16).cuda()
    o, go = materialize(dict(VARIANTS[vi]), E, seed=vi)
    gi, gw, gc, logits, ws = M.router_topk(x, wr, k, renorm, want_logits=True, **go)
    torch.cuda.synchronize()
    assert M.device_status(ws) == 0
    gi = gi.cpu().numpy()
    check_router(gi, gw.cpu(), logits.cpu().numpy(), k, renorm, o)
    assert np.array_equal(gc.cpu().numpy(), np.bincount(gi.ravel(), minlength=E))
