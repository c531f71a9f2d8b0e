"""GPU parity of the shared expert ([HP] MoE.forward: the routed output plus
shared_expert(x_flat), a dense SwiGLU FeedForward on every token) against
the oracle, at the tolerances of the other parity tests (bf16:
max|err| <= 3e-2 (1 + |ref|), ||err||_F <= 1e-2 ||ref||_F; fp32: 1e-5)."""
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


def weights(shape_list, seed, dtype, fan_in):
    g = torch.Generator().manual_seed(seed)
    return [(torch.randn(*s, generator=g) / fi ** 0.5).to(dtype) for s, fi in zip(shape_list,
                                                                                    fan_in)]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("before", [False, True])
def test_shared_expert_full_oracle(M, dtype, before):
    T, d, E, k, h, hs = 300, 128, 16, 4, 192, 256
    g = torch.Generator().manual_seed(7)
    x = torch.randn(T, d, generator=g).to(dtype)
    w1, w3, w2, s1, s3, s2 = weights([(E, h, d), (E, h, d), (E, d, h), (hs, d), (hs, d), (d, hs)],
                                     8, dtype, [d, d, h, d, d, hs])
    L = W.make_logits(T, E, k, seed=9)
    res = M.forward(x.cuda(), None, w1.cuda(), w3.cuda(), w2.cuda(), k, True,
                    logits_in=torch.from_numpy(L).cuda(), want_router=True,
                    shared=(s1.cuda(), s3.cuda(), s2.cuda()), score_before_experts=before)
    assert M.device_status(res["ws"]) == 0
    ref = O.moe_forward(x, None, w1, w3, w2, k, True, logits=L, shared=(s1, s3, s2),
                        score_before_experts=before)
    assert np.array_equal(res["topk_idx"].cpu().numpy(), ref["topk_idx"])
    close(res["out"].cpu(), ref["out"], dtype)


def test_shared_expert_full_size_sampled(M):
    """Qwen3-30B-A3B layer sizes plus a 2048-wide shared expert; 128 sampled
    tokens against the token-by-token definition."""
    c = W.config(1)
    lay = W.make_layer(c, "cuda")
    hs = 2048
    s1, s3, s2 = weights([(hs, c.d), (hs, c.d), (c.d, hs)], 31, torch.bfloat16, [c.d, c.d, hs])
    L = W.make_logits(c.T, c.E, c.top_k, seed=12)
    res = M.forward(lay["x"], lay["w_router"], lay["w1"], lay["w3"], lay["w2"], c.top_k, True,
                    logits_in=torch.from_numpy(L).cuda(), want_router=True,
                    shared=(s1.cuda(), s3.cuda(), s2.cuda()))
    assert M.device_status(res["ws"]) == 0
    idx, w, _, _ = O.router_topk(c.top_k, True, logits=L)
    assert np.array_equal(res["topk_idx"].cpu().numpy(), idx)
    toks = np.sort(np.random.default_rng(3).choice(c.T, size=128, replace=False))
    xs = lay["x"].cpu()[torch.from_numpy(toks)]
    ref = O.moe_tokens(xs, idx[toks], w[toks], lay["w1"].cpu(), lay["w3"].cpu(),
                       lay["w2"].cpu()) + O.swiglu_ffn(xs, s1, s3, s2)
    close(res["out"].cpu()[torch.from_numpy(toks)], ref, torch.bfloat16)


def test_shared_expert_ep_equals_single_device_bitwise(M):
    c = W.config(4)
    lay = W.make_layer(c, "cuda")
    s1, s3, s2 = weights([(1024, c.d), (1024, c.d), (c.d, 1024)], 5, torch.bfloat16,
                         [c.d, c.d, 1024])
    sh = (s1.cuda(), s3.cuda(), s2.cuda())
    args = (lay["x"], lay["w_router"], lay["w1"], lay["w3"], lay["w2"], c.top_k, True)
    a = M.forward(*args, ep_ranks=8, shared=sh)
    b = M.forward(*args, ep_ranks=1, shared=sh)
    assert torch.equal(a, b)


@pytest.mark.parametrize("T", [0, 1, 130])
def test_shared_expert_edge_sizes(M, T):
    d, E, k, h, hs = 128, 8, 2, 128, 64
    g = torch.Generator().manual_seed(T)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16)
    wr = (torch.randn(E, d, generator=g) * 0.02).to(torch.bfloat16)
    w1, w3, w2, s1, s3, s2 = weights([(E, h, d), (E, h, d), (E, d, h), (hs, d), (hs, d), (d, hs)],
                                     T + 1, torch.bfloat16, [d, d, h, d, d, hs])
    res = M.forward(x.cuda(), wr.cuda(), w1.cuda(), w3.cuda(), w2.cuda(), k, True,
                    want_router=True, shared=(s1.cuda(), s3.cuda(), s2.cuda()))
    assert M.device_status(res["ws"]) == 0
    assert res["out"].shape == (T, d)
    if T == 0:
        return
    gi = res["topk_idx"].cpu().numpy()
    gw = res["topk_w"].cpu().numpy()
    ref = O.moe_tokens(x, gi, gw, w1, w3, w2) + O.swiglu_ffn(x, s1, s3, s2)
    close(res["out"].cpu(), ref, torch.bfloat16)
