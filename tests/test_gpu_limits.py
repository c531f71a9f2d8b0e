"""GPU parity at the limits of the C ABI (include/moe.h): the largest expert
count and top_k (E = 512, top_k = 16), a million routed copies in one
dispatch, and fp32 layers with d and h that are multiples of 4 but not of
64.  Integers bit-exact, floats within the layer tolerances of the other
parity tests."""
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


def layer(T, d, E, h, seed, dtype):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, d, generator=g).to(dtype)
    w1 = (torch.randn(E, h, d, generator=g) / d ** 0.5).to(dtype)
    w3 = (torch.randn(E, h, d, generator=g) / d ** 0.5).to(dtype)
    w2 = (torch.randn(E, d, h, generator=g) / h ** 0.5).to(dtype)
    return x, w1, w3, w2


def test_forward_max_experts_and_topk(M):
    """E = 512 experts, top_k = 16 (MOE_MAX_EXPERTS, MOE_MAX_TOPK), bf16,
    generated logits: every integer output exact, 256 sampled tokens."""
    T, d, E, k, h = 2048, 256, 512, 16, 128
    x, w1, w3, w2 = layer(T, d, E, h, 1, torch.bfloat16)
    L = W.make_logits(T, E, k, seed=41)
    res = M.forward(x.cuda(), None, w1.cuda(), w3.cuda(), w2.cuda(), k, True,
                    logits_in=torch.from_numpy(L).cuda(), want_router=True)
    assert M.device_status(res["ws"]) == 0
    idx, w, counts, _ = O.router_topk(k, True, logits=L)
    assert np.array_equal(res["topk_idx"].cpu().numpy(), idx)
    assert np.array_equal(res["counts"].cpu().numpy(), counts)
    close(res["topk_w"].cpu(), w, torch.float32)
    toks = np.sort(np.random.default_rng(0).choice(T, size=256, replace=False))
    ref = O.moe_tokens(x[torch.from_numpy(toks)], idx[toks], w[toks], w1, w3, w2)
    close(res["out"].cpu()[torch.from_numpy(toks)], ref, torch.bfloat16)


def test_dispatch_a_million_copies(M):
    """T = 131072 tokens x top_k = 8 = 1,048,576 routed copies over E = 256
    experts with a Zipf-like skew: counts, offsets, src_row and dst_pos are
    the oracle's stable expert-major order bit for bit; x_perm is the exact
    row gather."""
    T, d, E, k = 131072, 64, 256, 8
    rng = np.random.default_rng(7)
    p = 1.0 / np.arange(1, E + 1) ** 1.1
    p /= p.sum()
    idx = np.empty((T, k), dtype=np.int64)
    for t0 in range(0, T, 16384):          # k distinct experts per token
        n = min(16384, T - t0)
        keys = rng.gumbel(size=(n, E)) + np.log(p)[None, :]
        idx[t0:t0 + n] = np.argsort(-keys, axis=1, kind="stable")[:, :k]
    x = torch.randn(T, d, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    counts, offsets, src_row, dst_pos, x_perm, ws = M.dispatch(
        x.cuda(), torch.from_numpy(idx.astype(np.int32)).cuda(), E)
    assert M.device_status(ws) == 0
    c, off, src, dst = O.dispatch(idx, E)
    assert np.array_equal(counts.cpu().numpy(), c)
    assert np.array_equal(offsets.cpu().numpy(), off)
    assert np.array_equal(src_row.cpu().numpy(), src)
    assert np.array_equal(dst_pos.cpu().numpy(), dst)
    assert torch.equal(x_perm.cpu(), x[torch.from_numpy(src)])


@pytest.mark.parametrize("d,h", [(68, 36), (132, 4)])
def test_forward_fp32_unaligned_to_tiles(M, d, h):
    """fp32 layers whose d and h are multiples of 4 but not of the 64-wide
    tiles (the CUDA-core path), against the full oracle at 1e-5."""
    T, E, k = 300, 6, 2
    x, w1, w3, w2 = layer(T, d, E, h, d + h, torch.float32)
    g = torch.Generator().manual_seed(d)
    wr = torch.randn(E, d, generator=g) * 0.5
    res = M.forward(x.cuda(), wr.cuda(), w1.cuda(), w3.cuda(), w2.cuda(), k, True,
                    want_router=True)
    assert M.device_status(res["ws"]) == 0
    gi = res["topk_idx"].cpu().numpy()
    idx, w, _, L64 = O.router_topk(k, True, x=x, w_router=wr)
    srt = -np.sort(-L64, axis=1)
    sure = (srt[:, k - 1] - srt[:, k]) > 1e-4 * (1 + np.abs(srt[:, k - 1]))
    assert sure.mean() > 0.9
    assert np.array_equal(gi[sure], idx[sure])
    ref = O.moe_tokens(x, gi, res["topk_w"].cpu().numpy(), w1, w3, w2)
    close(res["out"].cpu(), ref, torch.float32)
