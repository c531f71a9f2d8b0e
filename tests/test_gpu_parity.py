"""GPU parity: every entry point of libmoe against the fp64 CPU oracle.

Integer outputs (top-k indices, counts, offsets, permutations) must match
bit for bit; copies (x_perm, regroup rows) must be bitwise identical;
floating-point outputs must meet the layer tolerance:

* bf16 I/O, fp32 accumulation: max|err| <= 3e-2 (1 + |ref|) and
  ||err||_F <= 1e-2 ||ref||_F
* fp32 layers (and the fp32 routing weights): max|err| <= 1e-5 (1 + |ref|)
  and ||err||_F <= 1e-5 ||ref||_F

Top-k decisions taken on fp32 logits computed by the GPU's own contraction
are compared where the oracle's fp64 gap between the k-th and (k+1)-th
logit exceeds the fp32 dot-product error bound; elsewhere only validity of
the GPU's choice is checked.  With logits supplied as input (gap >= 1e-3)
the indices must match everywhere.
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


def close(got, ref, dtype):
    g = f64(got)
    ref = np.asarray(ref, dtype=np.float64)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    tol_max, tol_fro = (3e-2, 1e-2) if dtype == torch.bfloat16 else (1e-5, 1e-5)
    err = np.abs(g - ref)
    bad = err > tol_max * (1 + np.abs(ref))
    assert not bad.any(), f"{bad.sum()} elements off, worst {err.max()}"
    den = np.linalg.norm(ref)
    if den > 0:
        assert np.linalg.norm(g - ref) <= tol_fro * den, np.linalg.norm(g - ref) / den


def small_layer(T, d, E, k, h, seed, dtype=torch.bfloat16, device="cuda"):
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn(T, d, generator=g).to(dtype)
    wr = (torch.randn(E, d, generator=g) * 0.02).to(dtype)
    w1 = (torch.randn(E, h, d, generator=g) / math.sqrt(d)).to(dtype)
    w3 = (torch.randn(E, h, d, generator=g) / math.sqrt(d)).to(dtype)
    w2 = (torch.randn(E, d, h, generator=g) / math.sqrt(h)).to(dtype)
    return [t.to(device) for t in (x, wr, w1, w3, w2)]


def i32(a, device="cuda"):
    return torch.as_tensor(np.asarray(a), dtype=torch.int32, device=device)


ROUTER_SHAPES = [(c.T, c.E, c.top_k) for c in W.CONFIGS] + [(1, 1, 1), (37, 8, 8), (129, 300, 16)]


# ----------------------------------------------------------------- router
@pytest.mark.parametrize("T,E,k", ROUTER_SHAPES)
@pytest.mark.parametrize("renorm", [True, False])
def test_router_from_logits_exact(M, T, E, k, renorm):
    L = W.make_logits(T, E, k, seed=T + E + k)
    idx, w, counts, _ = O.router_topk(k, renorm, logits=L)
    gi, gw, gc, _, _ = M.router_topk(top_k=k, renormalize=renorm,
                                     logits_in=torch.from_numpy(L).cuda())
    assert np.array_equal(gi.cpu().numpy(), idx)
    assert np.array_equal(gc.cpu().numpy(), counts)
    close(gw, w, torch.float32)


def router_gemm_check(M, x, wr, k, renorm, dtype):
    T, d = x.shape
    E = wr.shape[0]
    gi, gw, gc, gl, _ = M.router_topk(x, wr, top_k=k, renormalize=renorm, want_logits=True)
    L64 = O.router_logits(x, wr)
    # fp32 dot-product error bound (products of bf16 values are exact in fp32)
    absdot = np.abs(f64(x)) @ np.abs(f64(wr)).T
    bound = (d + 2) * 2.0 ** -23 * absdot + 1e-30
    err = np.abs(f64(gl) - L64)
    assert np.all(err <= bound), (err / bound).max()
    idx, w, counts, _ = O.router_topk(k, renorm, logits=L64)
    gi = gi.cpu().numpy()
    margin = 2 * bound.max(axis=1)
    sure = compare_topk(gi, idx, L64, margin)
    assert gc.cpu().numpy().sum() == T * k
    assert np.array_equal(gc.cpu().numpy(), np.bincount(gi.ravel(), minlength=E))
    # weights compared per expert (the order of two near-equal experts may differ)
    gw = gw.cpu().numpy()
    for t in np.nonzero(sure)[0]:
        got = dict(zip(gi[t].tolist(), gw[t].tolist()))
        ref = np.array([got[e] for e in idx[t].tolist()])
        assert np.all(np.abs(ref - w[t]) <= 1e-5 * (1 + np.abs(w[t])))
    return sure


def compare_topk(gi, idx, L64, margin):
    """Top-k indices from GPU-computed fp32 logits vs the oracle's fp64 ones.

    ``margin[t]`` bounds twice the logit error of token t.  Where the k-th and
    (k+1)-th fp64 logits are more than ``margin`` apart the selected SET must
    be the oracle's; inside the set, two experts whose logits are more than
    ``margin`` apart must keep the oracle's order.  Elsewhere the GPU's choice
    must be valid: k distinct experts, none below the k-th logit by more than
    ``margin``.  Returns the mask of tokens whose set is decided."""
    T, k = idx.shape
    E = L64.shape[1]
    srt = -np.sort(-L64, axis=1)
    sure = (srt[:, k - 1] - srt[:, k] > margin) if k < E else np.ones(T, dtype=bool)
    for t in range(T):
        g = gi[t].tolist()
        assert len(set(g)) == k and all(0 <= e < E for e in g)
        assert np.all(L64[t, g] >= srt[t, k - 1] - margin[t])
        if sure[t]:
            assert sorted(g) == sorted(idx[t].tolist()), t
            lg = L64[t, g]
            for a in range(k):
                for b in range(a + 1, k):
                    # GPU order a before b: b's logit must not exceed a's by > margin
                    assert lg[b] <= lg[a] + margin[t], (t, g)
    return sure


def test_router_gemm_integer_logits_exact_with_ties(M):
    """Integer-valued x and w_router: every fp32 partial sum is exact, so the
    GPU logits equal the fp64 ones bit for bit and the top-k (with many
    ties) must match the oracle everywhere, order and tie-break included."""
    for (T, d, E, k) in [(300, 64, 128, 8), (129, 128, 64, 16), (64, 256, 32, 4)]:
        g = torch.Generator().manual_seed(T)
        x = torch.randint(-2, 3, (T, d), generator=g).to(torch.bfloat16)
        wr = torch.randint(-1, 2, (E, d), generator=g).to(torch.bfloat16)
        gi, gw, gc, gl, _ = M.router_topk(x.cuda(), wr.cuda(), top_k=k, renormalize=True,
                                          want_logits=True)
        idx, w, counts, L64 = O.router_topk(k, True, x=x, w_router=wr)
        assert np.array_equal(f64(gl), L64)
        assert np.array_equal(gi.cpu().numpy(), idx)
        assert np.array_equal(gc.cpu().numpy(), counts)
        close(gw, w, torch.float32)


# Tokens of each workload (inputs drawn on the CPU) whose top-k set the fp32
# dot-product error bound decides: the k-th and (k+1)-th fp64 logits are
# more than twice the bound apart.  Their indices must equal the oracle's;
# the others are checked for validity only.  The counts depend on the
# inputs and the bound alone, not on the GPU, and are asserted exactly.
DECIDED_TOKENS = {0: 256, 1: 3258, 2: 14589, 3: 34, 4: 6563}


@pytest.mark.parametrize("cfg", [0, 1, 2, 3, 4])
def test_router_gemm_configs(M, cfg):
    c = W.config(cfg)
    lay = W.make_layer(c, "cpu", experts=False)
    sure = router_gemm_check(M, lay["x"].cuda(), lay["w_router"].cuda(), c.top_k,
                             c.renormalize, c.torch_dtype())
    print(f"{c.name}: top-k set decided by the error bound on {sure.sum()} of {c.T} tokens "
          f"({sure.mean():.3f})")
    assert int(sure.sum()) == DECIDED_TOKENS[cfg]


@pytest.mark.parametrize("T,d,E,k", [(1, 64, 8, 2), (130, 72, 8, 3), (300, 256, 32, 4),
                                     (257, 128, 200, 16), (64, 64, 256, 8), (50, 96, 300, 5)])
def test_router_gemm_shapes(M, T, d, E, k):
    x, wr, *_ = small_layer(T, d, E, k, 64, seed=T + d + E)
    wr = (wr.float() * 50).to(torch.bfloat16)   # spread the logits
    sure = router_gemm_check(M, x, wr, k, True, torch.bfloat16)
    assert sure.mean() >= 0.25


# --------------------------------------------------------------- dispatch
DISPATCH_CASES = [(c.T, c.d, c.E, c.top_k, c.dtype) for c in W.CONFIGS] + [
    (1, 64, 4, 1, "bf16"), (33, 64, 8, 8, "bf16"), (1000, 16, 512, 16, "f32"), (5, 8, 3, 2, "bf16")]


@pytest.mark.parametrize("T,d,E,k,dt", DISPATCH_CASES)
def test_dispatch_exact(M, T, d, E, k, dt):
    dtype = torch.float32 if dt == "f32" else torch.bfloat16
    L = W.make_logits(T, E, k, seed=T * 3 + E)
    idx, *_ = O.router_topk(k, True, logits=L)
    x = torch.randn(T, d, generator=torch.Generator().manual_seed(T)).to(dtype)
    c, off, src, dst = O.dispatch(idx, E)
    gc, goff, gsrc, gdst, gxp, ws = M.dispatch(x.cuda(), i32(idx), E)
    assert np.array_equal(gc.cpu().numpy(), c)
    assert np.array_equal(goff.cpu().numpy(), off)
    assert np.array_equal(gsrc.cpu().numpy(), src)
    assert np.array_equal(gdst.cpu().numpy(), dst)
    assert torch.equal(gxp.cpu(), x[torch.from_numpy(src)])
    assert M.device_status(ws) == 0


def test_dispatch_skewed_with_empty_experts(M):
    T, E, k = 5000, 64, 4
    rng = np.random.default_rng(0)
    p = rng.dirichlet(np.full(E, 0.05))
    p[[3, 17, 40]] = 0
    p /= p.sum()
    idx = np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)])
    x = torch.randn(T, 128).to(torch.bfloat16)
    c, off, src, dst = O.dispatch(idx, E)
    gc, goff, gsrc, gdst, gxp, ws = M.dispatch(x.cuda(), i32(idx), E)
    assert (c == 0).sum() >= 3
    assert np.array_equal(gc.cpu().numpy(), c) and np.array_equal(goff.cpu().numpy(), off)
    assert np.array_equal(gsrc.cpu().numpy(), src) and np.array_equal(gdst.cpu().numpy(), dst)
    assert torch.equal(gxp.cpu(), x[torch.from_numpy(src)])


def test_dispatch_bad_expert_id_sets_status(M):
    T, E, k = 40, 8, 2
    L = W.make_logits(T, E, k, seed=5)
    idx, *_ = O.router_topk(k, True, logits=L)
    idx[3, 1] = E
    idx[7, 0] = -1
    x = torch.randn(T, 64).to(torch.bfloat16).cuda()
    gc, goff, gsrc, gdst, gxp, ws = M.dispatch(x, i32(idx), E)
    assert M.device_status(ws) & M.MOE_DEV_BAD_EXPERT
    gdst = gdst.cpu().numpy()
    assert gdst[3, 1] == -1 and gdst[7, 0] == -1
    valid = (idx >= 0) & (idx < E)
    assert np.array_equal(gc.cpu().numpy(), np.bincount(idx[valid], minlength=E))
    assert goff.cpu().numpy()[-1] == valid.sum()
    assert np.all(gsrc.cpu().numpy()[valid.sum():] == -1)


# ------------------------------------------------------ EP layout / regroup
@pytest.mark.parametrize("T,d,E,k,R", [(8192, 2880, 128, 4, 8), (203, 64, 16, 3, 4),
                                       (7, 32, 8, 2, 8), (1000, 64, 64, 8, 2)])
def test_ep_dispatch_then_regroup(M, T, d, E, k, R):
    L = W.make_logits(T, E, k, seed=R + T)
    idx, *_ = O.router_topk(k, True, logits=L)
    x = torch.randn(T, d, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    crm, src_rm, dst_rm = O.ep_dispatch_rank_major(idx, E, R)
    gcrm, goffrm, gsrc, gdst, gxrm, ws = M.ep_dispatch_rank_major(x.cuda(), i32(idx), E, R)
    assert np.array_equal(gcrm.cpu().numpy(), crm)
    assert np.array_equal(gsrc.cpu().numpy(), src_rm)
    assert np.array_equal(gdst.cpu().numpy(), dst_rm)
    assert torch.equal(gxrm.cpu(), x[torch.from_numpy(src_rm)])
    # regroup of the GPU's rank-major buffer
    perm, cem, oem = O.ep_local_regroup(crm)
    out, gcem, goem, gperm, ginv, ws2 = M.ep_local_regroup(gxrm, gcrm)
    assert np.array_equal(gperm.cpu().numpy(), perm)
    assert np.array_equal(gcem.cpu().numpy(), cem) and np.array_equal(goem.cpu().numpy(), oem)
    assert torch.equal(out.cpu(), gxrm.cpu()[torch.from_numpy(perm)])
    inv = np.empty_like(perm)
    inv[perm] = np.arange(len(perm))
    assert np.array_equal(ginv.cpu().numpy(), inv)
    # the EP identity: regrouped rank-major layout == single-device dispatch
    c, off, src, dst = O.dispatch(idx, E)
    assert np.array_equal(gsrc.cpu().numpy()[perm], src)
    assert np.array_equal(inv[gdst.cpu().numpy()], dst)
    assert M.device_status(ws2) == 0


@pytest.mark.parametrize("G,R,L,rows_mean", [(8, 8, 16, 32), (1, 2, 2, 3), (3, 5, 7, 1), (8, 16, 64, 1),
                                             (2, 4, 3, 0)])
def test_regroup_random_counts(M, G, R, L, rows_mean):
    crm = W.make_rank_counts(G, R, L, rows_mean * G * R * L, seed=G * R + L)
    rows = int(crm.sum())
    inp = torch.randn(max(rows, 1), 48).to(torch.bfloat16)[:rows].contiguous()
    perm, cem, oem = O.ep_local_regroup(crm)
    if rows == 0:
        inp = torch.empty(0, 48, dtype=torch.bfloat16)
    out, gcem, goem, gperm, ginv, ws = M.ep_local_regroup(inp.cuda(), i32(crm))
    assert np.array_equal(gcem.cpu().numpy(), cem) and np.array_equal(goem.cpu().numpy(), oem)
    if rows:
        assert np.array_equal(gperm.cpu().numpy(), perm)
        assert torch.equal(out.cpu(), inp[torch.from_numpy(perm)])


def test_regroup_bad_counts_sets_status(M):
    crm = np.array([[[1, 2], [2, 1]]], dtype=np.int32)
    inp = torch.randn(5, 16).to(torch.bfloat16).cuda()     # counts say 6 rows
    out = torch.full_like(inp, 7.0)
    G, R, L = crm.shape
    cem = torch.empty(G * L, dtype=torch.int32, device="cuda")
    oem = torch.empty(G * L + 1, dtype=torch.int32, device="cuda")
    perm = torch.full((5,), -5, dtype=torch.int32, device="cuda")
    ws = torch.empty(M.regroup_workspace_size(G, R, L), dtype=torch.uint8, device="cuda")
    M.moe_ep_local_regroup(inp, i32(crm), G, R, L, 5, 16, M.MOE_BF16, out, cem, oem, perm, None,
                           ws)
    assert M.device_status(ws) & M.MOE_DEV_BAD_COUNTS
    assert torch.all(out == 7.0) and torch.all(perm == -5)


# ----------------------------------------------------------- grouped SwiGLU
def swiglu_case(M, T, d, E, k, h, seed, dtype, row_scale=False, logits=None, sample=None,
                gather=False):
    x, wr, w1, w3, w2 = small_layer(T, d, E, k, h, seed, dtype, device="cpu")
    L = W.make_logits(T, E, k, seed=seed) if logits is None else logits
    idx, w, *_ = O.router_topk(k, True, logits=L)
    c, off, src, dst = O.dispatch(idx, E)
    xp = x[torch.from_numpy(src)].contiguous()
    rs = torch.rand(T * k, generator=torch.Generator().manual_seed(seed)) if row_scale else None
    if gather:
        gy, ws = M.grouped_swiglu_gather(x.cuda(), i32(src), i32(off), w1.cuda(), w3.cuda(),
                                         w2.cuda(), None if rs is None else rs.cuda())
    else:
        gy, ws = M.grouped_swiglu(xp.cuda(), i32(off), w1.cuda(), w3.cuda(), w2.cuda(),
                                  None if rs is None else rs.cuda())
    assert M.device_status(ws) == 0
    if sample is None:
        ref = O.grouped_swiglu(xp, off, w1, w3, w2, None if rs is None else rs.numpy())
        close(gy.cpu(), ref, dtype)
    else:
        rows = np.random.default_rng(seed).choice(T * k, size=sample, replace=False)
        seg = np.searchsorted(off, rows, side="right") - 1
        ref = np.zeros((sample, d))
        for e in np.unique(seg):
            q = seg == e
            ref[q] = O.swiglu_ffn(xp[torch.from_numpy(rows[q])], w1[e], w3[e], w2[e])
        if rs is not None:
            ref *= rs.numpy()[rows][:, None]
        close(gy.cpu()[torch.from_numpy(rows)], ref, dtype)


@pytest.mark.parametrize("T,d,E,k,h", [
    (300, 128, 4, 2, 192),      # ragged m-tiles, h not a multiple of 128
    (64, 64, 8, 2, 64),         # K = one block, tiny segments
    (1, 128, 16, 1, 128),       # a single row
    (700, 320, 6, 3, 256),      # several k-blocks, partial down n-tile (320 = 256 + 64)
    (2048, 256, 1, 1, 512),     # one expert, 16 m-tiles
    (517, 192, 130, 4, 128),    # many experts, empty experts
])
@pytest.mark.parametrize("row_scale", [False, True])
@pytest.mark.parametrize("gather", [False, True])
def test_grouped_swiglu_bf16_shapes(M, T, d, E, k, h, row_scale, gather):
    swiglu_case(M, T, d, E, k, h, seed=T + d, dtype=torch.bfloat16, row_scale=row_scale,
                gather=gather)


@pytest.mark.parametrize("row_scale", [False, True])
@pytest.mark.parametrize("gather", [False, True])
def test_grouped_swiglu_f32(M, row_scale, gather):
    swiglu_case(M, 256, 128, 8, 2, 256, seed=0, dtype=torch.float32, row_scale=row_scale,
                gather=gather)
    swiglu_case(M, 77, 36, 5, 3, 20, seed=1, dtype=torch.float32, row_scale=row_scale,
                gather=gather)


@pytest.mark.parametrize("cfg", [1, 3, 4])
def test_grouped_swiglu_gather_full_size_sampled(M, cfg):
    """Workload sizes, the launch the forward uses (rows gathered from x),
    checked on 256 sampled output rows."""
    c = W.config(cfg)
    swiglu_case(M, c.T, c.d, c.E, c.top_k, c.h, seed=c.seed, dtype=torch.bfloat16, sample=256,
                gather=True)


@pytest.mark.parametrize("counts,d,h", [
    # full 256-row pair tiles, short and long tails (pair tiles mostly or
    # half padding), empty experts, h and d that leave partial n-tiles
    ([256, 128, 129, 1, 0, 31, 32, 33, 384, 511], 192, 320),
    ([600, 200, 90], 320, 448),
    # last blocks of 1, 44 and 128 rows after full pair tiles (computed with
    # their pair tile), one of 129 rows (a pair tile of its own)
    ([257, 300, 640, 385, 130, 2], 128, 192),
])
@pytest.mark.parametrize("row_scale", [False, True])
def test_grouped_swiglu_pair_tile_mix(M, counts, d, h, row_scale):
    g = torch.Generator().manual_seed(sum(counts) + d)
    E, N = len(counts), int(sum(counts))
    bf = torch.bfloat16
    xp = torch.randn(N, d, generator=g).to(bf)
    w1 = (torch.randn(E, h, d, generator=g) / math.sqrt(d)).to(bf)
    w3 = (torch.randn(E, h, d, generator=g) / math.sqrt(d)).to(bf)
    w2 = (torch.randn(E, d, h, generator=g) / math.sqrt(h)).to(bf)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    rs = torch.rand(N, generator=g) if row_scale else None
    gy, ws = M.grouped_swiglu(xp.cuda(), i32(off), w1.cuda(), w3.cuda(), w2.cuda(),
                              None if rs is None else rs.cuda())
    assert M.device_status(ws) == 0
    ref = O.grouped_swiglu(xp, off, w1, w3, w2, None if rs is None else rs.numpy())
    close(gy.cpu(), ref, bf)


def test_grouped_swiglu_long_reduction_tails(M):
    """Reductions of 2624 in both GEMMs (the long-reduction path): a
    segment's short last block after its full 256-row pair tiles runs in the
    single-CTA launch (last blocks of 1, 44, 64, 65 and 128 rows), a
    129-row last block and segments of at most 128 rows are pair tiles of
    their own; 2624 hidden units and output columns leave partial n-tiles.
    Sampled rows (every segment's first and last rows, the rows around each
    256-row boundary, a random few) against the oracle's per-expert SwiGLU,
    with a row scale."""
    counts = [257, 300, 320, 321, 384, 385, 640, 130, 2, 0]
    d = h = 2624
    g = torch.Generator().manual_seed(11)
    E, N = len(counts), int(sum(counts))
    bf = torch.bfloat16
    xp = torch.randn(N, d, generator=g).to(bf)
    w1 = (torch.randn(E, h, d, generator=g) / math.sqrt(d)).to(bf)
    w3 = (torch.randn(E, h, d, generator=g) / math.sqrt(d)).to(bf)
    w2 = (torch.randn(E, d, h, generator=g) / math.sqrt(h)).to(bf)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    rs = torch.rand(N, generator=g)
    gy, ws = M.grouped_swiglu(xp.cuda(), i32(off), w1.cuda(), w3.cuda(), w2.cuda(), rs.cuda())
    assert M.device_status(ws) == 0
    gy = gy.cpu()
    assert torch.isfinite(gy.float()).all()
    rng = np.random.default_rng(3)
    for e in range(E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi == lo:
            continue
        rows = {lo, hi - 1, min(lo + 1, hi - 1), max(hi - 2, lo)}
        for b in range(256, hi - lo, 256):
            rows |= {lo + b - 1, lo + b, min(lo + b + 63, hi - 1), min(lo + b + 64, hi - 1)}
        rows |= set(rng.integers(lo, hi, size=4).tolist())
        r = torch.tensor(sorted(rows))
        ref = O.grouped_swiglu(xp[r], np.array([0, len(r)]), w1[e:e + 1], w3[e:e + 1],
                               w2[e:e + 1], rs[r].numpy())
        close(gy[r], ref, bf)


def test_grouped_swiglu_all_rows_one_expert(M):
    T, E, k = 1500, 8, 1
    L = W.make_logits(T, E, k, seed=3)
    L[:, 5] += 100.0
    swiglu_case(M, T, 128, E, k, 128, seed=3, dtype=torch.bfloat16, logits=L)


def test_grouped_swiglu_bad_offsets_sets_status(M):
    x, wr, w1, w3, w2 = small_layer(10, 64, 2, 1, 64, 0)
    y = torch.full((10, 64), 3.0, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(M.grouped_swiglu_workspace_size(10, 64, 64, 2, M.MOE_BF16), dtype=torch.uint8,
                     device="cuda")
    for off in ([0, 7, 5], [1, 5, 10], [0, 5, 9]):
        M.moe_grouped_swiglu(x, i32(off), w1, w3, w2, None, 10, 64, 64, 2, M.MOE_BF16, y, ws)
        assert M.device_status(ws) & M.MOE_DEV_BAD_OFFSETS
    assert torch.all(y == 3.0)


# ------------------------------------------------------------------ combine
@pytest.mark.parametrize("k", [1, 2, 4, 8, 16])
def test_combine_identity_exact(M, k):
    T, E, d = 333, 16, 256
    x = torch.randn(T, d).to(torch.bfloat16)
    L = W.make_logits(T, E, k, seed=k)
    idx, *_ = O.router_topk(k, True, logits=L)
    c, off, src, dst = O.dispatch(idx, E)
    xp = x[torch.from_numpy(src)].cuda()
    w = torch.full((T, k), 1.0 / k, device="cuda")
    out = M.combine(xp, i32(dst), w)
    assert torch.equal(out.cpu(), x)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_combine_weighted(M, dtype):
    T, E, k, d = 1000, 32, 6, 512
    L = W.make_logits(T, E, k, seed=2)
    idx, w, *_ = O.router_topk(k, True, logits=L)
    c, off, src, dst = O.dispatch(idx, E)
    y = torch.randn(T * k, d).to(dtype)
    out = M.combine(y.cuda(), i32(dst), torch.from_numpy(w).float().cuda())
    close(out.cpu(), O.combine(y, dst, w.astype(np.float32)), dtype)
    if dtype == torch.float32:
        assert torch.equal(M.combine(y.cuda(), i32(dst), None).cpu(),
                           M.combine(y.cuda(), i32(dst), torch.ones(T, k, device="cuda")).cpu())


# ------------------------------------------------------------------ forward
def forward_check(M, x, wr, w1, w3, w2, k, renorm=True, ep=1, logits_in=None, sample=256,
                  seed=0):
    """GPU forward vs the oracle's token-by-token definition on (a sample of)
    the tokens whose top-k set is unambiguous; all integer outputs checked."""
    T, d = x.shape
    E = w1.shape[0]
    dtype = x.dtype
    res = M.forward(x, wr, w1, w3, w2, k, renorm, ep_ranks=ep, want_router=True,
                    logits_in=None if logits_in is None else torch.from_numpy(logits_in).cuda())
    assert M.device_status(res["ws"]) == 0
    gi = res["topk_idx"].cpu().numpy()
    assert np.array_equal(res["counts"].cpu().numpy(), np.bincount(gi.ravel(), minlength=E))
    if T == 0:
        assert res["out"].shape == (0, d)
        return res
    xc, wrc = x.cpu(), wr.cpu()
    if logits_in is not None:
        idx, w, counts, _ = O.router_topk(k, renorm, logits=logits_in)
        assert np.array_equal(gi, idx)
        sure = np.ones(T, dtype=bool)
    else:
        idx, w, counts, L64 = O.router_topk(k, renorm, x=xc, w_router=wrc)
        absdot = np.abs(f64(xc)) @ np.abs(f64(wrc)).T
        margin = 2 * (d + 2) * 2.0 ** -23 * absdot.max(axis=1)
        sure = compare_topk(gi, idx, L64, margin)
    toks = np.nonzero(sure)[0]
    if sample is not None and len(toks) > sample:
        toks = np.sort(np.random.default_rng(seed).choice(toks, size=sample, replace=False))
    ref = O.moe_tokens(xc[torch.from_numpy(toks)], idx[toks], w[toks], w1.cpu(), w3.cpu(),
                       w2.cpu())
    close(res["out"].cpu()[torch.from_numpy(toks)], ref, dtype)
    return res


def test_forward_cfg0_full_oracle(M):
    c = W.config(0)
    lay = W.make_layer(c, "cpu")
    ref = O.moe_forward(lay["x"], lay["w_router"], lay["w1"], lay["w3"], lay["w2"], c.top_k,
                        c.renormalize)
    res = M.forward(*(lay[n].cuda() for n in ("x", "w_router", "w1", "w3", "w2")), c.top_k,
                    c.renormalize, want_router=True)
    assert np.array_equal(res["topk_idx"].cpu().numpy(), ref["topk_idx"])
    assert np.array_equal(res["counts"].cpu().numpy(), ref["counts"])
    close(res["topk_w"].cpu(), ref["topk_w"], torch.float32)
    close(res["out"].cpu(), ref["out"], torch.float32)


@pytest.mark.parametrize("cfg", [1, 2, 3, 4])
def test_forward_configs(M, cfg):
    c = W.config(cfg)
    lay = W.make_layer(c, "cuda")
    args = (lay["x"], lay["w_router"], lay["w1"], lay["w3"], lay["w2"], c.top_k, c.renormalize,
            c.ep_ranks)
    forward_check(M, *args, seed=c.seed)
    L = W.make_logits(c.T, c.E, c.top_k, seed=c.seed)
    forward_check(M, *args, logits_in=L, sample=128, seed=c.seed)


def test_forward_ep_equals_single_device_bitwise(M):
    c = W.config(4)
    lay = W.make_layer(c, "cuda")
    args = (lay["x"], lay["w_router"], lay["w1"], lay["w3"], lay["w2"], c.top_k)
    a = M.forward(*args, ep_ranks=8)
    b = M.forward(*args, ep_ranks=1)
    assert torch.equal(a, b)


def test_forward_is_deterministic(M):
    c = W.config(1)
    lay = W.make_layer(c, "cuda")
    args = (lay["x"], lay["w_router"], lay["w1"], lay["w3"], lay["w2"], c.top_k)
    assert torch.equal(M.forward(*args), M.forward(*args))


@pytest.mark.parametrize("T,d,E,k,h,ep", [(0, 128, 8, 2, 128, 1), (1, 128, 8, 2, 128, 1),
                                          (5, 64, 4, 4, 64, 2), (257, 192, 8, 8, 192, 4),
                                          (130, 128, 1, 1, 64, 1), (999, 64, 16, 3, 128, 8)])
def test_forward_edge_shapes(M, T, d, E, k, h, ep):
    x, wr, w1, w3, w2 = small_layer(T, d, E, k, h, seed=T + 1)
    wr = (wr.float() * 50).to(torch.bfloat16)
    forward_check(M, x, wr, w1, w3, w2, k, True, ep, sample=None)


# ---------------------------------------------------------- NaN scores
def test_router_nan_logits_from_logits(M):
    """Logits with NaN entries: a NaN score never wins over a number (it is
    taken as -inf for the selection), so the routing equals the oracle's on
    the same logits with NaN set to -inf; weights of rows with a finite
    winner stay finite."""
    T, E, k = 300, 64, 6
    L = W.make_logits(T, E, k, seed=21)
    rng = np.random.default_rng(21)
    mask = rng.random((T, E)) < 0.1
    L[mask] = np.nan
    gi, gw, gc, _, ws = M.router_topk(logits_in=torch.from_numpy(L).cuda(), top_k=k,
                                      renormalize=True)
    torch.cuda.synchronize()
    assert M.device_status(ws) == 0
    Lr = np.where(np.isnan(L), -np.inf, L)
    idx, w, counts, _ = O.router_topk(k, True, logits=Lr)
    assert np.array_equal(gi.cpu().numpy(), idx)
    assert np.array_equal(gc.cpu().numpy(), counts)
    close(gw, w, torch.float32)


def test_router_nan_tokens_fused_gate(M):
    """The fused router on tokens whose x holds a NaN (all their logits
    NaN): every key ties at -inf, so the k lowest expert ids are selected;
    the other tokens route as without them."""
    T, d, E, k = 512, 256, 32, 4
    g = torch.Generator().manual_seed(5)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16)
    wr = (torch.randn(E, d, generator=g) * 0.1).to(torch.bfloat16)
    bad = torch.tensor([0, 17, 255, 511])
    xn = x.clone()
    xn[bad, 3] = float("nan")
    gi, gw, gc, _, ws = M.router_topk(xn.cuda(), wr.cuda(), top_k=k, renormalize=True)
    gi0, gw0, _, _, _ = M.router_topk(x.cuda(), wr.cuda(), top_k=k, renormalize=True)
    torch.cuda.synchronize()
    assert M.device_status(ws) == 0
    gi, gi0 = gi.cpu().numpy(), gi0.cpu().numpy()
    assert (gi[bad.numpy()] == np.arange(k)[None, :]).all()
    good = np.setdiff1d(np.arange(T), bad.numpy())
    assert np.array_equal(gi[good], gi0[good])
    assert torch.equal(gw.cpu()[good], gw0.cpu()[good])
    assert np.array_equal(gc.cpu().numpy(), np.bincount(gi.ravel(), minlength=E))


def test_router_nan_expert_fused_gate(M):
    """A NaN in one row of w_router: that expert's logit is NaN for every
    token and is never selected; the routing equals the oracle's on the
    GPU's own logits with NaN set to -inf."""
    T, d, E, k = 700, 512, 48, 5
    g = torch.Generator().manual_seed(6)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16)
    wr = (torch.randn(E, d, generator=g) * 0.1).to(torch.bfloat16)
    wr[7, 11] = float("nan")
    gi, gw, gc, gl, ws = M.router_topk(x.cuda(), wr.cuda(), top_k=k, renormalize=True,
                                       want_logits=True)
    torch.cuda.synchronize()
    assert M.device_status(ws) == 0
    L = gl.cpu().numpy()
    assert np.isnan(L[:, 7]).all() and np.isfinite(np.delete(L, 7, axis=1)).all()
    idx, w, counts, _ = O.router_topk(k, True, logits=np.where(np.isnan(L), -np.inf, L))
    gi = gi.cpu().numpy()
    assert not (gi == 7).any()
    assert np.array_equal(gi, idx)
    assert np.array_equal(gc.cpu().numpy(), counts)
    close(gw, w, torch.float32)
