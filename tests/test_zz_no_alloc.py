"""moe_dispatch_noalloc: the dispatch entry point for callers that cannot
allocate device memory (an engine or plugin whose enqueue path must not
allocate, a server whose memory is all held by another framework's pool).
Its scratch lives in a fixed array inside libmoe.so instead of a caller
workspace.  These tests call it through the C ABI and compare it, bit for
bit, with moe_dispatch on the same inputs, for two calls in a row (the
second call must not see anything the first left in the shared array).

The file is named to be collected last; it works alone in a fresh process
as well as after the other tests.
"""
import ctypes

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


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _noalloc(M, x, idx, E):
    T, k = idx.shape
    d = x.shape[1]
    N = T * k
    dev = x.device
    counts = torch.full((E,), -7, dtype=torch.int32, device=dev)
    offsets = torch.full((E + 1,), -7, dtype=torch.int32, device=dev)
    src_row = torch.full((N,), -7, dtype=torch.int32, device=dev)
    dst_pos = torch.full((T, k), -7, dtype=torch.int32, device=dev)
    x_perm = torch.zeros(N, d, dtype=x.dtype, device=dev)
    stream = torch.cuda.current_stream().cuda_stream
    rc = M.lib().moe_dispatch_noalloc(
        _p(x), _p(idx), T, d, E, k, M.MOE_BF16 if x.dtype == torch.bfloat16 else M.MOE_F32,
        _p(counts), _p(offsets), _p(src_row), _p(dst_pos), _p(x_perm),
        ctypes.c_void_p(stream) if stream else None)
    assert rc == 0, M.lib().moe_last_error()
    torch.cuda.synchronize()
    return counts, offsets, src_row, dst_pos, x_perm


def _case(T, d, E, k, seed, dtype=torch.bfloat16):
    L = W.make_logits(T, E, k, seed=seed)
    idx, *_ = O.router_topk(k, True, logits=L)
    x = torch.randn(T, d, generator=torch.Generator().manual_seed(seed)).to(dtype)
    return x.cuda(), torch.as_tensor(idx, dtype=torch.int32).cuda()


def test_noalloc_matches_workspace_dispatch_twice(M):
    # two calls in a row with different sizes; each compared with moe_dispatch
    for (T, d, E, k, seed) in [(4096, 2048, 128, 8, 1), (777, 256, 64, 4, 2)]:
        x, idx = _case(T, d, E, k, seed)
        ref = M.dispatch(x, idx, E)[:5]
        got = _noalloc(M, x, idx, E)
        for a, b in zip(got, ref):
            assert torch.equal(a, b)


def test_noalloc_second_call_sees_no_stale_state(M):
    # the first call routes to every expert, the second leaves most experts
    # empty: a stale histogram in the shared array would corrupt the second
    x1, idx1 = _case(2000, 128, 32, 4, 5)
    _noalloc(M, x1, idx1, 32)
    L = W.make_logits(300, 32, 2, seed=6)
    L[:, 3] += 50.0
    idx2 = torch.as_tensor(O.router_topk(2, True, logits=L)[0], dtype=torch.int32).cuda()
    x2 = torch.randn(300, 128).to(torch.bfloat16).cuda()
    got = _noalloc(M, x2, idx2, 32)
    ref = M.dispatch(x2, idx2, 32)[:5]
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
