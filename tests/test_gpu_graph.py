"""moe_forward inside a CUDA graph: every step of the layer is a kernel (or
the status memset) on the caller's stream with no host synchronisation, so
one captured call replays the whole layer.  Checked: the replay's output is
bit-identical to a direct call, and a replay after new tokens are copied
into the captured input buffer computes the layer on the new tokens.
"""
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M(cuda_ok):
    from routing_dispatch_grouped_topk_b200 import build
    build.build()
    import routing_dispatch_grouped_topk_b200 as m
    m.lib()
    return m


@pytest.mark.parametrize("cfg", [1, 4])
def test_forward_replays_from_a_cuda_graph(M, cfg):
    c = W.config(cfg)
    lay = W.make_layer(c, "cuda")
    x, wr, w1, w3, w2 = (lay[n] for n in ("x", "w_router", "w1", "w3", "w2"))
    dt = M.MOE_BF16
    ws = torch.empty(M.forward_workspace_size(c.T, c.d, c.E, c.top_k, c.h, c.ep_ranks, dt),
                     dtype=torch.uint8, device="cuda")
    out = torch.empty(c.T, c.d, dtype=x.dtype, device="cuda")
    xin = x.clone()

    def call():
        M.moe_forward(xin, wr, None, w1, w3, w2, c.T, c.d, c.E, c.top_k, c.h,
                      M.MOE_SCORE_SOFTMAX, c.renormalize, c.ep_ranks, dt, out, None, None, None,
                      None, ws)

    call()                      # first call outside the capture (one-time setup)
    torch.cuda.synchronize()
    direct = out.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert M.device_status(ws) == 0
    assert torch.equal(out, direct)
    # new tokens in the captured buffer: the replay routes and computes them
    x2 = W.make_layer(W.config(cfg), "cuda", experts=False)["x"].flip(0).contiguous()
    xin.copy_(x2)
    g.replay()
    torch.cuda.synchronize()
    ref = M.forward(x2, wr, w1, w3, w2, c.top_k, c.renormalize, ep_ranks=c.ep_ranks)
    assert torch.equal(out, ref)
    del g
