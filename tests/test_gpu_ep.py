"""The expert-parallel forward (routing_dispatch_grouped_topk_b200.ep) on one
GPU: a one-rank NCCL group, so both all-to-alls are local copies and every
step of the path runs -- router, dispatch, counts exchange, row exchange,
regroup to expert-major and back, grouped SwiGLU, combine.  Every expert
sees its rows in the single-device order, so the result equals moe_forward
bit for bit (the multi-rank exchange logic is checked on CPU over gloo in
test_ep_exchange.py)."""
import math
import os
import socket

import pytest
import torch

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.fixture(scope="module")
def M(cuda_ok):
    from routing_dispatch_grouped_topk_b200 import build
    build.build()
    import routing_dispatch_grouped_topk_b200 as m
    m.lib()
    return m


@pytest.mark.parametrize("T,d,E,k,h", [(300, 256, 16, 4, 192), (1000, 512, 32, 8, 256)])
def test_ep_forward_one_rank_equals_forward(M, T, d, E, k, h):
    import datetime

    import torch.distributed as dist
    from routing_dispatch_grouped_topk_b200 import ep
    torch.cuda.set_device(0)
    store = dist.TCPStore("127.0.0.1", _free_port(), 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        g = torch.Generator().manual_seed(T + E)
        bf = torch.bfloat16
        x = torch.randn(T, d, generator=g).to(bf).cuda()
        wr = (torch.randn(E, d, generator=g) * 0.02).to(bf).cuda()
        w1 = (torch.randn(E, h, d, generator=g) / math.sqrt(d)).to(bf).cuda()
        w3 = (torch.randn(E, h, d, generator=g) / math.sqrt(d)).to(bf).cuda()
        w2 = (torch.randn(E, d, h, generator=g) / math.sqrt(h)).to(bf).cuda()
        out = ep.ep_forward(x, wr, w1, w3, w2, k, True)
        ref = M.forward(x, wr, w1, w3, w2, k, True)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    finally:
        dist.destroy_process_group()
