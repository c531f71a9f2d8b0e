"""Failure detection without a GPU fault: every pipeline wait of libmoe is
bounded.  moe_selftest_timeout waits, through the same bounded wait, on a
barrier that nothing arrives at; the test checks that the wait gives up
after its limit (about 2 s), that MOE_DEV_TIMEOUT reaches the host through
the status word, and that the context is still usable afterwards."""
import time

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


def test_bounded_wait_gives_up_and_reports(M):
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    M.moe_selftest_timeout(ws)
    code = M.device_status(ws)        # synchronises the stream
    elapsed = time.perf_counter() - t0
    assert code == M.MOE_DEV_TIMEOUT
    assert 1.5 < elapsed < 60, elapsed
    # the context is usable: a small layer still matches the oracle
    c = W.config(0)
    lay = W.make_layer(c, "cpu")
    ref = O.moe_forward(lay["x"], lay["w_router"], lay["w1"], lay["w3"], lay["w2"], c.top_k,
                        c.renormalize)
    res = M.forward(*(lay[n].cuda() for n in ("x", "w_router", "w1", "w3", "w2")), c.top_k,
                    c.renormalize, want_router=True)
    assert M.device_status(res["ws"]) == 0
    assert np.array_equal(res["topk_idx"].cpu().numpy(), ref["topk_idx"])
    np.testing.assert_allclose(res["out"].cpu().numpy(), ref["out"], rtol=1e-5, atol=1e-5)
