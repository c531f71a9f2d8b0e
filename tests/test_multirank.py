"""World-size-2 checks of the multi-rank bench logic on CPU (gloo): ranks get
independent token batches, the job time is the max over ranks, and the
whole-job throughput counts every rank's tokens.  No GPU is used."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, ws, port, q):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import workloads as W
        cfg = W.config(1)
        mine = bench.rank_workload(cfg, rank)
        x = W.make_layer(mine, "cpu", T=8, experts=False)["x"]
        xs = [torch.empty_like(x) for _ in range(ws)]
        dist.all_gather(xs, x)
        per_rank_ms = 100.0 + 50.0 * rank
        mx = bench.max_over_ranks(per_rank_ms, ws, device="cpu")
        val = bench.job_tokens_per_s(cfg.T, ws, 10, mx)
        if rank == 0:
            q.put((not torch.equal(xs[0], xs[1]), mx, val))
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    differ, mx, val = q.get(timeout=10)
    assert differ                       # independent token batches
    assert mx == 150.0                  # slowest rank sets the job time
    assert abs(val - 4096 * 2 * 10 / 0.150) < 1e-6


def _failing_worker(rank, ws, port, q):
    import datetime
    import time
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=10))
    import bench
    dist.barrier()
    if rank == 1:
        raise SystemExit(3)             # a rank that leaves between steps
    t0 = time.time()
    try:
        bench.max_over_ranks(1.0, ws, device="cpu")
        q.put(("no error", time.time() - t0))
    except Exception as e:              # the survivor's next collective fails
        q.put((type(e).__name__, time.time() - t0))


def test_a_rank_that_leaves_ends_the_others_collective():
    """A rank that exits between steps: the surviving rank's next collective
    (the max-over-ranks timing reduction) ends with an error within the
    process group's timeout instead of waiting for ever."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_failing_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert procs[1].exitcode == 3
    assert procs[0].exitcode == 0
    what, secs = q.get(timeout=10)
    assert what != "no error"
    assert secs < 60
