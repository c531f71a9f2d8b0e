"""World-size-2 check, on CPU over gloo, of the host side of the expert-
parallel forward (routing_dispatch_grouped_topk_b200.ep): the counts
all-to-all, the split sizes, the row all-to-all both ways and the transposed
counts of the reverse regroup.

The GPU kernels of the path (dispatch, regroup, grouped SwiGLU, combine) are
replaced here by the oracle's definitions of the same steps, and the experts
by a map that tags each row with its global expert (y = (e + 1) x), so the
test pins where every row travels: rank g must receive, from every source
rank in rank order, that rank's copies for g's experts in flat order; after
the local regroup every local expert's segment must be that expert's rows;
the reverse regroup and exchange must bring each output back to the slot it
was dispatched from, and the combine must then equal the per-token
definition.  The multi-GPU path itself is unmeasured on hardware (one GPU
per run here)."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

R, L, K, D, T = 2, 4, 2, 8, 37
E = R * L


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_inputs(rank):
    import oracle as O
    import workloads as W
    L_ = W.make_logits(T + 5 * rank, E, K, seed=40 + rank)
    idx, w, _, _ = O.router_topk(K, True, logits=L_)
    x = torch.randn(T + 5 * rank, D, generator=torch.Generator().manual_seed(rank)).double()
    return x, idx, w


def _worker(rank, port, q):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=R,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle as O
        from routing_dispatch_grouped_topk_b200 import ep
        x, idx, w = _rank_inputs(rank)
        # dispatch (oracle): expert-major rows = destination-rank-major
        counts, off, src_row, dst_pos = O.dispatch(idx, E)
        x_perm = x[torch.from_numpy(src_row)]
        counts_t = torch.from_numpy(counts.astype(np.int32))
        counts_recv = ep.exchange_counts(counts_t, R)
        send, recv = ep.split_sizes(counts_t, counts_recv)
        x_recv = ep.exchange_rows(x_perm, send, recv)
        # expected: every source rank's copies for this rank's experts
        want_c, want_rows = [], []
        for r in range(R):
            xr, ir, _ = _rank_inputs(r)
            c_r, off_r, src_r, _ = O.dispatch(ir, E)
            want_c.append(c_r[rank * L:(rank + 1) * L])
            want_rows.append(xr[torch.from_numpy(src_r[off_r[rank * L]:off_r[(rank + 1) * L]])])
        assert np.array_equal(counts_recv.numpy(), np.stack(want_c))
        assert send == [int(counts[g * L:(g + 1) * L].sum()) for g in range(R)]
        assert recv == [int(c.sum()) for c in want_c]
        assert torch.equal(x_recv, torch.cat(want_rows))
        # local regroup (oracle) to expert-major, experts tag rows with e + 1
        perm, cem, oem = O.ep_local_regroup(counts_recv.numpy()[None])
        x_em = x_recv[torch.from_numpy(perm)]
        y_em = torch.empty_like(x_em)
        for l in range(L):
            seg = slice(int(oem[l]), int(oem[l + 1]))
            y_em[seg] = (rank * L + l + 1) * x_em[seg]
        # the reverse regroup with transposed counts undoes the regroup
        perm2, _, _ = O.ep_local_regroup(ep.reverse_counts(counts_recv).numpy())
        y_rm = y_em[torch.from_numpy(perm2)]
        inv = np.empty_like(perm)
        inv[perm] = np.arange(len(perm))
        assert np.array_equal(perm2, inv)
        y = ep.exchange_rows(y_rm, recv, send)
        out = O.combine(y.numpy(), dst_pos, w)
        ref = np.stack([sum(w[t, j] * (idx[t, j] + 1) * x[t].numpy() for j in range(K))
                        for t in range(x.shape[0])])
        q.put((rank, float(np.abs(out - ref).max())))
    finally:
        dist.destroy_process_group()


def test_ep_exchange_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(R)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    errs = dict(q.get(timeout=10) for _ in range(R))
    assert set(errs) == {0, 1}
    assert max(errs.values()) < 1e-12


def test_reverse_counts_is_the_transpose():
    from routing_dispatch_grouped_topk_b200 import ep
    c = torch.arange(6, dtype=torch.int32).view(2, 3)
    rc = ep.reverse_counts(c)
    assert rc.shape == (1, 3, 2)
    assert torch.equal(rc[0], c.t())
