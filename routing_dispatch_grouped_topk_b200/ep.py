"""Expert parallelism across GPUs: the MoE layer forward with the experts
split over the ranks of a process group, one process per GPU.

This follows the exchange of [EP] (huggingface/transformers PR #41053
"Qwen3 moe", ``Ep2DpParallel._token_dispatch`` / ``_token_combine``): rank
g holds the L = E / R experts ``[g L, (g + 1) L)`` and its own tokens.  On
rank r:

1. the router top-k of its tokens (``moe_router_topk``);
2. the dispatch (``moe_dispatch``): expert-major order is destination-rank
   major, because the experts of a rank are contiguous, so the routed rows
   are already the send buffer of the all-to-all;
3. the counts exchange: an all-to-all of the per-expert counts ``[R, L]``
   gives ``counts_recv[r', l]``, the rows source rank r' sends for local
   expert l;
4. the split sizes of both all-to-alls, from one device-to-host copy of the
   two count arrays (the pages' ``.tolist()`` of the split sizes);
5. the all-to-all of the rows (NCCL over NVLink): the received buffer is
   source-rank major, (r' outer, l inner);
6. ``moe_ep_local_regroup`` (G = 1, R, L) reorders it expert-major, the
   reshuffle [EP] says the received buffer needs;
7. ``moe_grouped_swiglu`` over the L local experts;
8. the same regroup with the roles of R and L exchanged (counts transposed)
   puts the outputs back source-rank major;
9. the reverse all-to-all returns every row to the rank that routed it, in
   that rank's expert-major order;
10. ``moe_combine`` with the dispatch's ``dst_pos`` and the routing weights.

Every step on the data runs in libmoe's kernels or in the collective; the
host only turns counts into split sizes.  The exchanges are plain
``torch.distributed.all_to_all_single`` calls (NCCL on GPUs); no TMA
multicast is involved anywhere.

The host-side pieces (:func:`exchange_counts`, :func:`split_sizes`,
:func:`reverse_counts`, :func:`exchange_rows`) take and return torch
tensors on any device, so they run on CPU tensors over a ``gloo`` group as
well.
"""
from __future__ import annotations

from typing import List, Tuple

import torch
import torch.distributed as dist

__all__ = ["exchange_counts", "split_sizes", "reverse_counts", "exchange_rows", "ep_forward"]


def exchange_counts(counts: torch.Tensor, R: int, group=None) -> torch.Tensor:
    """All-to-all of per-expert counts.  ``counts`` [E] int32 of this rank's
    routed copies per global expert (E = R L); returns ``counts_recv`` [R, L]:
    row r' holds the counts rank r' routed to this rank's L experts."""
    E = counts.numel()
    assert E % R == 0, "the experts must split evenly over the ranks"
    L = E // R
    recv = torch.empty(R * L, dtype=counts.dtype, device=counts.device)
    dist.all_to_all_single(recv, counts.contiguous(), [L] * R, [L] * R, group=group)
    return recv.view(R, L)


def split_sizes(counts: torch.Tensor, counts_recv: torch.Tensor) -> Tuple[List[int], List[int]]:
    """Row split sizes of the dispatch all-to-all: ``send[g]`` = rows this
    rank sends to rank g (its copies for experts ``[g L, (g + 1) L)``),
    ``recv[r']`` = rows it receives from rank r'.  One host copy of both."""
    R, L = counts_recv.shape
    both = torch.cat([counts.view(R, L).sum(1), counts_recv.sum(1)]).to("cpu")
    return both[:R].tolist(), both[R:].tolist()


def reverse_counts(counts_recv: torch.Tensor) -> torch.Tensor:
    """Counts of the reverse regroup: the expert outputs sit local-expert
    major (l outer, r' inner); regrouping with R and L exchanged, i.e. with
    counts ``[1, L, R]`` = the transpose, restores source-rank-major order."""
    R, L = counts_recv.shape
    return counts_recv.t().contiguous().view(1, L, R)


def exchange_rows(send: torch.Tensor, send_splits: List[int], recv_splits: List[int],
                  group=None) -> torch.Tensor:
    """All-to-all of variable-size row blocks: rows ``[sum(send_splits[:g]),
    +send_splits[g])`` go to rank g; the result stacks what every rank sent
    here, in rank order."""
    recv = torch.empty((sum(recv_splits),) + tuple(send.shape[1:]), dtype=send.dtype,
                       device=send.device)
    dist.all_to_all_single(recv, send.contiguous(), recv_splits, send_splits, group=group)
    return recv


def ep_forward(x, w_router, w1_local, w3_local, w2_local, top_k, renormalize=True, group=None):
    """The layer forward on this rank's tokens with expert parallelism.

    ``x`` [T, d]: this rank's tokens; ``w_router`` [E, d] (the same on every
    rank); ``w1_local``, ``w3_local`` [L, h, d] and ``w2_local`` [L, d, h]:
    this rank's experts, global experts ``[rank L, (rank + 1) L)``.  Returns
    ``out`` [T, d].  Uses the process group's device (NCCL: one GPU per
    rank).  The result equals the single-device layer's on the same tokens:
    every expert sees its rows in the same order (source rank, then flat
    index), so each expert's segment is the one the single device forms.
    """
    import routing_dispatch_grouped_topk_b200 as M

    R = dist.get_world_size(group)
    L = w1_local.shape[0]
    E = w_router.shape[0]
    assert E == R * L, "w_router has E = R L rows"
    idx, w, counts, _, _ = M.router_topk(x, w_router, top_k, renormalize)
    _, _, _, dst_pos, x_perm, _ = M.dispatch(x, idx, E)
    counts_recv = exchange_counts(counts, R, group)
    send_splits, recv_splits = split_sizes(counts, counts_recv)
    x_recv = exchange_rows(x_perm, send_splits, recv_splits, group)
    if x_recv.shape[0] > 0:
        x_em, _, off_em, _, _, _ = M.ep_local_regroup(x_recv, counts_recv.view(1, R, L))
        y_em, _ = M.grouped_swiglu(x_em, off_em, w1_local, w3_local, w2_local)
        y_rm, _, _, _, _, _ = M.ep_local_regroup(y_em, reverse_counts(counts_recv))
    else:
        y_rm = x_recv
    y = exchange_rows(y_rm, recv_splits, send_splits, group)
    return M.combine(y, dst_pos, w)
