"""Plain fp64 CPU oracle of the single-device MoE layer forward.

TEST INFRASTRUCTURE.  Nothing on the product path may import, call or run
this module: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it.  It is written for a reader who wants to check it
against the pages by eye: every step is the textbook definition, one expert
or one token at a time, with NumPy float64 matmuls and sorts as the only
library primitives.  No blocking, fusion or reordering beyond that.

Sources (page title, then the function or section on it):

* [HP]  hyper_parallel ``platform/torch/common/moe.py`` coverage page --
  ``TokenChoiceTopKRouter.forward``, ``MoE.permutation``,
  ``MoE.unpermutation``, ``_run_experts_for_loop``, ``MoE.forward``.
* [QO]  QwenLM/Qwen3-Omni issue #115 "Training: Extremely Slow Deepspeed
  Engine initialization ..." -- ``SpeedupMoeExperts.forward`` (training
  branch: per-expert ``index_add_``; eval branch: dense ``bmm`` over all
  experts) and ``SpeedupMoeSparseMoeBlock.forward`` (``norm_topk_prob``).
* [EP]  huggingface/transformers PR #41053 "Qwen3 moe" --
  ``Ep2DpParallel._token_dispatch`` (per-rank counts, all-to-all, the
  received buffer that "needs to be reshuffled back").

Readings taken where the pages are silent or disagree (each is repeated in
the design notes):

* top-k order: descending score, ties to the lower expert index; selection is
  on the router logits (softmax is strictly increasing, so the selected set
  and its order are the same as on the probabilities).
* the order of copies inside one expert's segment is the order of the flat
  index ``t*k + j`` ([HP] ``MoE.permutation`` uses a stable argsort).
* the routing weight multiplies the expert output (after ``w2``), as in [QO]
  ``weighted_output``; [HP] applies it to the hidden activation before ``w2``,
  which is the same number by linearity of ``w2``.
* ``offsets`` has ``E + 1`` entries (exclusive scan including the total).
* the received EP buffer is source-rank-major: for each destination block,
  source rank outer and local expert inner; the regroup output is local
  expert outer and source rank inner.

Parity pins: every function here is pinned by a ``-m "not gpu"`` test that
does not re-derive it (hand cases, closed forms, brute force, invariants, a
second formulation).  No function is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "as_f64", "router_logits", "topk_select", "softmax", "router_topk", "sigmoid",
    "node_limited_mask", "router_topk_general", "load_balance_loss",
    "expert_counts", "dispatch", "permute_rows", "ep_dispatch_rank_major",
    "ep_local_regroup", "apply_row_perm", "silu", "swiglu_ffn",
    "grouped_swiglu", "combine", "moe_forward", "dense_moe", "moe_tokens",
    "silu_grad", "grouped_preactivations", "combine_backward", "grouped_swiglu_backward",
    "dispatch_backward", "router_backward", "load_balance_loss_grad",
    "scaled_dispatch_backward", "capacity_drop",
]


def as_f64(a) -> np.ndarray:
    """Exact conversion of a torch tensor (fp32/bf16) or array to float64."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().to("cpu")
            if a.dtype in (torch.bfloat16, torch.float16):
                a = a.to(torch.float32)          # exact widening
            return a.numpy().astype(np.float64)
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(a, dtype=np.float64)


def _i64(a) -> np.ndarray:
    try:
        import torch
        if isinstance(a, torch.Tensor):
            return a.detach().to("cpu").numpy().astype(np.int64)
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(a, dtype=np.int64)


# --------------------------------------------------------------------------
# Router  ([HP] TokenChoiceTopKRouter.forward; [QO] SpeedupMoeSparseMoeBlock)
# --------------------------------------------------------------------------

def router_logits(x, w_router) -> np.ndarray:
    """Gate logits ``x @ w_router^T`` in fp64 (the gate is a bias-free
    ``nn.Linear(d, E)`` whose weight is ``w_router[E, d]``)."""
    return as_f64(x) @ as_f64(w_router).T


def topk_select(scores, top_k: int) -> np.ndarray:
    """Indices of the ``top_k`` largest scores per row, largest first, ties
    broken towards the lower expert index.  ``int64 [T, k]``.

    A stable sort of the negated scores keeps equal scores in index order.
    """
    s = as_f64(scores)
    order = np.argsort(-s, axis=1, kind="stable")
    return order[:, :top_k]


def softmax(L) -> np.ndarray:
    """Row softmax ``exp(L - max) / sum`` in fp64."""
    L = as_f64(L)
    z = np.exp(L - L.max(axis=1, keepdims=True))
    return z / z.sum(axis=1, keepdims=True)


def router_topk(top_k: int, renormalize: bool, x=None, w_router=None, logits=None):
    """Token-choice top-k router.

    Scores are the fp32 gate logits if ``logits`` is given (consumed exactly),
    else the fp64 ``x @ w_router^T``.  Returns ``(idx[T,k] int64,
    w[T,k] fp64, counts[E] int64, logits[T,E] fp64)``.

    [HP] ``TokenChoiceTopKRouter.forward``: softmax over all experts, top-k,
    gather of the (unbiased) probabilities, bincount.  [QO]
    ``SpeedupMoeSparseMoeBlock.forward``: with ``norm_topk_prob`` the k
    weights are divided by their sum.
    """
    L = as_f64(logits) if logits is not None else router_logits(x, w_router)
    idx = topk_select(L, top_k)
    p = softmax(L)
    w = np.take_along_axis(p, idx, axis=1)
    if renormalize:
        w = w / w.sum(axis=1, keepdims=True)
    counts = expert_counts(idx, L.shape[1])
    return idx, w, counts, L


def sigmoid(L) -> np.ndarray:
    """``1 / (1 + exp(-L))`` in fp64."""
    L = as_f64(L)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-L))


def node_limited_mask(scores, num_groups: int, topk_groups: int) -> np.ndarray:
    """Node-limited routing ([HP] ``_get_node_limited_routing_scores``): the
    experts form ``num_groups`` equal consecutive groups; per token, the
    ``topk_groups`` groups with the largest maximum score are kept (ties to
    the lower group) and every expert of the other groups gets -inf."""
    s = as_f64(scores)
    T, E = s.shape
    gs = E // num_groups
    gmax = s.reshape(T, num_groups, gs).max(axis=2)
    keep = topk_select(gmax, topk_groups)
    mask = np.zeros((T, num_groups), dtype=bool)
    mask[np.arange(T)[:, None], keep] = True
    return np.where(np.repeat(mask, gs, axis=1), s, -np.inf)


def router_topk_general(top_k: int, x=None, w_router=None, logits=None, score: str = "softmax",
                        renormalize: bool = False, route_scale: float = 1.0, expert_bias=None,
                        num_groups: int = 0, topk_groups: int = 0, capacity: int = 0,
                        sel_scores=None):
    """Token-choice router with every option of [HP] ``TokenChoiceTopKRouter``,
    in its order: gate logits -> ``score_func`` (softmax over the experts or
    sigmoid) -> times ``route_scale`` -> node-limited group masking ->
    plus ``expert_bias`` (selection only) -> top-k -> gather of the unbiased
    scores as weights -> bincount.  With ``renormalize`` ([QO]
    ``norm_topk_prob``) the gathered weights are divided by their sum; the
    scale is applied after that division (so that it survives it; without
    renormalisation this equals gathering the scaled scores).  With
    ``capacity`` > 0 the capacity drop policy (:func:`capacity_drop`) then
    marks the dropped copies ``idx = -1`` with weight 0; it ranks by
    ``sel_scores`` [T, k] when given (a caller's copy of the selected scores
    in its own precision), else by this function's.  Returns ``(idx, w,
    counts, logits)`` like :func:`router_topk`."""
    L = as_f64(logits) if logits is not None else router_logits(x, w_router)
    E = L.shape[1]
    s = softmax(L) if score == "softmax" else sigmoid(L)
    scaled = s * route_scale
    for_topk = node_limited_mask(scaled, num_groups, topk_groups) if num_groups else scaled
    keys = for_topk + as_f64(expert_bias)[None, :] if expert_bias is not None else for_topk
    idx = topk_select(keys, top_k)
    w = np.take_along_axis(s, idx, axis=1)
    sel = w.copy()
    if renormalize:
        w = w / w.sum(axis=1, keepdims=True)
    w = w * route_scale
    if capacity > 0:
        keep = capacity_drop(idx, sel if sel_scores is None else sel_scores, capacity)
        idx = np.where(keep, idx, -1)
        w = np.where(keep, w, 0.0)
    return idx, w, expert_counts(idx, E), L


def load_balance_loss(top_scores, selected_experts, E: int) -> float:
    """Auxiliary load-balance loss of one router call ([HP]
    ``_compute_load_balance_loss``, without the sequence-partition
    all-reduce): with ``f_e`` the fraction of the ``T*k`` routed copies that
    go to expert e and ``P_e`` the sum of those copies' routing weights
    divided by T, the loss is ``E * sum_e f_e * P_e``; 0 for no tokens.
    The caller multiplies it by its coefficient."""
    w = as_f64(top_scores)
    idx = _i64(selected_experts)
    T, k = idx.shape
    if T == 0:
        return 0.0
    frac = np.zeros(E)
    prob = np.zeros(E)
    for t in range(T):
        for j in range(k):
            frac[idx[t, j]] += 1.0
            prob[idx[t, j]] += w[t, j]
    frac /= T * k
    prob /= T
    return float(E * np.sum(frac * prob))


def load_balance_loss_grad(selected_experts, E: int) -> np.ndarray:
    """Gradient of :func:`load_balance_loss` with respect to the routing
    weights ``top_scores`` [T, k]: the loss is linear in them through
    ``P_e`` and the fractions ``f_e`` are counts (no gradient), so the entry
    for a copy routed to expert e is ``E * f_e / T``.  A trainer that adds
    ``coef * loss`` to its objective ([HP] adds the auxiliary loss to the
    training loss) adds ``coef`` times this to the upstream gradient of the
    routing weights."""
    idx = _i64(selected_experts)
    T, k = idx.shape
    g = np.zeros((T, k))
    if T == 0:
        return g
    frac = np.zeros(E)
    for t in range(T):
        for j in range(k):
            frac[idx[t, j]] += 1.0
    frac /= T * k
    for t in range(T):
        for j in range(k):
            g[t, j] = E * frac[idx[t, j]] / T
    return g


def expert_counts(idx, E: int) -> np.ndarray:
    """``counts[e] = #{(t, j): idx[t, j] == e}`` ([HP] ``torch.bincount``);
    copies marked -1 (dropped by :func:`capacity_drop`) are not counted."""
    flat = _i64(idx).ravel()
    return np.bincount(flat[flat >= 0], minlength=E).astype(np.int64)


def capacity_drop(idx, sel_scores, capacity: int) -> np.ndarray:
    """Capacity drop policy ([PF] PaddleFormers ``moe_gate.py``,
    ``_probs_drop_policy``): a token keeps its assignment to an expert when
    it is routed there and its score for that expert is among the top
    ``capacity`` scores for that expert.  Reading taken: the ranking is over
    the copies routed to the expert (unrouted pairs rank below every routed
    one), by the router's score of the pair before renormalisation and
    scale, higher first, equal scores in increasing token order.  Returns
    the keep mask ``[T, k]``.  ``sel_scores[t, j]`` is the score of the
    copy ``(t, j)``."""
    idx = _i64(idx)
    s = as_f64(sel_scores)
    T, k = idx.shape
    keep = np.zeros((T, k), dtype=bool)
    for e in np.unique(idx):
        if e < 0:
            continue
        tt, jj = np.nonzero(idx == e)
        order = sorted(range(len(tt)), key=lambda q: (-s[tt[q], jj[q]], tt[q]))
        for q in order[:max(capacity, 0)]:
            keep[tt[q], jj[q]] = True
    return keep


# --------------------------------------------------------------------------
# Dispatch  ([HP] MoE.permutation and the gather in MoE.forward)
# --------------------------------------------------------------------------

def dispatch(idx, E: int):
    """Expert-major permutation of the routed copies.

    Flattening ``idx[T, k]`` gives flat index ``f = t*k + j``; a stable sort of
    the flat expert ids lists the copies expert by expert, and inside one
    expert in increasing ``f`` ([HP] ``MoE.permutation``).  Returns

    * ``counts[E]``, ``offsets[E+1]`` (exclusive scan, ``offsets[E] = T*k``),
    * ``src_row[N]``: the token of each expert-major slot (``f // k``),
    * ``dst_pos[T, k]``: the slot of each copy (inverse of the sort).

    Copies marked -1 (dropped by the capacity policy) get no slot: their
    ``dst_pos`` is -1, and ``offsets[E]`` counts the kept copies only.
    """
    idx = _i64(idx)
    T, k = idx.shape
    flat = idx.ravel()
    kept = np.nonzero(flat >= 0)[0]
    order = kept[np.argsort(flat[kept], kind="stable")]   # slot -> flat index
    counts = np.bincount(flat[kept], minlength=E).astype(np.int64)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    src_row = order // k
    dst = np.full(T * k, -1, dtype=np.int64)
    dst[order] = np.arange(len(order))
    return counts, offsets, src_row, dst.reshape(T, k)


def permute_rows(x, src_row) -> np.ndarray:
    """``x_perm[s] = x[src_row[s]]`` ([HP] ``routed_x = x_flat[token_indices]``)."""
    return as_f64(x)[_i64(src_row)]


# --------------------------------------------------------------------------
# Expert-parallel layout and local regroup ([EP] Ep2DpParallel._token_dispatch)
# --------------------------------------------------------------------------

def ep_dispatch_rank_major(idx, E: int, R: int):
    """Layout of the routed copies as EP ranks would receive them.

    Source rank ``r`` owns the contiguous token shard
    ``[r*S, min(T, (r+1)*S))`` with ``S = ceil(T / R)`` and dispatches it into
    its own expert-major order.  Destination block ``g`` owns the local
    experts ``g*L .. g*L + L - 1`` (``L = E // R``); the all-to-all
    concatenates, for every ``g``, source rank after source rank, the rows each
    source holds for those experts (source rank outer, local expert inner).

    Returns ``counts_rm[G, R, L]``, ``src_row[N]`` (token of every received
    row), ``dst_pos[T, k]`` (received row of every copy).
    """
    idx = _i64(idx)
    T, k = idx.shape
    G = R
    L = E // G
    S = -(-T // R) if T else 0
    counts_rm = np.zeros((G, R, L), dtype=np.int64)
    src_row = []
    dst_pos = np.full((T, k), -1, dtype=np.int64)
    local = []
    for r in range(R):
        t0, t1 = min(T, r * S), min(T, (r + 1) * S)
        c, off, srow, dpos = dispatch(idx[t0:t1], E)
        local.append((t0, c, off, srow, dpos))
    pos = 0
    for g in range(G):
        for r in range(R):
            t0, c, off, srow, dpos = local[r]
            for l in range(L):
                e = g * L + l
                counts_rm[g, r, l] = c[e]
            lo, hi = off[g * L], off[(g + 1) * L]
            # rows [lo, hi) of rank r's buffer land at [pos, pos + hi - lo)
            src_row.append(srow[lo:hi] + t0)
            sel = (dpos >= lo) & (dpos < hi)
            tt, jj = np.nonzero(sel)
            dst_pos[tt + t0, jj] = dpos[tt, jj] - lo + pos
            pos += hi - lo
    src_row = np.concatenate(src_row) if src_row else np.zeros(0, np.int64)
    return counts_rm, src_row, dst_pos


def ep_local_regroup(counts_rm):
    """Regroup of a rank-major received buffer into expert-major order.

    For each destination block ``g`` and local expert ``l``, the segments of
    source ranks ``r = 0 .. R-1`` are appended in order.  Returns
    ``perm[rows]`` (output row -> input row), ``counts_em[G*L]`` (summed over
    source ranks) and ``offsets_em[G*L + 1]``.
    """
    c = _i64(counts_rm)
    G, R, L = c.shape
    in_off = np.zeros(G * R * L + 1, dtype=np.int64)
    in_off[1:] = np.cumsum(c.ravel())              # (g, r, l) order
    perm = []
    for g in range(G):
        for l in range(L):
            for r in range(R):
                s = (g * R + r) * L + l
                perm.append(np.arange(in_off[s], in_off[s + 1]))
    perm = np.concatenate(perm) if perm else np.zeros(0, np.int64)
    counts_em = c.sum(axis=1).reshape(G * L)
    offsets_em = np.zeros(G * L + 1, dtype=np.int64)
    offsets_em[1:] = np.cumsum(counts_em)
    return perm, counts_em, offsets_em


def apply_row_perm(rows, perm) -> np.ndarray:
    """``out[i] = rows[perm[i]]``."""
    return np.asarray(rows)[_i64(perm)]


# --------------------------------------------------------------------------
# Experts ([HP] _run_experts_for_loop / FeedForward; [QO] training branch)
# --------------------------------------------------------------------------

def silu(z) -> np.ndarray:
    """``silu(z) = z / (1 + exp(-z))``."""
    z = as_f64(z)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def swiglu_ffn(S, w1e, w3e, w2e) -> np.ndarray:
    """One expert: ``(silu(S w1^T) * (S w3^T)) w2^T`` with ``[out, in]``
    weights ([HP] ``FeedForward.forward``)."""
    S = as_f64(S)
    A = silu(S @ as_f64(w1e).T) * (S @ as_f64(w3e).T)
    return A @ as_f64(w2e).T


def grouped_swiglu(x_perm, offsets, w1, w3, w2, row_scale=None) -> np.ndarray:
    """Per-expert SwiGLU over expert-major segments ([HP]
    ``_run_experts_for_loop``): experts with no rows are skipped; an optional
    per-row ``row_scale`` multiplies the hidden activation before ``w2``.
    Converts one expert's weights to fp64 at a time."""
    xp = as_f64(x_perm)
    off = _i64(offsets)
    E = len(off) - 1
    d = w2.shape[1]
    y = np.zeros((xp.shape[0], d), dtype=np.float64)
    rs = None if row_scale is None else as_f64(row_scale)
    for e in range(E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi == lo:
            continue
        S = xp[lo:hi]
        A = silu(S @ as_f64(w1[e]).T) * (S @ as_f64(w3[e]).T)
        if rs is not None:
            A = A * rs[lo:hi, None]
        y[lo:hi] = A @ as_f64(w2[e]).T
    return y


# --------------------------------------------------------------------------
# Combine ([QO] index_add_; [HP] MoE.unpermutation scatter_add)
# --------------------------------------------------------------------------

def combine(y, dst_pos, topk_w=None) -> np.ndarray:
    """``out[t] = sum_j w[t, j] * y[dst_pos[t, j]]`` (``w = 1`` if None).

    The sum over ``j`` is the scatter-add of every copy's output into its
    token row.
    """
    y = as_f64(y)
    dp = _i64(dst_pos)
    T, k = dp.shape
    out = np.zeros((T, y.shape[1]), dtype=np.float64)
    w = np.ones((T, k)) if topk_w is None else as_f64(topk_w)
    for j in range(k):
        live = dp[:, j] >= 0           # a dropped copy (-1) adds nothing
        out[live] += w[live, j:j + 1] * y[dp[live, j]]
    return out


# --------------------------------------------------------------------------
# Whole layer ([HP] MoE.forward with score_before_experts=False)
# --------------------------------------------------------------------------

def moe_forward(x, w_router, w1, w3, w2, top_k: int, renormalize: bool = True,
                logits=None, ep_ranks: int = 1, router=None, score_before_experts=False,
                shared=None):
    """Router -> dispatch -> (EP regroup) -> grouped SwiGLU -> combine.

    Returns a dict with every intermediate (fp64 / int64).  With
    ``ep_ranks > 1`` the routed rows are first laid out as received by
    ``ep_ranks`` simulated EP ranks and regrouped before the experts.
    ``router`` (a dict of :func:`router_topk_general` options) selects the
    general router.  With ``score_before_experts`` ([HP] ``MoE.forward``)
    every routed row is multiplied by its routing weight before the experts
    and the combine adds the expert outputs unweighted.  ``shared`` =
    ``(ws1 [hs, d], ws3 [hs, d], ws2 [d, hs])`` adds the shared expert, a
    dense SwiGLU ``FeedForward`` on every token ([HP] ``MoE.forward``:
    ``out = unpermutation(...) + shared_expert(x_flat)``).
    """
    res = _moe_routed(x, w_router, w1, w3, w2, top_k, renormalize, logits, ep_ranks, router,
                      score_before_experts)
    if shared is not None:
        res["shared_out"] = swiglu_ffn(x, *shared)
        res["out"] = res["out"] + res["shared_out"]
    return res


def _moe_routed(x, w_router, w1, w3, w2, top_k, renormalize, logits, ep_ranks, router,
                score_before_experts):
    E = w1.shape[0]
    if router is None:
        idx, w, counts, L = router_topk(top_k, renormalize, x=x, w_router=w_router,
                                        logits=logits)
    else:
        idx, w, counts, L = router_topk_general(top_k, x=x, w_router=w_router, logits=logits,
                                                renormalize=renormalize, **router)
    res = {"logits": L, "topk_idx": idx, "topk_w": w}
    if ep_ranks == 1:
        c, off, src_row, dst_pos = dispatch(idx, E)
        res.update(counts=c, offsets=off, src_row=src_row, dst_pos=dst_pos)
        x_perm = permute_rows(x, src_row)
        if score_before_experts:
            slot_w = np.empty(len(src_row))
            slot_w[_i64(dst_pos).ravel()] = w.ravel()
            x_perm = x_perm * slot_w[:, None]
        y = grouped_swiglu(x_perm, off, w1, w3, w2)
        out = combine(y, dst_pos, None if score_before_experts else w)
        res.update(x_perm=x_perm, y=y, out=out)
        return res
    assert not score_before_experts, "score_before_experts is defined on the single-device path"
    counts_rm, src_rm, dst_rm = ep_dispatch_rank_major(idx, E, ep_ranks)
    x_rm = permute_rows(x, src_rm)
    perm, counts_em, off_em = ep_local_regroup(counts_rm)
    x_em = apply_row_perm(x_rm, perm)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(len(perm))
    dst_em = inv[dst_rm]
    y = grouped_swiglu(x_em, off_em, w1, w3, w2)
    res.update(counts_rm=counts_rm, src_row_rm=src_rm, dst_pos_rm=dst_rm,
               perm=perm, counts=counts_em, offsets=off_em, dst_pos=dst_em,
               src_row=src_rm[perm], x_perm=x_em, y=y,
               out=combine(y, dst_em, w))
    return res


# --------------------------------------------------------------------------
# Backward (the training path: [HP] MoE.forward and _run_experts_for_loop
# differentiated by the chain rule; [QO] training branch)
# --------------------------------------------------------------------------

def silu_grad(z) -> np.ndarray:
    """``d silu(z) / dz = s(z) (1 + z (1 - s(z)))`` with ``s`` the logistic
    sigmoid (derivative of ``z s(z)`` by the product rule, ``s' = s(1-s)``)."""
    s = sigmoid(z)
    z = as_f64(z)
    return s * (1.0 + z * (1.0 - s))


def grouped_preactivations(x_perm, offsets, w1, w3):
    """The two first-layer products of every expert segment, ``G = S w1^T``
    and ``U = S w3^T`` ([HP] ``FeedForward.forward`` before the SiLU), as
    ``[N, h]`` fp64 arrays (what a training forward keeps for the
    backward)."""
    xp = as_f64(x_perm)
    off = _i64(offsets)
    h = w1.shape[1]
    G = np.zeros((xp.shape[0], h))
    U = np.zeros((xp.shape[0], h))
    for e in range(len(off) - 1):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi > lo:
            G[lo:hi] = xp[lo:hi] @ as_f64(w1[e]).T
            U[lo:hi] = xp[lo:hi] @ as_f64(w3[e]).T
    return G, U


def combine_backward(dout, y, dst_pos, topk_w=None):
    """Gradients of ``out[t] = sum_j w[t, j] y[dst_pos[t, j]]``.

    Returns ``(dy, dw)``: ``dy[dst_pos[t, j]] = w[t, j] dout[t]`` (every slot
    is the copy of exactly one ``(t, j)``) and ``dw[t, j] = <dout[t],
    y[dst_pos[t, j]]>`` (``dw`` is None when the combine is unweighted).
    """
    dout = as_f64(dout)
    y = as_f64(y)
    dp = _i64(dst_pos)
    T, k = dp.shape
    w = np.ones((T, k)) if topk_w is None else as_f64(topk_w)
    dy = np.zeros_like(y)
    dw = np.zeros((T, k))
    for t in range(T):
        for j in range(k):
            dy[dp[t, j]] = w[t, j] * dout[t]
            dw[t, j] = float(dout[t] @ y[dp[t, j]])
    return dy, (None if topk_w is None else dw)


def grouped_swiglu_backward(x_perm, offsets, w1, w3, w2, dy):
    """Gradients of :func:`grouped_swiglu` (no row scale) for an upstream
    gradient ``dy [N, d]``, one expert segment at a time.

    With ``S`` the expert's rows, ``G = S w1^T``, ``U = S w3^T``,
    ``A = silu(G) * U`` and ``Y = A w2^T``:
    ``dA = dY w2``, ``dU = dA * silu(G)``, ``dG = dA * U * silu'(G)``,
    ``dw2 = dY^T A``, ``dw1 = dG^T S``, ``dw3 = dU^T S``,
    ``dS = dG w1 + dU w3``.  Experts with no rows get zero weight gradients.
    Returns ``(dx_perm, dw1, dw3, dw2)`` in fp64.
    """
    xp = as_f64(x_perm)
    g = as_f64(dy)
    off = _i64(offsets)
    E = len(off) - 1
    h, d = w1.shape[1], w1.shape[2]
    dxp = np.zeros_like(xp)
    dw1 = np.zeros((E, h, d))
    dw3 = np.zeros((E, h, d))
    dw2 = np.zeros((E, d, h))
    for e in range(E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi == lo:
            continue
        S, dY = xp[lo:hi], g[lo:hi]
        W1, W3, W2 = as_f64(w1[e]), as_f64(w3[e]), as_f64(w2[e])
        G, U = S @ W1.T, S @ W3.T
        A = silu(G) * U
        dA = dY @ W2
        dU = dA * silu(G)
        dG = dA * U * silu_grad(G)
        dw2[e] = dY.T @ A
        dw1[e] = dG.T @ S
        dw3[e] = dU.T @ S
        dxp[lo:hi] = dG @ W1 + dU @ W3
    return dxp, dw1, dw3, dw2


def dispatch_backward(dx_perm, dst_pos) -> np.ndarray:
    """Gradient of ``x_perm = x[src_row]`` with respect to ``x``: every token
    collects the gradients of its copies, ``dx[t] = sum_j dx_perm[dst_pos[t,
    j]]`` (the adjoint of the row gather is the scatter-add)."""
    return combine(dx_perm, dst_pos, None)


def scaled_dispatch_backward(dx_perm, dst_pos, topk_w, x):
    """Gradients of the scaled row gather of ``score_before_experts`` ([HP]
    ``MoE.forward``): the copy in slot ``p = dst_pos[t, j]`` is
    ``x_perm[p] = topk_w[t, j] * x[t]``, so ``dx[t] = sum_j topk_w[t, j] *
    dx_perm[p]`` and ``d_topk_w[t, j] = <dx_perm[p], x[t]>``.  Returns
    ``(dx [T, d], d_topk_w [T, k])`` in fp64."""
    g = as_f64(dx_perm)
    xx = as_f64(x)
    dp = _i64(dst_pos)
    w = as_f64(topk_w)
    T, k = dp.shape
    dx = np.zeros_like(xx)
    dw = np.zeros((T, k))
    for t in range(T):
        for j in range(k):
            dx[t] += w[t, j] * g[dp[t, j]]
            dw[t, j] = float(g[dp[t, j]] @ xx[t])
    return dx, dw


def router_backward(logits, topk_idx, d_topk_w, score: str = "softmax",
                    renormalize: bool = False, route_scale: float = 1.0, x=None, w_router=None):
    """Gradient of the routing weights of :func:`router_topk_general` with
    respect to the gate logits, for upstream gradients ``d_topk_w [T, k]``
    and the experts it selected (selection itself has no gradient; the
    expert bias and the group masking only select).

    Per token, with ``s`` the scores (softmax or sigmoid of the logits), ``S``
    the selected set and ``c`` the route scale: ``w_j = c s_j / sum_S s``
    (renormalised) or ``w_j = c s_j``, so ``ds_j = c (g_j - sum_S g s /
    sum_S s) / sum_S s`` or ``ds_j = c g_j`` on ``S`` and 0 elsewhere; then
    ``dz = s * (ds - <s, ds>)`` (softmax) or ``dz = ds * s (1 - s)``
    (sigmoid).  Returns ``dz [T, E]``; with ``x`` and ``w_router`` also the
    gate's gradients ``(dz, dw_router = dz^T x, dx = dz w_router)``.
    """
    L = as_f64(logits)
    idx = _i64(topk_idx)
    g = as_f64(d_topk_w)
    T, E = L.shape
    s = softmax(L) if score == "softmax" else sigmoid(L)
    dz = np.zeros((T, E))
    for t in range(T):
        sel = s[t, idx[t]]
        ds = np.zeros(E)
        if renormalize:
            tot = sel.sum()
            ds[idx[t]] = route_scale * (g[t] - float(g[t] @ sel) / tot) / tot
        else:
            ds[idx[t]] = route_scale * g[t]
        if score == "softmax":
            dz[t] = s[t] * (ds - float(s[t] @ ds))
        else:
            dz[t] = ds * s[t] * (1.0 - s[t])
    if x is None:
        return dz
    return dz, dz.T @ as_f64(x), dz @ as_f64(w_router)


def dense_moe(x, idx, w, w1, w3, w2) -> np.ndarray:
    """Brute-force dense formulation ([QO] eval branch): every expert runs
    on every token and the outputs are summed with the mask
    ``M[t, e] = sum_j w[t, j] [idx[t, j] == e]``."""
    x = as_f64(x)
    idx = _i64(idx)
    w = as_f64(w)
    T = x.shape[0]
    E = w1.shape[0]
    M = np.zeros((T, E))
    for j in range(idx.shape[1]):
        np.add.at(M, (np.arange(T), idx[:, j]), w[:, j])
    out = np.zeros((T, w2.shape[1]))
    for e in range(E):
        out += M[:, e:e + 1] * swiglu_ffn(x, w1[e], w3[e], w2[e])
    return out


def moe_tokens(x_rows, idx_rows, w_rows, w1, w3, w2) -> np.ndarray:
    """Token-by-token definition for a sample of tokens:
    ``out[t] = sum_j w[t, j] * FFN_{idx[t, j]}(x[t])``.  Used to check sampled
    outputs of layers too large for the full oracle.  Each expert's weights
    are widened to fp64 once, for all sampled copies routed to it."""
    x_rows = as_f64(x_rows)
    idx_rows = _i64(idx_rows)
    w_rows = as_f64(w_rows)
    out = np.zeros((x_rows.shape[0], w2.shape[1]))
    for e in np.unique(idx_rows):
        tt, jj = np.nonzero(idx_rows == e)
        ye = swiglu_ffn(x_rows[tt], w1[int(e)], w3[int(e)], w2[int(e)])
        for q in range(len(tt)):
            out[tt[q]] += w_rows[tt[q], jj[q]] * ye[q]
    return out
