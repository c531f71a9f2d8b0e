"""B200 (sm_100a) MoE layer forward: thin Python binding of libmoe.so.

Every step of the layer (router, dispatch, EP regroup, grouped SwiGLU,
combine) runs in the CUDA kernels of ``libmoe.so``; this module only
marshals torch tensors into the C ABI of ``include/moe.h`` (pointers, sizes,
the current CUDA stream) and raises on a non-zero status.  There is no CPU
fallback: importing the binding without the built library raises.

Two layers of API:

* ``moe_router_topk``, ``moe_router_topk_ex``, ``moe_dispatch``,
  ``moe_ep_dispatch_rank_major``, ``moe_ep_local_regroup``,
  ``moe_grouped_swiglu``, ``moe_combine``, ``moe_forward``,
  ``moe_forward_ex`` -- same names and argument order as the C functions,
  with torch tensors (or None) in place of pointers and a
  ``RouterOptions`` structure for ``moe_router_options_t``; outputs are
  caller-allocated.
* ``router_topk``, ``dispatch``, ``ep_dispatch_rank_major``,
  ``ep_local_regroup``, ``grouped_swiglu``, ``combine``, ``forward`` --
  allocate their outputs and workspace with torch and return them.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = [
    "MoEError", "lib", "LIB_PATH", "MOE_F32", "MOE_BF16", "MOE_SCORE_SOFTMAX",
    "MOE_SCORE_SIGMOID", "RouterOptions", "router_options", "moe_router_options_init",
    "SharedExpert", "shared_expert", "forward_ex_workspace_size",
    "moe_router_topk_ex", "moe_forward_ex",
    "MOE_DEV_BAD_EXPERT", "MOE_DEV_BAD_COUNTS", "MOE_DEV_BAD_OFFSETS", "MOE_DEV_TIMEOUT",
    "EXPORTED_SYMBOLS",
    "moe_router_topk", "moe_dispatch", "moe_ep_dispatch_rank_major", "moe_ep_local_regroup",
    "moe_grouped_swiglu", "moe_grouped_swiglu_gather", "moe_combine", "moe_forward",
    "moe_get_device_status", "grouped_swiglu_gather", "moe_grouped_swiglu_combine",
    "grouped_swiglu_combine",
    "router_workspace_size", "dispatch_workspace_size", "ep_dispatch_workspace_size",
    "regroup_workspace_size", "grouped_swiglu_workspace_size", "forward_workspace_size",
    "router_topk", "dispatch", "ep_dispatch_rank_major", "ep_local_regroup",
    "grouped_swiglu", "combine", "forward", "device_status",
    "moe_grouped_swiglu_train", "moe_grouped_swiglu_backward", "moe_combine_backward",
    "moe_dispatch_backward", "grouped_swiglu_backward_workspace_size",
    "grouped_swiglu_train", "grouped_swiglu_backward", "combine_backward", "dispatch_backward",
    "moe_router_backward", "router_backward_workspace_size", "router_backward",
    "moe_train_state_size", "moe_forward_train", "moe_backward_workspace_size", "moe_backward",
    "moe_train_state_size_ex", "moe_forward_train_ex", "moe_backward_workspace_size_ex",
    "moe_backward_ex", "forward_train", "backward",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe.so")

MOE_F32, MOE_BF16 = 0, 1
MOE_SCORE_SOFTMAX, MOE_SCORE_SIGMOID = 0, 1
MOE_DEV_BAD_EXPERT, MOE_DEV_BAD_COUNTS, MOE_DEV_BAD_OFFSETS, MOE_DEV_TIMEOUT = 1, 2, 4, 8

EXPORTED_SYMBOLS = [
    "moe_router_workspace_size", "moe_router_topk", "moe_router_options_init",
    "moe_router_topk_ex",
    "moe_dispatch_workspace_size", "moe_dispatch", "moe_dispatch_noalloc",
    "moe_ep_dispatch_workspace_size", "moe_ep_dispatch_rank_major",
    "moe_regroup_workspace_size", "moe_ep_local_regroup",
    "moe_grouped_swiglu_workspace_size", "moe_grouped_swiglu", "moe_grouped_swiglu_gather",
    "moe_grouped_swiglu_combine_workspace_size", "moe_grouped_swiglu_combine",
    "moe_combine",
    "moe_grouped_swiglu_train", "moe_grouped_swiglu_backward_workspace_size",
    "moe_grouped_swiglu_backward", "moe_combine_backward", "moe_dispatch_backward",
    "moe_router_backward_workspace_size", "moe_router_backward",
    "moe_train_state_size", "moe_forward_train", "moe_backward_workspace_size", "moe_backward",
    "moe_train_state_size_ex", "moe_forward_train_ex", "moe_backward_workspace_size_ex",
    "moe_backward_ex",
    "moe_forward_workspace_size", "moe_forward", "moe_forward_ex_workspace_size",
    "moe_forward_ex", "moe_get_device_status", "moe_selftest_timeout", "moe_status_string",
    "moe_last_error", "moe_version",
]


class MoEError(RuntimeError):
    pass


class RouterOptions(ctypes.Structure):
    """``moe_router_options_t`` of include/moe.h (device pointers as ints)."""
    _fields_ = [
        ("score", ctypes.c_int),
        ("renormalize", ctypes.c_int),
        ("route_scale", ctypes.c_float),
        ("expert_bias", ctypes.c_void_p),
        ("num_groups", ctypes.c_int),
        ("topk_groups", ctypes.c_int),
        ("tokens_per_expert", ctypes.c_void_p),
        ("score_before_experts", ctypes.c_int),
        ("aux_loss", ctypes.c_void_p),
        ("aux_loss_coef", ctypes.c_float),
        ("capacity", ctypes.c_int),
        ("topk_scores", ctypes.c_void_p),
    ]


class SharedExpert(ctypes.Structure):
    """``moe_shared_expert_t`` of include/moe.h (device pointers as ints)."""
    _fields_ = [
        ("w1", ctypes.c_void_p),
        ("w3", ctypes.c_void_p),
        ("w2", ctypes.c_void_p),
        ("h", ctypes.c_int),
    ]


_P = ctypes.c_void_p
_I = ctypes.c_int
_Z = ctypes.c_size_t
_SIGS = {
    "moe_router_workspace_size": (_Z, [_I, _I, _I, _I]),
    "moe_router_topk": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _Z, _P]),
    "moe_router_options_init": (None, [ctypes.POINTER(RouterOptions)]),
    "moe_router_topk_ex": (_I, [_P, _P, _P, _I, _I, _I, _I, ctypes.POINTER(RouterOptions), _I,
                                _P, _P, _P, _P, _P, _Z, _P]),
    "moe_dispatch_workspace_size": (_Z, [_I, _I, _I]),
    "moe_dispatch": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _Z, _P]),
    "moe_dispatch_noalloc": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "moe_ep_dispatch_workspace_size": (_Z, [_I, _I, _I, _I]),
    "moe_ep_dispatch_rank_major": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P,
                                        _Z, _P]),
    "moe_regroup_workspace_size": (_Z, [_I, _I, _I]),
    "moe_ep_local_regroup": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _Z,
                                  _P]),
    "moe_grouped_swiglu_workspace_size": (_Z, [_I, _I, _I, _I, _I]),
    "moe_grouped_swiglu": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _Z, _P]),
    "moe_grouped_swiglu_gather": (_I, [_P, _I, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P,
                                       _P, _Z, _P]),
    "moe_grouped_swiglu_combine_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I]),
    "moe_grouped_swiglu_combine": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P,
                                        _P, _Z, _P]),
    "moe_combine": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P]),
    "moe_grouped_swiglu_train": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _Z,
                                      _P]),
    "moe_grouped_swiglu_backward_workspace_size": (_Z, [_I, _I, _I, _I, _I]),
    "moe_grouped_swiglu_backward": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P,
                                         _P, _P, _P, _P, _Z, _P]),
    "moe_combine_backward": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P]),
    "moe_dispatch_backward": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P]),
    "moe_router_backward_workspace_size": (_Z, [_I, _I, _I]),
    "moe_train_state_size": (_Z, [_I, _I, _I, _I, _I]),
    "moe_forward_train": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _I, _P, _P, _Z,
                               _P]),
    "moe_backward_workspace_size": (_Z, [_I, _I, _I, _I, _I]),
    "moe_backward": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _I, _P, _P, _P, _P, _P,
                          _P, _P, _P, _Z, _P]),
    "moe_router_backward": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _I, _P, _P, _P, _P, _Z,
                                 _P]),
    "moe_train_state_size_ex": (_Z, [_I, _I, _I, _I, _I, _I]),
    "moe_forward_train_ex": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P,
                                  ctypes.POINTER(SharedExpert), _I, _P, _P, _Z, _P]),
    "moe_backward_workspace_size_ex": (_Z, [_I, _I, _I, _I, _I, _I]),
    "moe_backward_ex": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P,
                             ctypes.POINTER(SharedExpert), _I, _P, _P, _P, _P, _P, _P, _P, _P,
                             _P, _P, _P, _Z, _P]),
    "moe_forward_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I, _I]),
    "moe_forward": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P,
                         _P, _P, _P, _Z, _P]),
    "moe_forward_ex_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I, _I, _I]),
    "moe_forward_ex": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I,
                            ctypes.POINTER(RouterOptions), ctypes.POINTER(SharedExpert), _I, _I,
                            _P, _P, _P, _P, _P, _P, _Z, _P]),
    "moe_selftest_timeout": (_I, [_P, _Z, _P]),
    "moe_get_device_status": (_I, [_P, ctypes.POINTER(_I), _P]),
    "moe_status_string": (ctypes.c_char_p, [_I]),
    "moe_last_error": (ctypes.c_char_p, []),
    "moe_version": (_I, []),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libmoe.so.  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise MoEError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m routing_dispatch_grouped_topk_b200.build` (there is no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


# ------------------------------------------------------------------ helpers
def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return MOE_BF16
    if t.dtype == torch.float32:
        return MOE_F32
    raise MoEError(f"unsupported dtype {t.dtype}")


def _ptr(t: Optional[torch.Tensor], dtype=None, name="tensor") -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise MoEError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise MoEError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise MoEError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr() or None


def _stream(stream=None) -> Optional[int]:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream or None


def _check(code: int, fn: str):
    if code != 0:
        L = lib()
        msg = L.moe_last_error().decode()
        raise MoEError(f"{fn}: {L.moe_status_string(code).decode()} ({msg})")


def _nbytes(t: Optional[torch.Tensor]) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def _ws(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


# ------------------------------------------------------ C-ABI mirror (1:1)
def router_workspace_size(T, d, E, dt) -> int:
    return lib().moe_router_workspace_size(T, d, E, dt)


def dispatch_workspace_size(T, E, top_k) -> int:
    return lib().moe_dispatch_workspace_size(T, E, top_k)


def ep_dispatch_workspace_size(T, E, top_k, R) -> int:
    return lib().moe_ep_dispatch_workspace_size(T, E, top_k, R)


def regroup_workspace_size(G, R, L) -> int:
    return lib().moe_regroup_workspace_size(G, R, L)


def grouped_swiglu_workspace_size(N, d, h, E, dt) -> int:
    return lib().moe_grouped_swiglu_workspace_size(N, d, h, E, dt)


def forward_workspace_size(T, d, E, top_k, h, ep_ranks, dt) -> int:
    return lib().moe_forward_workspace_size(T, d, E, top_k, h, ep_ranks, dt)


def forward_ex_workspace_size(T, d, E, top_k, h, ep_ranks, dt, h_shared=0) -> int:
    return lib().moe_forward_ex_workspace_size(T, d, E, top_k, h, ep_ranks, dt, h_shared)


def moe_router_topk(x, w_router, logits_in, T, d, E, top_k, score, renormalize, dt, logits_out,
                    topk_idx, topk_w, counts, ws, stream=None):
    _check(lib().moe_router_topk(
        _ptr(x, name="x"), _ptr(w_router, name="w_router"),
        _ptr(logits_in, torch.float32, "logits_in"), T, d, E, top_k, score, int(renormalize), dt,
        _ptr(logits_out, torch.float32, "logits_out"), _ptr(topk_idx, torch.int32, "topk_idx"),
        _ptr(topk_w, torch.float32, "topk_w"), _ptr(counts, torch.int32, "counts"),
        _ptr(ws, name="ws"), _nbytes(ws), _stream(stream)), "moe_router_topk")


def moe_router_options_init() -> RouterOptions:
    o = RouterOptions()
    lib().moe_router_options_init(ctypes.byref(o))
    return o


def router_options(score="softmax", renormalize=False, route_scale=1.0, expert_bias=None,
                   num_groups=0, topk_groups=0, tokens_per_expert=None,
                   score_before_experts=False, aux_loss=None,
                   aux_loss_coef=0.0, capacity=0, topk_scores=None) -> RouterOptions:
    """A RouterOptions from keyword values ([HP] TokenChoiceTopKRouter's
    settings).  expert_bias / tokens_per_expert are fp32 CUDA tensors [E],
    aux_loss an fp32 CUDA tensor of one element, topk_scores an fp32 CUDA
    tensor [T, k] (output), or None; they must stay alive while the call
    that takes the options runs.  aux_loss_coef (the backward entry points)
    adds the gradient of aux_loss_coef times the load-balance loss to the
    routing weights' gradient.  capacity > 0 applies the capacity drop
    policy (dropped copies: topk_idx -1, weight 0)."""
    o = moe_router_options_init()
    o.score = {"softmax": MOE_SCORE_SOFTMAX, "sigmoid": MOE_SCORE_SIGMOID}[score]
    o.renormalize = int(bool(renormalize))
    o.route_scale = float(route_scale)
    o.expert_bias = _ptr(expert_bias, torch.float32, "expert_bias")
    o.num_groups = int(num_groups or 0)
    o.topk_groups = int(topk_groups or 0)
    o.tokens_per_expert = _ptr(tokens_per_expert, torch.float32, "tokens_per_expert")
    o.score_before_experts = int(bool(score_before_experts))
    o.aux_loss = _ptr(aux_loss, torch.float32, "aux_loss")
    o.aux_loss_coef = float(aux_loss_coef)
    o.capacity = int(capacity or 0)
    o.topk_scores = _ptr(topk_scores, torch.float32, "topk_scores")
    return o


def _opts(o: Optional[RouterOptions]):
    return None if o is None else ctypes.byref(o)


def moe_router_topk_ex(x, w_router, logits_in, T, d, E, top_k, opts, dt, logits_out, topk_idx,
                       topk_w, counts, ws, stream=None):
    _check(lib().moe_router_topk_ex(
        _ptr(x, name="x"), _ptr(w_router, name="w_router"),
        _ptr(logits_in, torch.float32, "logits_in"), T, d, E, top_k, _opts(opts), dt,
        _ptr(logits_out, torch.float32, "logits_out"), _ptr(topk_idx, torch.int32, "topk_idx"),
        _ptr(topk_w, torch.float32, "topk_w"), _ptr(counts, torch.int32, "counts"),
        _ptr(ws, name="ws"), _nbytes(ws), _stream(stream)), "moe_router_topk_ex")


def moe_dispatch(x, topk_idx, T, d, E, top_k, dt, counts, offsets, src_row, dst_pos, x_perm, ws,
                 stream=None):
    _check(lib().moe_dispatch(
        _ptr(x, name="x"), _ptr(topk_idx, torch.int32, "topk_idx"), T, d, E, top_k, dt,
        _ptr(counts, torch.int32, "counts"), _ptr(offsets, torch.int32, "offsets"),
        _ptr(src_row, torch.int32, "src_row"), _ptr(dst_pos, torch.int32, "dst_pos"),
        _ptr(x_perm, name="x_perm"), _ptr(ws, name="ws"), _nbytes(ws), _stream(stream)),
        "moe_dispatch")


def moe_ep_dispatch_rank_major(x, topk_idx, T, d, E, top_k, R, dt, counts_rm, offsets_rm,
                               src_row, dst_pos, x_rm, ws, stream=None):
    _check(lib().moe_ep_dispatch_rank_major(
        _ptr(x, name="x"), _ptr(topk_idx, torch.int32, "topk_idx"), T, d, E, top_k, R, dt,
        _ptr(counts_rm, torch.int32, "counts_rm"), _ptr(offsets_rm, torch.int32, "offsets_rm"),
        _ptr(src_row, torch.int32, "src_row"), _ptr(dst_pos, torch.int32, "dst_pos"),
        _ptr(x_rm, name="x_rm"), _ptr(ws, name="ws"), _nbytes(ws), _stream(stream)),
        "moe_ep_dispatch_rank_major")


def moe_ep_local_regroup(inp, counts_rm, G, R, L, rows, d, dt, out, counts_em, offsets_em, perm,
                         perm_inv, ws, stream=None):
    _check(lib().moe_ep_local_regroup(
        _ptr(inp, name="in"), _ptr(counts_rm, torch.int32, "counts_rm"), G, R, L, rows, d, dt,
        _ptr(out, name="out"), _ptr(counts_em, torch.int32, "counts_em"),
        _ptr(offsets_em, torch.int32, "offsets_em"), _ptr(perm, torch.int32, "perm"),
        _ptr(perm_inv, torch.int32, "perm_inv"), _ptr(ws, name="ws"), _nbytes(ws),
        _stream(stream)), "moe_ep_local_regroup")


def moe_grouped_swiglu(x_perm, offsets, w1, w3, w2, row_scale, N, d, h, E, dt, y, ws,
                       stream=None):
    _check(lib().moe_grouped_swiglu(
        _ptr(x_perm, name="x_perm"), _ptr(offsets, torch.int32, "offsets"), _ptr(w1, name="w1"),
        _ptr(w3, name="w3"), _ptr(w2, name="w2"), _ptr(row_scale, torch.float32, "row_scale"),
        N, d, h, E, dt, _ptr(y, name="y"), _ptr(ws, name="ws"), _nbytes(ws), _stream(stream)),
        "moe_grouped_swiglu")


def moe_grouped_swiglu_gather(x, T, src_row, offsets, w1, w3, w2, row_scale, N, d, h, E, dt, y,
                              ws, stream=None):
    _check(lib().moe_grouped_swiglu_gather(
        _ptr(x, name="x"), T, _ptr(src_row, torch.int32, "src_row"),
        _ptr(offsets, torch.int32, "offsets"), _ptr(w1, name="w1"), _ptr(w3, name="w3"),
        _ptr(w2, name="w2"), _ptr(row_scale, torch.float32, "row_scale"), N, d, h, E, dt,
        _ptr(y, name="y"), _ptr(ws, name="ws"), _nbytes(ws), _stream(stream)),
        "moe_grouped_swiglu_gather")


def moe_grouped_swiglu_combine(x_perm, offsets, w1, w3, w2, dst_pos, topk_w, T, top_k, d, h, E,
                               dt, out, ws, stream=None):
    _check(lib().moe_grouped_swiglu_combine(
        _ptr(x_perm, name="x_perm"), _ptr(offsets, torch.int32, "offsets"), _ptr(w1, name="w1"),
        _ptr(w3, name="w3"), _ptr(w2, name="w2"), _ptr(dst_pos, torch.int32, "dst_pos"),
        _ptr(topk_w, torch.float32, "topk_w"), T, top_k, d, h, E, dt, _ptr(out, name="out"),
        _ptr(ws, name="ws"), _nbytes(ws), _stream(stream)), "moe_grouped_swiglu_combine")


def moe_combine(y, dst_pos, row_map, topk_w, T, d, N, top_k, dt, out, stream=None):
    _check(lib().moe_combine(
        _ptr(y, name="y"), _ptr(dst_pos, torch.int32, "dst_pos"),
        _ptr(row_map, torch.int32, "row_map"), _ptr(topk_w, torch.float32, "topk_w"), T, d, N,
        top_k, dt, _ptr(out, name="out"), _stream(stream)), "moe_combine")


def moe_grouped_swiglu_train(x_perm, offsets, w1, w3, w2, N, d, h, E, dt, y, h_act, gu, ws,
                             stream=None):
    _check(lib().moe_grouped_swiglu_train(
        _ptr(x_perm, name="x_perm"), _ptr(offsets, torch.int32, "offsets"), _ptr(w1, name="w1"),
        _ptr(w3, name="w3"), _ptr(w2, name="w2"), N, d, h, E, dt, _ptr(y, name="y"),
        _ptr(h_act, name="h_act"), _ptr(gu, name="gu"), _ptr(ws, name="ws"), _nbytes(ws),
        _stream(stream)), "moe_grouped_swiglu_train")


def moe_grouped_swiglu_backward(x_perm, offsets, w1, w3, w2, h_act, gu, dy, N, d, h, E, dt,
                                dx_perm, dw1, dw3, dw2, ws, stream=None):
    _check(lib().moe_grouped_swiglu_backward(
        _ptr(x_perm, name="x_perm"), _ptr(offsets, torch.int32, "offsets"), _ptr(w1, name="w1"),
        _ptr(w3, name="w3"), _ptr(w2, name="w2"), _ptr(h_act, name="h_act"), _ptr(gu, name="gu"),
        _ptr(dy, name="dy"), N, d, h, E, dt, _ptr(dx_perm, name="dx_perm"),
        _ptr(dw1, name="dw1"), _ptr(dw3, name="dw3"), _ptr(dw2, name="dw2"),
        _ptr(ws, name="ws"), _nbytes(ws), _stream(stream)), "moe_grouped_swiglu_backward")


def moe_combine_backward(dout, y, dst_pos, topk_w, T, d, N, top_k, dt, dy, d_topk_w,
                         stream=None):
    _check(lib().moe_combine_backward(
        _ptr(dout, name="dout"), _ptr(y, name="y"), _ptr(dst_pos, torch.int32, "dst_pos"),
        _ptr(topk_w, torch.float32, "topk_w"), T, d, N, top_k, dt, _ptr(dy, name="dy"),
        _ptr(d_topk_w, torch.float32, "d_topk_w"), _stream(stream)), "moe_combine_backward")


def moe_dispatch_backward(dx_perm, dst_pos, dx_add, T, d, N, top_k, dt, dx, stream=None):
    _check(lib().moe_dispatch_backward(
        _ptr(dx_perm, name="dx_perm"), _ptr(dst_pos, torch.int32, "dst_pos"),
        _ptr(dx_add, name="dx_add"), T, d, N, top_k, dt, _ptr(dx, name="dx"), _stream(stream)),
        "moe_dispatch_backward")


def moe_router_backward(logits, topk_idx, d_topk_w, x, w_router, T, d, E, top_k, opts, dt,
                        d_logits, dw_router, dx, ws, stream=None):
    _check(lib().moe_router_backward(
        _ptr(logits, torch.float32, "logits"), _ptr(topk_idx, torch.int32, "topk_idx"),
        _ptr(d_topk_w, torch.float32, "d_topk_w"), _ptr(x, name="x"),
        _ptr(w_router, name="w_router"), T, d, E, top_k, _opts(opts), dt,
        _ptr(d_logits, torch.float32, "d_logits"), _ptr(dw_router, name="dw_router"),
        _ptr(dx, name="dx"), _ptr(ws, name="ws"), _nbytes(ws), _stream(stream)),
        "moe_router_backward")


def moe_forward_train(x, w_router, logits_in, w1, w3, w2, T, d, E, top_k, h, opts, dt, out,
                      state, stream=None):
    _check(lib().moe_forward_train(
        _ptr(x, name="x"), _ptr(w_router, name="w_router"),
        _ptr(logits_in, torch.float32, "logits_in"), _ptr(w1, name="w1"), _ptr(w3, name="w3"),
        _ptr(w2, name="w2"), T, d, E, top_k, h, _opts(opts), dt, _ptr(out, name="out"),
        _ptr(state, name="state"), _nbytes(state), _stream(stream)), "moe_forward_train")


def moe_backward(dout, x, w_router, w1, w3, w2, T, d, E, top_k, h, opts, dt, state, dx,
                 d_logits, dw_router, dw1, dw3, dw2, ws, stream=None):
    _check(lib().moe_backward(
        _ptr(dout, name="dout"), _ptr(x, name="x"), _ptr(w_router, name="w_router"),
        _ptr(w1, name="w1"), _ptr(w3, name="w3"), _ptr(w2, name="w2"), T, d, E, top_k, h,
        _opts(opts), dt, _ptr(state, name="state"), _ptr(dx, name="dx"),
        _ptr(d_logits, torch.float32, "d_logits"), _ptr(dw_router, name="dw_router"),
        _ptr(dw1, name="dw1"), _ptr(dw3, name="dw3"), _ptr(dw2, name="dw2"),
        _ptr(ws, name="ws"), _nbytes(ws), _stream(stream)), "moe_backward")


def moe_forward_train_ex(x, w_router, logits_in, w1, w3, w2, T, d, E, top_k, h, opts, shared,
                         dt, out, state, stream=None):
    _check(lib().moe_forward_train_ex(
        _ptr(x, name="x"), _ptr(w_router, name="w_router"),
        _ptr(logits_in, torch.float32, "logits_in"), _ptr(w1, name="w1"), _ptr(w3, name="w3"),
        _ptr(w2, name="w2"), T, d, E, top_k, h, _opts(opts),
        None if shared is None else ctypes.byref(shared), dt, _ptr(out, name="out"),
        _ptr(state, name="state"), _nbytes(state), _stream(stream)), "moe_forward_train_ex")


def moe_backward_ex(dout, x, w_router, w1, w3, w2, T, d, E, top_k, h, opts, shared, dt, state,
                    dx, d_logits, dw_router, dw1, dw3, dw2, dws1, dws3, dws2, ws, stream=None):
    _check(lib().moe_backward_ex(
        _ptr(dout, name="dout"), _ptr(x, name="x"), _ptr(w_router, name="w_router"),
        _ptr(w1, name="w1"), _ptr(w3, name="w3"), _ptr(w2, name="w2"), T, d, E, top_k, h,
        _opts(opts), None if shared is None else ctypes.byref(shared), dt,
        _ptr(state, name="state"), _ptr(dx, name="dx"),
        _ptr(d_logits, torch.float32, "d_logits"), _ptr(dw_router, name="dw_router"),
        _ptr(dw1, name="dw1"), _ptr(dw3, name="dw3"), _ptr(dw2, name="dw2"),
        _ptr(dws1, name="dws1"), _ptr(dws3, name="dws3"), _ptr(dws2, name="dws2"),
        _ptr(ws, name="ws"), _nbytes(ws), _stream(stream)), "moe_backward_ex")


def moe_forward(x, w_router, logits_in, w1, w3, w2, T, d, E, top_k, h, score, renormalize,
                ep_ranks, dt, out, logits_out, topk_idx, topk_w, counts, ws, stream=None):
    _check(lib().moe_forward(
        _ptr(x, name="x"), _ptr(w_router, name="w_router"),
        _ptr(logits_in, torch.float32, "logits_in"), _ptr(w1, name="w1"), _ptr(w3, name="w3"),
        _ptr(w2, name="w2"), T, d, E, top_k, h, score, int(renormalize), ep_ranks, dt,
        _ptr(out, name="out"), _ptr(logits_out, torch.float32, "logits_out"),
        _ptr(topk_idx, torch.int32, "topk_idx"), _ptr(topk_w, torch.float32, "topk_w"),
        _ptr(counts, torch.int32, "counts"), _ptr(ws, name="ws"), _nbytes(ws), _stream(stream)),
        "moe_forward")


def shared_expert(w1, w3, w2) -> SharedExpert:
    """A SharedExpert for weights w1, w3 [hs, d] and w2 [d, hs] (CUDA
    tensors that must stay alive while the call that takes it runs)."""
    return SharedExpert(_ptr(w1, name="shared w1"), _ptr(w3, name="shared w3"),
                        _ptr(w2, name="shared w2"), int(w1.shape[0]))


def moe_forward_ex(x, w_router, logits_in, w1, w3, w2, T, d, E, top_k, h, opts, shared,
                   ep_ranks, dt, out, logits_out, topk_idx, topk_w, counts, ws, stream=None):
    _check(lib().moe_forward_ex(
        _ptr(x, name="x"), _ptr(w_router, name="w_router"),
        _ptr(logits_in, torch.float32, "logits_in"), _ptr(w1, name="w1"), _ptr(w3, name="w3"),
        _ptr(w2, name="w2"), T, d, E, top_k, h, _opts(opts),
        None if shared is None else ctypes.byref(shared), ep_ranks, dt,
        _ptr(out, name="out"), _ptr(logits_out, torch.float32, "logits_out"),
        _ptr(topk_idx, torch.int32, "topk_idx"), _ptr(topk_w, torch.float32, "topk_w"),
        _ptr(counts, torch.int32, "counts"), _ptr(ws, name="ws"), _nbytes(ws), _stream(stream)),
        "moe_forward_ex")


def moe_selftest_timeout(ws, stream=None):
    _check(lib().moe_selftest_timeout(_ptr(ws, name="ws"), _nbytes(ws), _stream(stream)),
           "moe_selftest_timeout")


def moe_get_device_status(ws, stream=None) -> int:
    code = _I(0)
    _check(lib().moe_get_device_status(_ptr(ws, name="ws"), ctypes.byref(code), _stream(stream)),
           "moe_get_device_status")
    return code.value


device_status = moe_get_device_status


# --------------------------------------------------- allocating wrappers
def router_topk(x=None, w_router=None, top_k=1, renormalize=True, logits_in=None,
                want_logits=False, E=None, **options):
    """Returns (topk_idx int32 [T,k], topk_w fp32 [T,k], counts int32 [E],
    logits fp32 [T,E] or None, ws).  ``options`` are router_options()
    keywords (score, route_scale, expert_bias, num_groups, topk_groups,
    tokens_per_expert)."""
    src = logits_in if logits_in is not None else x
    dev = src.device
    if logits_in is not None:
        T, E = logits_in.shape
        d = x.shape[1] if x is not None else 8
        dt = _dt(x) if x is not None else MOE_BF16
    else:
        T, d = x.shape
        E = w_router.shape[0]
        dt = _dt(x)
    idx = torch.empty(T, top_k, dtype=torch.int32, device=dev)
    w = torch.empty(T, top_k, dtype=torch.float32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    logits = torch.empty(T, E, dtype=torch.float32, device=dev) if (
        want_logits and logits_in is None) else None
    ws = _ws(router_workspace_size(T, d, E, dt), dev)
    opts = router_options(renormalize=renormalize, **options)
    moe_router_topk_ex(x, w_router, logits_in, T, d, E, top_k, opts, dt, logits, idx, w, counts,
                       ws)
    return idx, w, counts, logits, ws


def dispatch(x, topk_idx, E, materialize=True):
    """Returns (counts [E], offsets [E+1], src_row [N], dst_pos [T,k], x_perm [N,d] or None, ws)."""
    T, k = topk_idx.shape
    d = x.shape[1]
    dev = topk_idx.device
    N = T * k
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    src_row = torch.empty(N, dtype=torch.int32, device=dev)
    dst_pos = torch.empty(T, k, dtype=torch.int32, device=dev)
    x_perm = torch.empty(N, d, dtype=x.dtype, device=dev) if materialize else None
    ws = _ws(dispatch_workspace_size(T, E, k), dev)
    moe_dispatch(x, topk_idx, T, d, E, k, _dt(x), counts, offsets, src_row, dst_pos, x_perm, ws)
    return counts, offsets, src_row, dst_pos, x_perm, ws


def ep_dispatch_rank_major(x, topk_idx, E, R, materialize=True):
    """Returns (counts_rm [R,R,E/R], offsets_rm, src_row, dst_pos, x_rm or None, ws)."""
    T, k = topk_idx.shape
    d = x.shape[1]
    dev = topk_idx.device
    N = T * k
    counts = torch.empty(R, R, E // R, dtype=torch.int32, device=dev)
    offsets = torch.empty(E * R + 1, dtype=torch.int32, device=dev)
    src_row = torch.empty(N, dtype=torch.int32, device=dev)
    dst_pos = torch.empty(T, k, dtype=torch.int32, device=dev)
    x_rm = torch.empty(N, d, dtype=x.dtype, device=dev) if materialize else None
    ws = _ws(ep_dispatch_workspace_size(T, E, k, R), dev)
    moe_ep_dispatch_rank_major(x, topk_idx, T, d, E, k, R, _dt(x), counts, offsets, src_row,
                               dst_pos, x_rm, ws)
    return counts, offsets, src_row, dst_pos, x_rm, ws


def ep_local_regroup(inp, counts_rm):
    """Returns (out [rows,d], counts_em [G*L], offsets_em [G*L+1], perm, perm_inv, ws)."""
    G, R, L = counts_rm.shape
    rows, d = inp.shape
    dev = inp.device
    out = torch.empty_like(inp)
    counts_em = torch.empty(G * L, dtype=torch.int32, device=dev)
    offsets_em = torch.empty(G * L + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(rows, dtype=torch.int32, device=dev)
    perm_inv = torch.empty(rows, dtype=torch.int32, device=dev)
    ws = _ws(regroup_workspace_size(G, R, L), dev)
    moe_ep_local_regroup(inp, counts_rm, G, R, L, rows, d, _dt(inp), out, counts_em, offsets_em,
                         perm, perm_inv, ws)
    return out, counts_em, offsets_em, perm, perm_inv, ws


def grouped_swiglu(x_perm, offsets, w1, w3, w2, row_scale=None):
    """Returns (y [N,d], ws)."""
    N, d = x_perm.shape
    E, h, _ = w1.shape
    y = torch.empty(N, d, dtype=x_perm.dtype, device=x_perm.device)
    ws = _ws(grouped_swiglu_workspace_size(N, d, h, E, _dt(x_perm)), x_perm.device)
    moe_grouped_swiglu(x_perm, offsets, w1, w3, w2, row_scale, N, d, h, E, _dt(x_perm), y, ws)
    return y, ws


def grouped_swiglu_combine(x_perm, offsets, w1, w3, w2, dst_pos, topk_w=None):
    """The grouped SwiGLU with the combine folded into GEMM2.  Returns
    (out [T, d], ws)."""
    T, k = dst_pos.shape
    d = x_perm.shape[1]
    E, h, _ = w1.shape
    dt = _dt(x_perm)
    out = torch.empty(T, d, dtype=x_perm.dtype, device=x_perm.device)
    ws = _ws(lib().moe_grouped_swiglu_combine_workspace_size(T, k, d, h, E, dt), x_perm.device)
    moe_grouped_swiglu_combine(x_perm, offsets, w1, w3, w2, dst_pos, topk_w, T, k, d, h, E, dt,
                               out, ws)
    return out, ws


def grouped_swiglu_gather(x, src_row, offsets, w1, w3, w2, row_scale=None):
    """Grouped SwiGLU reading the rows of x through src_row.  Returns (y, ws)."""
    T, d = x.shape
    N = src_row.numel()
    E, h, _ = w1.shape
    y = torch.empty(N, d, dtype=x.dtype, device=x.device)
    ws = _ws(grouped_swiglu_workspace_size(N, d, h, E, _dt(x)), x.device)
    moe_grouped_swiglu_gather(x, T, src_row, offsets, w1, w3, w2, row_scale, N, d, h, E, _dt(x),
                              y, ws)
    return y, ws


def combine(y, dst_pos, topk_w=None, row_map=None):
    T, k = dst_pos.shape
    N, d = y.shape
    out = torch.empty(T, d, dtype=y.dtype, device=y.device)
    moe_combine(y, dst_pos, row_map, topk_w, T, d, N, k, _dt(y), out)
    return out


def grouped_swiglu_backward_workspace_size(N, d, h, E, dt) -> int:
    return lib().moe_grouped_swiglu_backward_workspace_size(N, d, h, E, dt)


def grouped_swiglu_train(x_perm, offsets, w1, w3, w2):
    """Training forward of the experts.  Returns (y [N, d], h_act [N, h],
    gu [N, 2h], ws)."""
    N, d = x_perm.shape
    E, h, _ = w1.shape
    dev = x_perm.device
    y = torch.empty(N, d, dtype=x_perm.dtype, device=dev)
    h_act = torch.empty(N, h, dtype=x_perm.dtype, device=dev)
    gu = torch.empty(N, 2 * h, dtype=x_perm.dtype, device=dev)
    ws = _ws(256, dev)
    moe_grouped_swiglu_train(x_perm, offsets, w1, w3, w2, N, d, h, E, _dt(x_perm), y, h_act, gu,
                             ws)
    return y, h_act, gu, ws


def grouped_swiglu_backward(x_perm, offsets, w1, w3, w2, h_act, gu, dy):
    """Backward of the experts.  Returns (dx_perm, dw1, dw3, dw2, ws)."""
    N, d = x_perm.shape
    E, h, _ = w1.shape
    dev = x_perm.device
    dx_perm = torch.empty(N, d, dtype=x_perm.dtype, device=dev)
    dw1 = torch.empty_like(w1)
    dw3 = torch.empty_like(w3)
    dw2 = torch.empty_like(w2)
    ws = _ws(grouped_swiglu_backward_workspace_size(N, d, h, E, _dt(x_perm)), dev)
    moe_grouped_swiglu_backward(x_perm, offsets, w1, w3, w2, h_act, gu, dy, N, d, h, E,
                                _dt(x_perm), dx_perm, dw1, dw3, dw2, ws)
    return dx_perm, dw1, dw3, dw2, ws


def combine_backward(dout, y, dst_pos, topk_w=None, want_dw=True):
    """Backward of combine.  Returns (dy [N, d], d_topk_w [T, k] fp32 or None)."""
    T, k = dst_pos.shape
    N, d = y.shape
    dy = torch.empty(N, d, dtype=y.dtype, device=y.device)
    dw = torch.empty(T, k, dtype=torch.float32, device=y.device) if want_dw else None
    moe_combine_backward(dout, y, dst_pos, topk_w, T, d, N, k, _dt(y), dy, dw)
    return dy, dw


def dispatch_backward(dx_perm, dst_pos, dx_add=None):
    """dx [T, d]: every token's sum of its copies' gradients (plus dx_add)."""
    T, k = dst_pos.shape
    N, d = dx_perm.shape
    dx = torch.empty(T, d, dtype=dx_perm.dtype, device=dx_perm.device)
    moe_dispatch_backward(dx_perm, dst_pos, dx_add, T, d, N, k, _dt(dx_perm), dx)
    return dx


def router_backward_workspace_size(T, d, E) -> int:
    return lib().moe_router_backward_workspace_size(T, d, E)


def router_backward(logits, topk_idx, d_topk_w, x=None, w_router=None, want_d_logits=True,
                    **options):
    """Router backward.  Returns (d_logits fp32 [T, E] or None, dw_router
    [E, d] or None, dx [T, d] or None, ws); the gate gradients are computed
    when x / w_router are given.  ``options`` are router_options() keywords
    (score, renormalize, route_scale)."""
    T, E = logits.shape
    k = topk_idx.shape[1]
    dev = logits.device
    d = x.shape[1] if x is not None else (w_router.shape[1] if w_router is not None else 8)
    dt = _dt(x) if x is not None else (_dt(w_router) if w_router is not None else MOE_BF16)
    dl = torch.empty(T, E, dtype=torch.float32, device=dev) if want_d_logits else None
    dwr = torch.empty(E, d, dtype=x.dtype, device=dev) if x is not None else None
    dx = torch.empty(T, d, dtype=w_router.dtype, device=dev) if w_router is not None else None
    ws = _ws(router_backward_workspace_size(T, d, E), dev)
    opts = router_options(**options)
    moe_router_backward(logits, topk_idx, d_topk_w, x, w_router, T, d, E, k, opts, dt, dl, dwr,
                        dx, ws)
    return dl, dwr, dx, ws


def forward_train(x, w_router, w1, w3, w2, top_k, renormalize=True, logits_in=None,
                  shared=None, **options):
    """Training forward of the whole layer.  Returns (out [T, d], state), the
    state to hand to :func:`backward` (it records the sizes and options).
    ``shared`` = (ws1 [hs, d], ws3 [hs, d], ws2 [d, hs]) adds a shared
    expert; ``options`` are router_options() keywords."""
    T, d = x.shape
    E, h, _ = w1.shape
    sh = None if shared is None else shared_expert(*shared)
    hs = 0 if sh is None else sh.h
    st = _ws(lib().moe_train_state_size_ex(T, d, E, top_k, h, hs), x.device)
    out = torch.empty(T, d, dtype=x.dtype, device=x.device)
    opts = router_options(renormalize=renormalize, **options)
    moe_forward_train_ex(x, w_router, logits_in, w1, w3, w2, T, d, E, top_k, h, opts, sh, _dt(x),
                         out, st)
    state = {"state": st, "T": T, "d": d, "E": E, "k": top_k, "h": h, "hs": hs,
             "options": dict(options, renormalize=renormalize)}
    return out, state


def backward(state, dout, x, w_router, w1, w3, w2, router_grads=True, want_d_logits=False,
             shared=None):
    """Backward of the whole layer for dout [T, d].  Returns a dict with dx,
    dw1, dw3, dw2, dw_router (None unless router_grads), d_logits (None
    unless asked), the shared expert's dws1, dws3, dws2 (None without one)
    and ws.  ``shared`` must be the forward's."""
    T, d, E, k, h = (state[n] for n in ("T", "d", "E", "k", "h"))
    dev = dout.device
    sh = None if shared is None else shared_expert(*shared)
    hs = 0 if sh is None else sh.h
    dx = torch.empty(T, d, dtype=dout.dtype, device=dev)
    dw1, dw3, dw2 = torch.empty_like(w1), torch.empty_like(w3), torch.empty_like(w2)
    dwr = torch.empty_like(w_router) if router_grads else None
    dl = torch.empty(T, E, dtype=torch.float32, device=dev) if want_d_logits else None
    ds = [torch.empty_like(t) for t in shared] if shared is not None else [None] * 3
    ws = _ws(lib().moe_backward_workspace_size_ex(T, d, E, k, h, hs), dev)
    opts = router_options(**state["options"])
    moe_backward_ex(dout, x, w_router, w1, w3, w2, T, d, E, k, h, opts, sh, _dt(dout),
                    state["state"], dx, dl, dwr, dw1, dw3, dw2, ds[0], ds[1], ds[2], ws)
    return {"dx": dx, "dw1": dw1, "dw3": dw3, "dw2": dw2, "dw_router": dwr, "d_logits": dl,
            "dws1": ds[0], "dws3": ds[1], "dws2": ds[2], "ws": ws}


def forward(x, w_router, w1, w3, w2, top_k, renormalize=True, ep_ranks=1, logits_in=None,
            want_router=False, ws=None, out=None, shared=None, **options):
    """Whole layer.  Returns ``out`` ([T, d], x's dtype), or with
    ``want_router`` a dict with out, topk_idx, topk_w, counts, logits, ws.
    ``shared`` = (ws1 [hs, d], ws3 [hs, d], ws2 [d, hs]) adds a shared
    expert.  ``options`` are router_options() keywords (score, route_scale,
    expert_bias, num_groups, topk_groups, tokens_per_expert,
    score_before_experts)."""
    T, d = x.shape
    E, h, _ = w1.shape
    dt = _dt(x)
    dev = x.device
    sh = None if shared is None else shared_expert(*shared)
    need = forward_ex_workspace_size(T, d, E, top_k, h, ep_ranks, dt, 0 if sh is None else sh.h)
    if ws is None or _nbytes(ws) < need:
        ws = _ws(need, dev)
    if out is None:
        out = torch.empty(T, d, dtype=x.dtype, device=dev)
    idx = w = counts = logits = None
    if want_router:
        idx = torch.empty(T, top_k, dtype=torch.int32, device=dev)
        w = torch.empty(T, top_k, dtype=torch.float32, device=dev)
        counts = torch.empty(E, dtype=torch.int32, device=dev)
        logits = torch.empty(T, E, dtype=torch.float32, device=dev) if logits_in is None else None
    opts = router_options(renormalize=renormalize, **options)
    moe_forward_ex(x, w_router, logits_in, w1, w3, w2, T, d, E, top_k, h, opts, sh, ep_ranks, dt,
                   out, logits, idx, w, counts, ws)
    if want_router:
        return {"out": out, "topk_idx": idx, "topk_w": w, "counts": counts, "logits": logits,
                "ws": ws}
    return out
