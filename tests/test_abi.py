"""Host-only checks of the C ABI: the library loads, exports every function
include/moe.h declares, and rejects bad arguments before touching the GPU.
No kernel is launched here.

The argument checks pass made-up device addresses: every call must be
rejected on the host.  So that a regressed check cannot turn into a launch
on those addresses, the checks only run in a process that sees no CUDA
device; where this process sees one, the module re-runs itself in a child
process with CUDA_VISIBLE_DEVICES="" (a launch there fails with "no
device" instead of touching memory)."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def _device_visible() -> bool:
    if os.environ.get("CUDA_VISIBLE_DEVICES") == "":
        return False
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="module")
def L():
    if _device_visible():
        pytest.skip("argument checks with made-up addresses run in a child process without a "
                    "CUDA device (test_checks_in_a_process_without_a_device)")
    from routing_dispatch_grouped_topk_b200 import build
    build.build()
    import routing_dispatch_grouped_topk_b200 as m
    return m.lib()


def test_checks_in_a_process_without_a_device():
    if not _device_visible():
        pytest.skip("this process sees no CUDA device: the checks run here directly")
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.abspath(__file__), "-q", "-x",
                        "-p", "no:cacheprovider", "-m", "not gpu"], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ["moe_router_topk", "moe_dispatch", "moe_ep_local_regroup", "moe_grouped_swiglu",
              "moe_combine", "moe_forward"]:
        assert n in names


def test_library_exports_every_declared_symbol(L):
    import routing_dispatch_grouped_topk_b200 as m
    names = declared_functions()
    for n in names:
        assert hasattr(L, n), n
    assert sorted(m.EXPORTED_SYMBOLS) == names
    out = subprocess.run(["nm", "-D", "--defined-only", m.LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = set(re.findall(r"\bT (moe_[a-z0-9_]+)", out))
    assert set(names) <= exported
    # plain C names: nothing C++-mangled with the moe_ prefix leaks out
    assert not re.search(r"\bT _Z\S*moe_", out)


def test_version_and_strings(L):
    assert L.moe_version() == 10000
    assert L.moe_status_string(0) == b"ok"
    assert L.moe_status_string(1) == b"invalid argument"


def test_workspace_sizes_are_host_only(L):
    assert L.moe_dispatch_workspace_size(4096, 128, 8) >= 256
    # x_perm and y [N, d] and H [N, h] in bf16 at least
    N = 4096 * 8
    assert L.moe_forward_workspace_size(4096, 2048, 128, 8, 768, 1, 1) > N * (2 * 2048 + 768) * 2
    assert L.moe_router_workspace_size(64, 4096, 128, 1) >= 256 + 64 * 128 * 4
    assert L.moe_forward_workspace_size(8192, 2880, 128, 4, 2880, 8, 1) > \
        L.moe_forward_workspace_size(8192, 2880, 128, 4, 2880, 1, 1)
    assert L.moe_regroup_workspace_size(8, 8, 16) >= 256
    assert L.moe_grouped_swiglu_workspace_size(100, 64, 128, 4, 1) >= 256 + 100 * 128 * 2


@pytest.mark.parametrize("case", [
    dict(top_k=0), dict(top_k=17), dict(E=0), dict(E=513), dict(T=-1), dict(dt=7), dict(score=2),
    dict(top_k=9, E=8),
])
def test_router_rejects_bad_arguments(L, case):
    a = dict(T=4, d=64, E=8, top_k=2, score=0, dt=1)
    a.update(case)
    p = ctypes.c_void_p(16)
    r = L.moe_router_topk(p, p, None, a["T"], a["d"], a["E"], a["top_k"], a["score"], 1, a["dt"],
                          None, p, p, None, p, 1 << 20, None)
    assert r == 1, L.moe_last_error()
    assert L.moe_last_error() != b""


def test_router_rejects_unaligned_and_null(L):
    p = ctypes.c_void_p(16)
    q = ctypes.c_void_p(18)
    assert L.moe_router_topk(q, p, None, 4, 64, 8, 2, 0, 1, 1, None, p, p, None, p, 1 << 20,
                             None) == 1
    assert L.moe_router_topk(None, p, None, 4, 64, 8, 2, 0, 1, 1, None, p, p, None, p, 1 << 20,
                             None) == 1
    # d not a whole number of 16-byte vectors for bf16
    assert L.moe_router_topk(p, p, None, 4, 60, 8, 2, 0, 1, 1, None, p, p, None, p, 1 << 20,
                             None) == 1


def test_grouped_swiglu_shape_rules(L):
    p = ctypes.c_void_p(256)
    # bf16 tensor-core path needs d, h multiples of 64
    assert L.moe_grouped_swiglu(p, p, p, p, p, None, 10, 96, 128, 4, 1, p, p, 1 << 30, None) == 2
    assert L.moe_grouped_swiglu(p, p, p, p, p, None, 10, 128, 96, 4, 1, p, p, 1 << 30, None) == 2
    # workspace too small
    assert L.moe_grouped_swiglu(p, p, p, p, p, None, 10, 128, 128, 4, 1, p, p, 16, None) == 4


def test_grouped_swiglu_combine_rules(L):
    """The folded combine runs only on the bf16 CTA-pair path (segments
    averaging >= 64 rows); every rule is checked before any launch."""
    p = ctypes.c_void_p(256)
    big = 1 << 30
    ws = L.moe_grouped_swiglu_combine_workspace_size(512, 4, 128, 128, 8, 1)
    assert ws >= 256 + 512 * 4 * 128 * 2 + 512 * 128 * 4
    # fp32 layers, decode-sized segments (N = 16 < 64 E), d not a multiple of 64
    assert L.moe_grouped_swiglu_combine(p, p, p, p, p, p, None, 512, 4, 128, 128, 8, 0, p, p,
                                        big, None) == 2
    assert L.moe_grouped_swiglu_combine(p, p, p, p, p, p, None, 4, 4, 128, 128, 8, 1, p, p, big,
                                        None) == 2
    assert L.moe_grouped_swiglu_combine(p, p, p, p, p, p, None, 512, 4, 96, 128, 8, 1, p, p, big,
                                        None) == 2
    # bad top_k, missing dst_pos, workspace too small
    assert L.moe_grouped_swiglu_combine(p, p, p, p, p, p, None, 512, 0, 128, 128, 8, 1, p, p, big,
                                        None) == 1
    assert L.moe_grouped_swiglu_combine(p, p, p, p, p, None, None, 512, 4, 128, 128, 8, 1, p, p,
                                        big, None) == 1
    assert L.moe_grouped_swiglu_combine(p, p, p, p, p, p, None, 512, 4, 128, 128, 8, 1, p, p, 16,
                                        None) == 4


def test_dispatch_and_regroup_argument_rules(L):
    p = ctypes.c_void_p(256)
    # R must divide E
    assert L.moe_ep_dispatch_rank_major(p, p, 8, 64, 10, 2, 3, 1, p, p, p, p, p, p, 1 << 20,
                                        None) == 1
    # E * R above the bin limit
    assert L.moe_ep_dispatch_rank_major(p, p, 8, 64, 512, 2, 32, 1, p, p, p, p, p, p, 1 << 20,
                                        None) == 1
    assert L.moe_ep_local_regroup(p, p, 0, 2, 2, 10, 64, 1, p, p, p, p, None, p, 1 << 20,
                                  None) == 1
    assert L.moe_dispatch(p, p, 8, 64, 8, 2, 1, p, p, p, p, p, p, 8, None) == 4
    assert L.moe_combine(p, p, None, None, 4, 64, 8, 0, 1, p, None) == 1


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    import routing_dispatch_grouped_topk_b200 as m
    monkeypatch.setattr(m, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(m, "_lib", None)
    with pytest.raises(m.MoEError, match="no CPU fallback"):
        m.lib()


@pytest.mark.parametrize("case", [
    dict(score=2), dict(route_scale=0.0), dict(route_scale=float("nan")),
    dict(route_scale=float("inf")), dict(num_groups=3), dict(num_groups=64, E=128),
    dict(num_groups=4, topk_groups=0), dict(num_groups=4, topk_groups=5),
    dict(num_groups=4, topk_groups=1, top_k=3), dict(num_groups=-1),
])
def test_router_options_are_checked(L, case):
    """Options the router cannot honour (include/moe.h, moe_router_options_t
    rules) are rejected on the host before anything is launched."""
    import routing_dispatch_grouped_topk_b200 as m
    E = case.pop("E", 8)
    top_k = case.pop("top_k", 2)
    o = m.RouterOptions()
    L.moe_router_options_init(ctypes.byref(o))
    for k, v in case.items():
        setattr(o, k, v)
    p = ctypes.c_void_p(16)
    r = L.moe_router_topk_ex(p, p, None, 4, 64, E, top_k, ctypes.byref(o), 1, None, p, p, None, p,
                             1 << 20, None)
    assert r == 1, L.moe_last_error()
    r = L.moe_forward_ex(p, p, None, p, p, p, 4, 64, E, top_k, 64, ctypes.byref(o), None, 1, 1, p, None,
                         None, None, None, p, 1 << 30, None)
    assert r == 1, L.moe_last_error()


def test_router_options_defaults(L):
    import routing_dispatch_grouped_topk_b200 as m
    o = m.RouterOptions()
    o.route_scale = 7.0
    o.num_groups = 3
    o.aux_loss_coef = 2.0
    o.capacity = 5
    o.topk_scores = 64
    L.moe_router_options_init(ctypes.byref(o))
    assert (o.score, o.renormalize, o.route_scale, o.expert_bias, o.num_groups, o.topk_groups,
            o.tokens_per_expert, o.score_before_experts, o.aux_loss, o.aux_loss_coef,
            o.capacity, o.topk_scores) == (0, 0, 1.0, None, 0, 0, None, 0, None, 0.0, 0, None)


def test_capacity_rules(L):
    """A negative capacity is rejected; the layer forward takes the capacity
    policy only in bf16 with ep_ranks = 1, the training forward not at all
    (all before any launch)."""
    import routing_dispatch_grouped_topk_b200 as m
    o = m.RouterOptions()
    L.moe_router_options_init(ctypes.byref(o))
    p = ctypes.c_void_p(256)
    o.capacity = -1
    assert L.moe_router_topk_ex(p, p, None, 4, 64, 8, 2, ctypes.byref(o), 1, None, p, p, None, p,
                                1 << 20, None) == 1
    o.capacity = 3
    assert L.moe_forward_ex(p, p, None, p, p, p, 4, 64, 8, 2, 64, ctypes.byref(o), None, 2, 1, p,
                            None, None, None, None, p, 1 << 30, None) == 2
    assert L.moe_forward_ex(p, p, None, p, p, p, 4, 64, 8, 2, 64, ctypes.byref(o), None, 1, 0, p,
                            None, None, None, None, p, 1 << 30, None) == 2
    assert L.moe_forward_train(p, p, None, p, p, p, 4, 64, 8, 2, 64, ctypes.byref(o), 1, p, p,
                               1 << 30, None) == 2


def test_shared_expert_workspace_and_checks(L):
    """moe_forward_ex_workspace_size with h_shared = 0 is moe_forward's;
    a shared expert adds its [T, hs] hidden and [T, d] output; bad shared
    experts are rejected before any launch."""
    import routing_dispatch_grouped_topk_b200 as m
    base = L.moe_forward_workspace_size(4096, 2048, 128, 8, 768, 1, 1)
    assert L.moe_forward_ex_workspace_size(4096, 2048, 128, 8, 768, 1, 1, 0) == base
    assert L.moe_forward_ex_workspace_size(4096, 2048, 128, 8, 768, 1, 1, 1024) >= \
        base + 4096 * (1024 + 2048) * 2
    p = ctypes.c_void_p(256)
    for sh, code in [(m.SharedExpert(256, 256, 256, 0), 1), (m.SharedExpert(256, 256, 256, 96), 2),
                     (m.SharedExpert(None, 256, 256, 128), 1), (m.SharedExpert(264, 256, 256, 128), 1)]:
        r = L.moe_forward_ex(p, p, None, p, p, p, 4, 64, 8, 2, 64, None, ctypes.byref(sh), 1, 1, p,
                             None, None, None, None, p, 1 << 30, None)
        assert r == code, (sh.h, r, L.moe_last_error())


def test_selftest_timeout_checks_its_workspace(L):
    assert L.moe_selftest_timeout(None, 1 << 10, None) == 1
    assert L.moe_selftest_timeout(ctypes.c_void_p(256), 16, None) == 1


def test_training_entry_points_check_their_arguments(L):
    """Whole-layer training: host-only sizes, and the rules of include/moe.h
    (bf16 only, E % 8 == 0, no score_before_experts) enforced before any
    launch."""
    import routing_dispatch_grouped_topk_b200 as m
    T, d, E, k, h = 4096, 2048, 128, 8, 768
    N = T * k
    assert L.moe_train_state_size(T, d, E, k, h) >= N * (2 * d + 3 * h) * 2 + T * E * 4
    assert L.moe_backward_workspace_size(T, d, E, k, h) >= N * (2 * d + 2 * h) * 2
    p = ctypes.c_void_p(256)
    big = 1 << 40
    # fp32 is not supported
    assert L.moe_forward_train(p, p, None, p, p, p, 4, 64, 8, 2, 64, None, 0, p, p, big,
                               None) == 2
    # E not a multiple of 8
    assert L.moe_forward_train(p, p, None, p, p, p, 4, 64, 12, 2, 64, None, 1, p, p, big,
                               None) == 2
    # a shared expert: h % 64 != 0 is unsupported, its weight gradients are
    # required by the backward, the sizes grow by its state
    assert L.moe_train_state_size_ex(T, d, E, k, h, 0) == L.moe_train_state_size(T, d, E, k, h)
    assert L.moe_train_state_size_ex(T, d, E, k, h, 1024) >= \
        L.moe_train_state_size(T, d, E, k, h) + T * (d + 3 * 1024) * 2
    assert L.moe_backward_workspace_size_ex(T, d, E, k, h, 1024) >= \
        L.moe_backward_workspace_size(T, d, E, k, h) + T * (d + 2 * 1024) * 2
    bad = m.SharedExpert(256, 256, 256, 96)
    assert L.moe_forward_train_ex(p, p, None, p, p, p, 4, 64, 8, 2, 64, None, ctypes.byref(bad), 1,
                                  p, p, big, None) == 2
    sh = m.SharedExpert(256, 256, 256, 64)
    assert L.moe_backward_ex(p, p, p, p, p, p, 4, 64, 8, 2, 64, None, ctypes.byref(sh), 1, p, p,
                             None, p, p, p, p, None, None, None, p, big, None) == 1
    # state / workspace too small
    assert L.moe_forward_train(p, p, None, p, p, p, 4, 64, 8, 2, 64, None, 1, p, p, 16,
                               None) == 4
    assert L.moe_backward(p, p, p, p, p, p, 4, 64, 8, 2, 64, None, 1, p, p, None, p, p, p, p, p,
                          16, None) == 4


def test_router_backward_gate_rules(L):
    """The bf16 gate gradients need E % 8 == 0 and d % 64 == 0 (the tcgen05
    epilogue writes 32-column chunks); the fp32 ones (CUDA cores) and d
    logits alone have no such rule (those run on the GPU tests)."""
    p = ctypes.c_void_p(256)
    big = 1 << 30
    assert L.moe_router_backward(p, p, p, p, p, 4, 96, 8, 2, None, 1, None, p, None, p, big,
                                 None) == 2
    assert L.moe_router_backward(p, p, p, p, p, 4, 64, 12, 2, None, 1, None, p, None, p, big,
                                 None) == 2
    assert L.moe_router_backward(p, p, p, p, p, 4, 96, 12, 2, None, 0, p, None, None, p, 16,
                                 None) == 4


DISPATCH_BAD = [
    dict(dt=7), dict(T=-1), dict(E=0), dict(E=513), dict(top_k=0), dict(top_k=9, E=8),
    dict(top_k=17, E=64), dict(counts=None), dict(offsets=None), dict(idx=None),
    dict(src_row=None), dict(dst_pos=None), dict(x=None), dict(x=18), dict(x_perm=24),
    dict(d=60), dict(d=0),
]


@pytest.mark.parametrize("case", DISPATCH_BAD)
def test_dispatch_entry_points_share_their_argument_rules(L, case):
    """moe_dispatch and moe_dispatch_noalloc reject the same arguments with
    the same status and the same text (one copy of the rules)."""
    a = dict(x=256, idx=256, T=8, d=64, E=8, top_k=2, dt=1, counts=256, offsets=256,
             src_row=256, dst_pos=256, x_perm=512)
    a.update(case)

    def p(v):
        return None if v is None else ctypes.c_void_p(v)
    r1 = L.moe_dispatch(p(a["x"]), p(a["idx"]), a["T"], a["d"], a["E"], a["top_k"], a["dt"],
                        p(a["counts"]), p(a["offsets"]), p(a["src_row"]), p(a["dst_pos"]),
                        p(a["x_perm"]), ctypes.c_void_p(256), 1 << 30, None)
    m1 = L.moe_last_error()
    r2 = L.moe_dispatch_noalloc(p(a["x"]), p(a["idx"]), a["T"], a["d"], a["E"], a["top_k"],
                                a["dt"], p(a["counts"]), p(a["offsets"]), p(a["src_row"]),
                                p(a["dst_pos"]), p(a["x_perm"]), None)
    m2 = L.moe_last_error()
    assert r1 == 1 and r2 == 1, (r1, r2, m1, m2)
    assert m1 == m2


def test_noalloc_rejects_sizes_beyond_its_array(L):
    """Sizes whose scratch exceeds the fixed array are refused on the host
    with MOE_ERR_UNSUPPORTED before anything is launched."""
    T, E, k = 1 << 22, 512, 16
    need = L.moe_dispatch_workspace_size(T, E, k)
    assert need > (4 << 20)
    p = ctypes.c_void_p(256)
    rc = L.moe_dispatch_noalloc(p, p, T, 64, E, k, 1, p, p, p, p, None, None)
    assert rc == 2
    assert b"fixed array" in L.moe_last_error()
