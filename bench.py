"""Benchmark of the MoE layer forward on B200 (one JSON line on rank 0).

A step is one pass of the whole hot path over one batch of synthetic tokens
resident in HBM: router top-k -> dispatch -> (EP regroup) -> grouped SwiGLU
-> combine.  The headline workload is the gpt-oss-120b-shaped layer with
8 simulated EP ranks (T=8192, d=2880, E=128, k=4, h=2880), the largest
single-GPU one and the one that runs the regroup.  Timed region 1 (the
headline ``value``) calls the public moe_forward once per step.  Timed
region 2 runs the same layer as the sequence of entry points
(moe_router_topk, moe_ep_dispatch_rank_major, moe_ep_local_regroup,
moe_grouped_swiglu, moe_combine), each bracketed by CUDA events on the
launching stream, for the per-stage breakdown and the grouped-GEMM duration
of the roofline.  L2 is flushed (256 MB write) between timed steps, outside
the step's events.  ``value`` is tokens/s of the whole job (all ranks; ranks
run independent token batches, weak scaling, no data-path collective).
On one GPU the same run then measures every other workload (moe_forward
and the staged entry points) into ``other_configs``, with the grouped
SwiGLU against HBM and against the burst and sustained bf16 peaks.

``--impl reference`` times the fp64 CPU oracle on the host cores instead
(a bounded token sample per step) and prints the same metric.

``--training`` times the training step instead (its own JSON line): the
forward with the experts' training variant (which keeps G | U) and the
router's logits, then the backward of the combine, of the grouped SwiGLU
(data and weight gradients), of the router (logits, gate weight, its share
of dx) and of the dispatch, each stage bracketed by CUDA events.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "MoE-layer routed tokens/s (bf16); grouped-GEMM TFLOP/s as % of tensor peak"
UNIT = "tokens/s"
FLUSH_BYTES = 256 << 20


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.t:
            self.t.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(n_gpus):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, ws, device="cuda"):
    """Max of a per-rank float over all ranks (the job's device time)."""
    if ws == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_workload(cfg, rank):
    """Workload of one rank: the same experts, an independent token batch."""
    if rank == 0:
        return cfg
    return W.MoEConfig(**{**cfg.__dict__, "seed": cfg.seed + 1000 * rank})


def job_tokens_per_s(T, ws, steps, total_ms_max):
    """Whole-job throughput: every rank processed T tokens per step."""
    return T * ws * steps / (total_ms_max / 1e3)


def stage_algorithmic_bytes(cfg) -> dict:
    """Unique HBM bytes each staged entry point must move (read + write):
    router: x and w_router read, indices and weights written (the fp32
    partial logits stay on chip / in L2 and are not counted); dispatch: x
    read, the routed rows written, the four int32 index arrays; regroup:
    the routed rows read and written; combine: the expert outputs read,
    the output written, indices and weights read."""
    esz = 2 if cfg.dtype == "bf16" else 4
    T, d, E, k, N = cfg.T, cfg.d, cfg.E, cfg.top_k, cfg.N
    out = {"router": esz * (T * d + E * d) + 8 * N,
           "dispatch": esz * (T * d + N * d) + 4 * (2 * N + N + N),
           "combine": esz * (N * d + T * d) + 8 * N}
    if cfg.ep_ranks > 1:
        out["regroup"] = esz * 2 * N * d + 4 * 2 * N
    return out


def swiglu_algorithmic_bytes(cfg) -> int:
    """Unique HBM bytes of one grouped SwiGLU launch: the routed rows read
    (N x d) and the output written (N x d), the hidden activation written and
    read back (2 x N x h), and every expert's three weight matrices once
    (all experts are touched on the multi-token workloads)."""
    esz = 2 if cfg.dtype == "bf16" else 4
    return esz * (2 * cfg.N * cfg.d + 2 * cfg.N * cfg.h + 3 * cfg.E * cfg.h * cfg.d)


# Sources each profiled kernel is compiled from: a recorded DRAM traffic
# figure is used only while these files are byte-identical to the capture.
KERNEL_SOURCES = {
    "grouped_swiglu": ["tc_gemm.cu", "common.cuh"],
}


def source_digest(kernel: str) -> str:
    """Hash of the CUDA sources of `kernel` (KERNEL_SOURCES)."""
    import hashlib
    hsh = hashlib.sha256()
    csrc = os.path.join(ROOT, "routing_dispatch_grouped_topk_b200", "csrc")
    for f in KERNEL_SOURCES[kernel]:
        hsh.update(f.encode())
        hsh.update(open(os.path.join(csrc, f), "rb").read())
    return hsh.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch measured by ncu (profiles/ncu_traffic.json), or
    None when the kernel's sources changed since the capture."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get("traffic", {}).get(workload, {}).get(kernel)
    if not rec or rec.get("source_digest") != source_digest(kernel):
        return None
    return rec.get("dram_bytes_per_launch")


# --------------------------------------------------------------- CPU oracle
def cpu_oracle_step(cfg, lay_cpu, tokens):
    """One oracle pass (router -> dispatch -> experts -> combine) on `tokens`
    rows; returns wall seconds."""
    import oracle as O
    x = lay_cpu["x"][:tokens]
    t0 = time.perf_counter()
    O.moe_forward(x, lay_cpu["w_router"], lay_cpu["w1"], lay_cpu["w3"], lay_cpu["w2"],
                  cfg.top_k, cfg.renormalize, ep_ranks=cfg.ep_ranks)
    return time.perf_counter() - t0


def cpu_layer(cfg, tokens):
    lay = W.make_layer(cfg, "cpu", T=tokens)
    return lay


def cpu_baseline(cfg, tokens=256, reps=1):
    lay = cpu_layer(cfg, tokens)
    cpu_oracle_step(cfg, lay, min(tokens, 16))          # warm-up (BLAS init)
    secs = [cpu_oracle_step(cfg, lay, tokens) for _ in range(reps)]
    s = sum(secs)
    return {"value": tokens * reps / s, "unit": UNIT, "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{tokens} tokens of {cfg.name} per pass, {reps} pass(es), fp64 NumPy "
                      f"(BLAS threads = all host cores), {s:.1f} s"}


def run_reference(args, ws, rank):
    """Reference arm: the fp64 CPU oracle, rank 0 only."""
    if rank != 0:
        return
    cfg = W.config(args.config)
    tokens = args.ref_tokens
    lay = cpu_layer(cfg, tokens)
    for _ in range(args.warmup):
        cpu_oracle_step(cfg, lay, tokens)
    secs = [cpu_oracle_step(cfg, lay, tokens) for _ in range(args.steps)]
    total = sum(secs)
    value = tokens * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": cfg.name, "T": cfg.T, "d": cfg.d, "E": cfg.E, "top_k": cfg.top_k,
                   "h": cfg.h, "sample_tokens_per_step": tokens},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": os.cpu_count(), "kind": "oracle",
                         "sample": f"{tokens} tokens of {cfg.name} per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------- GPU arm
# kernels of libmoe that one moe_forward step launches: router (one fused
# kernel: gate GEMM, top-k, dispatch histogram), dispatch (column scan,
# scatter), regroup on the EP layout (one kernel), grouped SwiGLU (GEMM1,
# GEMM2), combine
def grouped_gemm_launches(cfg) -> int:
    """Launches of the grouped SwiGLU: GEMM1 and GEMM2, one each, plus a
    single-CTA launch over the segments' short last blocks for each GEMM that
    runs on CTA pairs (bf16, segments averaging >= 64 rows) with a reduction
    of >= 2560 (d for GEMM1, h for GEMM2)."""
    if cfg.dtype != "bf16" or cfg.N < 64 * cfg.E:
        return 2
    return 2 + (cfg.d >= 2560) + (cfg.h >= 2560)


def forward_launches(cfg) -> int:
    # router (its kernel also writes the dispatch histogram), dispatch column
    # scan and scatter, [regroup], the grouped SwiGLU, combine
    return 1 + 2 + (1 if cfg.ep_ranks > 1 else 0) + grouped_gemm_launches(cfg) + 1


class Layer:
    """Device buffers of one workload and its two step functions: the public
    moe_forward call, and the same layer as the sequence of entry points
    (moe_router_topk, moe_dispatch / moe_ep_dispatch_rank_major,
    moe_ep_local_regroup, moe_grouped_swiglu, moe_combine)."""

    def __init__(self, M, cfg, dev, rank=0):
        self.M, self.cfg, self.dev = M, cfg, dev
        T, d, E, k, h, R = cfg.T, cfg.d, cfg.E, cfg.top_k, cfg.h, cfg.ep_ranks
        N = T * k
        lay = W.make_layer(cfg, dev)
        if rank:   # independent token batch per rank
            lay["x"] = W.make_layer(rank_workload(cfg, rank), dev, experts=False)["x"]
        self.x, self.wr, self.w1, self.w3, self.w2 = (lay["x"], lay["w_router"], lay["w1"],
                                                      lay["w3"], lay["w2"])
        self.dt = M.MOE_BF16 if cfg.dtype == "bf16" else M.MOE_F32
        x = self.x
        self.idx = torch.empty(T, k, dtype=torch.int32, device=dev)
        self.w = torch.empty(T, k, dtype=torch.float32, device=dev)
        self.rws = torch.empty(M.router_workspace_size(T, d, E, self.dt), dtype=torch.uint8,
                               device=dev)
        nb = E * R
        self.counts = torch.empty(nb, dtype=torch.int32, device=dev)
        self.offsets = torch.empty(nb + 1, dtype=torch.int32, device=dev)
        self.src_row = torch.empty(N, dtype=torch.int32, device=dev)
        self.dst_pos = torch.empty(T, k, dtype=torch.int32, device=dev)
        self.x_perm = torch.empty(N, d, dtype=x.dtype, device=dev)
        self.dws = torch.empty(M.ep_dispatch_workspace_size(T, E, k, R), dtype=torch.uint8,
                               device=dev)
        if R > 1:
            self.x_em = torch.empty_like(self.x_perm)
            self.cem = torch.empty(E, dtype=torch.int32, device=dev)
            self.oem = torch.empty(E + 1, dtype=torch.int32, device=dev)
            self.perm = torch.empty(N, dtype=torch.int32, device=dev)
            self.pinv = torch.empty(N, dtype=torch.int32, device=dev)
            self.gws = torch.empty(M.regroup_workspace_size(R, R, E // R), dtype=torch.uint8,
                                   device=dev)
        self.y = torch.empty(N, d, dtype=x.dtype, device=dev)
        self.sws = torch.empty(M.grouped_swiglu_workspace_size(N, d, h, E, self.dt),
                               dtype=torch.uint8, device=dev)
        self.out = torch.empty(T, d, dtype=x.dtype, device=dev)
        self.fws = torch.empty(M.forward_workspace_size(T, d, E, k, h, R, self.dt),
                               dtype=torch.uint8, device=dev)
        self.fout = torch.empty_like(self.out)
        self.stages = (["router", "dispatch"] + (["regroup"] if R > 1 else [])
                       + ["grouped_swiglu", "combine"])

    def forward(self, x=None, out=None):
        c, M = self.cfg, self.M
        M.moe_forward(self.x if x is None else x, self.wr, None, self.w1, self.w3, self.w2, c.T,
                      c.d, c.E, c.top_k, c.h, M.MOE_SCORE_SOFTMAX, c.renormalize, c.ep_ranks,
                      self.dt, self.fout if out is None else out, None, None, None, None,
                      self.fws)

    def staged(self, stream, ev=None):
        c, M = self.cfg, self.M
        T, d, E, k, h, R, N, dt = c.T, c.d, c.E, c.top_k, c.h, c.ep_ranks, c.N, self.dt

        def mark(i):
            if ev is not None:
                ev[i].record(stream)
        mark(0)
        M.moe_router_topk(self.x, self.wr, None, T, d, E, k, M.MOE_SCORE_SOFTMAX,
                          c.renormalize, dt, None, self.idx, self.w, None, self.rws)
        mark(1)
        if R == 1:
            M.moe_dispatch(self.x, self.idx, T, d, E, k, dt, self.counts, self.offsets,
                           self.src_row, self.dst_pos, self.x_perm, self.dws)
        else:
            M.moe_ep_dispatch_rank_major(self.x, self.idx, T, d, E, k, R, dt, self.counts,
                                         self.offsets, self.src_row, self.dst_pos, self.x_perm,
                                         self.dws)
        mark(2)
        i = 2
        xe, off, rmap = self.x_perm, self.offsets, None
        if R > 1:
            M.moe_ep_local_regroup(self.x_perm, self.counts, R, R, E // R, N, d, dt, self.x_em,
                                   self.cem, self.oem, self.perm, self.pinv, self.gws)
            i += 1
            mark(i)
            xe, off, rmap = self.x_em, self.oem, self.pinv
        M.moe_grouped_swiglu(xe, off, self.w1, self.w3, self.w2, None, N, d, h, E, dt, self.y,
                             self.sws)
        mark(i + 1)
        M.moe_combine(self.y, self.dst_pos, rmap, self.w, T, d, N, k, dt, self.out)
        mark(i + 2)


def timed_next_rows(layer, stream, flush, steps):
    """CUDA-event medians (us; L2 flushed after every call, calls of one kind
    back to back) of the layer's NEXT-row options at its sizes: the router
    entry point with each router option ([HP] TokenChoiceTopKRouter's score
    function, selection-only bias, node-limited groups) and with the capacity
    drop policy ([PF] moe_gate _probs_drop_policy), and the single-device layer
    forward (ep_ranks = 1) with and without the capacity.  The capacity is the
    mean load per expert, so the copies routed past it to busier experts are
    dropped.  None for fp32 layers."""
    c, M = layer.cfg, layer.M
    if layer.dt != M.MOE_BF16:
        return None
    T, d, E, k, h, dt, dev = c.T, c.d, c.E, c.top_k, c.h, layer.dt, layer.dev
    cap = -(-T * k // E)
    bias = torch.linspace(-0.05, 0.05, E, device=dev)
    idx = torch.empty(T, k, dtype=torch.int32, device=dev)
    w = torch.empty(T, k, dtype=torch.float32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    rws = torch.empty(M.router_workspace_size(T, d, E, dt), dtype=torch.uint8, device=dev)
    out1 = torch.empty_like(layer.out)
    fws = torch.empty(M.forward_ex_workspace_size(T, d, E, k, h, 1, dt), dtype=torch.uint8,
                      device=dev)

    def timed(fn):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps + 1)]
        torch.cuda.synchronize()
        for a_ev, b_ev in ev:
            a_ev.record(stream)
            fn()
            b_ev.record(stream)
            flush.zero_()
        torch.cuda.synchronize()
        return 1e3 * statistics.median(a.elapsed_time(b) for a, b in ev[1:])

    router = {}
    variants = {"softmax": {}, "sigmoid": {"score": "sigmoid"}, "expert_bias": {"expert_bias": bias},
                "node_limited_groups": {"num_groups": 8, "topk_groups": 4}, "capacity": {"capacity": cap}}
    for name, o in variants.items():
        if name == "node_limited_groups" and E % 8:
            continue
        opts = M.router_options(renormalize=c.renormalize, **o)
        router[name] = timed(lambda opts=opts: M.moe_router_topk_ex(
            layer.x, layer.wr, None, T, d, E, k, opts, dt, None, idx, w, counts, rws))
    M.moe_router_topk_ex(layer.x, layer.wr, None, T, d, E, k,
                         M.router_options(renormalize=c.renormalize, capacity=cap), dt, None, idx,
                         w, counts, rws)
    torch.cuda.synchronize()
    dropped = int((idx < 0).sum())
    fwd = {}
    for name, o in (("forward_ep1_us", {}), ("forward_ep1_capacity_us", {"capacity": cap})):
        opts = M.router_options(renormalize=c.renormalize, **o)
        fwd[name] = timed(lambda opts=opts: M.moe_forward_ex(
            layer.x, layer.wr, None, layer.w1, layer.w3, layer.w2, T, d, E, k, h, opts, None, 1,
            dt, out1, None, None, None, None, fws))
    return {"router_us": router,
            "capacity": dict(capacity=cap, dropped_copies=dropped, copies=T * k, **fwd),
            "what": "moe_router_topk_ex with each option and moe_forward_ex (ep_ranks 1) with and "
                    "without the capacity at the headline sizes; medians of calls of one kind, "
                    "L2 flushed after each call"}


def timed_folded(layer, stream, flush, steps):
    """CUDA-event times (ms) of moe_grouped_swiglu_combine (the combine folded
    into GEMM2) and of the unfused moe_grouped_swiglu + moe_combine on the
    layer's routed rows, alternating in blocks, L2 flushed between calls;
    None where the folded path does not apply (fp32, decode-sized segments).
    Its dst_pos addresses the expert-major rows the experts read (through
    the regroup's inverse permutation under simulated EP), composed once
    before timing from the last staged step."""
    c, M = layer.cfg, layer.M
    if layer.dt != M.MOE_BF16 or c.N < 64 * c.E:
        return None
    R = c.ep_ranks
    xe, off = (layer.x_em, layer.oem) if R > 1 else (layer.x_perm, layer.offsets)
    rmap = layer.pinv if R > 1 else None
    dst = layer.pinv[layer.dst_pos.long()].int() if R > 1 else layer.dst_pos
    ws = torch.empty(M.lib().moe_grouped_swiglu_combine_workspace_size(c.T, c.top_k, c.d, c.h,
                                                                       c.E, layer.dt),
                     dtype=torch.uint8, device=layer.dev)
    out = torch.empty_like(layer.out)

    def folded():
        M.moe_grouped_swiglu_combine(xe, off, layer.w1, layer.w3, layer.w2, dst, layer.w, c.T,
                                     c.top_k, c.d, c.h, c.E, layer.dt, out, ws)

    def unfused():
        M.moe_grouped_swiglu(xe, off, layer.w1, layer.w3, layer.w2, None, c.N, c.d, c.h, c.E,
                             layer.dt, layer.y, layer.sws)
        M.moe_combine(layer.y, layer.dst_pos, rmap, layer.w, c.T, c.d, c.N, c.top_k, layer.dt,
                      layer.out)

    times = {"folded": [], "unfused": []}
    for blk in range(4):
        order = (("folded", folded), ("unfused", unfused))
        for name, fn in (order if blk % 2 == 0 else order[::-1]):
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(steps + 1)]
            torch.cuda.synchronize()
            for a_ev, b_ev in ev:
                a_ev.record(stream)
                fn()
                b_ev.record(stream)
                flush.zero_()
            torch.cuda.synchronize()
            times[name] += [a.elapsed_time(b) for a, b in ev[1:]]
    # the folded output against the unfused one (rounding differs: y is not
    # rounded to bf16 on the folded path)
    err = (out.float() - layer.out.float()).abs().max().item()
    ref = layer.out.float().abs().max().item()
    return times, err / max(ref, 1e-30)


def timed_forward(layer, stream, flush, steps):
    """CUDA-event time (ms) of each moe_forward step; L2 flushed between
    steps, outside the events."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    torch.cuda.synchronize()
    for a_ev, b_ev in ev:
        a_ev.record(stream)
        layer.forward()
        b_ev.record(stream)
        flush.zero_()
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def timed_staged(layer, stream, flush, steps):
    """Per-stage CUDA-event times (ms lists) of the entry-point sequence and
    the whole staged step; L2 flushed between steps."""
    n = len(layer.stages) + 1
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(n)] for _ in range(steps)]
    torch.cuda.synchronize()
    for s in range(steps):
        layer.staged(stream, events[s])
        flush.zero_()
    torch.cuda.synchronize()
    per_stage = {nm: [ev[i].elapsed_time(ev[i + 1]) for ev in events]
                 for i, nm in enumerate(layer.stages)}
    whole = [ev[0].elapsed_time(ev[-1]) for ev in events]
    return per_stage, whole


def gemm_views(cfg, sw_ms, pk):
    """The grouped SwiGLU against HBM (its algorithmic bytes) and against the
    bf16 tensor peak, burst and sustained."""
    flops = cfg.gemm_flops()
    alg_bytes = swiglu_algorithmic_bytes(cfg)
    tflops = flops / (sw_ms / 1e3) / 1e12
    gbs = alg_bytes / (sw_ms / 1e3) / 1e9
    return {"launch_us": 1e3 * sw_ms, "algorithmic_bytes_per_launch": alg_bytes,
            "algorithmic_flops_per_launch": flops,
            "hbm": {"achieved_GBps": gbs, "frac": gbs / pk["hbm_gbs"]},
            "tensor_burst": {"achieved_TFLOPs": tflops, "frac": tflops / pk["bf16_tflops"]},
            "tensor_sustained": {"achieved_TFLOPs": tflops,
                                 "frac": tflops / pk["bf16_tflops_sustained"]}}


def stage_report(cfg, stage_ms, pk):
    return {n: {"us": 1e3 * stage_ms[n], "algorithmic_bytes": b,
                "GBps": b / (stage_ms[n] * 1e-3) / 1e9,
                "frac": b / (stage_ms[n] * 1e-3) / 1e9 / pk["hbm_gbs"]}
            for n, b in stage_algorithmic_bytes(cfg).items() if n in stage_ms}


def other_config(M, idx, dev, stream, flush, pk, steps=10, warmup=3):
    """One other workload: moe_forward and the staged entry points, timed
    like the headline (L2 flushed between steps)."""
    cfg = W.config(idx)
    layer = Layer(M, cfg, dev)
    for _ in range(warmup):
        layer.forward()
        flush.zero_()
        layer.staged(stream)
        flush.zero_()
    fwd = timed_forward(layer, stream, flush, steps)
    per_stage, _ = timed_staged(layer, stream, flush, steps)
    fwd_ms = statistics.median(fwd)
    stage_ms = {n: statistics.median(v) for n, v in per_stage.items()}
    rec = {"workload": cfg.name, "T": cfg.T, "d": cfg.d, "E": cfg.E, "top_k": cfg.top_k,
           "h": cfg.h, "dtype": cfg.dtype, "moe_forward_us": 1e3 * fwd_ms,
           "tokens_per_s": cfg.T / (fwd_ms / 1e3),
           "forward_matches_staged": bool(torch.equal(layer.fout, layer.out)),
           "grouped_swiglu": gemm_views(cfg, stage_ms["grouped_swiglu"], pk),
           "stages": stage_report(cfg, stage_ms, pk)}
    if cfg.T < 1024:
        # weight-bandwidth view: every touched expert's three matrices once
        touched = int((layer.counts.view(cfg.ep_ranks, -1).sum(0) > 0).sum().item()
                      if cfg.ep_ranks > 1 else (layer.counts > 0).sum().item())
        wbytes = touched * 3 * cfg.d * cfg.h * (2 if cfg.dtype == "bf16" else 4)
        rec["touched_weight_bytes"] = wbytes
        rec["weights_GBps"] = wbytes / (stage_ms["grouped_swiglu"] * 1e-3) / 1e9
        rec["weights_frac_of_hbm"] = rec["weights_GBps"] / pk["hbm_gbs"]
    del layer
    torch.cuda.empty_cache()
    return rec


def profile_stage(args):
    """For ncu captures of one kernel family on a small device footprint:
    run one stage of the layer three times (no timing, no JSON).  router:
    only x and w_router are allocated; grouped_swiglu: the layer is routed
    and dispatched once, then the experts run three times."""
    import dataclasses
    import routing_dispatch_grouped_topk_b200 as M
    M.lib()
    cfg = W.config(args.config)
    if args.profile_experts:
        # the same layer with fewer experts and as many rows per expert (the
        # same kernels, reduction lengths and segment tails on a device
        # footprint small enough for multi-pass captures)
        E2 = args.profile_experts
        cfg = dataclasses.replace(cfg, E=E2, T=cfg.T * E2 // cfg.E, ep_ranks=1,
                                  name=f"{cfg.name}_E{E2}")
    dev = torch.device("cuda", 0)
    T, d, E, k = cfg.T, cfg.d, cfg.E, cfg.top_k
    dt = M.MOE_BF16 if cfg.dtype == "bf16" else M.MOE_F32
    if args.profile_stage == "router":
        lay = W.make_layer(cfg, dev, experts=False)
        idx = torch.empty(T, k, dtype=torch.int32, device=dev)
        w = torch.empty(T, k, dtype=torch.float32, device=dev)
        rws = torch.empty(M.router_workspace_size(T, d, E, dt), dtype=torch.uint8, device=dev)
        for _ in range(3):
            M.moe_router_topk(lay["x"], lay["w_router"], None, T, d, E, k, M.MOE_SCORE_SOFTMAX,
                              cfg.renormalize, dt, None, idx, w, None, rws)
    else:
        lay = W.make_layer(cfg, dev)
        idx, w, _, _, _ = M.router_topk(lay["x"], lay["w_router"], k, cfg.renormalize)
        _, off, _, _, xp, _ = M.dispatch(lay["x"], idx, E)
        for _ in range(3):
            M.grouped_swiglu(xp, off, lay["w1"], lay["w3"], lay["w2"])
    torch.cuda.synchronize()


def run_ours(args, ws, rank, local):
    import routing_dispatch_grouped_topk_b200 as M
    M.lib()  # fails loudly if the CUDA library is missing
    if args.profile and args.profile_stage != "all":
        profile_stage(args)
        return
    cfg = W.config(args.config)
    T, d, E, k, h, R = cfg.T, cfg.d, cfg.E, cfg.top_k, cfg.h, cfg.ep_ranks
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    layer = Layer(M, cfg, dev, rank)
    x, out = layer.x, layer.out
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    if args.profile:
        # Kernel order per staged step: router (fused), dispatch histogram,
        # column scan, scatter, [regroup], GEMM1, GEMM2, combine.
        for _ in range(2):
            layer.staged(stream)
        layer.forward()
        torch.cuda.synchronize()
        return

    # The clock sampler runs from the start of the warm-up (which lasts at
    # least ~1.5 s of back-to-back steps) to the end of the timed regions, so
    # nvidia-smi has samples under load even when a timed region is short.
    sampler = ClockSampler(local)
    if rank == 0:
        sampler.start()
    t_warm = time.perf_counter()
    n_warm = 0
    while n_warm < args.warmup or time.perf_counter() - t_warm < 1.5:
        layer.forward()
        flush.zero_()
        layer.staged(stream)
        flush.zero_()
        n_warm += 1
        if n_warm % 16 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()

    # Timed region 1 (headline): the public moe_forward, one call per step.
    barrier(ws)
    fwd_ms = timed_forward(layer, stream, flush, args.steps)
    barrier(ws)
    total_ms_max = max_over_ranks(sum(fwd_ms), ws)
    ms_per_step = total_ms_max / args.steps
    value = job_tokens_per_s(T, ws, args.steps, total_ms_max)

    # Timed region 2 (breakdown): the same layer as the sequence of entry
    # points, each bracketed by events; gives the grouped-GEMM duration.
    barrier(ws)
    per_stage, staged_whole = timed_staged(layer, stream, flush, args.steps)
    barrier(ws)
    staged_ms_per_step = statistics.mean(staged_whole)
    forward_matches_staged = bool(torch.equal(layer.fout, out))

    # e2e through the public moe_forward with host buffers: every step copies
    # its input from pinned host memory, runs the layer and copies the output
    # back, in sequence on one stream; L2 flushed between steps (outside the
    # events).  This per-call cost is the headline e2e value.
    x_host = x.cpu().pin_memory()
    out_host = torch.empty(T, d, dtype=x.dtype).pin_memory()
    x_dev = torch.empty_like(x)
    out_dev = torch.empty_like(out)

    def e2e_step():
        x_dev.copy_(x_host, non_blocking=True)
        layer.forward(x_dev, out_dev)
        out_host.copy_(out_dev, non_blocking=True)

    for _ in range(args.warmup):
        e2e_step()
        flush.zero_()
    torch.cuda.synchronize()
    e2e_ev = []
    barrier(ws)
    for _ in range(args.steps):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        e2e_step()
        b.record(stream)
        flush.zero_()
        e2e_ev.append((a, b))
    torch.cuda.synchronize()
    barrier(ws)
    e2e_seq_total = max_over_ranks(sum(a.elapsed_time(b) for a, b in e2e_ev), ws)
    e2e_seq_value = job_tokens_per_s(T, ws, args.steps, e2e_seq_total)
    # the e2e output equals the device-resident step's output
    e2e_match = bool(torch.equal(out_host.to(dev), out))

    # Pipelined e2e (a stream of batches): the H2D copy of step i+1 and the
    # D2H copy of step i-1 run on copy streams while step i's forward runs;
    # every step still copies its input in and its output out.  Double
    # buffers on the device, events order the reuse.  No L2 flush between
    # steps here (the copies run concurrently with the forward), so this is
    # a sub-key, not the e2e value.
    xb = [torch.empty_like(x) for _ in range(2)]
    ob = [torch.empty_like(out) for _ in range(2)]
    oh = [torch.empty(T, d, dtype=x.dtype).pin_memory() for _ in range(2)]
    s_in = torch.cuda.Stream(device=dev)
    s_out = torch.cuda.Stream(device=dev)

    def pipelined(nsteps, t_start=None, t_end=None):
        h2d = [torch.cuda.Event() for _ in range(nsteps)]
        fwd = [torch.cuda.Event() for _ in range(nsteps)]
        d2h = [torch.cuda.Event() for _ in range(nsteps)]
        if t_start is not None:
            t_start.record(s_in)
        for i in range(nsteps + 1):
            if i < nsteps:                       # input of step i
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(fwd[i - 2])   # buffer i%2 no longer read
                    xb[i % 2].copy_(x_host, non_blocking=True)
                    h2d[i].record(s_in)
            if i >= 1:                           # forward of step i-1
                j = i - 1
                stream.wait_event(h2d[j])
                if j >= 2:
                    stream.wait_event(d2h[j - 2])     # out buffer j%2 copied out
                layer.forward(xb[j % 2], ob[j % 2])
                fwd[j].record(stream)
                with torch.cuda.stream(s_out):       # output of step j
                    s_out.wait_event(fwd[j])
                    oh[j % 2].copy_(ob[j % 2], non_blocking=True)
                    d2h[j].record(s_out)
        if t_end is not None:
            t_end.record(s_out)

    pipelined(args.warmup)
    torch.cuda.synchronize()
    barrier(ws)
    t0e = torch.cuda.Event(enable_timing=True)
    t1e = torch.cuda.Event(enable_timing=True)
    s_in.wait_stream(stream)
    pipelined(args.steps, t0e, t1e)
    torch.cuda.synchronize()
    barrier(ws)
    e2e_pipe_total = max_over_ranks(t0e.elapsed_time(t1e), ws)
    e2e_pipe_value = job_tokens_per_s(T, ws, args.steps, e2e_pipe_total)
    e2e_match = e2e_match and bool(torch.equal(oh[(args.steps - 1) % 2].to(dev), out))
    # The combine folded into GEMM2 (moe_grouped_swiglu_combine), timed beside
    # the unfused grouped SwiGLU + combine of the staged step.
    folded = timed_folded(layer, stream, flush, min(args.steps, 5))
    clocks = sampler.stop() if rank == 0 else None
    next_rows = timed_next_rows(layer, stream, flush, min(args.steps, 5))

    if rank != 0:
        return
    pk = peaks()
    stage_ms = {n: statistics.mean(v) for n, v in per_stage.items()}
    sw_ms = stage_ms["grouped_swiglu"]
    views = gemm_views(cfg, sw_ms, pk)
    flops, alg_bytes = views["algorithmic_flops_per_launch"], views["algorithmic_bytes_per_launch"]
    # The grouped SwiGLU is timed as one launch pair inside a ~ms step (not
    # a seconds-long loop): the burst peaks apply.  Its binding roofline is
    # the larger lower bound on its time; the other views stand beside it.
    t_mem = alg_bytes / (pk["hbm_gbs"] * 1e9)
    t_flop = flops / (pk["bf16_tflops"] * 1e12)
    traffic = profiled_traffic("grouped_swiglu", cfg.name)
    if t_mem >= t_flop:
        main = {"bound": "hbm", "achieved": views["hbm"]["achieved_GBps"],
                "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": views["hbm"]["frac"],
                "peak_kind": f"HBM copy, {pk['source']}"}
    else:
        main = {"bound": "tensor", "achieved": views["tensor_burst"]["achieved_TFLOPs"],
                "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": views["tensor_burst"]["frac"],
                "peak_kind": f"bf16 dense burst, {pk['source']}"}
    roofline = {"kernel": "moe_grouped_swiglu (GEMM1 w1|w3 + SiLU*up, GEMM2 w2)", **main,
                "traffic": traffic, "launch_ms": sw_ms,
                "algorithmic_bytes_per_launch": alg_bytes,
                "algorithmic_flops_per_launch": flops,
                "views": {"hbm": views["hbm"], "tensor_burst": views["tensor_burst"],
                          "tensor_sustained": views["tensor_sustained"]}}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
        "config": {"workload": cfg.name, "T": T, "d": d, "E": E, "top_k": k, "h": h,
                   "ep_ranks": R, "global_batch": T * ws, "parallelism": f"dp{ws}",
                   "l2": "flushed between steps (256 MB write, outside step events)",
                   "inputs": "seeded synthetic, resident in HBM"},
        "roofline": roofline,
        "grouped_gemm_tflops": views["tensor_burst"]["achieved_TFLOPs"],
        "grouped_gemm_frac_of_tensor_peak": views["tensor_burst"]["frac"],
        "grouped_gemm_frac_of_tensor_peak_sustained": views["tensor_sustained"]["frac"],
        "stage_ms": stage_ms,
        "stage_hbm": stage_report(cfg, stage_ms, pk),
        "staged_ms_per_step": staged_ms_per_step,
        "forward_matches_staged": forward_matches_staged,
        "copies_per_s": value * k,
        "e2e": {"value": e2e_seq_value, "unit": UNIT,
                "h2d_bytes_per_step": x.numel() * x.element_size(),
                "d2h_bytes_per_step": out.numel() * out.element_size(),
                "mode": "sequential: every step copies x from pinned host memory, runs "
                        "moe_forward and copies out back, on one stream; L2 flushed between "
                        "steps",
                "pipelined_value": e2e_pipe_value,
                "pipelined_mode": "step i+1's H2D and step i-1's D2H overlap step i's "
                                  "moe_forward on copy streams (two device buffers); no L2 "
                                  "flush between steps",
                "output_matches_device_step": e2e_match},
        "gpu_launches": args.steps * forward_launches(cfg),
        "gpu_launches_note": "kernels of libmoe in timed region 1 (moe_forward per step)",
        "clocks": clocks,
        "peaks": pk,
    }
    if folded is not None:
        line["folded_combine"] = {
            "us": 1e3 * statistics.median(folded[0]["folded"]),
            "unfused_us": 1e3 * statistics.median(folded[0]["unfused"]),
            "max_diff_vs_unfused_rel": folded[1],
            "what": "moe_grouped_swiglu_combine (fp32 reductions in GEMM2's epilogue, then one "
                    "bf16 rounding) against moe_grouped_swiglu + moe_combine, medians of "
                    "calls alternating in blocks, L2 flushed between calls"}
    if next_rows is not None:
        line["next_rows"] = next_rows
    if ws == 1 and not args.no_other_configs:
        del layer
        torch.cuda.empty_cache()
        line["other_configs"] = [other_config(M, i, dev, stream, flush, pk)
                                 for i in range(len(W.CONFIGS)) if i != args.config]
    if not args.no_cpu_baseline and ws == 1:
        line["cpu_baseline"] = cpu_baseline(cfg, tokens=args.cpu_tokens)
    print(json.dumps(line), flush=True)


TRAIN_STAGES = ["router", "dispatch", "grouped_swiglu_train", "combine", "combine_backward",
                "grouped_swiglu_backward", "router_backward", "dispatch_backward"]
def train_launches(cfg) -> int:
    """Kernels of ours per two-call training step: router 2 (its top-k kernel
    also writes the dispatch histogram), dispatch 2, the training GEMMs (as
    the forward's grouped SwiGLU), combine 1, combine backward 1, backward
    GEMMs 4, router backward 6 (scores, token segments, gate weight-gradient
    partials, their sum, one segment, gate data gradient), dispatch
    backward 1."""
    return 17 + grouped_gemm_launches(cfg)


def run_training(args, ws, rank, local):
    import routing_dispatch_grouped_topk_b200 as M
    M.lib()
    cfg = W.config(args.config)
    if cfg.dtype != "bf16" or cfg.ep_ranks != 1:
        raise SystemExit("--training runs the bf16 single-device layouts (configs 1-3)")
    T, d, E, k, h = cfg.T, cfg.d, cfg.E, cfg.top_k, cfg.h
    N = T * k
    dev = torch.device("cuda", local)
    lay = W.make_layer(cfg, dev)
    if rank:
        lay["x"] = W.make_layer(rank_workload(cfg, rank), dev, experts=False)["x"]
    x, wr, w1, w3, w2 = lay["x"], lay["w_router"], lay["w1"], lay["w3"], lay["w2"]
    dt = M.MOE_BF16
    stream = torch.cuda.current_stream()
    bf = torch.bfloat16
    g = torch.Generator(device=dev).manual_seed(cfg.seed * 7 + rank)
    dout = torch.randn(T, d, generator=g, device=dev).to(bf)
    idx = torch.empty(T, k, dtype=torch.int32, device=dev)
    w = torch.empty(T, k, dtype=torch.float32, device=dev)
    rws = torch.empty(M.router_workspace_size(T, d, E, dt), dtype=torch.uint8, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    src_row = torch.empty(N, dtype=torch.int32, device=dev)
    dst_pos = torch.empty(T, k, dtype=torch.int32, device=dev)
    x_perm = torch.empty(N, d, dtype=bf, device=dev)
    dws = torch.empty(M.dispatch_workspace_size(T, E, k), dtype=torch.uint8, device=dev)
    y = torch.empty(N, d, dtype=bf, device=dev)
    h_act = torch.empty(N, h, dtype=bf, device=dev)
    gu = torch.empty(N, 2 * h, dtype=bf, device=dev)
    tws = torch.empty(256, dtype=torch.uint8, device=dev)
    out = torch.empty(T, d, dtype=bf, device=dev)
    dy = torch.empty(N, d, dtype=bf, device=dev)
    dtw = torch.empty(T, k, dtype=torch.float32, device=dev)
    dxp = torch.empty(N, d, dtype=bf, device=dev)
    dw1, dw3, dw2 = torch.empty_like(w1), torch.empty_like(w3), torch.empty_like(w2)
    bws = torch.empty(M.grouped_swiglu_backward_workspace_size(N, d, h, E, dt),
                      dtype=torch.uint8, device=dev)
    dx = torch.empty(T, d, dtype=bf, device=dev)
    logits = torch.empty(T, E, dtype=torch.float32, device=dev)
    dwr = torch.empty_like(wr)
    dxr = torch.empty(T, d, dtype=bf, device=dev)
    rbws = torch.empty(M.router_backward_workspace_size(T, d, E), dtype=torch.uint8, device=dev)
    ropts = M.router_options(renormalize=cfg.renormalize)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    # the public two-call training step: moe_forward_train + moe_backward
    tstate = torch.empty(M.lib().moe_train_state_size(T, d, E, k, h), dtype=torch.uint8,
                         device=dev)
    tws = torch.empty(M.lib().moe_backward_workspace_size(T, d, E, k, h), dtype=torch.uint8,
                      device=dev)
    tout = torch.empty(T, d, dtype=bf, device=dev)
    tdx = torch.empty(T, d, dtype=bf, device=dev)
    tdw1, tdw3, tdw2 = torch.empty_like(w1), torch.empty_like(w3), torch.empty_like(w2)
    tdwr = torch.empty_like(wr)

    def train_step():
        M.moe_forward_train(x, wr, None, w1, w3, w2, T, d, E, k, h, ropts, dt, tout, tstate)
        M.moe_backward(dout, x, wr, w1, w3, w2, T, d, E, k, h, ropts, dt, tstate, tdx, None,
                       tdwr, tdw1, tdw3, tdw2, tws)

    def step(ev=None):
        def mark(i):
            if ev is not None:
                ev[i].record(stream)
        mark(0)
        M.moe_router_topk(x, wr, None, T, d, E, k, M.MOE_SCORE_SOFTMAX, cfg.renormalize, dt,
                          logits, idx, w, None, rws)
        mark(1)
        M.moe_dispatch(x, idx, T, d, E, k, dt, counts, offsets, src_row, dst_pos, x_perm, dws)
        mark(2)
        M.moe_grouped_swiglu_train(x_perm, offsets, w1, w3, w2, N, d, h, E, dt, y, h_act, gu, tws)
        mark(3)
        M.moe_combine(y, dst_pos, None, w, T, d, N, k, dt, out)
        mark(4)
        M.moe_combine_backward(dout, y, dst_pos, w, T, d, N, k, dt, dy, dtw)
        mark(5)
        M.moe_grouped_swiglu_backward(x_perm, offsets, w1, w3, w2, h_act, gu, dy, N, d, h, E, dt,
                                      dxp, dw1, dw3, dw2, bws)
        mark(6)
        M.moe_router_backward(logits, idx, dtw, x, wr, T, d, E, k, ropts, dt, None, dwr, dxr, rbws)
        mark(7)
        M.moe_dispatch_backward(dxp, dst_pos, dxr, T, d, N, k, dt, dx)
        mark(8)

    if args.profile:
        for _ in range(2):
            step()
        torch.cuda.synchronize()
        return
    sampler = ClockSampler(local)
    if rank == 0:
        sampler.start()
    t_warm = time.perf_counter()
    n_warm = 0
    while n_warm < args.warmup or time.perf_counter() - t_warm < 1.5:
        train_step()
        flush.zero_()
        step()
        flush.zero_()
        n_warm += 1
        if n_warm % 8 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    # Timed region 1 (the value): the two public calls per step.
    tev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    barrier(ws)
    torch.cuda.synchronize()
    for a_ev, b_ev in tev:
        a_ev.record(stream)
        train_step()
        b_ev.record(stream)
        flush.zero_()
    torch.cuda.synchronize()
    barrier(ws)
    two_call_ms = sum(a.elapsed_time(b) for a, b in tev)
    two_call_ms_max = max_over_ranks(two_call_ms, ws)
    # Timed region 2 (breakdown): the per-step entry points, each bracketed.
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(len(TRAIN_STAGES) + 1)]
              for _ in range(args.steps)]
    barrier(ws)
    torch.cuda.synchronize()
    for s_ in range(args.steps):
        step(events[s_])
        flush.zero_()          # L2 flush between steps, outside the step's events
    torch.cuda.synchronize()
    barrier(ws)
    clocks = sampler.stop() if rank == 0 else None
    total_ms = sum(ev[0].elapsed_time(ev[-1]) for ev in events)
    total_ms_max = max_over_ranks(total_ms, ws)
    status = int(bws[:4].view(torch.int32)[0].item()) | int(tws[:4].view(torch.int32)[0].item())
    matches = bool(torch.equal(tdx, dx) and torch.equal(tdw1, dw1) and torch.equal(tdwr, dwr))
    if rank != 0:
        return
    pk = peaks()
    stage_ms = {n: statistics.mean(ev[i].elapsed_time(ev[i + 1]) for ev in events)
                for i, n in enumerate(TRAIN_STAGES)}
    bwd_flops = 2 * cfg.gemm_flops()   # dgrad 2Ndh + 4Ndh, wgrad 2Ndh + 4Ndh
    fwd_flops = cfg.gemm_flops()
    bwd_ms = stage_ms["grouped_swiglu_backward"]
    tflops = bwd_flops / (bwd_ms / 1e3) / 1e12
    line = {
        "metric": "MoE-layer training step (forward + backward) routed tokens/s (bf16)",
        "value": job_tokens_per_s(T, ws, args.steps, two_call_ms_max), "unit": UNIT,
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": two_call_ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": cfg.name, "T": T, "d": d, "E": E, "top_k": k, "h": h,
                   "global_batch": T * ws, "parallelism": f"dp{ws}",
                   "l2": "flushed between steps (256 MB write, outside step events)",
                   "inputs": "seeded synthetic, resident in HBM; dout ~ N(0,1)"},
        "roofline": {"kernel": "moe_grouped_swiglu_backward (4 tcgen05 GEMMs: dgrad w2 + "
                               "SwiGLU', dgrad w1|w3, wgrad w2, wgrad w1|w3)",
                     "bound": "tensor", "achieved": tflops,
                     "peak": pk["bf16_tflops_sustained"], "unit": "TFLOP/s",
                     "frac": tflops / pk["bf16_tflops_sustained"], "traffic": None,
                     "launch_ms": bwd_ms, "algorithmic_flops_per_launch": bwd_flops,
                     "peak_kind": f"bf16 sustained, {pk['source']}"},
        "forward_experts_tflops": fwd_flops / (stage_ms["grouped_swiglu_train"] / 1e3) / 1e12,
        "stage_ms": stage_ms,
        "staged_ms_per_step": total_ms_max / args.steps,
        "two_call_matches_staged": matches,
        "device_status": status,
        "gpu_launches": args.steps * train_launches(cfg),
        "gpu_launches_note": "kernels of libmoe per moe_forward_train + moe_backward step: "
                             "router 2, dispatch 2, experts forward "
                             f"{grouped_gemm_launches(cfg)}, combine 1, combine backward 1, "
                             "experts backward 4, router backward 6, dispatch backward 1",
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=4, help="headline workload index (default: "
                    "the gpt-oss-120b-shaped EP8 layer, T=8192, the largest single-GPU one)")
    ap.add_argument("--cpu-tokens", type=int, default=64,
                    help="tokens of the fp64 oracle's CPU-baseline sample")
    ap.add_argument("--ref-tokens", type=int, default=8,
                    help="tokens of the oracle per step of the reference arm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="skip the per-workload measurements of the other configs")
    ap.add_argument("--training", action="store_true",
                    help="time the training step (forward + backward) instead")
    ap.add_argument("--profile", action="store_true",
                    help="for ncu captures: run the staged step twice, then moe_forward "
                         "once, and exit (no timing, no JSON)")
    ap.add_argument("--profile-stage", default="all", choices=["all", "router", "grouped_swiglu"],
                    help="with --profile: run only this stage three times (small device "
                         "footprint for multi-pass captures)")
    ap.add_argument("--profile-experts", type=int, default=0,
                    help="with --profile-stage: the workload with this many experts and the "
                         "token count scaled to keep the rows per expert")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        ws = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, ws, rank)
        return
    ws, rank, local = dist_setup(args.gpus)
    try:
        if args.training:
            run_training(args, ws, rank, local)
        else:
            run_ours(args, ws, rank, local)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
