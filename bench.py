#!/usr/bin/env python
"""Routed-MoE SwiGLU layer forward benchmark (B200, sm_100a).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload: the mid MoE layer (T=4096 tokens, hidden 2048, 64 experts,
top_k=6, expert intermediate 1408, shared intermediate 2816, swiglu_limit 7,
routed_scaling_factor 2.5, renormalised top-k), seeded synthetic inputs with
random-init weights.  One step = one full layer forward (router -> permute ->
grouped gate/up+SwiGLU -> grouped down -> combine) over T tokens.

For N > 1 (torchrun, one process per GPU) every rank runs its own replica on
its own tokens (weak scaling; the forward has no collective).  Timing: W
untimed warm-up steps, then K steps between a barrier + synchronize, CUDA
events on the launching stream, max over ranks.  Rank 0 prints one JSON line.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import threading
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "routed-MoE layer tokens/s; grouped-GEMM TFLOP/s as % of B200 bf16 dense peak"
CONFIG_NAME = "mid"


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--stage-iters", type=int, default=50)
    ap.add_argument("--workload", default=CONFIG_NAME,
                    help="layer to time (default: the mid layer the metric is quoted on)")
    ap.add_argument("--graph", action="store_true", help="replay the forward from a captured CUDA graph")
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the W4A16 decode-layer measurement added beside the mid layer's line")
    ap.add_argument("--mode", default="replicas", choices=["replicas", "ep"],
                    help="replicas: every rank runs the whole layer on its own tokens (weak scaling); "
                         "ep: expert parallelism, every rank holds E/N experts and 1/N of the shared expert for "
                         "the same tokens, one all-reduce per step (strong scaling)")
    return ap.parse_args(argv)


# ------------------------------------------------------------ utilities ----

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi samples (50 ms) of SM clock and throttle reasons."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_id: str):
        self.proc = None
        self.lines = []
        self.reader = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        if self.proc is not None:
            # drain the pipe as it fills: a full pipe would stall the sampler
            # (and lose every later sample) about half a minute into a long run
            self.reader = threading.Thread(target=self._drain, daemon=True)
            self.reader.start()
        self.windows = []

    def _drain(self):
        try:
            for line in self.proc.stdout:
                self.lines.append(line)
        except (OSError, ValueError):
            pass

    def mark(self, t0, t1):
        self.windows.append((t0, t1))

    def finish(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                pass  # leave it; the samples read so far are enough
        self.reader.join(timeout=5)
        mhz, max_mhz, reasons = [], None, set()
        for line in list(self.lines):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 7:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                sm, smax = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            if not any(a - 0.06 <= ts <= b + 0.06 for a, b in self.windows):
                continue
            mhz.append(sm)
            max_mhz = smax
            for name, v in zip(self.REASONS, parts[3:]):
                if v.lower() == "active":
                    reasons.add(name)
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": max_mhz, "reasons": sorted(reasons), "samples": 0}
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": max_mhz, "reasons": sorted(reasons),
                "samples": len(mhz)}


def gpu_uuid(dev):
    import torch
    try:
        u = torch.cuda.get_device_properties(dev).uuid
        return "GPU-" + str(u)
    except Exception:
        return str(dev)


def traffic_from_profile(kernel_key: str):
    """DRAM bytes per call of the timed FFN kernels, from the committed ncu
    summary, only while the kernel source still matches the profiled one."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    ent = d.get(kernel_key)
    if not ent:
        return None
    src = os.path.join(ROOT, ent["source"])
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] if os.path.exists(src) else None
    if h != ent.get("source_sha256_16"):
        return None
    return ent["dram_bytes_per_call"]


# ------------------------------------------------------------ workloads ----

def make_inputs(name=CONFIG_NAME):
    import moe_inputs
    from moe_inputs.configs import CONFIGS
    cfg = CONFIGS[name]
    # the multi-GB layers draw their weights on the GPU (same draws as the tests)
    wdev = "cpu" if name in ("tiny", "mid") else "cuda"
    return cfg, moe_inputs.make_layer(cfg, seed=0, weight_device=wdev)


def gemm_flops(cfg):
    R = cfg.T * cfg.k
    routed = 6.0 * R * cfg.H * cfg.I
    shared = 6.0 * cfg.T * cfg.H * cfg.I_s
    return routed, shared


def run_cpu_baseline(inp, min_seconds=10.0, max_passes=20, gpu_out=None, gpu_ids=None):
    """The oracle as it stands, on the host cores: whole-layer passes until
    about `min_seconds` of CPU work (at least one, at most `max_passes`).
    The last pass also checks the timed GPU run's result: expert ids against
    the oracle's (near-ties, where the k-th and (k+1)-th biased scores are
    within 1e-6, counted apart) and the layer output within the bf16
    tolerance max|gpu - oracle| <= 2e-2 max|oracle|."""
    import torch
    import oracle
    cores = torch.get_num_threads()
    t0 = time.perf_counter()
    passes = 0
    res = None
    while passes < max_passes:
        res = oracle.moe_forward(inp)
        passes += 1
        if time.perf_counter() - t0 >= min_seconds:
            break
    dt = time.perf_counter() - t0
    line = {"value": passes * inp.cfg.T / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{passes} passes of the full {inp.cfg.name} layer ({inp.cfg.T} tokens each), fp64 torch "
                      f"CPU, {dt:.1f} s"}
    if gpu_out is not None and gpu_ids is not None:
        sel = res.selection
        tie = sel.gap < 1e-6
        mism = (gpu_ids.to(torch.int64) != sel.ids).any(dim=1)
        ok = not bool((mism & ~tie).any())
        if ok:  # near-tie tokens are re-evaluated with the GPU's (equally valid) selection
            ref = oracle.moe_forward(inp, ids_override=gpu_ids).out if bool(mism.any()) else res.out
            err = float((gpu_out.double() - ref).abs().max() / ref.abs().max())
        else:
            err = None
        line["parity"] = {"near_ties": int(tie.sum()), "near_ties_chosen_differently": int((mism & tie).sum()),
                          "ids_mismatched_outside_near_ties": int((mism & ~tie).sum()),
                          "out_max_rel_err": err, "tolerance": 2e-2,
                          "checked": "every token of the timed run's output"}
    return line


def w4a16_bytes(cfg, ids):
    """HBM bytes the 4-bit expert FFN call must move: codes + scales of every
    touched expert (W4A16: bf16 per 128; NVFP4: one byte per 16 and two fp32
    tensor scales), the bf16 shared expert, and its activations (the T*k
    gathered token rows and x read, y_perm and the shared output written)."""
    touched = int(len(set(ids.reshape(-1).tolist())))
    codes = 2 * cfg.I * cfg.H // 2 + cfg.H * cfg.I // 2
    if cfg.nvfp4:
        per_expert = codes + (2 * cfg.I * cfg.H // 16 + cfg.H * cfg.I // 16) + 2 * 4
    else:
        per_expert = codes + 2 * (2 * cfg.I * cfg.H // 128 + cfg.H * cfg.I // 128)
    shared = 2 * (2 * cfg.I_s * cfg.H + cfg.H * cfg.I_s)
    acts = 2 * cfg.T * cfg.H * (2 + 2 * cfg.k)
    return touched, touched * per_expert + shared + acts


def launches_per_step(cfg):
    """Kernels one forward launches: router 3 (weight split, tensor-core
    logits, top-k), permute 2 (count/rank with the scan in its last block,
    then the scatter into x_perm, or for 4-bit experts the maps alone, their
    activation conversion gathering the rows), combine 1, plus the expert
    FFN path and the shared expert's launches when it does not ride in the
    routed ones."""
    n = 6
    four = cfg.w4a16 or cfg.nvfp4
    prefill = four and cfg.T * cfg.k >= 32 * cfg.E       # 4-bit codes dequantised in shared memory, tensor cores
    gemv = four and not prefill                           # 4-bit codes dequantised in registers
    shared = 0
    if cfg.I_s > 0:
        if gemv and cfg.T <= 32:
            shared = 0      # in the two GEMV launches
        elif cfg.T <= 32:
            shared = 4      # split-K GEMMs + ordered slice sums
        elif cfg.w4a16 or cfg.nvfp4:
            shared = 2      # its own tcgen05 gate/up and down launches
        else:
            shared = 0      # one more problem of the routed tcgen05 launches
    if prefill:
        return n + 3 + shared  # token prep + dequantising gate/up and down
    if gemv:
        return n + 4 + shared  # (activation prep + GEMV) x 2
    return n + 2 + shared      # gate/up + down


def base_line(args, n_gpus, cfg):
    bytes_per_weight = 0.5 + 1 / 16 if cfg.nvfp4 else 0.5 + 2 / 128 if cfg.w4a16 else 2
    l2 = ("inputs larger than L2 (expert weights streamed per step: %.2f GB)"
          % ((cfg.E * 3 * cfg.H * cfg.I * bytes_per_weight + 6 * cfg.H * cfg.I_s) / 1e9))
    return {
        "metric": METRIC, "unit": "tokens/s", "n_gpus": n_gpus, "steps": args.steps, "warmup": args.warmup,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "data": "synthetic",
        "config": {"workload": f"{cfg.name} MoE layer: T={cfg.T} tokens/GPU, hidden={cfg.H}, E={cfg.E}, "
                               f"top_k={cfg.k}, I={cfg.I}, I_s={cfg.I_s}, swiglu_limit={cfg.swiglu_limit}, "
                               f"alpha={cfg.alpha}, renorm={cfg.renorm}",
                   "tokens_per_gpu_step": cfg.T, "global_tokens_per_step": cfg.T * n_gpus,
                   "parallelism": f"replicas x{n_gpus} (no collective in the forward)",
                   "l2": l2},
    }


# ------------------------------------------------------- replicas (N > 1) ----

def rank_barrier(world):
    """Barrier over the job's ranks (no-op for one rank)."""
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def rank_max(v, world, device):
    """Max of a per-rank float over the job's ranks: every timed figure is
    the slowest rank's."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_tokens_per_s(world, tokens_per_rank, ms_per_step):
    """Whole-job throughput of N replicas: every rank processes its own
    tokens each step; the step time is the max over ranks."""
    return world * tokens_per_rank / (ms_per_step / 1e3)


# ------------------------------------------------- W4A16 decode layer ----

DECODE_NAME = "decode_w4a16"


def measure_decode(dev, iters, clocks, max_over_ranks):
    """The W4A16 decode layer (T=32, H=6144, E=256, k=8, int4 g128 experts)
    beside the mid layer's line: its expert FFN call (the HBM-bound part:
    codes and scales of every touched expert, the bf16 shared expert) and
    its whole forward, each timed with CUDA events over `iters` calls after
    warm-up, a burst of at most 50 (the HBM peak it is compared with is a
    copy timed on its own; the call is bound by its instruction stream, so
    a longer loop measures how far the power cap pulls the clock down).  The
    touched experts' codes alone (about 2.9 GB) exceed L2, so every call
    streams them from HBM."""
    import torch
    import routed_swiglu_experts_b200 as rse
    cfg, inp = make_inputs(DECODE_NAME)
    c = cfg

    def mv(t):
        return None if t is None else t.to(dev)
    layer = rse.MoELayer(hidden=c.H, num_experts=c.E, top_k=c.k, expert_inter=c.I, shared_inter=c.I_s,
                         swiglu_limit=c.swiglu_limit, routed_scaling_factor=c.alpha, renormalize=c.renorm,
                         router_w=mv(inp.router_w), correction_bias=mv(inp.correction_bias),
                         w_gate_up=mv(inp.w_gate_up), w_down=mv(inp.w_down), s_gate_up=mv(inp.s_gate_up),
                         s_down=mv(inp.s_down), shared_w_gate_up=mv(inp.shared_w_gate_up),
                         shared_w_down=mv(inp.shared_w_down), g_gate_up=mv(inp.g_gate_up),
                         g_down=mv(inp.g_down), max_tokens=c.T)
    x = inp.x.to(dev)
    T, k, E, H = c.T, c.k, c.E, c.H
    R = T * k
    stream = torch.cuda.current_stream()
    ids = torch.empty(T, k, dtype=torch.int32, device=dev)
    tw = torch.empty(T, k, dtype=torch.float32, device=dev)
    offs = torch.empty(E + 1, dtype=torch.int32, device=dev)
    row_of = torch.empty(R, dtype=torch.int32, device=dev)
    src = torch.empty(R, dtype=torch.int32, device=dev)
    w_perm = torch.empty(R, dtype=torch.float32, device=dev)
    y_perm = torch.empty(R, H, dtype=torch.bfloat16, device=dev)
    sh = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    rse.moe_router_topk(layer.cfg, layer.w, x, T, ids, tw, layer.ws)
    rse.moe_permute(layer.cfg, ids, tw, None, T, offs, row_of, src, w_perm, None, layer.ws)

    def ffn():  # the FFN call moe_forward makes: the permute's gather fused into its loads
        rse.moe_grouped_swiglu_ffn_gather(layer.cfg, layer.w, x, T, src, offs, w_perm, y_perm, sh, layer.ws)

    def fwd():
        layer.forward(x, out=out)

    res = {}
    for name, fn in (("ffn", ffn), ("forward", fwd)):
        for _ in range(5):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        w0 = time.time()
        e0.record(stream)
        for _ in range(iters):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        clocks.mark(w0, time.time())
        res[name] = max_over_ranks(e0.elapsed_time(e1)) / iters
    assert layer.device_error() == 0
    touched, nbytes = w4a16_bytes(c, ids.cpu())
    peaks = measured_peaks()
    gbs = nbytes / (res["ffn"] / 1e3) / 1e9
    return {
        "workload": f"{c.name} MoE layer: T={c.T}, hidden={c.H}, E={c.E}, top_k={c.k}, I={c.I}, I_s={c.I_s}, "
                    f"int4 group-128 experts (bf16 scales), bf16 shared expert",
        "forward_ms": res["forward"], "tokens_per_s": c.T / (res["forward"] / 1e3),
        "ffn_ms": res["ffn"], "ffn_bytes": nbytes, "touched_experts": touched,
        "ffn_gbs": gbs, "hbm_peak_gbs": peaks["hbm_gbs"], "ffn_frac_of_hbm": gbs / peaks["hbm_gbs"],
        "peak_source": f"{peaks['source']} HBM copy", "iters": iters,
        "note": "HBM-bound W4A16 expert FFN call (the decode layer's roofline); "
                "L2 not flushed: its 2.9 GB of touched codes exceed L2",
    }


# --------------------------------------------------------------- our arm ----

def bench_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import routed_swiglu_experts_b200 as rse

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    rse.load_library()
    cfg, inp = make_inputs(args.workload)
    c = cfg

    def mv(t):
        return None if t is None else t.to(dev)
    layer = rse.MoELayer(hidden=c.H, num_experts=c.E, top_k=c.k, expert_inter=c.I, shared_inter=c.I_s,
                         swiglu_limit=c.swiglu_limit, routed_scaling_factor=c.alpha, renormalize=c.renorm,
                         router_w=mv(inp.router_w), correction_bias=mv(inp.correction_bias),
                         w_gate_up=mv(inp.w_gate_up), w_down=mv(inp.w_down), s_gate_up=mv(inp.s_gate_up),
                         s_down=mv(inp.s_down), shared_w_gate_up=mv(inp.shared_w_gate_up),
                         shared_w_down=mv(inp.shared_w_down), g_gate_up=mv(inp.g_gate_up),
                         g_down=mv(inp.g_down), max_tokens=c.T)
    x = inp.x.to(dev)
    out = torch.empty(c.T, c.H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    clocks = ClockSampler(gpu_uuid(dev))

    def barrier():
        rank_barrier(world)

    def max_over_ranks(v):
        return rank_max(v, world, dev)

    for _ in range(args.warmup):
        layer.forward(x, out=out)
    torch.cuda.synchronize()
    step = lambda: layer.forward(x, out=out)  # noqa: E731
    graph = None
    if args.graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            layer.forward(x, out=out)
        graph.replay()
        torch.cuda.synchronize()
        step = graph.replay

    # --- device-resident timing of K whole-layer steps
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0 = time.time()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    w1 = time.time()
    barrier()
    clocks.mark(w0, w1)
    ms = max_over_ranks(e0.elapsed_time(e1))
    ms_per_step = ms / args.steps

    # --- per-stage durations (the kernels the forward launches, one C-ABI call
    # per stage, events between).  As in moe_forward: bf16 experts permute
    # into x_perm; 4-bit experts write the maps only and gather in the FFN.
    T, k, E, H = c.T, c.k, c.E, c.H
    R = T * k
    ids = torch.empty(T, k, dtype=torch.int32, device=dev)
    tw = torch.empty(T, k, dtype=torch.float32, device=dev)
    offs = torch.empty(E + 1, dtype=torch.int32, device=dev)
    row_of = torch.empty(R, dtype=torch.int32, device=dev)
    src = torch.empty(R, dtype=torch.int32, device=dev)
    w_perm = torch.empty(R, dtype=torch.float32, device=dev)
    x_perm = None if (c.w4a16 or c.nvfp4) else torch.empty(R, H, dtype=torch.bfloat16, device=dev)

    def permute():
        rse.moe_permute(layer.cfg, ids, tw, x, T, offs, row_of, src, w_perm, x_perm, layer.ws)

    def ffn():
        if x_perm is None:
            rse.moe_grouped_swiglu_ffn_gather(layer.cfg, layer.w, x, T, src, offs, w_perm, y_perm, sh, layer.ws)
        else:
            rse.moe_grouped_swiglu_ffn(layer.cfg, layer.w, x_perm, offs, w_perm, T, y_perm, x, sh, layer.ws)
    y_perm = torch.empty(R, H, dtype=torch.bfloat16, device=dev)
    sh = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    n_it = max(3, min(args.stage_iters, args.steps))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(n_it)]
    w0 = time.time()
    for it in range(n_it + 3):
        ev = evs[it - 3] if it >= 3 else None
        if ev:
            ev[0].record(stream)
        rse.moe_router_topk(layer.cfg, layer.w, x, T, ids, tw, layer.ws)
        if ev:
            ev[1].record(stream)
        permute()
        if ev:
            ev[2].record(stream)
        ffn()
        if ev:
            ev[3].record(stream)
        rse.moe_combine(layer.cfg, y_perm, row_of, None, sh, T, out)
        if ev:
            ev[4].record(stream)
    torch.cuda.synchronize()
    clocks.mark(w0, time.time())
    stage_ms = {name: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs)
                for i, name in enumerate(["router", "permute", "grouped_ffn", "combine"])}
    stage_ms = {kname: max_over_ranks(v) for kname, v in stage_ms.items()}

    # --- end to end through the public API with host buffers, pipelined as a
    # serving loop runs it: every step copies its input from pinned host
    # memory and its result back, on their own streams, so step i's input
    # copy and step i-1's result copy overlap step i's forward (two buffers
    # of each; events keep a buffer from being overwritten while in use)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    x_host = [inp.x.pin_memory() for _ in range(2)]
    out_host = [torch.empty(T, H, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(x) for _ in range(2)]
    out_dev = [torch.empty_like(out) for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_fwd = [torch.cuda.Event() for _ in range(2)]
    ev_back = [torch.cuda.Event() for _ in range(2)]

    def e2e_steps(n):
        for i in range(n):
            b = i % 2
            if i >= 2:
                s_in.wait_event(ev_fwd[b])    # step i-2's forward has read x_dev[b]
            with torch.cuda.stream(s_in):
                x_dev[b].copy_(x_host[b], non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_back[b])  # step i-2's result copy has read out_dev[b]
            layer.forward(x_dev[b], out=out_dev[b], stream=stream)
            ev_fwd[b].record(stream)
            s_out.wait_event(ev_fwd[b])
            with torch.cuda.stream(s_out):
                out_host[b].copy_(out_dev[b], non_blocking=True)
                ev_back[b].record(s_out)

    e2e_steps(2)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    w0 = time.time()
    e0.record(s_in)
    s_in.wait_event(e0)
    e2e_steps(args.steps)
    e1.record(s_out)
    torch.cuda.synchronize()
    clocks.mark(w0, time.time())
    barrier()
    assert torch.equal(out_host[(args.steps - 1) % 2], out.cpu()), "end-to-end result differs from the device run"
    e2e_ms = max_over_ranks(e0.elapsed_time(e1)) / args.steps
    assert layer.device_error() == 0
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and c.name == CONFIG_NAME:
        cpu = run_cpu_baseline(inp, gpu_out=out.cpu(), gpu_ids=ids.cpu())
    decode = None
    if c.name == CONFIG_NAME and not args.no_decode:
        # the decode layer's FFN call is compared with an HBM copy timed on its
        # own, so it is timed after the host-side oracle baseline (about 10 s
        # with the GPU idle), not in the clock state the mid layer's long runs
        # leave behind under the power cap
        decode = measure_decode(dev, max(20, min(args.steps, 50)), clocks, max_over_ranks)
    clk = clocks.finish()

    peaks = measured_peaks()
    routed_f, shared_f = gemm_flops(c)
    ffn_s = stage_ms["grouped_ffn"] / 1e3
    if (c.w4a16 or c.nvfp4) and c.T * c.k < 32 * c.E:  # the GEMV path: HBM-bound
        touched, nbytes = w4a16_bytes(c, ids.cpu())
        achieved = nbytes / ffn_s / 1e9
        roof = {"kernel": ("NVFP4" if c.nvfp4 else "W4A16") + " expert FFN (register-dequant gate/up and down GEMV "
                          "launches with their activation preps) + bf16 shared expert", "bound": "hbm",
                "achieved": achieved,
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                "traffic": traffic_from_profile(f"grouped_ffn_{c.name}"),
                "peak_source": f"{peaks['source']} HBM copy", "bytes_per_call": nbytes,
                "touched_experts": touched}
    else:
        achieved = (routed_f + shared_f) / ffn_s / 1e12
        roof = {"kernel": ("grouped W4A16 FFN (int4 dequantised to fp16 in shared memory, tcgen05 gate/up+SwiGLU "
                           "and down+weight launches) + bf16 shared expert") if c.w4a16 else
                          ("grouped NVFP4 FFN (E2M1 x E4M3 dequantised to fp16 in shared memory, tcgen05 "
                           "gate/up+SwiGLU and down+weight launches, fp32 tensor scales in the epilogues) + bf16 "
                           "shared expert") if c.nvfp4 else
                          "grouped SwiGLU FFN (tcgen05 gate/up+SwiGLU and down+weight launches, "
                          "routed + shared expert)",
                "bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"],
                "traffic": traffic_from_profile(f"grouped_ffn_{c.name}"),
                "peak_source": f"{peaks['source']} bf16 burst",
                "frac_of_sustained": (achieved / peaks["bf16_tflops_sustained"]
                                      if peaks.get("bf16_tflops_sustained") else None),
                "flops_per_call": routed_f + shared_f, "routed_flops_per_call": routed_f,
                "routed_tflops": routed_f / ffn_s / 1e12}
    line = base_line(args, world, c)
    line.update({
        "value": replica_tokens_per_s(world, c.T, ms_per_step), "ms_per_step": ms_per_step, "dtype": "bf16",
        "roofline": roof,
        "stage_ms": stage_ms,
        "e2e": {"value": world * c.T / (e2e_ms / 1e3), "unit": "tokens/s",
                "method": "moe_forward per step with its input copied from pinned host memory and its result "
                          "copied back, on separate streams with two buffers (copies of neighbouring steps "
                          "overlap the forward)",
                "h2d_bytes_per_step": c.T * c.H * 2, "d2h_bytes_per_step": c.T * c.H * 2},
        "gpu_launches": launches_per_step(c) * args.steps,
        "clocks": clk,
    })
    if decode is not None:
        line["decode_w4a16"] = decode
    if args.graph:
        line["config"]["launch"] = "CUDA graph replay of the forward"
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if graph is not None:
        del graph
    return line


# ------------------------------------------------ expert parallel arm ----

def bench_ep(args, rank, world, local_rank):
    """Expert parallelism: every rank holds the full router, its contiguous
    range of E/N experts and 1/N of the shared expert's intermediate
    features, runs moe_forward_ep on all T tokens and joins the ranks'
    partial sums with one NCCL all-reduce (page "Module glm5next_mlp",
    §One all-reduce for both EP and TP).  Total work per step is fixed
    (strong scaling): value = T / step time."""
    import torch
    import torch.distributed as dist
    import routed_swiglu_experts_b200 as rse
    from routed_swiglu_experts_b200 import ep

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    rse.load_library()
    cfg, inp = make_inputs(args.workload)
    c = cfg

    def mv(t):
        return None if t is None else t.to(dev)
    group = dist.group.WORLD if world > 1 else None
    layer = ep.ExpertParallelLayer(
        hidden=c.H, num_experts=c.E, top_k=c.k, expert_inter=c.I, shared_inter=c.I_s,
        swiglu_limit=c.swiglu_limit, routed_scaling_factor=c.alpha, renormalize=c.renorm,
        router_w=mv(inp.router_w), correction_bias=mv(inp.correction_bias), w_gate_up=mv(inp.w_gate_up),
        w_down=mv(inp.w_down), s_gate_up=mv(inp.s_gate_up), s_down=mv(inp.s_down),
        shared_w_gate_up=mv(inp.shared_w_gate_up), shared_w_down=mv(inp.shared_w_down),
        g_gate_up=mv(inp.g_gate_up), g_down=mv(inp.g_down),
        rank=rank, world=world, max_tokens=c.T, group=group)
    x = inp.x.to(dev)
    out = torch.empty(c.T, c.H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    clocks = ClockSampler(gpu_uuid(dev))
    for _ in range(args.warmup):
        layer.forward(x, out=out)
    torch.cuda.synchronize()
    rank_barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0 = time.time()
    e0.record(stream)
    for _ in range(args.steps):
        layer.forward(x, out=out)
    e1.record(stream)
    torch.cuda.synchronize()
    clocks.mark(w0, time.time())
    rank_barrier(world)
    ms_per_step = rank_max(e0.elapsed_time(e1), world, dev) / args.steps

    # end to end: the step's tokens from pinned host memory, its result back
    x_host = inp.x.pin_memory()
    out_host = torch.empty(c.T, c.H, dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(x)
    for _ in range(2):
        x_dev.copy_(x_host, non_blocking=True)
        layer.forward(x_dev, out=out)
        out_host.copy_(out, non_blocking=True)
    torch.cuda.synchronize()
    rank_barrier(world)
    torch.cuda.synchronize()
    w0 = time.time()
    e0.record(stream)
    for _ in range(args.steps):
        x_dev.copy_(x_host, non_blocking=True)
        layer.forward(x_dev, out=out)
        out_host.copy_(out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    clocks.mark(w0, time.time())
    rank_barrier(world)
    e2e_ms = rank_max(e0.elapsed_time(e1), world, dev) / args.steps
    clk = clocks.finish()
    assert layer.device_error() == 0
    b, e = layer.expert_range
    line = base_line(args, world, c)
    line["scaling"] = "strong"
    line["config"]["tokens_per_gpu_step"] = c.T
    line["config"]["global_tokens_per_step"] = c.T
    line["config"]["parallelism"] = (f"ep{world}: experts split in contiguous ranges (rank 0: [{b}, {e})), shared "
                                     f"expert split by intermediate features, router replicated, one NCCL "
                                     f"all-reduce of the bf16 [T, H] partials per step")
    line.update({
        "mode": "ep", "value": c.T / (ms_per_step / 1e3), "ms_per_step": ms_per_step, "dtype": "bf16",
        "e2e": {"value": c.T / (e2e_ms / 1e3), "unit": "tokens/s",
                "method": "per step: input copied from pinned host memory, moe_forward_ep + all-reduce, result "
                          "copied back, one stream",
                "h2d_bytes_per_step": c.T * c.H * 2, "d2h_bytes_per_step": c.T * c.H * 2},
        "gpu_launches": launches_per_step(c) * args.steps,
        "clocks": clk,
        "roofline": None,
        "note": "the roofline object is reported by the replicas mode (one GPU runs the whole layer)",
    })
    return line


# -------------------------------------------------------- reference arm ----

def bench_reference(args):
    """The CPU oracle, as it stands, on a bounded sample of the same layer per
    step (the only other place bench.py runs oracle/)."""
    import torch
    import oracle
    cfg, inp = make_inputs(args.workload)
    # per-step sample sized so the whole run stays within a few minutes
    sample = min(512, cfg.T)
    t0 = time.perf_counter()
    oracle.moe_forward(inp, tokens=range(sample))
    est = time.perf_counter() - t0
    budget = 150.0
    while sample > 16 and est * (args.steps + args.warmup) > budget:
        sample //= 2
        est /= 1.6
    toks = list(range(sample))
    for _ in range(args.warmup):
        oracle.moe_forward(inp, tokens=toks)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.moe_forward(inp, tokens=toks)
    dt = time.perf_counter() - t0
    value = args.steps * sample / dt
    line = base_line(args, 1, cfg)
    line.update({
        "impl": "reference", "value": value, "ms_per_step": dt / args.steps * 1e3, "dtype": "f64",
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": torch.get_num_threads(), "kind": "oracle",
                         "sample": f"{sample} of the {cfg.T} tokens of the {cfg.name} layer per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    })
    return line


def main(argv=None):
    args = parse_args(argv)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(bench_reference(args)), flush=True)
        return 0
    import torch
    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        line = bench_ep(args, rank, world, local_rank) if args.mode == "ep" else bench_ours(args, rank, world,
                                                                                           local_rank)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
