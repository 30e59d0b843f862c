#!/usr/bin/env python
"""Throughput of the MoE expert layer on B200: prints one JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
    python bench.py --router-sweep     # the router alone at the gate-epilogue page's shapes

A step is one full layer pass (router, permute, GEMM1 + SwiGLU, GEMM2, combine) over
one batch of T synthetic tokens already resident in HBM. The default workload is the
largest single-GPU configuration: the GLM-style FP8 prefill (T = 8192, H = 4096,
I = 1536, 288 routed experts top-8 plus one shared expert, E4M3 weights with 128x128
block scales, 1x128 activation scales, L = 10). Under torchrun each rank runs its own
batch with replicated weights (weak scaling, no data-path collective); the step time is
the maximum over ranks. L2 is flushed (a 512 MiB write) between timed steps, outside
the timed events.

--impl reference times the fp64 CPU oracle on the host cores instead (rank 0 only),
each step a bounded sample of the same workload's tokens.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE layer tokens/s"
UNIT = "tokens/s"


def parse():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="glm_fp8")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the timed oracle sample")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target length of the oracle sample")
    ap.add_argument("--tokens", type=int, default=None, help="override the workload's T (profiling runs)")
    ap.add_argument("--experts", type=int, default=None, help="override the workload's E (profiling runs)")
    ap.add_argument("--mode", choices=["dp", "ep", "tp"], default="dp",
                    help="dp: every rank runs the whole layer on its own tokens (default); ep: the routed "
                         "experts split over the ranks, rows exchanged with all_to_all; tp: every expert's "
                         "intermediate size split over the ranks, outputs all-reduced")
    ap.add_argument("--router-sweep", action="store_true",
                    help="time the router alone at fp32 [T, 258] (256 routed + 2 sinks), k = 6, "
                         "T in 1, 8, 64, 512, 4096, 8192, and print one JSON line")
    return ap.parse_args()


KERNEL_SOURCES = ("gemm.cu", "ptx.cuh", "internal.h")  # the grouped-GEMM kernel and what it includes


def strip_comments(text: str) -> str:
    """C/C++ source without comments and with whitespace runs collapsed (string and
    character literals kept as they are)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_code_digest() -> str:
    """sha1 of the grouped-GEMM kernel's sources without their comments: a comment edit
    keeps a capture's counters, any code edit retires them."""
    import hashlib
    h = hashlib.sha1()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "grouped_gemm_swiglu_b200", "csrc", name)) as f:
            h.update(strip_comments(f.read()).encode())
    return h.hexdigest()


def profiled_traffic(workload: str):
    """DRAM bytes per launch of the grouped-GEMM kernel from the committed ncu capture,
    or None when the kernel's code changed since that capture."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)
        if rec.get("kernel_code_sha1") != kernel_code_digest():
            return None
        return rec.get("workloads", {}).get(workload)
    except Exception:
        return None


def peaks():
    """(HBM GB/s, bf16 TFLOP/s burst, bf16 TFLOP/s sustained, source)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return (float(p["hbm_gbs"]), float(p["bf16_tflops"]),
                float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured")
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def w_bytes_all(wl) -> float:
    """Bytes of every expert's weights (not only the touched ones)."""
    welt = {1: 1.0, 2: 0.5 + 2.0 / 32, 3: 0.5 + 1.0 / 16}.get(wl.wdtype, 2.0)
    return wl.G * 3 * wl.I * wl.H * welt


def kernel_work(wl, offsets):
    """Algorithmic work of one grouped-GEMM launch (both GEMMs) for group offsets [G+1]:
    FLOPs 2*A*H*2I + 2*A*I*H over the A permuted rows; bytes = the weights (and block or
    group scales) of every group with at least one row, each read once; and, apart, the
    implementation's own traffic: x_perm read, h written and read back (+ FP8 scales), y
    written. Returns (flops, weight_bytes, impl_bytes)."""
    used = int(((offsets[1:] - offsets[:-1]) > 0).sum())
    A = int(offsets[-1])
    fp8 = wl.wdtype == 1
    H, I = wl.H, wl.I
    elt = 1 if fp8 else 2  # activations (x_perm, h)
    # weight bytes per element: INT4 a nibble + a bf16 scale per 32; NVFP4 a nibble + an E4M3 scale per 16
    welt = {2: 0.5 + 2.0 / 32, 3: 0.5 + 1.0 / 16}.get(wl.wdtype, elt)
    flops = 2.0 * A * H * 2 * I + 2.0 * A * I * H
    w_bytes = used * 3 * I * H * welt
    if fp8:
        w_bytes += used * ((2 * I // 128) * (H // 128) + (H // 128) * (I // 128)) * 4
    impl_bytes = A * H * elt + 2 * A * I * elt + A * H * 2
    if fp8:
        impl_bytes += A * (H // 128 + 2 * (I // 128)) * 4
    return flops, w_bytes, impl_bytes


def stats(xs):
    """mean / median / min of a list of times (ms)."""
    return {"mean": sum(xs) / len(xs), "median": statistics.median(xs), "min": min(xs), "n": len(xs)}


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ["uuid", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]

    def __init__(self, uuid: str):
        self.uuid = uuid.lower().replace("gpu-", "")
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"moe_b200_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + ",".join(self.FIELDS),
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != len(self.FIELDS) or self.uuid not in parts[0].lower():
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        try:
            os.remove(self.path)
        except OSError:
            pass
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ oracle timing
def oracle_rate(wl, inp_host, seconds: float, max_tokens: int | None = None):
    """Tokens/s of the fp64 oracle on a sample sized to take about `seconds`."""
    import numpy as np
    import oracle
    from oracle.torch_io import oracle_layer_from_inputs
    L = oracle_layer_from_inputs(wl, inp_host)
    t0 = time.perf_counter()
    L.moe_rows(np.array([0], dtype=np.int32))
    one = max(time.perf_counter() - t0, 1e-4)
    n = int(max(1, min(max_tokens or wl.T, wl.T, math.ceil(seconds / one))))
    toks = np.arange(n, dtype=np.int32)
    # whole passes over the sample until about `seconds` of work (small workloads take
    # several passes; a pass is never cut short)
    passes, dt = 0, 0.0
    while passes == 0 or dt < seconds:
        t0 = time.perf_counter()
        L.moe_rows(toks)
        dt += time.perf_counter() - t0
        passes += 1
    return passes * n / dt, n, dt, oracle.num_threads(), passes


# ------------------------------------------------------------------ reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import numpy as np
    import oracle
    from grouped_gemm_swiglu_b200 import workloads as W
    from oracle.torch_io import oracle_layer_from_inputs, host_inputs
    wl = workload_of(args)
    inp = host_inputs(W.make_inputs(wl, "cpu"))
    L = oracle_layer_from_inputs(wl, inp)
    t0 = time.perf_counter()
    L.moe_rows(np.array([0], dtype=np.int32))
    one = max(time.perf_counter() - t0, 1e-4)
    budget = 150.0 / max(1, args.steps + args.warmup)
    n = int(max(1, min(wl.T, round(budget / one))))
    rng = np.random.default_rng(0)
    times = []
    for s in range(args.warmup + args.steps):
        toks = np.sort(rng.choice(wl.T, n, replace=False)).astype(np.int32)
        t0 = time.perf_counter()
        L.moe_rows(toks)
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            times.append(dt)
    sec = sum(times) / len(times)
    value = n / sec
    line = {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(wl),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": f"{n} random tokens of {wl.T} per step ({wl.name}), fp64 oracle"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_of(args):
    from grouped_gemm_swiglu_b200 import workloads as W
    wl = W.WORKLOADS[args.workload]
    if args.tokens is not None:
        wl = wl.with_(T=args.tokens)
    if args.experts is not None:
        wl = wl.with_(E=args.experts)
    return wl


def config_of(wl):
    return {"workload": wl.name, "T": wl.T, "H": wl.H, "I": wl.I, "E": wl.E, "top_k": wl.k,
            "n_sink": wl.n_sink, "n_shared": wl.n_shared,
            "weights": {1: "fp8_e4m3_block128", 2: "int4_group32_bf16_scales",
                        3: "nvfp4_e2m1_e4m3_scales_per16"}.get(wl.wdtype, "bf16"),
            "score": "sigmoid_logsigmoid_lse" if wl.score == 1 else "softmax_renorm",
            "alpha": wl.alpha, "beta": wl.beta, "limit": None if math.isinf(wl.limit) else wl.limit,
            "seed": wl.seed, "l2": "device-timed steps: flushed before each step (512 MiB write, outside the timed events); "
                                  "e2e: weights larger than L2, else flushed before each pass"}


# ------------------------------------------------------------------ ranks
class Ranks:
    """One process per GPU as torchrun starts them (RANK, LOCAL_RANK, WORLD_SIZE, MASTER_*).

    The layer is token-parallel: every rank runs its own batch with replicated weights and
    there is no data-path collective; the only collectives are the barriers around the
    timed region and a MAX all-reduce of each timing, so the reported time is the slowest
    rank's and the whole-job rate counts every rank's tokens. `backend` is "nccl" on GPUs;
    the tests drive the same logic with "gloo" on CPU."""

    def __init__(self, backend: str = "nccl", device=None, timeout_s: float = 180.0):
        import torch
        import torch.distributed as dist
        self.dist = dist
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.device = device if device is not None else torch.device("cpu")
        self.backend = backend
        if self.world > 1:
            from datetime import timedelta
            kw = {"device_id": self.device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=timedelta(seconds=timeout_s), **kw)

    def barrier(self):
        if self.world > 1:
            if self.backend == "nccl":
                self.dist.barrier(device_ids=[self.local])
            else:
                self.dist.barrier()

    def max_over_ranks(self, v: float) -> float:
        if self.world == 1:
            return v
        import torch
        t = torch.tensor([v], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def rate(self, tokens_per_rank: int, ms_per_step: float) -> float:
        """Whole-job tokens/s: every rank's tokens over the slowest rank's step time."""
        return self.world * tokens_per_rank / (ms_per_step / 1e3)

    def close(self):
        if self.world > 1:
            self.dist.destroy_process_group()


# ------------------------------------------------------------------ our arm
def run_ours(args):
    import numpy as np
    import torch
    import grouped_gemm_swiglu_b200 as moe
    from grouped_gemm_swiglu_b200 import workloads as W

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks("nccl", dev)
    world, rank = ranks.world, ranks.rank
    barrier, max_over_ranks = ranks.barrier, ranks.max_over_ranks

    wl = workload_of(args)
    inp = W.make_inputs(wl, dev)
    d = moe.MoeDims.of(wl)
    fp8 = wl.wdtype == W.WDTYPE_FP8
    A, G, T = d.A, d.G, wl.T
    layer = moe.MoELayer(d, inp["w1"], inp["w2"], inp["w1_scale"], inp["w2_scale"], inp["gate_scale"],
                         inp["up_scale"])
    out = torch.empty((T, wl.H), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    K, Wm = args.steps, args.warmup

    # The layer pass as its four public calls: router, permutation, both grouped GEMMs
    # (one persistent kernel), weighted combine. moe_forward runs the same kernels.
    ids = torch.empty((T, wl.k), dtype=torch.int32, device=dev)
    tw = torch.empty((T, wl.k), dtype=torch.float32, device=dev)
    sw = torch.empty((T, wl.n_sink), dtype=torch.float32, device=dev) if wl.n_sink else None
    offsets = torch.empty((G + 1,), dtype=torch.int32, device=dev)
    perm = torch.empty((A,), dtype=torch.int32, device=dev)
    inv = torch.empty((T, wl.k), dtype=torch.int32, device=dev)
    xp = torch.empty((A, wl.H), dtype=torch.uint8 if fp8 else torch.bfloat16, device=dev)
    xs = torch.empty((wl.H // 128, A), dtype=torch.float32, device=dev) if fp8 else None
    h = torch.empty((A, wl.I), dtype=torch.uint8 if fp8 else torch.bfloat16, device=dev)
    hs = torch.empty((wl.I // 128, A), dtype=torch.float32, device=dev) if fp8 else None
    y = torch.empty((A, wl.H), dtype=torch.bfloat16, device=dev)
    ws_p = moe.alloc_workspace(d, moe.MOE_WS_PERMUTE, dev)
    ws_e = moe.alloc_workspace(d, moe.MOE_WS_EXPERTS, dev)
    ws_c = moe.alloc_workspace(d, moe.MOE_WS_COMBINE, dev)
    stages = {
        "route": lambda: moe.moe_route_topk(inp["logits"], d, None, ids, tw, sw),
        "permute": lambda: moe.moe_permute(ids, inp["x"], d, offsets, perm, inv, xp, xs, ws_p),
        "experts": lambda: moe.moe_experts(xp, xs, offsets, inp["w1"], inp["w1_scale"], inp["gate_scale"],
                                           inp["up_scale"], None, inp["w2"], inp["w2_scale"], d, h, hs, y, ws_e),
        "combine": lambda: moe.moe_combine(y, offsets, inv, tw, sw, d, out, ws_c),
    }
    launches_per_step = 5  # router 1, permutation 2, grouped GEMMs 1, combine 1

    def run_stages(marks):
        marks[0].record(stream)
        for i, fn in enumerate(stages.values()):
            fn()
            marks[i + 1].record(stream)

    # Eager warm-up (first calls set kernel attributes and look up the driver entry point).
    for _ in range(Wm):
        flush.zero_()
        run_stages([torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)])
        layer.forward(inp["logits"], inp["x"], out=out)
    torch.cuda.synchronize(dev)
    for ws in (ws_p, ws_e, ws_c, layer.ws):
        assert moe.moe_read_status(ws) == 0, moe.status_string(moe.moe_read_status(ws))

    # Deployment mode: the layer pass captured in CUDA graphs and replayed, so the timed
    # region holds the GPU's work without host launch gaps. Every step replays the whole
    # moe_forward graph (the layer throughput), then the four public calls (router,
    # permutation, grouped GEMMs, combine) as four graphs with device events between them
    # (per-stage times; the grouped-GEMM launch is the roofline kernel).
    g_fwd = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_fwd):
        layer.forward(inp["logits"], inp["x"], out=out)
    g_st = {}
    for k, fn in stages.items():
        g_st[k] = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_st[k]):
            fn()
    stream = torch.cuda.current_stream(dev)
    for _ in range(3):
        flush.zero_()
        g_fwd.replay()
        for g in g_st.values():
            g.replay()
    torch.cuda.synchronize(dev)

    # ---- timed region: K steps. Each step is one whole layer pass (the moe_forward graph:
    # `value`), then the four public calls as four graphs with device events between them
    # (`stages_ms`), then one eager moe_experts launch bracketed by events on its stream
    # (`roofline.kernel_ms`: the grouped-GEMM kernel alone, without a graph launch), each
    # after its own L2 flush.
    sampler = ClockSampler(str(torch.cuda.get_device_properties(dev).uuid))
    sampler.start()
    time.sleep(0.4)  # let the sampler start before the timed region
    steps = []
    barrier()
    torch.cuda.synchronize(dev)
    wall0 = time.perf_counter()
    for _ in range(K):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 + len(stages) + 1 + 2)]
        flush.zero_()
        ev[0].record(stream)
        g_fwd.replay()
        ev[1].record(stream)
        flush.zero_()
        ev[2].record(stream)
        for i, g in enumerate(g_st.values()):
            g.replay()
            ev[3 + i].record(stream)
        flush.zero_()
        ev[-2].record(stream)
        stages["experts"]()
        ev[-1].record(stream)
        steps.append(ev)
    torch.cuda.synchronize(dev)
    barrier()
    wall = time.perf_counter() - wall0
    clocks = sampler.stop()
    fwd_t = [ev[0].elapsed_time(ev[1]) for ev in steps]
    st_t = {k: [ev[2 + i].elapsed_time(ev[3 + i]) for ev in steps] for i, k in enumerate(stages)}
    kern_t = [ev[-2].elapsed_time(ev[-1]) for ev in steps]
    st = {k: max_over_ranks(sum(v) / K) for k, v in st_t.items()}
    ms = max_over_ranks(sum(fwd_t) / K)
    kern_ms = max_over_ranks(sum(kern_t) / K)
    value = ranks.rate(T, ms)
    fwd_ms = ms
    for ws in (ws_p, ws_e, ws_c, layer.ws):
        assert moe.moe_read_status(ws) == 0, moe.status_string(moe.moe_read_status(ws))

    # ---- end to end: pinned host inputs in, result out, every step, through moe_forward
    # (MoELayer.forward), pipelined as a serving loop: step s's host-to-device copies run on
    # a copy stream, its layer pass on the compute stream and its device-to-host copy on a
    # third stream, with two device buffer sets, so step s + 1's inputs and step s - 1's
    # output move while step s computes. Every step copies its whole input in and its whole
    # output out. The timed region runs from the first timed step's first copy to the last
    # one's output copy (events on the copy streams); per-step time = that / the steps.
    # Layers whose weights fit in L2 flush it on the compute stream before each pass.
    x_h = inp["x"].cpu().pin_memory()
    lg_h = inp["logits"].cpu().pin_memory()
    out_h = torch.empty((T, wl.H), dtype=torch.bfloat16).pin_memory()
    x_d = [torch.empty_like(inp["x"]) for _ in range(2)]
    lg_d = [torch.empty_like(inp["logits"]) for _ in range(2)]
    out_d = [torch.empty((T, wl.H), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    comp = stream
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    small = w_bytes_all(wl) < 2 * 126e6
    Ke = max(1, min(K, 200))

    def e2e_steps(n):
        first = last = None
        for s in range(n):
            b = s % 2
            if s >= 2:  # buffer set b was last used by step s - 2
                s_in.wait_event(ev_comp[b])
            with torch.cuda.stream(s_in):
                if s == 0:
                    first = torch.cuda.Event(enable_timing=True)
                    first.record(s_in)
                x_d[b].copy_(x_h, non_blocking=True)
                lg_d[b].copy_(lg_h, non_blocking=True)
                ev_in[b].record(s_in)
            comp.wait_event(ev_in[b])
            if s >= 2:
                comp.wait_event(ev_out[b])
            with torch.cuda.stream(comp):
                if small:
                    flush.zero_()
                layer.forward(lg_d[b], x_d[b], out=out_d[b])
                ev_comp[b].record(comp)
            s_out.wait_event(ev_comp[b])
            with torch.cuda.stream(s_out):
                out_h.copy_(out_d[b], non_blocking=True)
                ev_out[b].record(s_out)
                if s == n - 1:
                    last = torch.cuda.Event(enable_timing=True)
                    last.record(s_out)
        last.synchronize()
        return first.elapsed_time(last)

    e2e_steps(3)  # warm-up
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e2e_steps(Ke) / Ke)
    h2d = x_h.numel() * x_h.element_size() + lg_h.numel() * lg_h.element_size()
    d2h = out_h.numel() * out_h.element_size()

    # ---- the fused gate GEMV + router (decode-sized batches, outside the layer step): x . W_gate
    # with a seeded bf16 gate weight [E + n_sink][H], then the routing, in one launch
    gate = None
    if T <= 16:
        gg = torch.Generator(device=dev).manual_seed(1)
        w_gate = (torch.randn((wl.E + wl.n_sink, wl.H), generator=gg, device=dev) * 0.05).to(torch.bfloat16)
        ws_g = moe.alloc_workspace(d, moe.MOE_WS_GATE_ROUTE, dev)
        lg_g = torch.empty((T, wl.E + wl.n_sink), dtype=torch.float32, device=dev)
        gate_fn = lambda: moe.moe_gate_route(inp["x"], w_gate, d, None, lg_g, ids, tw, sw, None, ws_g)  # noqa: E731
        for _ in range(3):
            gate_fn()
        g_gate = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_gate):
            gate_fn()
        gt = []
        for _ in range(max(1, min(K, 200))):
            flush.zero_()
            a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a_.record(stream)
            g_gate.replay()
            b_.record(stream)
            gt.append((a_, b_))
        torch.cuda.synchronize(dev)
        assert moe.moe_read_status(ws_g) == 0
        gate = {"ms": max_over_ranks(sum(x.elapsed_time(y) for x, y in gt) / len(gt)),
                "what": "moe_gate_route: gate GEMV over E + n_sink columns fused with the router, one launch, "
                        "graph replay, L2 flushed; compare stages_ms.route (router alone, logits given)",
                "w_gate_bytes": w_gate.numel() * 2}
        del g_gate

    # ---- roofline of the dominant kernel: both grouped GEMMs (moe_experts, one launch).
    # Algorithmic bytes of the kernel: the weights (and block scales) of every expert that
    # has at least one row, each read once. Its other traffic -- x_perm read, h written and
    # read back, y written -- is the implementation's choice of materialising the
    # intermediates and is reported apart as impl_bytes.
    hbm, bf16_tf, bf16_sus, peak_src = peaks()
    H_ = wl.H
    off = offsets.cpu().numpy()
    used = int(((off[1:] - off[:-1]) > 0).sum())
    flops, w_bytes, impl_bytes = kernel_work(wl, off)
    t_k = kern_ms / 1e3
    tensor_peak = bf16_tf * (2.0 if fp8 else 1.0)
    tensor_sus = bf16_sus * (2.0 if fp8 else 1.0)
    # the roof that bounds the kernel is the one giving the longer time for its algorithmic work
    if w_bytes / (hbm * 1e9) >= flops / (tensor_peak * 1e12):
        roof = {"bound": "hbm", "achieved": w_bytes / t_k / 1e9, "peak": hbm, "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": flops / t_k / 1e12, "peak": tensor_peak, "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = profiled_traffic(wl.name)
    roof["kernel"] = "moe_gemm_kernel (GEMM1 + SwiGLU and GEMM2, one persistent launch)"
    roof["kernel_ms"] = kern_ms
    roof["kernel_ms_stats"] = stats(kern_t)
    roof["timing"] = ("achieved = algorithmic work per launch / mean duration of an eager moe_experts launch "
                      "bracketed by CUDA events on its stream, L2 flushed before each")
    roof["peak_source"] = peak_src + " burst" + (" (E4M3 = 2x measured bf16, the nominal ratio)" if fp8 else "")
    roof["algorithmic_bytes"] = w_bytes
    roof["algorithmic_bytes_what"] = "weights + block scales of the experts with at least one row, read once"
    roof["impl_bytes"] = impl_bytes
    roof["impl_bytes_what"] = "x_perm read, h written and read (+ scales), y written"
    roof["algorithmic_flops"] = flops
    roof["hbm_frac"] = w_bytes / t_k / 1e9 / hbm
    roof["tensor_frac"] = flops / t_k / 1e12 / tensor_peak
    roof["tensor_frac_of_sustained"] = flops / t_k / 1e12 / tensor_sus
    roof["other_roof_frac"] = roof["tensor_frac"] if roof["bound"] == "hbm" else roof["hbm_frac"]
    roof["stage_graph_ms"] = st["experts"]
    # the whole layer step against its own algorithmic bytes: touched weights, x in, out,
    # logits in, routing outputs (ids, weights, sink weights) out
    layer_bytes = (w_bytes + T * H_ * 2 + T * H_ * 2 + T * (wl.E + wl.n_sink) * 4 + T * wl.k * 8
                   + T * wl.n_sink * 4)
    layer_roof = {"algorithmic_bytes": layer_bytes, "flops": flops,
                  "hbm_frac": layer_bytes / (fwd_ms / 1e3) / 1e9 / hbm,
                  "tensor_frac": flops / (fwd_ms / 1e3) / 1e12 / tensor_peak,
                  "tflops": flops / (fwd_ms / 1e3) / 1e12, "gbs": layer_bytes / (fwd_ms / 1e3) / 1e9}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": Wm,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp8_e4m3" if fp8 else "bf16", "data": "synthetic", "config": config_of(wl),
            "e2e": {"value": ranks.rate(T, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": Ke,
                    "how": "moe_forward (MoELayer.forward) fed from pinned host memory every step, pipelined: the "
                           "next step's host-to-device copies and the previous step's device-to-host copy overlap "
                           "the layer pass on separate streams; timed from the first copy to the last"},
            "roofline": roof, "clocks": clocks, "gpu_launches": (2 * launches_per_step + 1) * K,
            "stages_ms": st, "forward_ms_per_step": fwd_ms, "forward_ms_stats": stats(fwd_t),
            "stages_ms_stats": {k: stats(v) for k, v in st_t.items()},
            "experts_touched": used, "gate_route": gate, "layer_roofline": layer_roof,
            "timing": "CUDA graph replays: value from the moe_forward graph (mean over the steps); stages from "
                      "one graph per public call with device events between the launches; the roofline kernel "
                      "from an eager launch between events",
            "layer_tflops": wl.flops() / (ms / 1e3) / 1e12,
            "wall_s_timed_region": wall}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle.torch_io import host_inputs
        rate, n, dt, cores, passes = oracle_rate(wl, host_inputs(inp), args.cpu_seconds)
        line["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": f"{passes} pass(es) over the first {n} of {wl.T} tokens of {wl.name} "
                                          f"({dt:.1f} s, fp64)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    ranks.close()
    return 0


# ------------------------------------------------------------------ expert / tensor parallel
def parallel_bench(mode, wl, ranks, dev, K, Wm, ops=None, inputs=None, exchange=None):
    """Times the expert-parallel (mode "ep") or tensor-parallel ("tp") layer, one rank per
    GPU, and returns the JSON line (rank 0 prints it). ep: every rank routes its own T
    tokens (the workload's tokens rolled by 17 * rank rows, so ranks route differently)
    and the routed experts are split in contiguous blocks; value = all ranks' tokens / the
    slowest rank's step (weak scaling). tp: every rank runs all T tokens on an I/R slice
    of every expert and the outputs are all-reduced; value = T / the slowest rank's step
    (strong scaling). A step is one eager forward (the expert-parallel pass reads its row
    counts on the host, so it is not graph-captured), between CUDA events on its stream
    and barriers. `ops`, `inputs` and `exchange` let the plumbing run with stand-ins."""
    import torch
    from grouped_gemm_swiglu_b200 import ep as EP
    from grouped_gemm_swiglu_b200 import tp as TP
    from grouped_gemm_swiglu_b200 import workloads as W
    from grouped_gemm_swiglu_b200._lib import MoeDims
    import grouped_gemm_swiglu_b200 as moe
    ops = ops if ops is not None else moe._lib
    world, rank = ranks.world, ranks.rank
    inp = inputs if inputs is not None else W.make_inputs(wl, dev)
    d = inp["dims"] if "dims" in inp else MoeDims.of(wl)
    if exchange is None:
        exchange = EP.TorchExchange() if world > 1 else EP.LocalExchange(1).for_rank(0)
    T = wl.T
    if mode == "ep":
        if d.E % world:
            raise SystemExit(f"--mode ep: E = {d.E} does not split over {world} ranks")
        sh = lambda t: EP.shard(t, rank, world, d.E, d.n_shared)  # noqa: E731
        layer = EP.ExpertParallelMoE(d, rank, world, sh(inp["w1"]), sh(inp["w2"]), sh(inp.get("w1_scale")),
                                     sh(inp.get("w2_scale")), sh(inp.get("gate_scale")), sh(inp.get("up_scale")),
                                     exchange=exchange, ops=ops, max_tokens=T)
        x = torch.roll(inp["x"], 17 * rank, 0).contiguous()
        logits = torch.roll(inp["logits"], 17 * rank, 0).contiguous()
    else:
        if d.I % (128 * world):
            raise SystemExit(f"--mode tp: I = {d.I} does not split into multiples of 128 over {world} ranks")
        layer = TP.TensorParallelMoE(d, rank, world, TP.shard_w1(inp["w1"], rank, world),
                                     TP.shard_w2(inp["w2"], rank, world), TP.shard_w1(inp.get("w1_scale"), rank, world),
                                     TP.shard_w2(inp.get("w2_scale"), rank, world), inp.get("gate_scale"),
                                     inp.get("up_scale"), exchange=exchange, ops=ops)
        x, logits = inp["x"], inp["logits"]
    out = torch.empty((T, d.H), dtype=torch.bfloat16, device=dev)
    cuda = torch.device(dev).type == "cuda"
    for _ in range(Wm):
        layer.forward(logits, x, out=out)
    if cuda:
        torch.cuda.synchronize(dev)
    times = []
    for _ in range(K):
        ranks.barrier()
        if cuda:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            layer.forward(logits, x, out=out)
            b.record()
            b.synchronize()
            times.append(a.elapsed_time(b))
        else:
            t0 = time.perf_counter()
            layer.forward(logits, x, out=out)
            times.append((time.perf_counter() - t0) * 1e3)
    ranks.barrier()
    st = layer.status()
    ms = ranks.max_over_ranks(sum(times) / len(times))
    tokens = world * T if mode == "ep" else T
    return {"metric": METRIC, "value": tokens / (ms / 1e3), "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": Wm, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak" if mode == "ep" else "strong", "vs_baseline": None,
            "dtype": {1: "fp8_e4m3", 2: "int4_w4a16", 3: "nvfp4_w4a16"}.get(wl.wdtype, "bf16"),
            "data": "synthetic", "config": dict(config_of(wl), mode=mode, parallelism=f"{mode}{world}"),
            "status": st, "roofline": None, "cpu_baseline": None,
            "timing": "eager forward between CUDA events on its stream, barrier before each step, mean over "
                      "the steps, max over ranks",
            "ms_stats": stats(times)}


def run_parallel(args):
    import torch
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks("nccl", dev)
    line = parallel_bench(args.mode, workload_of(args), ranks, dev, args.steps, args.warmup)
    if ranks.rank == 0:
        print(json.dumps(line), flush=True)
    ranks.close()
    return 0


# ------------------------------------------------------------------ router sweep
ROUTER_SWEEP_T = (1, 8, 64, 512, 4096, 8192)


def run_router_sweep(args):
    """The router alone (moe_route_topk) at the gate-epilogue page's shapes: an fp32 gate
    row of 258 columns (256 routed + 2 shared sinks), top-6, logsigmoid-LSE weights over
    the selected and sink columns (sglang PR #36385 "Performance"). Device time per launch
    from CUDA events around a graph of 200 back-to-back launches (so host submission is
    not in the figure), the minimum of 5 replays."""
    import torch
    import grouped_gemm_swiglu_b200 as moe
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    N, S, k, reps, n = 256, 2, 6, 5, 200
    rows = []
    for T in ROUTER_SWEEP_T:
        d = moe.MoeDims(T=T, H=128, I=128, E=N, k=k, n_sink=S, n_shared=0, wdtype=0, score=moe.MOE_SCORE_SIGMOID,
                        alpha=1.0, beta=0.0, limit=float("inf"), route_scale=1.0)
        g = torch.Generator(device=dev).manual_seed(T)
        logits = torch.randn((T, N + S), generator=g, device=dev)
        ids = torch.empty((T, k), dtype=torch.int32, device=dev)
        w = torch.empty((T, k), dtype=torch.float32, device=dev)
        sw = torch.empty((T, S), dtype=torch.float32, device=dev)
        for _ in range(10):
            moe.moe_route_topk(logits, d, None, ids, w, sw)
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _ in range(n):
                moe.moe_route_topk(logits, d, None, ids, w, sw)
        graph.replay()
        torch.cuda.synchronize(dev)
        best = float("inf")
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            graph.replay()
            b.record()
            b.synchronize()
            best = min(best, a.elapsed_time(b) * 1e3 / n)
        del graph
        nbytes = T * (N + S) * 4 + T * k * 8 + T * S * 4
        rows.append({"T": T, "us_per_launch": best, "gbs": nbytes / (best * 1e-6) / 1e9, "bytes": nbytes})
    line = {"metric": "router device time per launch", "unit": "us", "impl": "ours",
            "config": {"workload": "router_sweep", "N": N, "n_sink": S, "top_k": k,
                       "score": "sigmoid_logsigmoid_lse", "logits": "fp32 N(0,1), seed T"},
            "timing": f"min over {reps} replays of a CUDA graph of {n} back-to-back launches, CUDA events around "
                      "each replay; logits L2-resident (as in a model's decode loop)",
            "rows": rows,
            "pages_context": {"hardware": "Intel Arc Pro B60 (sglang PR #36385)",
                              "us": {"1": 2.43, "8": 2.46, "64": 2.77, "512": 3.40, "4096": 15.64, "8192": 28.02}}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.router_sweep:
        return run_router_sweep(args)
    if args.impl == "reference":
        return run_reference(args)
    if args.mode != "dp":
        return run_parallel(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
