"""Benchmark of the routed MoE FFN forward on B200: tokens/s and roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one ``moe_forward`` (router -> grouping -> grouped gate/up GEMM with
GLU epilogue -> down GEMM -> shared expert -> combine) over one batch of
seeded synthetic tokens already resident in HBM.  L2 is flushed (a 256 MiB
write) before every timed step, outside the timed interval.  Under torchrun
(N > 1) every rank runs an independent replica on its own GPU and its own
tokens (the layer does not shard here; no collective on the data path); the
reported time is the max over ranks.

Rank 0 prints one JSON line.  ``--impl reference`` times the float64 CPU
oracle on the same workload (the reference arm): one full-size forward per
step for the bf16 workloads; for the INT4 decode workload, whose float64
experts do not fit in host memory at once, one token of the batch per step.
The default workload is ``granular`` (T=32768, d=768, 192 experts top-4, SwiGLU
hidden 256, shared expert 512, capacity factor 1.25).
"""

from __future__ import annotations

import argparse
import ctypes
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE-layer fwd tokens/s on 1 B200; % of bf16 tensor-core or HBM roofline"
DEFAULT_WORKLOAD = "granular"
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of the expert GEMM launches of one forward (routed
# gate/up, routed down, shared gate/up, shared down), from an `ncu --set full --clock-control none
# -k regex:k_grouped_gemm -s 5 -c 5` capture of `bench.py --workload <name> --steps 1 --warmup 1
# --no-cpu-baseline` on the current kernels; workloads without a complete capture report null.
GEMM_TRAFFIC_BYTES = {"small": 12628736 + 21004032,
                      "granular": (380192256 + 151918592 + 51950848 + 34377472) + (55830784 + 150960896 + 5970432 + 4317440)}
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(PEAKS_FALLBACK)
    d["source"] = "fallback"
    return d


def hbm_roofline_tokens_per_s(bandwidth_bytes_per_s: float, active_bytes_per_token: float) -> float:
    """Ideal bandwidth-bound decode rate: bandwidth / bytes of active weights per token."""
    return bandwidth_bytes_per_s / active_bytes_per_token


def bench_config(wl, capacity: int, world: int) -> dict:
    """The ``config`` object of the JSON line, identical for both arms on the same workload."""
    return {"workload": wl.name, "T": wl.T, "d": wl.d, "E": wl.E, "k": wl.k, "H": wl.H, "H_s": wl.H_s,
            "capacity": capacity, "act": "geglu" if wl.act else "swiglu",
            "wfmt": "int4_g128" if wl.wfmt else "bf16", "router": "fp32", "skew": wl.skew,
            "l2": "GPU arm: a 256 MiB write flushes L2 before every timed step, outside the timed interval",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


def int4_step_bytes(wl, touched: int) -> int:
    """Algorithmic HBM bytes of one INT4 forward: touched experts' packed weights and scales, the shared
    expert, the router weight, x in and out."""
    per_expert = (2 * wl.H * wl.d + wl.d * wl.H) // 2 + (2 * wl.H * wl.d + wl.d * wl.H) // 128 * 2
    shared = ((2 * wl.H_s * wl.d + wl.d * wl.H_s) // 2 + (2 * wl.H_s * wl.d + wl.d * wl.H_s) // 128 * 2) if wl.H_s else 0
    return touched * per_expert + shared + wl.E * wl.d * 4 + 2 * wl.T * wl.d * 2


def gemm_step_bytes(wl, kept: int, touched: int) -> int:
    """Algorithmic HBM bytes of the bf16 expert GEMMs of one forward: routed gate/up reads the grouped rows and
    the touched experts' w13 and writes h; down reads h and w2 and writes y; the shared expert likewise on all T
    tokens."""
    routed = kept * wl.d * 2 + touched * 2 * wl.H * wl.d * 2 + 2 * kept * wl.H * 2 \
        + touched * wl.d * wl.H * 2 + kept * wl.d * 2
    shared = (wl.T * wl.d * 2 + 2 * wl.H_s * wl.d * 2 + 2 * wl.T * wl.H_s * 2 + wl.d * wl.H_s * 2 + wl.T * wl.d * 2) \
        if wl.H_s else 0
    return routed + shared


def max_over_ranks(value: float, world: int) -> float:
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.15)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ workload setup


def setup(wl, seed, device):
    import torch

    import sparse_mixture_experts_expert_b200 as moe
    import synth
    inp = synth.make_inputs(wl, seed=0, device=device)                # weights: same on every replica
    if seed:
        inp["x"] = synth.make_inputs(wl, seed=seed, device=device, with_expert_weights=False)["x"]
    if wl.wfmt == synth.WFMT_INT4_G128:
        inp.update(int4_weights(moe, wl, 0, device))
    C = moe.moe_capacity(wl.T, wl.k, wl.E, wl.capacity_factor)
    s = moe.MoeShape(T=wl.T, d=wl.d, E=wl.E, k=wl.k, H=wl.H, H_s=wl.H_s, capacity=C, act=wl.act, wfmt=wl.wfmt,
                     renorm=wl.renorm)
    ws = moe.workspace(s, device)
    out = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device=device)
    return s, inp, ws, out


def int4_weights(moe, wl, seed, device):
    """Experts drawn in fp32 one at a time (synth) and packed by the library's INT4 quantiser."""
    import torch

    import synth
    E, d, H = wl.E, wl.d, wl.H
    out = dict(w13=torch.empty(E, 2 * H, d // 2, dtype=torch.uint8, device=device),
               s13=torch.empty(E, 2 * H, d // 128, dtype=torch.bfloat16, device=device),
               w2=torch.empty(E, d, H // 2, dtype=torch.uint8, device=device),
               s2=torch.empty(E, d, H // 128, dtype=torch.bfloat16, device=device))
    for e in range(E):
        a, b = synth.expert_weights_f32(wl, seed, e, device)
        moe.moe_quantize_int4(a, q=out["w13"][e], scales=out["s13"][e])
        moe.moe_quantize_int4(b, q=out["w2"][e], scales=out["s2"][e])
    if wl.H_s:
        a, b = synth.expert_weights_f32(wl, seed, E, device)
        q13, s13 = moe.moe_quantize_int4(a)
        q2, s2 = moe.moe_quantize_int4(b)
        out.update(w13_sh=q13[None], s13_sh=s13[None], w2_sh=q2[None], s2_sh=s2[None])
    torch.cuda.synchronize()
    return out


def run_forward(moe, s, inp, ws, out, aux, side=None):
    return moe.moe_forward(s, inp["x"], inp["w_router"], inp["w13"], inp["w2"], bias=inp["bias"],
                           s13=inp.get("s13"), s2=inp.get("s2"), w13_sh=inp.get("w13_sh"),
                           s13_sh=inp.get("s13_sh"), w2_sh=inp.get("w2_sh"), s2_sh=inp.get("s2_sh"), out=out,
                           ws=ws, aux=aux, side_stream=side)


def stage_times(moe, s, inp, ws, wl, flush, reps=10):
    """Per-stage device time (us): each stage of the pipeline is captured through its component entry point
    (moe_route, moe_permute, moe_expert_ffn routed / shared, moe_combine) into its own CUDA graph; the
    graphs are replayed back to back with events between them, L2 flushed before each repetition."""
    import torch
    names = ["route", "permute", "expert_ffn", "shared_ffn", "combine"]
    ws2 = torch.empty_like(ws)   # the permute reads the chunk table the route left in its own workspace
    state = {}

    def st_route():
        state["r"] = moe.moe_route(s, inp["x"], inp["w_router"], inp["bias"], ws=ws)

    pout = moe.permute_outputs(s, inp["x"].device)   # allocated and filled once, outside the timed graphs

    def st_permute():
        state["p"] = moe.moe_permute(s, inp["x"], state["r"]["topk_idx"], ws=ws2, out=pout)

    def st_ffn():
        p = state["p"]
        state["y"] = moe.moe_expert_ffn(s, p["x_perm"], inp["w13"], inp["w2"], group_start=p["offsets"],
                                        group_rows=p["kept"], s13=inp.get("s13"), s2=inp.get("s2"))[1]

    def st_shared():
        state["ysh"] = None
        if wl.H_s:
            state["ysh"] = moe.moe_expert_ffn(s, inp["x"], inp["w13_sh"], inp["w2_sh"], hidden=wl.H_s,
                                              s13=inp.get("s13_sh"), s2=inp.get("s2_sh"))[1]

    def st_combine():
        state["out"] = moe.moe_combine(s, state["y"], state["p"]["slot_pos"], state["r"]["topk_w"], state["ysh"])

    fns = [st_route, st_permute, st_ffn, st_shared, st_combine]
    if not wl.H_s:                      # no shared expert: no stage (an empty graph would still cost a replay)
        names.remove("shared_ffn")
        fns.remove(st_shared)
        state["ysh"] = None
    for f in fns:                       # eager warm-up (allocations, attributes)
        f()
    torch.cuda.synchronize()
    graphs = []
    for f in fns:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            f()
        graphs.append(g)
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(fns) + 1)]
    acc = {k: [] for k in names}
    for _ in range(reps):
        flush()
        ev[0].record(st)
        for i, g in enumerate(graphs):
            g.replay()
            ev[i + 1].record(st)
        torch.cuda.synchronize()
        for i, k in enumerate(names):
            acc[k].append(ev[i].elapsed_time(ev[i + 1]) * 1e3)
    kept = int(state["p"]["kept"].sum())
    touched = int((state["p"]["kept"] > 0).sum())
    del graphs
    out = {k: statistics.median(v) for k, v in acc.items()}
    if not wl.H_s:
        out["shared_ffn"] = 0.0
    return out, kept, touched


def _blas_threads(cores):
    try:
        from threadpoolctl import threadpool_info
        n = max([i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"] or [0])
        return min(cores, n) if n else cores
    except Exception:  # noqa: BLE001
        return cores


class OracleRunner:
    """The float64 oracle on one workload, inputs drawn once (seed 0, CPU generators).

    bf16 workloads: one call = one full-size forward of the whole batch (T tokens).  INT4 decode workload:
    the whole batch is routed once at set-up; one call = the next token of the batch, whose k experts and
    the shared expert are drawn, quantised, dequantised and applied by the oracle (the float64 experts of
    the whole layer would not fit in host memory)."""

    def __init__(self, wl):
        import torch

        import oracle as O
        import synth
        self.wl, self.O, self.synth = wl, O, synth
        self.cap = O.capacity(wl.T, wl.k, wl.E, wl.capacity_factor)
        f64 = lambda t: t.to(torch.float64).numpy() if t is not None else None  # noqa: E731
        if wl.wfmt == 0:
            inp = synth.make_inputs(wl, seed=0, device="cpu")
            self.args = {k: f64(inp.get(k)) for k in ("x", "w_router", "bias", "w13", "w2", "w13_sh", "w2_sh")}
        else:
            inp = synth.make_inputs(wl, seed=0, device="cpu", with_expert_weights=False)
            self.x = f64(inp["x"])
            self.r = O.route(self.x, f64(inp["w_router"]), f64(inp["bias"]), wl.k, bool(wl.renorm))
            self.next_t = 0

    def _expert(self, e):
        O = self.O
        a, b = self.synth.expert_weights_f32(self.wl, 0, e, "cpu")
        qa, sa = O.quantize_int4_g128(a.numpy())
        qb, sb = O.quantize_int4_g128(b.numpy())
        return O.dequantize_int4_g128(O.pack_int4(qa), sa), O.dequantize_int4_g128(O.pack_int4(qb), sb)

    def __call__(self) -> int:
        """One unit of oracle work; returns the tokens it covered."""
        import numpy as np
        wl, O = self.wl, self.O
        if wl.wfmt == 0:
            a = self.args
            O.moe_forward(a["x"], a["w_router"], a["bias"], a["w13"], a["w2"], k=wl.k, act=wl.act,
                          renorm=bool(wl.renorm), cap=self.cap, w13_sh=a["w13_sh"], w2_sh=a["w2_sh"])
            return wl.T
        t = self.next_t
        self.next_t = (t + 1) % wl.T
        out = np.zeros(wl.d)
        for j in range(wl.k):
            w13, w2 = self._expert(int(self.r["idx"][t, j]))
            out += self.r["w"][t, j] * O.expert_ffn(self.x[t:t + 1], w13, w2, wl.act)[0]
        if wl.H_s:
            w13, w2 = self._expert(wl.E)
            out += O.expert_ffn(self.x[t:t + 1], w13, w2, wl.act)[0]
        return 1

    def describe(self, done, el):
        if self.wl.wfmt == 0:
            return f"{done} tokens ({done // self.wl.T} full {self.wl.T}-token forwards of the {self.wl.name} " \
                   f"workload) in {el:.1f} s"
        return f"{done} tokens of the {self.wl.name} workload (batch routed once; each token's {self.wl.k} experts " \
               f"and the shared expert drawn, quantised and dequantised per token) in {el:.1f} s"


def cpu_oracle_sample(wl, budget_s=12.0, single_thread=False):
    """Time the float64 oracle on the workload for about ``budget_s`` seconds (at least one call).
    Returns (tokens/s, sample description, threads used)."""
    cores = len(os.sched_getaffinity(0))
    run = OracleRunner(wl)
    limit = None
    if single_thread:
        from threadpoolctl import threadpool_limits
        limit = threadpool_limits(limits=1)
    try:
        threads = 1 if single_thread else _blas_threads(cores)
        done, t0 = 0, time.perf_counter()
        while True:
            done += run()
            el = time.perf_counter() - t0
            if el >= budget_s:
                break
    finally:
        if limit is not None:
            limit.restore_original_limits()
    return done / el, run.describe(done, el), threads


# ------------------------------------------------------------------ main


def run_ep(args, wl, world, rank, device):
    """Expert-parallel timing: rank r holds experts [r E/N, (r + 1) E/N) and its own T tokens (weak scaling);
    without a capacity moe_forward_ep runs eagerly (its splits reach the host); with one the exchange has static
    shapes and the step is captured as a CUDA graph.  L2 flushed before every step; the step time is the max over
    ranks of the mean device time between events around each forward."""
    import socket
    from datetime import timedelta

    import torch
    import torch.distributed as dist

    import sparse_mixture_experts_expert_b200 as moe
    import synth
    from sparse_mixture_experts_expert_b200.ep import moe_forward_ep
    if wl.wfmt != synth.WFMT_BF16 or wl.E % world:
        raise SystemExit("--ep takes bf16 workloads whose experts split evenly over the ranks")
    own = not dist.is_initialized()
    if own:   # one rank: a process group of one, the exchanges are local copies
        sk = socket.socket()
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
        sk.close()
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                                timeout=timedelta(seconds=120), device_id=device)
    s, inp, _, _ = setup(wl, rank, device)
    E_loc = wl.E // world
    mine = slice(rank * E_loc, (rank + 1) * E_loc)
    w13, w2 = inp["w13"][mine].contiguous(), inp["w2"][mine].contiguous()
    flushbuf = torch.empty(256 << 20, dtype=torch.uint8, device=device)

    def step():
        return moe_forward_ep(s, inp["x"], inp["w_router"], w13, w2, bias=inp["bias"], w13_sh=inp.get("w13_sh"),
                              w2_sh=inp.get("w2_sh"))

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    run = step
    graph = None
    if s.capacity > 0:   # static shapes, no host synchronisation: the whole step replays as one CUDA graph
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        run = graph.replay
        run()
        torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        for a, b in evs:
            flushbuf.fill_(1)
            a.record()
            run()
            b.record()
        torch.cuda.synchronize()
    dist.barrier()
    status, site = moe.moe_get_status()
    if status != 0:
        raise RuntimeError(f"device status {status} at {site:#x} in the timed region")
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs) / args.steps, world)
    if rank == 0:
        cfg = bench_config(wl, s.capacity, world)
        cfg["parallelism"] = (f"expert-parallel x{world} (E/N experts per rank, NCCL all-to-all"
                              + (", static shapes with the capacity)" if s.capacity else "-v)"))
        print(json.dumps({"metric": METRIC, "value": world * wl.T / (ms * 1e-3), "unit": "tokens/s",
                          "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                          "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                          "data": "synthetic", "config": cfg,
                          "mode": "expert-parallel" + (", CUDA graph" if graph is not None else ", eager"),
                          "clocks": clk.summary()}), flush=True)
    del graph   # before the process group goes: a graph that holds NCCL calls is released first
    if own:
        dist.destroy_process_group()


def run_backward(args, wl, world, rank, device):
    """Backward timing: one moe_backward (forward recompute, input and weight gradients) captured as a CUDA graph
    and replayed per step, L2 flushed before every step; tokens/s and the bf16 GEMM work over the step time."""
    import torch

    import sparse_mixture_experts_expert_b200 as moe
    import synth
    if wl.wfmt != synth.WFMT_BF16:
        raise SystemExit("--backward takes bf16 workloads")
    s, inp, _, _ = setup(wl, rank, device)
    g = torch.Generator(device=device).manual_seed(1234 + rank)
    dout = torch.randn(wl.T, wl.d, generator=g, device=device).to(torch.bfloat16)
    t13, t2 = moe.moe_transpose_experts(inp["w13"]), moe.moe_transpose_experts(inp["w2"])
    t13s = moe.moe_transpose_experts(inp["w13_sh"]) if wl.H_s else None
    t2s = moe.moe_transpose_experts(inp["w2_sh"]) if wl.H_s else None
    n = ctypes.c_size_t(0)
    moe.load().moe_backward_workspace_size(ctypes.byref(s), ctypes.byref(n))
    ws = torch.empty(int(n.value), dtype=torch.uint8, device=device)

    side = torch.cuda.Stream() if not args.one_stream else None   # the shared expert's chain runs beside

    def step():
        return moe.moe_backward(s, inp["x"], inp["w_router"], inp["w13"], inp["w2"], dout, bias=inp["bias"],
                                w13t=t13, w2t=t2, w13_sh=inp.get("w13_sh"), w2_sh=inp.get("w2_sh"),
                                w13t_sh=t13s, w2t_sh=t2s, aux_coef=0.01, ws=ws, side_stream=side)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    launches0 = moe.moe_launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    per_step = moe.moe_launch_count() - launches0
    flushbuf = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        for a, b in evs:
            flushbuf.fill_(1)
            a.record()
            graph.replay()
            b.record()
        torch.cuda.synchronize()
    status, site = moe.moe_get_status()
    if status != 0:
        raise RuntimeError(f"device status {status} at {site:#x} in the timed region")
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs) / args.steps, world)
    # bf16 GEMM work per row: the recomputed [g | u] (2 H d), dout W2 (H d), dx = [dg | du] W13 (2 H d), the
    # weight gradients dW13 (2 H d) and dW2 (H d), for the kept grouped rows and the shared expert's tokens;
    # the router's dz W_r and dW_r (E d each per token)
    kept = int(moe.moe_permute(s, inp["x"], moe.moe_route(s, inp["x"], inp["w_router"], inp["bias"])["topk_idx"])
               ["kept"].sum())
    flops = 2.0 * 8 * (kept * wl.H + wl.T * wl.H_s) * wl.d + 2.0 * 2 * wl.T * wl.E * wl.d
    peaks = load_peaks()
    if rank == 0:
        metric = "MoE-layer backward (input and weight gradients) tokens/s on 1 B200; % of bf16 tensor-core roofline"
        print(json.dumps({"metric": metric,
                          "value": world * wl.T / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world,
                          "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                          "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                          "config": bench_config(wl, s.capacity, world),
                          "mode": "backward (input and weight gradients)" + (", one stream" if args.one_stream else
                                                                            ", shared expert on a side stream"),
                          "roofline": {"bound": "tensor", "kernel": "whole moe_backward",
                                       "achieved": flops / (ms * 1e-3) / 1e12, "peak": peaks["bf16_tflops"],
                                       "unit": "TFLOP/s", "frac": flops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                                       "peak_source": peaks["source"] + " burst bf16", "alg_flops_per_step": flops},
                          "gpu_launches": per_step * args.steps, "clocks": clk.summary()}), flush=True)
    del graph


def run_tree(args, wl, world, rank, device):
    """Hierarchical router timing: moe_route_tree over branch**levels experts on the workload's tokens, captured
    as a CUDA graph and replayed per step, L2 flushed before every step.  tokens/s, and the HBM roofline of its
    algorithmic bytes (x, the level routers, the level logits written and read back, the picks)."""
    import torch

    import sparse_mixture_experts_expert_b200 as moe
    import synth
    B, L = args.tree_branch, args.tree_levels
    E = B ** L
    inp = synth.draw_tree_router(wl.T, wl.d, B, L, seed=1234 + rank, device=device)
    s = moe.MoeShape(T=wl.T, d=wl.d, E=E, k=wl.k, H=16, renorm=1)
    n = ctypes.c_size_t(0)
    moe.load().moe_route_tree_workspace_size(ctypes.byref(s), B, L, ctypes.byref(n))
    ws = torch.empty(int(n.value), dtype=torch.uint8, device=device)

    def step():
        return moe.moe_route_tree(s, B, L, inp["x"], inp["w_tree"], ws=ws)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    launches0 = moe.moe_launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    per_step = moe.moe_launch_count() - launches0
    flushbuf = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        for a, b in evs:
            flushbuf.fill_(1)
            a.record()
            graph.replay()
            b.record()
        torch.cuda.synchronize()
    status, site = moe.moe_get_status()
    if status != 0:
        raise RuntimeError(f"device status {status} at {site:#x} in the timed region")
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs) / args.steps, world)
    nl = B * L
    alg = wl.T * wl.d * 2 + nl * wl.d * 4 + 2 * wl.T * nl * 4 + wl.T * wl.k * 8
    peaks = load_peaks()
    if rank == 0:
        cfg = bench_config(wl, 0, world)
        cfg.update(E=E, router=f"tree, branch {B}, levels {L} ({nl} level logits per token)", H=None, H_s=None)
        print(json.dumps({"metric": f"hierarchical router tokens/s over {E} experts on 1 B200",
                          "value": world * wl.T / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world,
                          "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                          "scaling": "weak", "vs_baseline": None, "dtype": "fp32", "data": "synthetic",
                          "config": cfg, "mode": "router only (moe_route_tree)",
                          "roofline": {"bound": "hbm", "kernel": "whole moe_route_tree",
                                       "achieved": alg / (ms * 1e-3) / 1e9, "peak": peaks["hbm_gbs"],
                                       "unit": "GB/s", "frac": alg / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                       "peak_source": peaks["source"] + " copy", "alg_bytes_per_step": alg},
                          "gpu_launches": per_step * args.steps, "clocks": clk.summary()}), flush=True)
    del graph


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ep", action="store_true",
                    help="expert-parallel forward instead of replicas: each of the N ranks holds E / N experts and "
                         "T tokens; the rows travel by NCCL all-to-all (bf16 workloads; with a capacity the "
                         "exchange has static shapes)")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward (moe_backward: input and weight gradients, bf16 experts) instead of the "
                         "forward")
    ap.add_argument("--one-stream", action="store_true",
                    help="keep the shared expert on the main stream (by default it runs on a side stream, "
                         "beside the routed path)")
    ap.add_argument("--tree", action="store_true",
                    help="time the hierarchical router (moe_route_tree) on the workload's tokens, d and k over "
                         "--tree-branch ** --tree-levels experts, instead of the forward")
    ap.add_argument("--tree-branch", type=int, default=16)
    ap.add_argument("--tree-levels", type=int, default=3)
    ap.add_argument("--experts", type=int, default=0,
                    help="profiling only: run the workload with this many experts (a small case for ncu); the "
                         "line's config names it")
    args = ap.parse_args()

    import synth
    wl = synth.get_workload(args.workload)
    if args.experts:
        wl = wl.replace(E=args.experts)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        cores = len(os.sched_getaffinity(0))
        run = OracleRunner(wl)
        threads = _blas_threads(cores)
        times, done = [], 0
        for i in range(args.warmup + args.steps):
            t0 = time.perf_counter()
            n = run()
            el = time.perf_counter() - t0
            if i >= args.warmup:
                times.append(el)
                done += n
        total = sum(times)
        val = done / total
        line = {"metric": METRIC, "value": val, "unit": "tokens/s", "impl": "reference", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / args.steps * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": bench_config(wl, run.cap, world),
                "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                 "sample": run.describe(done, total) + " (timed steps only)"},
                "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist

    import sparse_mixture_experts_expert_b200 as moe
    moe.load()
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    device = torch.device("cuda", torch.cuda.current_device())
    if args.ep:
        run_ep(args, wl, world, rank, device)
        return
    if args.backward:
        run_backward(args, wl, world, rank, device)
        return
    if args.tree:
        run_tree(args, wl, world, rank, device)
        return
    s, inp, ws, out = setup(wl, rank, device)
    flushbuf = torch.empty(256 << 20, dtype=torch.uint8, device=device)

    def flush():
        flushbuf.fill_(1)

    st = torch.cuda.current_stream()
    side = torch.cuda.Stream() if not args.one_stream else None   # the shared expert beside the routed path
    for _ in range(max(3, args.warmup)):
        run_forward(moe, s, inp, ws, out, wl.aux, side)
    torch.cuda.synchronize()
    status, site = moe.moe_get_status()
    if status != 0:
        raise RuntimeError(f"device status {status} at {site:#x} during warm-up")

    # One forward captured into a CUDA graph (the launch-bound small workloads would otherwise time the
    # host); the graph replays exactly the kernels moe_forward enqueues.
    launches0 = moe.moe_launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run_forward(moe, s, inp, ws, out, wl.aux, side)
    per_step_launches = moe.moe_launch_count() - launches0
    torch.cuda.synchronize()
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        for a, b in evs:
            flush()
            a.record(st)
            graph.replay()
            b.record(st)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    launches = per_step_launches * args.steps
    step_ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    status, site = moe.moe_get_status()
    if status != 0:
        raise RuntimeError(f"device status {status} at {site:#x} in the timed region")
    step_ms = max_over_ranks(step_ms, world)
    value = world * wl.T / (step_ms * 1e-3)

    # End to end through the public API with host buffers, as a serving loop runs it: every step copies its
    # input from pinned host memory, runs moe_forward (L2 flushed first) and copies its result back to pinned
    # host memory.  The copies run on their own streams with two device buffer sets, so step i + 1's input
    # copy and step i - 1's result copy overlap step i's forward.  Time: first copy in to last copy out.
    x_host = inp["x"].cpu().pin_memory()
    out_host = [torch.empty(wl.T, wl.d, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(inp["x"]) for _ in range(2)]
    out_dev = [torch.empty_like(out) for _ in range(2)]
    cs, hs, ds = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_run(nsteps):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        h2d_done = [torch.cuda.Event() for _ in range(nsteps)]
        fwd_done = [torch.cuda.Event() for _ in range(nsteps)]
        d2h_done = [torch.cuda.Event() for _ in range(nsteps)]
        t0.record(hs)
        for i in range(nsteps):
            b = i & 1
            with torch.cuda.stream(hs):
                if i >= 2:
                    hs.wait_event(fwd_done[i - 2])        # the forward of step i - 2 has read x_dev[b]
                x_dev[b].copy_(x_host, non_blocking=True)
                h2d_done[i].record(hs)
            with torch.cuda.stream(cs):
                cs.wait_event(h2d_done[i])
                if i >= 2:
                    cs.wait_event(d2h_done[i - 2])        # out_dev[b] of step i - 2 has been copied out
                flush()
                inp_i = dict(inp)
                inp_i["x"] = x_dev[b]
                run_forward(moe, s, inp_i, ws, out_dev[b], wl.aux, side)
                fwd_done[i].record(cs)
            with torch.cuda.stream(ds):
                ds.wait_event(fwd_done[i])
                out_host[b].copy_(out_dev[b], non_blocking=True)
                d2h_done[i].record(ds)
        ds.wait_event(d2h_done[-1])
        t1.record(ds)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    e2e_run(max(3, args.warmup))
    e2e_ms = max_over_ranks(e2e_run(args.steps) / args.steps, world)
    status, site = moe.moe_get_status()
    if status != 0:
        raise RuntimeError(f"device status {status} at {site:#x} in the end-to-end run")

    # stage breakdown and the roofline of the grouped expert GEMMs
    stages, kept, touched = stage_times(moe, s, inp, ws, wl, flush)
    peaks = load_peaks()
    flops = wl.flops_tc(kept)
    gemm_us = stages["expert_ffn"] + (stages["shared_ffn"] if wl.H_s else 0.0)
    if wl.wfmt == synth.WFMT_INT4_G128:
        alg_bytes = int4_step_bytes(wl, touched)
        achieved = alg_bytes / (step_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        roofline = {"bound": "hbm", "kernel": "whole moe_forward (INT4 weight streaming dominates)",
                    "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                    "peak_source": peaks["source"] + " HBM copy", "traffic": None,
                    "alg_bytes_per_step": alg_bytes, "touched_experts": touched,
                    "int4_gemm_GBps": (alg_bytes - wl.T * wl.d * 4 - wl.E * wl.d * 4) / (gemm_us * 1e-6) / 1e9}
    else:
        achieved_tf = flops / (gemm_us * 1e-6) / 1e12
        peak_tf = peaks["bf16_tflops"]
        gbytes = gemm_step_bytes(wl, kept, touched)
        roofline = {"bound": "tensor", "kernel": "k_grouped_gemm (gate/up + GLU, down; routed + shared)",
                    "achieved": achieved_tf, "peak": peak_tf, "unit": "TFLOP/s", "frac": achieved_tf / peak_tf,
                    "peak_source": peaks["source"] + " burst bf16",
                    "traffic": None if args.experts else GEMM_TRAFFIC_BYTES.get(wl.name),
                    "alg_flops_per_step": flops, "gemm_us": gemm_us,
                    # the same kernels against HBM: operands and results they must move (grouped rows, weights of
                    # the touched experts, h written and read back, y written)
                    "hbm_view": {"alg_bytes_per_step": gbytes, "achieved_GBps": gbytes / (gemm_us * 1e-6) / 1e9,
                                 "peak_GBps": peaks["hbm_gbs"],
                                 "frac": gbytes / (gemm_us * 1e-6) / 1e9 / peaks["hbm_gbs"]}}

    if rank == 0:
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            v, sample, cores = cpu_oracle_sample(wl, budget_s=12.0)
            cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample}
            if wl.name in ("tiny", "small"):
                v1, sample1, _ = cpu_oracle_sample(wl, budget_s=6.0, single_thread=True)
                cpu["single_thread"] = {"value": v1, "unit": "tokens/s", "cores": 1, "sample": sample1}
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": bench_config(wl, s.capacity, world),
                "roofline": roofline, "stages_us": stages, "cpu_baseline": cpu,
                "e2e": {"value": world * wl.T / (e2e_ms * 1e-3), "unit": "tokens/s",
                        "h2d_bytes_per_step": x_host.numel() * 2, "d2h_bytes_per_step": out_host[0].numel() * 2,
                        "ms_per_step": e2e_ms,
                        "overlap": "copy streams: step i+1's H2D and step i-1's D2H overlap step i's forward"},
                "gpu_launches": launches, "launches_per_step": per_step_launches,
                "timing": "CUDA graph of one moe_forward replayed per step (value); e2e calls the API eagerly, "
                          "copies pipelined with the forwards; shared expert "
                          + ("on the main stream" if args.one_stream else "on a side stream beside the routed path"),
                "clocks": clk.summary()}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
