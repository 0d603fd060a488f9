#!/usr/bin/env python
"""Benchmark of the NVFP4 routed-expert MoE layer on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload all|prefill|decode1|decode8|decode32|decode64|codec|layer|w4a4]

A step is one pass of the whole layer (route -> gate/up + SwiGLU -> down -> combine) over
one batch of the H=6144, I=2048, E=256, top-8 layer whose NVFP4 weights (5.4 GB, N(0,0.02)
bf16 quantized by the library) stay resident in HBM.  The headline line is the largest
single-GPU configuration, prefill of T=4096 tokens with Zipf-like routing (x ~ N(0,1); expert
e gets router-logit bias 1.5 ln(1/(e+1)) plus N(0,1) noise; top-8).  Every timed step routes
a NEW batch, so the expert bytes it reads are not left in the 126 MB L2 by the step before.
Steps are replayed from a CUDA graph and timed with CUDA events on the launching stream.

With --workload all (the default, one GPU) the line also carries `sub_records`: decode of
T = 1, 8, 32 and 64 tokens (HBM-bound GEMV path), the BF16 shared expert and the whole layer
(router + routed + shared) at T = 1 and 4096, the prefill batch on the FP4 tensor cores
(W4A4), and the whole-layer codec legs, each timed the same way with its own step count,
clock samples and roofline.

Keys beyond the base contract: `roofline` (dominant kernel; live CUDA-event durations of
each stage from a second, marked pass), `cpu_baseline` (the CPU oracle on a bounded
sample, rank 0 at N=1), `e2e` (the same metric through the C ABI with pinned host
buffers, copies inside the timed region), `clocks`, `gpu_launches`.

--impl reference times the CPU oracle itself on the host cores (the reference arm).
With torchrun (N>1) the layer runs expert parallel (--parallel ep, the default there):
rank r holds only the experts e % N == r, every rank routes the same batch of T tokens,
and one NCCL reduce-scatter sums the ranks' fp32 partial outputs (strong scaling: the job
processes T tokens per step).  --parallel replicas instead runs an independent token stream
per rank (weak scaling, no collective on the data path).  --parallel ep on one GPU runs the
same code with one rank.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "MoE-layer tokens/s"
H, I, K = 6144, 2048, 8
E = 256
GATEUP_BYTES_PER_EXPERT = 2 * I * (H // 2 + H // 16)      # 14,155,776
DOWN_BYTES_PER_EXPERT = H * (I // 2 + I // 16)            # 7,077,888
EXPERT_BYTES = GATEUP_BYTES_PER_EXPERT + DOWN_BYTES_PER_EXPERT


def measured_traffic(kernel):
    """DRAM bytes per launch of `kernel` from the committed ncu summary (profiles/), or None
    when no capture of the current kernel is recorded."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            return json.load(f).get(kernel, {}).get("dram_bytes_per_launch")
    except (OSError, ValueError):
        return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle sampling in the background during the timed region.

    Sampling starts `pre_s` seconds before the region; meanwhile `busy` (untimed replays of
    the same work on `stream`) keeps the GPU under the region's load, so the samples taken
    just before a short region describe the clocks it runs at."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, stream=None, busy=None, pre_s: float = 0.3):
        self.gpu = physical_gpu(gpu_index)
        self.stream, self.busy, self.pre_s = stream, busy, pre_s
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        t_end = time.perf_counter() + self.pre_s
        if self.busy is not None:
            with torch.cuda.stream(self.stream):
                while time.perf_counter() < t_end:
                    self.busy()
                    self.stream.synchronize()
        else:
            time.sleep(self.pre_s)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            out, _ = self.proc.communicate(timeout=10)
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def physical_gpu(local_index: int) -> str:
    """nvidia-smi's name for torch device `local_index` (CUDA_VISIBLE_DEVICES may remap)."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "").strip()
    if vis:
        parts = [p.strip() for p in vis.split(",") if p.strip()]
        if local_index < len(parts):
            return parts[local_index]
    return str(local_index)


# ----------------------------------------------------------------------------- setup
def build_layer(nv, device, seed=0, experts=None):
    """The layer's experts (all E, or the listed global ids in that order), bf16 N(0,0.02)
    drawn on the GPU per expert id and quantized by the library."""
    experts = list(range(E)) if experts is None else list(experts)
    dev = []
    for proj, shape in (("w_gu", (2 * I, H)), ("w_dn", (H, I))):
        x = torch.empty((len(experts),) + shape, dtype=torch.bfloat16, device=device)
        for n, e in enumerate(experts):
            x[n] = synth.normal_bf16(shape, seed, proj, e, std=0.02, device=device)
        dev += list(nv.nvfp4_quantize(x))
        del x
    torch.cuda.empty_cache()
    return dev


def workload_of(name):
    if name.startswith("decode"):
        T = int(name[len("decode"):])
        return synth.decode_batch(T) if T > 1 else synth.DECODE_T1
    if name == "prefill":
        return synth.PREFILL_T4096
    if name == "codec":
        return synth.CODEC_LAYER
    raise SystemExit(f"unknown workload {name}")


def make_batches(wl, n_batches, seed, device):
    """n_batches independent batches of T tokens: x, ids, w on the device."""
    T = wl.T
    xs = synth.activations_bf16(n_batches * T, H, seed, device=device).view(n_batches, T, H)
    ids, w = synth.routing(n_batches * T, E, K, seed=seed, zipf_bias=wl.zipf_bias)
    return xs, ids.view(n_batches, T, K).to(device), w.view(n_batches, T, K).to(device)


# ----------------------------------------------------------------------------- CPU baseline
def random_nvfp4_pool(pool, seed=11, i_rows=I):
    """NVFP4 weights for `pool` experts drawn directly as random E2M1 codes and E4M3 scales
    (for timing the oracle, whose cost does not depend on the values).  i_rows < I gives a
    slice of the layer: the first i_rows gate and up rows and the matching down columns."""
    rng = np.random.default_rng(seed)
    pg = rng.integers(0, 256, (pool, 2 * i_rows, H // 2), dtype=np.uint8)
    sg = rng.integers(0x30, 0x58, (pool, 2 * i_rows, H // 16), dtype=np.uint8)
    pd = rng.integers(0, 256, (pool, H, i_rows // 2), dtype=np.uint8)
    sd = rng.integers(0x30, 0x58, (pool, H, i_rows // 16), dtype=np.uint8)
    g = np.full((pool,), 1e-3, np.float32)
    return pg, sg, g, pd, sd, g.copy()


def cpu_baseline(wl, n_tokens=24, seed=7):
    """The CPU oracle on a bounded sample of the workload: n_tokens tokens of a batch routed
    like `wl` (Zipf bias for prefill) to 8 of a pool of 16 experts, as one oracle call."""
    import oracle
    pool = 16
    weights = random_nvfp4_pool(pool)
    ids, w = synth.routing(n_tokens, pool, K, seed=seed, zipf_bias=wl.zipf_bias)
    x = synth.activations_bf16(n_tokens, H, seed)
    t0 = time.perf_counter()
    oracle.moe_forward(x, ids, w, *weights)
    total = time.perf_counter() - t0
    return {"value": n_tokens / total, "unit": "tokens/s", "cores": oracle.threads(),
            "kind": "oracle",
            "sample": f"{n_tokens} tokens of the {wl.name} workload (routing over a pool of "
                      f"{pool} experts; fp64, {oracle.threads()} OpenMP threads)"}


# ----------------------------------------------------------------------------- ours
class Bench:
    """One device, one resident layer: times workloads of the layer and the codec."""

    def __init__(self, nv, args, rank, world, device):
        self.nv, self.args, self.rank, self.world, self.device = nv, args, rank, world, device
        self.peaks = load_peaks()
        self.layer = None

    def ensure_layer(self):
        if self.layer is None:
            self.layer = build_layer(self.nv, self.device)
        return self.layer

    def drop_layer(self):
        self.layer = None
        torch.cuda.empty_cache()

    def layer_record(self, name, steps, warmup, main):
        """Time `steps` steps of workload `name` (after `warmup` untimed steps)."""
        nv, args, world, device = self.nv, self.args, self.world, self.device
        peaks = self.peaks
        wl = workload_of(name)
        T = wl.T
        layer = self.ensure_layer()
        G = min(steps, args.graph_steps if T <= 64 else 2)   # steps per graph replay
        n_b = max(G, warmup)
        xs, ids, ws_ = make_batches(wl, n_b, seed=1000 + self.rank, device=device)
        ws = nv.alloc_moe_workspace(T, H, I, E, K, device)
        out = torch.empty((T, H), dtype=torch.bfloat16, device=device)
        path = args.path

        def step(i):
            nv.moe_nvfp4_forward(xs[i], ids[i], ws_[i], *layer, out=out, workspace=ws,
                                 path=path)

        for i in range(warmup):
            step(i % n_b)
        torch.cuda.synchronize()

        stream = torch.cuda.Stream(device)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            step(0)
            stream.synchronize()
            with torch.cuda.graph(graph, stream=stream):
                for i in range(G):
                    step(i)
        reps, rem = divmod(steps, G)
        tail_graph = None
        if rem:
            tail_graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(tail_graph, stream=stream):
                for i in range(rem):
                    step(i)
        graph.replay()
        torch.cuda.synchronize()

        barrier(world)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(torch.cuda.current_device(), stream, graph.replay) as clk:
            torch.cuda.synchronize()
            ev0.record(stream)
            with torch.cuda.stream(stream):
                for _ in range(reps):
                    graph.replay()
                if tail_graph is not None:
                    tail_graph.replay()
            ev1.record(stream)
            torch.cuda.synchronize()
        barrier(world)
        ms_total = max_over_ranks(ev0.elapsed_time(ev1), world, device)
        ms_step = ms_total / steps

        # marked pass: per-stage durations from events between the kernels
        n_mark = min(G, 64)
        marks = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(n_mark)]
        for m in marks:          # torch creates the CUDA event on its first record
            for e in m:
                e.record()
        torch.cuda.synchronize()
        mgraph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(mgraph, stream=stream):
                for i in range(n_mark):
                    nv.moe_nvfp4_forward_profiled(xs[i], ids[i], ws_[i], *layer, out, ws,
                                                  marks[i], path=path)
            mgraph.replay()
        torch.cuda.synchronize()
        stages = {n: statistics.mean(m[j].elapsed_time(m[j + 1]) for m in marks)
                  for j, n in enumerate(["route", "gate_up", "down", "combine"])}
        marked_step = statistics.mean(m[0].elapsed_time(m[4]) for m in marks)

        uniq = statistics.mean(len(set(ids[i].flatten().tolist())) for i in range(G))
        bytes_step = uniq * EXPERT_BYTES
        flops_step = 2 * T * K * (3 * H * I)
        value = T * steps * world / (ms_total / 1e3)

        gemv = path == 1 or (path == 0 and T <= 64)
        if gemv:   # HBM-bound: the gate/up GEMV streams 2/3 of the expert bytes
            gu_ms = stages["gate_up"]
            achieved = uniq * GATEUP_BYTES_PER_EXPERT / (gu_ms / 1e3) / 1e9
            kname = "gemv_gateup_kernel" if T == 1 else "gemv_mma_kernel<0>"
            roof = {"kernel": kname + " (gate/up + SwiGLU)", "bound": "hbm",
                    "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": achieved / peaks["hbm_gbs"], "traffic": measured_traffic(kname),
                    "algorithmic_bytes": uniq * GATEUP_BYTES_PER_EXPERT,
                    "peak_source": peaks["source"] + " (burst copy)"}
            launches = 2 if T == 1 else 3
        else:
            gu_ms = stages["gate_up"]
            fl = 2 * T * K * (2 * I * H)
            achieved = fl / (gu_ms / 1e3) / 1e12
            pk = peaks["bf16_tflops"]
            roof = {"kernel": "gemm_kernel mode 0 (tcgen05 grouped GEMM + SwiGLU)",
                    "bound": "tensor", "achieved": achieved, "peak": pk, "unit": "TFLOP/s",
                    "frac": achieved / pk, "traffic": measured_traffic("gemm_kernel_gateup"),
                    "algorithmic_flops": fl,
                    "peak_source": peaks["source"] + " (cuBLAS bf16 burst; the f16 MMA has the "
                                                     "same dense rate)"}
            launches = 5    # route, gather, gate/up GEMM, down GEMM, combine

        e2e = run_e2e(nv, layer, wl, args, device, ws, path)
        rec = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": steps, "warmup": warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f16/bf16 products of NVFP4 weights, f32 accumulation",
            "data": "synthetic (seeded N(0,1) tokens, N(0,0.02) bf16 weights quantized to NVFP4)",
            "config": {"workload": wl.name if E == 256 else wl.name.replace("E=256", f"E={E}"),
                       "T": T, "H": H, "I": I, "E": E, "K": K,
                       "weights": "NVFP4 (E2M1 + E4M3 per 16 + fp32 per tensor), "
                                  f"{E * EXPERT_BYTES / 1e9:.2f} GB resident",
                       "l2": "inputs larger than L2: every step routes new tokens over 5.4 GB "
                             "of expert weights (>126 MB L2)",
                       "timing": f"CUDA graph of {G} steps replayed, CUDA events",
                       "path": {0: "auto", 1: "gemv", 2: "gemm"}[path],
                       "parallelism": f"{world} independent replica(s), no data-path "
                                      "collective"},
            "hbm_gbs_step": bytes_step / (ms_step / 1e3) / 1e9,
            "tflops_step": flops_step / (ms_step / 1e3) / 1e12,
            "unique_experts_per_step": uniq,
            "stages_ms": stages, "marked_step_ms": marked_step,
            "roofline": roof,
            "e2e": e2e,
            "gpu_launches": launches * steps,
            "clocks": clk.summary(),
        }
        if main and self.rank == 0 and world == 1 and not args.no_cpu_baseline:
            rec["cpu_baseline"] = cpu_baseline(wl, args.cpu_tokens)
        del graph, tail_graph, mgraph, xs, ids, ws_, ws
        torch.cuda.empty_cache()
        return rec

    def ep_record(self, name, steps, warmup):
        """Expert parallelism over the `world` ranks: rank r holds only the experts
        e % world == r; every rank routes the same batch, runs its experts
        (moe_nvfp4_forward_ep), and an NCCL reduce-scatter sums the fp32 partials, leaving
        each rank T/world rows of the layer output (bf16, moe_nvfp4_ep_reduce).  A step is
        one batch of T tokens for the whole job (strong scaling)."""
        from bit_quantized_moe_nvfp4_b200 import ep
        nv, args, world, rank, device = self.nv, self.args, self.world, self.rank, self.device
        peaks = self.peaks
        wl = workload_of(name)
        T = wl.T
        mine = ep.local_experts(E, world, rank)
        layer = build_layer(nv, device, experts=mine)
        mode = "reduce_scatter" if T % world == 0 else "all_reduce"
        moe = ep.ExpertParallelMoE(E, layer, mode=mode, path=args.path)
        n_b = max(warmup, min(steps, 8))
        # the same tokens on every rank: one seed for the whole job
        xs, ids, ws_ = make_batches(wl, n_b, seed=1000, device=device)
        stream = torch.cuda.current_stream(device)

        def step(i):
            return moe.forward(xs[i], ids[i], ws_[i])

        for i in range(warmup):
            step(i % n_b)
        partial, summed, out, ws = moe._buffers(T, H, K, device)

        def busy():
            # this rank's experts only: the clock warm-up runs a different number of times
            # on each rank, so it must not hold a collective
            nv.moe_nvfp4_forward_ep(xs[0], ids[0], ws_[0], E, world, rank, *layer,
                                    out=partial, workspace=ws, path=args.path)

        barrier(world)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(torch.cuda.current_device(), stream, busy) as clk:
            torch.cuda.synchronize()
            ev0.record(stream)
            for i in range(steps):
                step(i % n_b)
            ev1.record(stream)
            torch.cuda.synchronize()
        barrier(world)
        ms_total = max_over_ranks(ev0.elapsed_time(ev1), world, device)
        ms_step = ms_total / steps

        # marked pass: this rank's experts, the exchange, the rounding
        marks = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        stage = {"experts": [], "exchange": [], "round": []}
        for i in range(min(steps, n_b)):
            marks[0].record(stream)
            nv.moe_nvfp4_forward_ep(xs[i], ids[i], ws_[i], E, world, rank, *layer,
                                    out=partial, workspace=ws, path=args.path)
            marks[1].record(stream)
            red = ep.reduce_partial(partial, mode=mode,
                                    out=summed if mode == "reduce_scatter" else None)
            marks[2].record(stream)
            nv.moe_nvfp4_ep_reduce([red], out=out)
            marks[3].record(stream)
            torch.cuda.synchronize()
            for j, k in enumerate(stage):
                stage[k].append(marks[j].elapsed_time(marks[j + 1]))
        stages = {k: statistics.mean(v) for k, v in stage.items()}
        stages = {k: max_over_ranks(v, world, device) for k, v in stages.items()}

        pairs = ids[:n_b].flatten().cpu()
        local_pairs = float((pairs % world == rank).sum()) / n_b
        fl_local = 2 * local_pairs * (3 * H * I)
        achieved = fl_local / (stages["experts"] / 1e3) / 1e12
        pk = peaks["bf16_tflops"]
        exch_bytes = T * H * 4 * (world - 1) / world   # reduce-scatter bytes out of a rank
        rec = {
            "metric": METRIC, "value": T * steps / (ms_total / 1e3), "unit": "tokens/s",
            "n_gpus": world, "steps": steps, "warmup": warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": "f16/bf16 products of NVFP4 weights, f32 accumulation",
            "data": "synthetic (seeded N(0,1) tokens, N(0,0.02) bf16 weights quantized to "
                    "NVFP4)",
            "config": {"workload": wl.name, "T": T, "H": H, "I": I, "E": E, "K": K,
                       "parallelism": f"expert parallel over {world} GPU(s): experts "
                                      f"e % {world} per rank, NCCL {mode} of fp32 partials",
                       "weights": f"{len(mine)} experts per rank "
                                  f"({len(mine) * EXPERT_BYTES / 1e9:.2f} GB)",
                       "l2": "every step routes a batch over the rank's expert weights "
                             "(>126 MB L2)",
                       "timing": "stream launches (no graph), CUDA events, max over ranks"},
            "stages_ms": stages,
            "roofline": {"kernel": "this rank's experts (route + tcgen05 GEMMs + combine)",
                         "bound": "tensor", "achieved": achieved, "peak": pk,
                         "unit": "TFLOP/s", "frac": achieved / pk, "traffic": None,
                         "algorithmic_flops": fl_local,
                         "peak_source": peaks["source"] + " (cuBLAS bf16 burst)"},
            "exchange": {"collective": f"NCCL {mode}", "bytes_out_per_rank": exch_bytes,
                         "ms": stages["exchange"],
                         "gbs": exch_bytes / (stages["exchange"] / 1e3) / 1e9
                         if stages["exchange"] > 0 else None},
            "gpu_launches": 6 * steps,   # route, gather, 2 GEMMs, combine, ep_reduce
            "clocks": clk.summary(),
        }
        rec["e2e"] = self.ep_e2e(moe, wl, mode)
        del moe, layer, xs, ids, ws_
        torch.cuda.empty_cache()
        return rec

    def ep_e2e(self, moe, wl, mode):
        """The expert-parallel step through the public API with host buffers: every rank
        copies the batch in from pinned memory and its kept rows of the output back."""
        from bit_quantized_moe_nvfp4_b200 import ep
        device, world, rank = self.device, self.world, self.rank
        T = wl.T
        n = 4
        xs = synth.activations_bf16(n * T, H, 77).view(n, T, H).pin_memory()
        ids, w = synth.routing(n * T, E, K, seed=77, zipf_bias=wl.zipf_bias)
        ids, w = ids.view(n, T, K).pin_memory(), w.view(n, T, K).pin_memory()
        rows = ep.kept_rows(T, world, rank, mode)
        out_h = torch.empty((n, rows.stop - rows.start, H), dtype=torch.bfloat16).pin_memory()
        xd = torch.empty((T, H), dtype=torch.bfloat16, device=device)
        idd = torch.empty((T, K), dtype=torch.int32, device=device)
        wd = torch.empty((T, K), dtype=torch.float32, device=device)

        def one(i):
            xd.copy_(xs[i], non_blocking=True)
            idd.copy_(ids[i], non_blocking=True)
            wd.copy_(w[i], non_blocking=True)
            out_h[i].copy_(moe.forward(xd, idd, wd), non_blocking=True)

        one(0)
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(n):
            one(i)
        e1.record()
        torch.cuda.synchronize()
        ms = max_over_ranks(e0.elapsed_time(e1), world, device)
        return {"value": n * T / (ms / 1e3), "unit": "tokens/s", "steps": n,
                "h2d_bytes_per_step": T * H * 2 + T * K * 4 * 2,
                "d2h_bytes_per_step": (rows.stop - rows.start) * H * 2}

    def codec_record(self, steps, warmup):
        """Whole-layer quantize + dequantize of all 256 experts (gate/up and down)."""
        nv, world, device, peaks = self.nv, self.world, self.device, self.peaks
        wl = synth.CODEC_LAYER
        xs = {}
        for proj, shape in (("w_gu", (2 * I, H)), ("w_dn", (H, I))):
            x = torch.empty((E,) + shape, dtype=torch.bfloat16, device=device)
            for e in range(E):
                x[e] = synth.normal_bf16(shape, wl.seed, proj, e, std=0.02, device=device,
                                         outlier_p=wl.outlier_p)
            xs[proj] = x
        outs = {p: nv.nvfp4_quantize(x) for p, x in xs.items()}
        qws = {p: torch.zeros((nv.nvfp4_quantize_workspace_size(*x.shape),), dtype=torch.uint8,
                              device=device) for p, x in xs.items()}
        deq = {p: torch.empty_like(x) for p, x in xs.items()}
        elts = sum(x.numel() for x in xs.values())
        stream = torch.cuda.current_stream(device)

        def q():
            for p, x in xs.items():
                nv.nvfp4_quantize(x, *outs[p], workspace=qws[p])

        def d():
            for p in xs:
                nv.nvfp4_dequantize(*outs[p], out=deq[p])

        # calibrated scales: the amax pass, and the quantizer with the amax given
        amx = {p: nv.nvfp4_amax(x) for p, x in xs.items()}

        def am():
            for p, x in xs.items():
                nv.nvfp4_amax(x, out=amx[p])

        def qa():
            for p, x in xs.items():
                nv.nvfp4_quantize_with_amax(x, amx[p], *outs[p])

        def q2():   # amax pass, then the quantizer with that amax
            am()
            qa()

        res = {}
        legs = (("quantize", q, 2.5625, "quantize_kernel"),
                ("dequantize", d, 2.5625, "dequantize_kernel"),
                ("amax", am, 2.0, "amax_kernel"),
                ("quantize_with_amax", qa, 2.5625, "quantize_amax_kernel"),
                ("quantize_two_pass", q2, 2.5625, "amax_kernel + quantize_amax_kernel"))
        for name, fn, bpe, kern in legs:
            for _ in range(warmup):
                fn()
            torch.cuda.synchronize()
            barrier(world)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with ClockSampler(torch.cuda.current_device(), stream, fn) as clk:
                torch.cuda.synchronize()
                e0.record(stream)
                for _ in range(steps):
                    fn()
                e1.record(stream)
                torch.cuda.synchronize()
            barrier(world)
            ms = max_over_ranks(e0.elapsed_time(e1), world, device) / steps
            gbs = elts * bpe / (ms / 1e3) / 1e9
            res[name] = {
                "ms_per_layer": ms, "GB/s": gbs,
                "roofline": {"kernel": kern, "bound": "hbm", "achieved": gbs,
                             "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": gbs / peaks["hbm_gbs"],
                             "traffic": measured_traffic(kern),
                             "algorithmic_bytes": elts * bpe,
                             "peak_source": peaks["source"] + " (burst copy)"},
                "clocks": clk.summary(),
                # per projection per layer: one launch, two for the two-pass quantizer
                "gpu_launches": (4 if name == "quantize_two_pass" else 2) * steps}
        del xs, outs, deq, qws, amx
        torch.cuda.empty_cache()
        return {"metric": "NVFP4 codec GB/s (whole layer)", "unit": "GB/s",
                "value": res["quantize"]["GB/s"], "steps": steps, "warmup": warmup,
                "higher_is_better": True, "dtype": "f32 (codec arithmetic), u8 codes",
                "config": {"workload": wl.name, "elements": elts,
                           "bytes_per_element": "2 (bf16) + 0.5625 (codes + scales)",
                           "l2": "inputs (19.3 GB bf16) larger than L2"},
                "roofline": res["quantize"]["roofline"],
                "ms_per_step": res["quantize"]["ms_per_layer"],
                "clocks": res["quantize"]["clocks"],
                "gpu_launches": res["quantize"]["gpu_launches"],
                **res}


SHARED_I = I                  # shared-expert intermediate size (one expert's, 2048)
SHARED_BYTES = 3 * H * SHARED_I * 2     # bf16 gate, up and down weights: 75.5 MB
SHARED_COPIES = 3                       # rotated so the 75.5 MB are not left in L2


def graph_timed(stream, fn, n_calls, steps, warmup):
    """Time `steps` calls of fn(i) (i cycles over n_calls prepared inputs) replayed from a
    CUDA graph of n_calls calls; returns (ms per call, clock summary)."""
    for i in range(warmup):
        fn(i % n_calls)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        fn(0)
        stream.synchronize()
        with torch.cuda.graph(graph, stream=stream):
            for i in range(n_calls):
                fn(i)
    reps = max(1, steps // n_calls)
    graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device(), stream, graph.replay) as clk:
        torch.cuda.synchronize()
        e0.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(reps):
                graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / (reps * n_calls)
    del graph
    return ms, clk.summary()


def shared_layer_records(b, warmup):
    """The BF16 shared expert alone and the whole layer (router + routed NVFP4 experts +
    shared expert, moe_nvfp4_layer) at one token and at the T = 4096 prefill batch."""
    nv, device, peaks = b.nv, b.device, b.peaks
    layer = b.ensure_layer()
    stream = torch.cuda.Stream(device)
    shared = [(synth.normal_bf16((2 * SHARED_I, H), c, "shared_gu", std=0.02, device=device),
               synth.normal_bf16((H, SHARED_I), c, "shared_dn", std=0.02, device=device))
              for c in range(SHARED_COPIES)]
    recs = []
    for T, steps, n_calls in ((1, 2048, 256), (4096, 10, 2)):
        wl = synth.PREFILL_T4096 if T > 1 else synth.DECODE_T1
        xs = synth.activations_bf16(n_calls * T, H, 31, device=device).view(n_calls, T, H)
        logits = synth.router_logits(n_calls * T, E, seed=31, zipf_bias=wl.zipf_bias)
        logits = logits.view(n_calls, T, E).to(device)
        routed = torch.randn(T, H, device=device) * 0.05
        out = torch.empty((T, H), dtype=torch.bfloat16, device=device)
        sws = torch.empty((max(16, T * SHARED_I * 2),), dtype=torch.uint8, device=device)
        lws = torch.zeros((nv.moe_nvfp4_layer_workspace_size(T, H, I, E, K, SHARED_I),),
                          dtype=torch.uint8, device=device)

        def shared_call(i):
            gu, dn = shared[i % SHARED_COPIES]
            nv.moe_nvfp4_shared_expert(xs[i], gu, dn, routed=routed, out=out, workspace=sws)

        def layer_call(i):
            gu, dn = shared[i % SHARED_COPIES]
            nv.moe_nvfp4_layer(xs[i], logits[i], K, *layer, gu, dn, out=out, workspace=lws)

        ms_s, clk_s = graph_timed(stream, shared_call, n_calls, steps, warmup)
        ms_l, clk_l = graph_timed(stream, layer_call, n_calls, steps, warmup)
        ids = torch.stack([nv.moe_nvfp4_router(logits[i], K)[0] for i in range(n_calls)])
        uniq = statistics.mean(len(set(ids[i].flatten().tolist())) for i in range(n_calls))
        if T == 1:
            ach_s = SHARED_BYTES / (ms_s / 1e3) / 1e9
            roof_s = {"kernel": "shared_gemv_gateup + shared_gemv_down", "bound": "hbm",
                      "achieved": ach_s, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                      "frac": ach_s / peaks["hbm_gbs"], "traffic": None,
                      "algorithmic_bytes": SHARED_BYTES,
                      "peak_source": peaks["source"] + " (burst copy)"}
            bytes_l = uniq * EXPERT_BYTES + SHARED_BYTES
            ach_l = bytes_l / (ms_l / 1e3) / 1e9
            roof_l = {"kernel": "whole layer step (router, routed GEMV pair, shared GEMV pair)",
                      "bound": "hbm", "achieved": ach_l, "peak": peaks["hbm_gbs"],
                      "unit": "GB/s", "frac": ach_l / peaks["hbm_gbs"], "traffic": None,
                      "algorithmic_bytes": bytes_l,
                      "peak_source": peaks["source"] + " (burst copy)"}
            launches = (2, 5)
        else:
            fl_s = 2 * T * 3 * H * SHARED_I
            ach_s = fl_s / (ms_s / 1e3) / 1e12
            roof_s = {"kernel": "shared_gemm_kernel (tcgen05, both projections)",
                      "bound": "tensor", "achieved": ach_s, "peak": peaks["bf16_tflops"],
                      "unit": "TFLOP/s", "frac": ach_s / peaks["bf16_tflops"], "traffic": None,
                      "algorithmic_flops": fl_s,
                      "peak_source": peaks["source"] + " (cuBLAS bf16 burst)"}
            fl_l = fl_s + 2 * T * K * 3 * H * I
            ach_l = fl_l / (ms_l / 1e3) / 1e12
            roof_l = {"kernel": "whole layer step (router, routed tcgen05 GEMMs, shared "
                                "tcgen05 GEMMs)", "bound": "tensor", "achieved": ach_l,
                      "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                      "frac": ach_l / peaks["bf16_tflops"], "traffic": None,
                      "algorithmic_flops": fl_l,
                      "peak_source": peaks["source"] + " (cuBLAS bf16 burst)"}
            launches = (2, 8)
        common = {"unit": "tokens/s", "higher_is_better": True,
                  "dtype": "bf16 shared expert (exact products, f32 sums); NVFP4 routed "
                           "experts", "data": "synthetic"}
        recs.append({"metric": "shared expert tokens/s", "value": T / (ms_s / 1e3),
                     "ms_per_step": ms_s, "steps": steps, "warmup": warmup, **common,
                     "config": {"workload": f"shared expert: H={H} Is={SHARED_I} bf16, T={T}",
                                "l2": f"{SHARED_COPIES} weight copies rotated "
                                      f"({SHARED_COPIES * SHARED_BYTES / 1e6:.0f} MB > L2)"},
                     "roofline": roof_s, "clocks": clk_s, "gpu_launches": launches[0] * steps})
        recs.append({"metric": METRIC + " (whole layer: router + routed + shared)",
                     "value": T / (ms_l / 1e3), "ms_per_step": ms_l, "steps": steps,
                     "warmup": warmup, **common,
                     "config": {"workload": f"layer: router logits -> top-8 of 256 NVFP4 "
                                            f"experts + BF16 shared expert (Is={SHARED_I}), "
                                            f"T={T}" + (", Zipf routing" if T > 1 else ""),
                                "unique_experts_per_step": uniq,
                                "l2": "new tokens every step; routed weights 5.4 GB, shared "
                                      f"weights rotated over {SHARED_COPIES} copies"},
                     "roofline": roof_l, "clocks": clk_l,
                     "gpu_launches": launches[1] * steps})
        del xs, logits, routed, out, sws, lws
    del shared
    torch.cuda.empty_cache()
    return recs


FP4_PER_BF16 = 4.0   # nominal dense FP4 : bf16 tensor-core rate (9 : 2.25 PFLOP/s)


def w4a4_record(b, steps, warmup):
    """The prefill batch on the block-scaled FP4 tensor cores (W4A4: NVFP4 activations)."""
    nv, device, peaks, world = b.nv, b.device, b.peaks, b.world
    wl = synth.PREFILL_T4096
    T = wl.T
    layer = b.ensure_layer()
    w_gu, s_gu, g_gu, w_dn, s_dn, g_dn = layer
    prep = (w_gu, nv.nvfp4_w4a4_prepare_scales(s_gu, gate_rows=I), g_gu,
            w_dn, nv.nvfp4_w4a4_prepare_scales(s_dn), g_dn)
    n_b = 2
    xs, ids, ws_ = make_batches(wl, n_b, seed=1000 + b.rank, device=device)
    ws = torch.zeros((nv.moe_nvfp4_w4a4_workspace_size(T, H, I, E, K),), dtype=torch.uint8,
                     device=device)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=device)
    stream = torch.cuda.Stream(device)

    def step(i):
        nv.moe_nvfp4_forward_w4a4(xs[i], ids[i], ws_[i], *prep, out=out, workspace=ws)

    ms, clk = graph_timed(stream, step, n_b, steps, warmup)
    marks = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(n_b)]
    for m in marks:
        for e in m:
            e.record()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(n_b):
            nv.moe_nvfp4_forward_w4a4_profiled(xs[i], ids[i], ws_[i], *prep, out, ws, marks[i])
    torch.cuda.synchronize()
    names = ["route_quantize_x", "gate_up", "quantize_h_down", "combine"]
    stages = {n: statistics.mean(m[j].elapsed_time(m[j + 1]) for m in marks)
              for j, n in enumerate(names)}
    fl_gu = 2 * T * K * (2 * I * H)
    pk = peaks["bf16_tflops"] * FP4_PER_BF16
    ach = fl_gu / (stages["gate_up"] / 1e3) / 1e12
    flops_step = 2 * T * K * (3 * H * I)
    rec = {"metric": METRIC + " (W4A4: NVFP4 activations, FP4 tensor cores)",
           "value": T / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
           "warmup": warmup, "higher_is_better": True,
           "dtype": "e2m1 x e2m1 products with e4m3 block scales (tcgen05 kind::mxf4nvf4), f32 "
                    "accumulation",
           "data": "synthetic (seeded N(0,1) tokens, N(0,0.02) bf16 weights quantized to NVFP4)",
           "config": {"workload": wl.name + ", W4A4 (each activation row quantized to NVFP4)",
                      "T": T, "H": H, "I": I, "E": E, "K": K,
                      "l2": "new tokens every step over 5.4 GB of resident weights",
                      "timing": f"CUDA graph of {n_b} steps replayed, CUDA events"},
           "stages_ms": stages, "tflops_step": flops_step / (ms / 1e3) / 1e12,
           "roofline": {"kernel": "w4a4_gemm_kernel mode 0 (block-scaled FP4 MMA + SwiGLU)",
                        "bound": "tensor", "achieved": ach, "peak": pk, "unit": "TFLOP/s",
                        "frac": ach / pk, "traffic": None, "algorithmic_flops": fl_gu,
                        "peak_source": peaks["source"] + " (cuBLAS bf16 burst x 4, the "
                                                         "nominal dense FP4:bf16 ratio)"},
           "clocks": clk, "gpu_launches": 6 * steps}
    del prep, xs, ids, ws_, ws, out
    torch.cuda.empty_cache()
    return rec


SUB_DECODE_STEPS = {"decode1": 4096, "decode8": 1024, "decode32": 512, "decode64": 256}


def run_ours(args, rank, world, device):
    import bit_quantized_moe_nvfp4_b200 as nv
    b = Bench(nv, args, rank, world, device)
    if args.workload == "w4a4":
        rec = w4a4_record(b, args.steps, args.warmup)
        return {**rec, "n_gpus": world, "scaling": "weak", "vs_baseline": None}
    if args.workload == "layer":
        recs = shared_layer_records(b, args.warmup)
        return {**recs[-1], "n_gpus": world, "scaling": "weak", "vs_baseline": None,
                "sub_records": recs}
    if args.workload == "codec":
        rec = b.codec_record(args.steps, args.warmup)
        rec.update({"n_gpus": world, "scaling": "weak", "vs_baseline": None,
                    "data": "synthetic", "ms_per_step": rec["quantize"]["ms_per_layer"],
                    "clocks": rec["quantize"]["clocks"],
                    "gpu_launches": rec["quantize"]["gpu_launches"]})
        return rec
    main = "prefill" if args.workload == "all" else args.workload
    if args.parallel == "ep":
        return b.ep_record(main, args.steps, args.warmup)
    line = b.layer_record(main, args.steps, args.warmup, main=True)
    if args.workload == "all" and world == 1 and not args.no_sub_records:
        subs = []
        for name, n in SUB_DECODE_STEPS.items():
            subs.append(b.layer_record(name, max(n, args.steps), args.warmup, main=False))
        subs += shared_layer_records(b, args.warmup)
        subs.append(w4a4_record(b, max(args.steps, 10), args.warmup))
        b.drop_layer()
        subs.append(b.codec_record(max(3, min(args.steps, 8)), args.warmup))
        line["sub_records"] = subs
    return line


def run_e2e(nv, layer, wl, args, device, ws, path):
    """Same metric through the public API with host buffers.  Every step copies its x, ids
    and weights in from pinned host memory, runs the layer (`moe_nvfp4_forward`) and copies
    its output back.  The copies run on a second stream: the inputs of step i+1 go in and the
    output of step i-1 comes back while step i computes, with two device buffer sets and
    events ordering each buffer's copy-in, use and copy-out.  At decode sizes (T <= 64) the
    host cost of issuing a step's copies and launches is larger than the step itself, so
    there the whole pipelined sequence is captured once as a CUDA graph and replayed; the
    copies stay in it, one per tensor and step."""
    T = wl.T
    n = max(1, min(args.e2e_steps, 256 if T <= 64 else 8))
    xs = synth.activations_bf16(n * T, H, 77).view(n, T, H).pin_memory()
    ids, w = synth.routing(n * T, E, K, seed=77, zipf_bias=wl.zipf_bias)
    ids = ids.view(n, T, K).pin_memory()
    w = w.view(n, T, K).pin_memory()
    out_h = torch.empty((n, T, H), dtype=torch.bfloat16).pin_memory()
    bufs = [(torch.empty((T, H), dtype=torch.bfloat16, device=device),
             torch.empty((T, K), dtype=torch.int32, device=device),
             torch.empty((T, K), dtype=torch.float32, device=device),
             torch.empty((T, H), dtype=torch.bfloat16, device=device)) for _ in range(2)]
    ks = torch.cuda.Stream(device)
    cs = torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]

    def copy_in(i):
        xd, idd, wd, _ = bufs[i % 2]
        with torch.cuda.stream(cs):
            xd.copy_(xs[i], non_blocking=True)
            idd.copy_(ids[i], non_blocking=True)
            wd.copy_(w[i], non_blocking=True)
            ev_in[i % 2].record(cs)

    def run(first, count):
        cs.wait_stream(ks)
        copy_in(first)
        for i in range(first, first + count):
            xd, idd, wd, od = bufs[i % 2]
            ks.wait_event(ev_in[i % 2])
            nv.moe_nvfp4_forward(xd, idd, wd, *layer, out=od, workspace=ws, path=path)
            ev_done[i % 2].record(ks)
            if i + 1 < first + count:
                copy_in(i + 1)   # after the copy-out of step i - 1 on the copy stream
            with torch.cuda.stream(cs):
                cs.wait_event(ev_done[i % 2])
                out_h[i].copy_(od, non_blocking=True)
        ks.wait_stream(cs)

    with torch.cuda.stream(ks):
        run(0, min(3, n))
        torch.cuda.synchronize()
        graph = None
        if T <= 64:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=ks):
                run(0, n)
            graph.replay()
            torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0 = time.perf_counter()
        e0.record(ks)
        if graph is not None:
            graph.replay()
        else:
            run(0, n)
        e1.record(ks)
        torch.cuda.synchronize()
        wall = time.perf_counter() - t0
    ms = e0.elapsed_time(e1)
    if graph is not None:
        ms = max(ms, wall * 1e3)   # the replay's host launch cost counts too
        del graph
    return {"value": n * T / (ms / 1e3), "unit": "tokens/s", "steps": n,
            "h2d_bytes_per_step": T * H * 2 + T * K * 4 * 2, "d2h_bytes_per_step": T * H * 2,
            "copies": "on a second stream, overlapped with the neighbouring steps' compute" +
                      ("; the n steps captured once as one CUDA graph" if T <= 64 else "")}


# ----------------------------------------------------------------------------- reference arm
REFERENCE_BUDGET_S = 150.0   # whole --impl reference run, warm-up included


def run_reference(args):
    """The CPU oracle as it stands, on the host cores, as the reference arm, on the headline
    workload (prefill, Zipf routing).  The unit of work is one token of that batch (routed to
    8 of a pool of 16 experts; NVFP4 weights drawn directly as random codes and scales, since
    the oracle's cost does not depend on values).  So that --steps K --warmup W ends within
    a few minutes, each step runs a slice of one token's work: the first i_rows of the
    I=2048 intermediate rows (gate, up and the matching down columns), i_rows a multiple of
    64 sized from a calibration run; the oracle's work is linear in i_rows, and the rate is
    scaled to whole tokens."""
    import oracle
    wl = synth.PREFILL_T4096
    pool = 16
    n = args.steps + args.warmup
    x = synth.activations_bf16(n, H, 5)
    ids, w = synth.routing(n, pool, K, seed=5, zipf_bias=wl.zipf_bias)
    # calibration (untimed): one step on a 64-row slice
    probe = random_nvfp4_pool(pool, i_rows=64)
    t0 = time.perf_counter()
    oracle.moe_forward(x[0:1], ids[0:1], w[0:1], *probe)
    t64 = max(time.perf_counter() - t0, 1e-4)
    per_step = REFERENCE_BUDGET_S / n
    i_rows = 64 * int(max(1, min(I // 64, per_step // t64)))
    weights = probe if i_rows == 64 else random_nvfp4_pool(pool, i_rows=i_rows)
    times = []
    for i in range(n):
        t0 = time.perf_counter()
        oracle.moe_forward(x[i:i + 1], ids[i:i + 1], w[i:i + 1], *weights)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    sec = sum(times)
    frac = i_rows / I                   # fraction of a token's work per step
    v = len(times) * frac / sec
    sample = (f"each step one token of the prefill batch (8 experts, Zipf routing) on the "
              f"first {i_rows} of {I} intermediate rows, i.e. {frac:.4f} of a token; rate "
              f"scaled to whole tokens")
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * sec / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": oracle.threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------- plumbing
def barrier(world, device=None):
    if world > 1:
        torch.distributed.barrier()
    if device is None or torch.device(device).type == "cuda":
        torch.cuda.synchronize()


def max_over_ranks(v, world, device):
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="all")
    ap.add_argument("--path", type=int, default=0)
    ap.add_argument("--graph-steps", type=int, default=512)
    ap.add_argument("--e2e-steps", type=int, default=256)
    ap.add_argument("--cpu-tokens", type=int, default=24)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sub-records", action="store_true")
    ap.add_argument("--parallel", choices=["ep", "replicas"], default=None,
                    help="N>1: expert parallel (default) or independent replicas; "
                         "ep also runs on one GPU (one rank)")
    ap.add_argument("--experts", type=int, default=256,
                    help="experts in the layer (a smaller layer is only for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    global E
    E = args.experts

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if args.parallel is None:
        args.parallel = "ep" if world > 1 else "replicas"
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1 or args.parallel == "ep":
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", "29511")
        os.environ.setdefault("RANK", str(rank))
        os.environ.setdefault("WORLD_SIZE", str(world))
        import datetime
        torch.distributed.init_process_group("nccl", device_id=device,
                                             timeout=datetime.timedelta(seconds=300))
    try:
        line = run_ours(args, rank, world, device)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
