"""Benchmark of the fused grouped W4A16 MoE layer on B200.

Default workload (one "step"): one decode step of a 16-layer stack of
OLMoE-shaped MoE layers (hidden 2048, expert intermediate 1024, 64 SwiGLU
experts, top-8; int4 group-128 experts, all resident, 3.32 GB packed) at
T=16 tokens, with the residual x + MoE(x) between layers. Every step runs
route -> group -> grouped W4A16 FFN -> combine for each layer through the
library's C ABI, replayed from one CUDA graph. The same step is also timed at
T = 1, 4, 64 (the rest of the decode sweep) and reported under "sweep".

metric: MoE-layer tokens/s = T * layers / step time (device time, CUDA events).
e2e:    the same metric with the activations copied host->device from pinned
        memory before and the output copied back after, inside the timed region.
roofline: the grouped FFN (gate/up + down kernels) per layer call: algorithmic
        bytes = active experts x 3,244,032 B of packed codes + scales, over the
        call's CUDA-event duration, against the measured HBM copy bandwidth.
cpu_baseline: the CPU oracle (plain C, fp64, OpenMP over experts and tokens)
        on a bounded sample of the workload: whole passes of layer 0 at the
        bench's T, repeated for about ten seconds.

The line also carries the rest of the decode sweep (T = 1, 4, 64), prefill
entries (tensor-core path, against the BF16 peak), the sequential-W4 and BF16
reference paths at T = 16, and slot-cache decode from a pinned host pool.

--impl reference runs that oracle as the reference arm (rank 0 only).
Multi-GPU: replicas only (each rank runs the whole workload on its own GPU;
the layer has no exchange step), timed as the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

H, I, E, K, LAYERS = 2048, 1024, 64, 8, 16
SWEEP_T = (1, 4, 16, 64)
METRIC = "MoE-layer tokens/s; HBM GB/s (decode) and TC TFLOP/s (prefill) vs B200 peak"
SHAPES = {"olmoe": (2048, 1024, 64, 8), "wide": (4096, 14336, 8, 2)}   # (H, I, E, k)

# DRAM bytes (read + write) of one decode FFN call per active expert, from an
# ncu capture of the shipped gate/up and down kernels (one-layer stack, T=16,
# 53 active experts: gate/up 119.04 MB read + 2.97 MB written, down 59.76 MB
# read + 0.08 MB written; 5.8 % above the 3,244,032 algorithmic bytes per
# expert). Reported as roofline.traffic, scaled to the bench's active experts.
DECODE_TRAFFIC_PER_ACTIVE_EXPERT = (119038464 + 2971648 + 59755776 + 76288) / 53

# Prefill entries of the default line: (shape, T).
# (shape, T, Zipf-skewed routing): every prefill configuration of the workload
PREFILL_CASES = (("olmoe", 512, False), ("olmoe", 2048, False), ("olmoe", 8192, False), ("wide", 512, False),
                 ("wide", 2048, False), ("wide", 8192, False), ("olmoe", 512, True))


def rec_bytes(h, i):
    """Bytes of one packed expert record: codes of three matrices + their scales."""
    return 3 * i * h // 2 + 3 * (i * h // 128) * 2


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--T", type=int, default=16)
    ap.add_argument("--layers", type=int, default=LAYERS)
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="leave the prefill entries out of the default line")
    ap.add_argument("--no-references", action="store_true",
                    help="leave the sequential-W4 and BF16 reference paths out of the default line")
    ap.add_argument("--no-slotcache", action="store_true",
                    help="leave the slot-cache decode entry out of the default line")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--path", default="auto", choices=["auto", "gemv", "tc", "seq"])
    ap.add_argument("--workload", default="decode", choices=["decode", "prefill", "slotcache"],
                    help="decode: the 16-layer stack sweep (default); prefill: one layer at large T; "
                         "slotcache: 16 layers decoding from a pinned host pool through S GPU slots per layer")
    ap.add_argument("--slots", default="8,16,32,64",
                    help="slotcache: slot counts per layer to sweep (comma list); the line's headline is 16")
    ap.add_argument("--shape", default="olmoe", choices=list(SHAPES))
    ap.add_argument("--skew", action="store_true", help="prefill with Zipf(1.2) log-bias routing")
    a = ap.parse_args()
    if a.workload == "prefill" and a.T == 16:
        a.T = 8192
    if a.workload == "prefill" and a.layers == LAYERS:
        a.layers = 1
    return a


def decode_config(T, L, world):
    """The decode workload's config, shared by both arms of the bench."""
    return {"workload": f"olmoe-{L}L-decode", "T": T, "layers": L, "H": H, "I": I, "E": E, "k": K,
            "weights": "int4 group-128 symmetric, all experts resident",
            "l2": "inputs larger than L2 (3.32 GB of packed experts read per step)",
            "parallelism": f"replicas{world}"}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------------------- distributed plumbing

def dist_setup(n):
    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world):
    """The largest of the ranks' values (device times: the job's time is the
    slowest rank's). The reduction runs on the GPU under NCCL, on the host
    under gloo."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v)], device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_value(units_per_rank, world, ms_max):
    """Whole-job throughput of `world` replicas: all ranks' units over the
    slowest rank's time (weak scaling: every rank runs the full workload)."""
    return units_per_rank * world / (ms_max / 1e3)


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        import torch
        self.idx = str(device_index)
        try:  # the UUID names the same GPU whatever CUDA_VISIBLE_DEVICES says
            u = str(torch.cuda.get_device_properties(device_index).uuid)
            self.idx = u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            pass
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)  # nvidia-smi needs a moment before its first sample
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
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
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
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
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- the stack

class Stack:
    """16 OLMoE-shaped layers: per layer a packed expert bank and a router, plus
    per-T buffers. Weights are drawn on the device with the seeded recipe."""

    def __init__(self, layers, path, shape="olmoe", renorm=False, skew=False):
        import torch

        import synth
        import w4a16_mixture_experts_moe_b200 as M
        from w4a16_mixture_experts_moe_b200.layer import ExpertBank
        self.M, self.torch, self.layers = M, torch, layers
        H, I, E, K = SHAPES[shape]
        self.H, self.I, self.E, self.K = H, I, E, K
        self.flags = M.MOE_RENORM if renorm else 0
        # skewed routing: log Zipf(1.2) per-expert offsets added to the logits
        self.bias = torch.from_numpy(synth.zipf_log_bias(E)).float().cuda() if skew else None
        self.path = {"auto": M.MOE_PATH_AUTO, "gemv": M.MOE_PATH_GEMV, "tc": M.MOE_PATH_TC,
                     "seq": M.MOE_PATH_SEQUENTIAL}[path]
        self.banks, self.routers = [], []
        for l in range(layers):
            gate, up, down = synth.expert_bank(l, E, H, I, device="cuda")
            bank = ExpertBank(E, H, I)
            bank.pack(gate, up, down)
            del gate, up, down
            self.banks.append(bank)
            self.routers.append(synth.router_weight(l, E, H, device="cuda"))
        torch.cuda.synchronize()

    def buffers(self, T):
        from w4a16_mixture_experts_moe_b200.layer import LayerBuffers
        torch = self.torch
        H, I, E, K = self.H, self.I, self.E, self.K
        bufs = [LayerBuffers(T, K, E, H, I, path=self.path) for _ in range(self.layers)]
        xs = [torch.empty(T, H, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
        return bufs, xs

    def forward(self, bufs, xs, x_in):
        """x_in -> layer 0 -> ... -> returns the output buffer."""
        from w4a16_mixture_experts_moe_b200.layer import moe_layer_forward
        cur = x_in
        for l in range(self.layers):
            out = xs[l % 2] if cur is not xs[l % 2] else xs[(l + 1) % 2]
            moe_layer_forward(cur, self.routers[l], self.banks[l], bufs[l], bias=self.bias, flags=self.flags,
                              residual=cur, out=out)
            cur = out
        return cur


def time_graph(torch, graph, steps, warmup):
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        graph.replay()
    e.record()
    torch.cuda.synchronize()
    return s.elapsed_time(e) / steps


def measure_T(stack, T, steps, warmup, world, want_e2e=True, want_roofline=True):
    """Device-timed step, e2e step and per-call FFN timing at T tokens."""
    import synth
    torch, M = stack.torch, stack.M
    H = stack.H
    bufs, xs = stack.buffers(T)
    x_dev = synth.activations(T, H, device="cuda")
    x_host = synth.activations(T, H).pin_memory()
    out_host = torch.empty(T, H, dtype=torch.bfloat16).pin_memory()
    x_in = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    x_in.copy_(x_dev)

    # eager warm-up (also loads kernels before capture)
    stack.forward(bufs, xs, x_in)
    torch.cuda.synchronize()
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    launches0 = M.moe_launch_counter()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        y = stack.forward(bufs, xs, x_in)
    launches_per_step = M.moe_launch_counter() - launches0
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g2, stream=stream):
        x_in.copy_(x_host, non_blocking=True)
        y2 = stack.forward(bufs, xs, x_in)
        out_host.copy_(y2, non_blocking=True)
    torch.cuda.synchronize()

    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        ms = time_graph(torch, g, steps, warmup)
    barrier(world)
    ms = max_over_ranks(ms, world)
    res = {"T": T, "ms_per_step": ms, "launches_per_step": int(launches_per_step), "clocks": clk.summary()}
    if want_e2e:
        barrier(world)
        ms_e2e = max_over_ranks(time_graph(torch, g2, steps, warmup), world)
        res["ms_e2e"] = ms_e2e
    if want_roofline:
        # The grouped FFN calls of all layers, replayed back to back from one
        # graph on the buffers the step left behind (same routing, same
        # launches as inside the step): CUDA events around the replays give
        # the FFN call's device time.
        g3 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g3, stream=stream):
            for l in range(stack.layers):
                b = bufs[l]
                x_ffn, path = b.ffn_input(x_in if l == 0 else xs[(l - 1) % 2])
                M.moe_grouped_w4a16_ffn(x_ffn, b.sorted_pair, b.offsets, stack.banks[l].ptr, stack.banks[l].rec,
                                        None, stack.E, T, stack.K, stack.E, stack.H, stack.I, path, b.y, b.ffn_ws,
                                        b.ffn_ws_bytes)
        ms_ffn_layers = time_graph(torch, g3, max(3, min(steps, 50)), 3)
        del g3
        n_act = [int((b.counts > 0).sum().item()) for b in bufs]
        res["ffn_ms_per_call"] = ms_ffn_layers / stack.layers
        res["n_active_mean"] = statistics.mean(n_act)
        res["counts_layer0"] = [int(c) for c in bufs[0].counts.tolist()]
        res["ffn_bytes_per_call"] = statistics.mean(n_act) * rec_bytes(stack.H, stack.I)
        res["ffn_flops_per_call"] = 6.0 * T * stack.K * stack.H * stack.I
    del g, g2
    return res


# ----------------------------------------------------------------------------- CPU oracle (baseline / reference)

def oracle_sample(T, seconds, shape="olmoe", tokens=None, skew=False, renorm=False, max_reps=200):
    """Time the C oracle on whole passes of one layer of `shape` for about
    `seconds` (at least one pass), on the first `tokens` of the T tokens
    (all of them by default). Returns (layer-tokens per second, threads,
    description). Quantisation (an offline step on both sides) is done before
    the clock starts."""
    import numpy as np
    import torch

    import synth
    from oracle import c_oracle as c
    H_, I_, E_, K_ = SHAPES[shape]
    Ts = T if tokens is None else min(T, tokens)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    mats = synth.expert_bank(0, E_, H_, I_, device=dev)
    bits = [m.view(torch.int16).cpu().numpy().view(np.uint16) for m in mats]
    del mats
    packs = c.pack_experts(*bits, bits=True)
    del bits
    wr = synth.router_weight(0, E_, H_).double().numpy()
    x = synth.activations(T, H_).double().numpy()[:Ts]
    bias = synth.zipf_log_bias(E_) if skew else None
    reps = 0
    t0 = time.perf_counter()
    while True:
        c.moe_layer(x, wr, packs, K_, bias, renorm, residual=True)
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= seconds or reps >= max_reps:
            break
    part = f"the first {Ts} of the T={T} tokens" if Ts < T else f"T={T}"
    return Ts * reps / dt, c.threads(), f"{reps} pass(es) of layer 0 ({shape}) at {part} by the C oracle " \
                                        f"(router + top-k + grouping + FFN with on-the-fly dequantisation + " \
                                        f"combine; quantisation not timed), {dt:.1f} s"


def run_reference(a):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    v, cores, desc = oracle_sample(a.T, seconds=min(60.0, 2.0 * max(1, a.steps)))
    # the same workload as the repo arm; the unit is per layer and every layer
    # has the same shape, so passes of layer 0 are a bounded sample of it
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "layer-tokens/s", "n_gpus": a.gpus,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": 1e3 * a.T * a.layers / v,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": decode_config(a.T, a.layers, a.gpus),
            "cpu_baseline": {"value": v, "unit": "layer-tokens/s", "cores": cores, "kind": "oracle", "sample": desc},
            "e2e": {"value": v, "unit": "layer-tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- main

def main():
    a = parse()
    if a.impl == "reference":
        run_reference(a)
        return
    import torch
    rank, world, local = dist_setup(a.gpus)
    P = peaks()
    if a.workload == "prefill":
        return main_prefill(a, rank, world, P)
    if a.workload == "slotcache":
        return main_slotcache(a, rank, world, P)
    stack = Stack(a.layers, a.path)
    head = measure_T(stack, a.T, a.steps, a.warmup, world)
    sweep = {}
    if not a.no_sweep:
        for T in SWEEP_T:
            if T == a.T:
                r = head
            else:
                r = measure_T(stack, T, a.steps, a.warmup, world, want_e2e=False)
            sweep[str(T)] = {"value": T * a.layers / (r["ms_per_step"] / 1e3) * world,
                             "ms_per_step": r["ms_per_step"],
                             "ffn_hbm_frac": (r["ffn_bytes_per_call"] / (r["ffn_ms_per_call"] / 1e3) / 1e9)
                             / P["hbm_gbs"],
                             "n_active_mean": r["n_active_mean"]}
    refs = {}
    if not a.no_references:
        refs = reference_paths(a, stack, head, world, P)
    del stack
    torch.cuda.empty_cache()
    prefill = {}
    if not a.no_prefill:
        for shape, Tp, skew in PREFILL_CASES:
            key = f"{shape}-T{Tp}" + ("-zipf1.2-skew" if skew else "")
            prefill[key] = prefill_entry(a, shape, Tp, rank, world, P, skew=skew)
            torch.cuda.empty_cache()
    slot = {}
    if not a.no_slotcache:
        slot = slotcache_entry(a)
        torch.cuda.empty_cache()
    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        v, cores, desc = oracle_sample(a.T, seconds=10.0)
        cpu = {"value": v, "unit": "layer-tokens/s", "cores": cores, "kind": "oracle", "sample": desc}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if rank == 0:
        T, L = a.T, a.layers
        value = replica_value(T * L, world, head["ms_per_step"])
        achieved = head["ffn_bytes_per_call"] / (head["ffn_ms_per_call"] / 1e3) / 1e9
        line = {
            "metric": METRIC, "value": value, "unit": "layer-tokens/s", "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": decode_config(T, L, world),
            "e2e": {"value": replica_value(T * L, world, head["ms_e2e"]), "unit": "layer-tokens/s",
                    "h2d_bytes_per_step": T * H * 2, "d2h_bytes_per_step": T * H * 2},
            "roofline": {"bound": "hbm", "kernel": "moe_grouped_w4a16_ffn (gate/up + down kernels), per layer call",
                         "achieved": achieved, "peak": P["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / P["hbm_gbs"],
                         "traffic": (DECODE_TRAFFIC_PER_ACTIVE_EXPERT * head["n_active_mean"]
                                     if DECODE_TRAFFIC_PER_ACTIVE_EXPERT and (T, H, I, E, K) == (16, 2048, 1024, 64, 8)
                                     else None),
                         "traffic_source": "ncu capture, scaled by active experts",
                         "peak_source": P["source"], "bytes_per_call": head["ffn_bytes_per_call"],
                         "ms_per_call": head["ffn_ms_per_call"], "n_active_mean": head["n_active_mean"]},
            "cpu_baseline": cpu,
            "gpu_launches": head["launches_per_step"] * a.steps,
            "clocks": head["clocks"],
            "sweep": sweep,
            "prefill": prefill,
            "references": refs,
            "slotcache": slot,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


# The pages' slot counts (Table 1) and their whole-model L4 hit rates, for context.
PAGES_HIT_RATE = {8: 0.388, 16: 0.563, 32: 0.814, 64: None}


def slotcache_runs(layers, runs, steps, warmup):
    """Decode with every expert in pinned host memory and S GPU slots per
    layer, for each (T, S) of `runs` (the pages' Table 1 sweeps S = 8, 16, 32
    and 64 = all experts). T tokens per step, each an independent routing
    stream that keeps each expert of its previous step with probability 0.5.
    Per layer and step: route (weights of the drawn ids), plan the step's
    experts in cache-sized waves, and per wave: host LRU lookup, H2D fill of
    the misses on a side stream, grouped FFN through the slot table (that
    wave's experts only), release; then the combine. Returns the per-run
    results, the pinned host -> device copy bandwidth measured in the same
    run, and the pool's size."""
    import numpy as np
    import torch

    import synth
    M = __import__("w4a16_mixture_experts_moe_b200")
    from w4a16_mixture_experts_moe_b200.layer import LayerBuffers
    L = layers
    stack = Stack(L, "auto")
    rec = stack.banks[0].rec
    pool = torch.empty(L * E * rec, dtype=torch.uint8, pin_memory=True)
    for l in range(L):
        pool[l * E * rec:(l + 1) * E * rec].copy_(stack.banks[l].buf)
    stack.banks = None                       # the experts now live only in the pinned pool
    torch.cuda.empty_cache()
    n_steps = warmup + steps
    side = torch.cuda.Stream()
    comp = torch.cuda.current_stream()

    # pinned host -> device copy bandwidth, same run, same size as a miss
    probe_n = 64
    dst = torch.empty(probe_n * rec, dtype=torch.uint8, device="cuda")
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(2):
        with torch.cuda.stream(side):
            ev0.record(side)
            for i in range(probe_n):
                dst[i * rec:(i + 1) * rec].copy_(pool[i * rec:(i + 1) * rec], non_blocking=True)
            ev1.record(side)
        side.synchronize()
    pinned_gbs = probe_n * rec / (ev0.elapsed_time(ev1) / 1e3) / 1e9
    del dst

    def run(T, S):
        # routing[l][s] = ids [T][K] of step s in layer l
        routing = [np.stack([synth.drawn_routing(l, E, K, n_steps, stream=t) for t in range(T)], axis=1)
                   for l in range(L)]
        ids_dev = torch.from_numpy(np.stack(routing, axis=1).astype(np.int32)).cuda()   # [step][layer][T][K]
        x0 = synth.activations(n_steps * T, H, device="cuda").view(n_steps, T, H)
        bufs = [LayerBuffers(T, K, E, H, I) for _ in range(L)]
        xs = [torch.empty(T, H, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
        slots = torch.empty(L * S * rec, dtype=torch.uint8, device="cuda")
        table = torch.full((L, E), -1, dtype=torch.int32, device="cuda")
        cache = M.SlotCache(L, E, S, rec, pool, slots, table)
        n_waves = [0]

        def step(si):
            cur = x0[si]
            for l in range(L):
                b = bufs[l]
                b.topk_ids.copy_(ids_dev[si, l])
                M.moe_route_topk_x16(cur, stack.routers[l], T, H, E, K, None, M.MOE_IDS_GIVEN, b.logits,
                                     b.topk_ids, b.topk_w, b.x16, b.ffn_ws)
                M.moe_group_tokens(b.topk_ids, T, K, E, b.counts, b.offsets, b.sorted_pair, b.pair_pos,
                                   b.group_ws, b.group_ws_bytes)
                x_ffn, path = b.ffn_input(cur)
                waves = cache.plan_waves(l, [int(v) for v in routing[l][si].reshape(-1)])
                n_waves[0] += len(waves)
                for w in waves:
                    _, miss = cache.lookup(l, w)
                    cache.fill(l, miss, side=side, compute=comp)
                    M.moe_grouped_w4a16_ffn(x_ffn, b.sorted_pair, b.offsets, slots.data_ptr() + l * S * rec, rec,
                                            table[l], S, T, K, E, H, I, path, b.y, b.ffn_ws, b.ffn_ws_bytes)
                    cache.release(l, comp)
                out = xs[l % 2]
                M.moe_combine(b.y, b.topk_w, b.pair_pos, cur, T, K, H, out)
                cur = out
            return cur

        for si in range(warmup):
            step(si)
        torch.cuda.synchronize()
        st0 = cache.stats()
        n_waves[0] = 0
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        launches0 = M.moe_launch_counter()
        with ClockSampler(torch.cuda.current_device()) as clk:
            s0.record()
            for si in range(warmup, n_steps):
                step(si)
            s1.record()
            torch.cuda.synchronize()
        launches = M.moe_launch_counter() - launches0
        ms = s0.elapsed_time(s1) / steps
        st1 = cache.stats()
        hits, misses = st1["hits"] - st0["hits"], st1["misses"] - st0["misses"]
        h2d = st1["h2d_bytes"] - st0["h2d_bytes"]
        err = sorted(set(M.moe_read_device_error(b.ffn_ws) for b in bufs))
        cache.close()
        del slots, table
        return {"T": T, "slots": S, "value": T * L / (ms / 1e3), "unit": "layer-tokens/s", "ms_per_step": ms,
                "decode_tokens_per_s": T * 1e3 / ms,
                "hit_rate": None if S >= E else hits / max(1, hits + misses),
                "pages_hit_rate_l4": PAGES_HIT_RATE.get(S) if T == 1 else None,
                "h2d_gb": h2d / 1e9, "h2d_gb_per_step": h2d / 1e9 / steps,
                "h2d_achieved_gbs": h2d / (ms * steps / 1e3) / 1e9,
                "waves_per_layer_step": n_waves[0] / (steps * L), "device_errors": err,
                "gpu_launches": launches, "clocks": clk.summary()}

    results = [run(T, S) for T, S in runs]
    del stack
    return results, pinned_gbs, L * E * rec


def main_slotcache(a, rank, world, P):
    """The slot-cache decode workload on its own line (--workload slotcache):
    T = --T (1 unless given), one run per slot count of --slots."""
    L, T = a.layers, a.T if a.T != 16 else 1
    slot_counts = [int(v) for v in str(a.slots).split(",")]
    steps = a.steps if a.steps >= 16 else 128
    results, pinned_gbs, pool_bytes = slotcache_runs(L, [(T, S) for S in slot_counts], steps, a.warmup)
    head = next((r for r in results if r["slots"] == 16), results[0])
    if rank == 0:
        line = {
            "metric": METRIC, "value": replica_value(T * L, world, head["ms_per_step"]), "unit": "layer-tokens/s",
            "n_gpus": world, "steps": steps, "warmup": a.warmup, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"olmoe-{L}L-slotcache-decode", "T": T, "layers": L,
                       "slots_per_layer": head["slots"], "H": H, "I": I, "E": E, "k": K,
                       "routing": "drawn per token stream, keep-probability 0.5",
                       "pool": f"{pool_bytes / 1e9:.2f} GB pinned host", "parallelism": f"replicas{world}"},
            "decode_tokens_per_s": head["decode_tokens_per_s"], "hit_rate": head["hit_rate"],
            "h2d_gb": head["h2d_gb"], "h2d_achieved_gbs": head["h2d_achieved_gbs"], "pinned_copy_gbs": pinned_gbs,
            "device_errors": head["device_errors"], "gpu_launches": head["gpu_launches"], "clocks": head["clocks"],
            "slot_sweep": {str(r["slots"]): r for r in results},
        }
        print(json.dumps(line), flush=True)


SLOTCACHE_STEPS = 128  # decode steps per slot-cache run (the workload's 128-step trace)


def slotcache_entry(a):
    """The slot-cache entry of the default line: the 16-layer stack decoding
    from the pinned pool at T = 1 for 8, 16, 32 and 64 slots per layer, and
    at T = 4 through 16 slots (about 27 distinct experts a step: two waves)."""
    runs = [(1, 8), (1, 16), (1, 32), (1, 64), (4, 16)]
    results, pinned_gbs, pool_bytes = slotcache_runs(LAYERS, runs, SLOTCACHE_STEPS, 4)
    out = {"pool_gb_pinned_host": pool_bytes / 1e9, "pinned_copy_gbs": pinned_gbs, "steps": SLOTCACHE_STEPS,
           "routing": "drawn per token stream, keep-probability 0.5"}
    for r in results:
        out[f"T{r['T']}-S{r['slots']}"] = r
    return out


# The pages' own ratios for these two comparisons, measured on one L4 on the
# whole OLMoE model (context only): fused grouped execution against the
# sequential W4 reference at 16 tokens, and W4A16 against BF16 decode.
PAGES_FUSED_OVER_SEQUENTIAL_L4 = 1.97
PAGES_W4_OVER_BF16_DECODE_L4 = 31.923 / 21.662


def reference_paths(a, stack, head, world, P):
    """The decode step at the bench's T through the two reference paths the
    pages compare against: the sequential W4 reference (the same GEMV kernels
    launched once per expert, MOE_PATH_SEQUENTIAL) and the BF16 grouped FFN
    on unquantised experts (moe_grouped_bf16_ffn; 12.6 MB per OLMoE expert,
    12.9 GB for the 16 layers). Route, group and combine are the same calls in
    all three; each step is replayed from a CUDA graph."""
    import torch

    import synth
    from w4a16_mixture_experts_moe_b200.layer import Bf16Bank
    M, T, L = stack.M, a.T, stack.layers
    steps = max(5, min(a.steps, 50))
    old = stack.path
    stack.path = M.MOE_PATH_SEQUENTIAL
    r = measure_T(stack, T, steps, a.warmup, world, want_e2e=False)
    stack.path = old
    seq = {"ms_per_step": r["ms_per_step"], "value": replica_value(T * L, world, r["ms_per_step"]),
           "unit": "layer-tokens/s", "ffn_ms_per_call": r["ffn_ms_per_call"],
           "launches_per_step": r["launches_per_step"],
           "fused_over_sequential_step": r["ms_per_step"] / head["ms_per_step"],
           "fused_over_sequential_ffn": r["ffn_ms_per_call"] / head["ffn_ms_per_call"],
           "pages_fused_over_sequential_l4": PAGES_FUSED_OVER_SEQUENTIAL_L4}

    banks = []
    for l in range(L):
        g, u, d = synth.expert_bank(l, E, H, I, device="cuda")
        b = Bf16Bank(E, H, I)
        b.load(g, u, d)
        del g, u, d
        banks.append(b)
    bufs, xs = stack.buffers(T)
    nb = M.moe_bf16_ffn_workspace_size(T, K, E, H, I)
    wss = [torch.zeros(nb, dtype=torch.uint8, device="cuda") for _ in range(L)]
    x_in = synth.activations(T, H, device="cuda")

    def ffn(l, cur):
        bb = bufs[l]
        M.moe_grouped_bf16_ffn(cur, bb.sorted_pair, bb.offsets, banks[l].ptr, banks[l].rec, T, K, E, H, I, bb.y,
                               wss[l], nb)

    def fwd():
        cur = x_in
        for l in range(L):
            bb = bufs[l]
            out = xs[l % 2] if cur is not xs[l % 2] else xs[(l + 1) % 2]
            M.moe_route_topk(cur, stack.routers[l], T, H, E, K, None, 0, bb.logits, bb.topk_ids, bb.topk_w)
            M.moe_group_tokens(bb.topk_ids, T, K, E, bb.counts, bb.offsets, bb.sorted_pair, bb.pair_pos,
                               bb.group_ws, bb.group_ws_bytes)
            ffn(l, cur)
            M.moe_combine(bb.y, bb.topk_w, bb.pair_pos, cur, T, K, H, out)
            cur = out
        return cur

    fwd()
    torch.cuda.synchronize()
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    g1 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g1, stream=stream):
        fwd()
    ms = max_over_ranks(time_graph(torch, g1, steps, a.warmup), world)
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g2, stream=stream):
        cur = x_in
        for l in range(L):
            ffn(l, x_in if l == 0 else xs[(l - 1) % 2])
    ms_ffn = time_graph(torch, g2, steps, 3) / L
    n_act = statistics.mean(int((b.counts > 0).sum().item()) for b in bufs)
    bf16_bytes = n_act * banks[0].rec
    del g1, g2, banks
    torch.cuda.empty_cache()
    bf = {"ms_per_step": ms, "value": replica_value(T * L, world, ms), "unit": "layer-tokens/s",
          "ffn_ms_per_call": ms_ffn, "n_active_mean": n_act, "ffn_bytes_per_call": bf16_bytes,
          "ffn_hbm_frac": bf16_bytes / (ms_ffn / 1e3) / 1e9 / P["hbm_gbs"],
          "w4_over_bf16_step": ms / head["ms_per_step"],
          "w4_over_bf16_ffn": ms_ffn / head["ffn_ms_per_call"],
          "pages_w4_over_bf16_decode_l4": PAGES_W4_OVER_BF16_DECODE_L4}
    return {"T": T, "sequential_w4": seq, "bf16_grouped": bf}


def prefill_entry(a, shape, T, rank, world, P, skew=False):
    """One prefill layer step (tensor-core path) at T tokens: layer-tokens/s,
    the grouped FFN call against the BF16 tensor peak, clocks, and the oracle
    on 64 of the tokens (rank 0, one GPU). Used by the default line."""
    H_, I_, E_, K_ = SHAPES[shape]
    renorm = shape == "wide"
    stack = Stack(1, "auto", shape, renorm=renorm, skew=skew)
    steps = max(5, min(a.steps, 50))
    r = measure_T(stack, T, steps, max(3, min(a.warmup, 10)), world)
    del stack
    achieved = r["ffn_flops_per_call"] / (r["ffn_ms_per_call"] / 1e3) / 1e12
    ent = {"value": replica_value(T, world, r["ms_per_step"]), "unit": "layer-tokens/s",
           "ms_per_step": r["ms_per_step"], "steps": steps,
           "e2e": {"value": replica_value(T, world, r["ms_e2e"]), "unit": "layer-tokens/s",
                   "h2d_bytes_per_step": T * H_ * 2, "d2h_bytes_per_step": T * H_ * 2},
           "config": {"workload": f"{shape}-prefill" + ("-zipf1.2-skew" if skew else ""), "T": T, "layers": 1,
                      "H": H_, "I": I_, "E": E_, "k": K_, "renorm": renorm,
                      "l2": f"inputs larger than L2 ({E_ * rec_bytes(H_, I_) / 1e6:.0f} MB of packed experts "
                            f"+ {T * H_ * 2 / 1e6:.0f} MB of activations)"},
           "roofline": {"bound": "tensor", "kernel": "moe_grouped_w4a16_ffn (tcgen05 gate/up + down), per call",
                        "achieved": achieved, "peak": P["bf16_tflops"], "unit": "TFLOP/s",
                        "frac": achieved / P["bf16_tflops"],
                        "frac_of_sustained": achieved / P["bf16_tflops_sustained"], "traffic": None,
                        "peak_source": P["source"], "flops_per_call": r["ffn_flops_per_call"],
                        "ms_per_call": r["ffn_ms_per_call"], "n_active_mean": r["n_active_mean"]},
           "gpu_launches": r["launches_per_step"] * steps,
           "clocks": r["clocks"]}
    if skew:  # the load imbalance the skewed router produces in layer 0
        counts = r["counts_layer0"]
        ent["groups"] = {"largest": max(counts), "empty": sum(1 for c in counts if c == 0),
                         "active": sum(1 for c in counts if c > 0)}
    ent["cpu_baseline"] = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        v, cores, desc = oracle_sample(T, seconds=5.0, shape=shape, tokens=64, skew=skew, renorm=renorm)
        ent["cpu_baseline"] = {"value": v, "unit": "layer-tokens/s", "cores": cores, "kind": "oracle",
                               "sample": desc}
    return ent


def main_prefill(a, rank, world, P):
    """One layer at large T (tensor-core path); roofline = FLOPs / FFN time."""
    H_, I_, E_, K_ = SHAPES[a.shape]
    stack = Stack(a.layers, a.path, a.shape, renorm=(a.shape == "wide"), skew=a.skew)
    r = measure_T(stack, a.T, a.steps, a.warmup, world)
    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        del stack
        v, cores, desc = oracle_sample(a.T, seconds=10.0, shape=a.shape, tokens=64, skew=a.skew,
                                       renorm=(a.shape == "wide"))
        cpu = {"value": v, "unit": "layer-tokens/s", "cores": cores, "kind": "oracle", "sample": desc}
    if rank == 0:
        T, L = a.T, a.layers
        achieved = r["ffn_flops_per_call"] / (r["ffn_ms_per_call"] / 1e3) / 1e12
        line = {
            "metric": METRIC, "value": replica_value(T * L, world, r["ms_per_step"]), "unit": "layer-tokens/s",
            "n_gpus": world, "steps": a.steps, "warmup": a.warmup, "ms_per_step": r["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"{a.shape}-prefill" + ("-zipf1.2-skew" if a.skew else ""), "T": T, "layers": L,
                       "H": H_, "I": I_, "E": E_, "k": K_,
                       "weights": "int4 group-128 symmetric, all experts resident",
                       "l2": f"inputs larger than L2 ({E_ * rec_bytes(H_, I_) / 1e6:.0f} MB of packed experts)",
                       "parallelism": f"replicas{world}"},
            "e2e": {"value": replica_value(T * L, world, r["ms_e2e"]), "unit": "layer-tokens/s",
                    "h2d_bytes_per_step": T * H_ * 2, "d2h_bytes_per_step": T * H_ * 2},
            "roofline": {"bound": "tensor", "kernel": "moe_grouped_w4a16_ffn (tcgen05 gate/up + down), per call",
                         "achieved": achieved, "peak": P["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": achieved / P["bf16_tflops"],
                         "frac_of_sustained": achieved / P["bf16_tflops_sustained"], "traffic": None,
                         "peak_source": P["source"], "flops_per_call": r["ffn_flops_per_call"],
                         "ms_per_call": r["ffn_ms_per_call"], "n_active_mean": r["n_active_mean"]},
            "cpu_baseline": cpu,
            "gpu_launches": r["launches_per_step"] * a.steps,
            "clocks": r["clocks"],
        }
        if a.skew:
            c = r["counts_layer0"]
            line["routing"] = {"bias": "log Zipf(s=1.2) per expert", "n_active": sum(1 for v in c if v > 0),
                               "max_group": max(c), "empty_groups": sum(1 for v in c if v == 0), "histogram": c}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
