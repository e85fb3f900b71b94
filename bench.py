#!/usr/bin/env python
"""Benchmark of the packed-MXFP4 W4A16 top-4 MoE expert FFN on B200.

Workload: the full expert stack at batch-1 decode -- 38 MoE layers, each
H=2048, I=1536, E=64, top-4 (12.19 GB of packed E2M1 codes + E8M0 scales
resident), per layer a weightless RMSNorm of the residual stream, routing,
the grouped expert FFN and the sequential BF16 combine with residual add;
one decode token = one CUDA-graph replay of all 38 layers.  One bench "step"
is a batch of 64 decode tokens (64 replays, each feeding its residual output
to the next).  Inputs are seeded synthetic data (no checkpoint exists here).

Prints ONE JSON line on rank 0.  ``--impl reference`` times the CPU oracle
(plain C, fp64) on the host cores on a bounded sample of the same workload.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time
from concurrent.futures import ThreadPoolExecutor

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import synth  # noqa: E402

METRIC = "MoE-FFN tokens/s and achieved HBM GB/s (fraction of B200 peak), 1 GPU"
TOKENS_PER_STEP = 64
SHAPE = synth.L24B
N_LAYERS = 38
WORKLOAD = ("stack24b: 38 MoE layers x (H=2048, I=1536, E=64, top-4) batch-1 decode, "
            "RMSNorm + route + experts + sequential BF16 combine + residual per layer, "
            "one CUDA graph per token, 64 tokens per step")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-pdl", action="store_true")
    ap.add_argument("--no-prefetch", action="store_true")
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--skip-sym8", action="store_true", help="skip the sym8 stack line")
    ap.add_argument("--skip-nvfp4", action="store_true",
                    help="skip the decode measurement of the stack with NVFP4 experts")
    ap.add_argument("--skip-batched", action="store_true",
                    help="skip the grouped-path measurements at batch sizes beyond decode")
    ap.add_argument("--layers", type=int, default=N_LAYERS,
                    help="layers in the stack (fewer: a smaller case for profiling; "
                         "the bench workload is the full stack)")
    ap.add_argument("--layered", action="store_true",
                    help="run the step one layer at a time (three launches per layer) instead "
                         "of the one-launch stack kernel")
    ap.add_argument("--skip-configs", action="store_true",
                    help="skip the tiny-layer, single-layer and 8B-stack measurements")
    ap.add_argument("--only-batched", default=None, metavar="T:ROUTING",
                    help="time one grouped-path case of one 24B layer only, e.g. 256:uniform "
                         "(a small command for profiler captures)")
    ap.add_argument("--only-main", action="store_true",
                    help="time the main line only (for profiler runs)")
    ap.add_argument("--only-sym8-prefill", action="store_true",
                    help="time the S = 64 chunk of one sym8 layer only (grouped products; a "
                         "small command for profiler captures)")
    return ap.parse_args()


def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def max_over_ranks(value, world, device):
    """The largest of every rank's value (the job ends when its slowest rank
    does); the value itself on a single rank."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank, world, t_ms):
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * world / (t_ms / 1e3)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def bytes_per_layer(shape, distinct_experts, T):
    """Algorithmic bytes of one layer: the touched experts' packed weights,
    the router matrix, and the activation vectors read/written once
    (residual in, normalised x out/in, h out/in, residual out)."""
    expert = 3 * shape.I * shape.H // 2 + 3 * shape.I * shape.H // 32
    router = shape.E * shape.H * 2
    act = T * shape.H * 2 * 4 + T * shape.top_k * shape.I * 2 * 2
    return distinct_experts * expert + router + act


# the translation unit of the stack kernel and every header it includes: a
# change to any of them may change the kernel
STACK_TU = ("stack.cu", "down.cuh", "gemv.cuh", "kernels.cuh", "common.cuh")


def csrc_digest():
    h = hashlib.sha256()
    d = os.path.join(ROOT, "packed_mxfp4_w4a16_b200", "csrc")
    for name in STACK_TU:
        with open(os.path.join(d, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def stored_traffic(n_layers):
    """DRAM bytes of one stack-kernel launch of n_layers from the committed
    ncu summary (taken on a smaller stack and scaled by layers: the traffic
    of a layer does not depend on the layer count), if it was taken from the
    current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "stack_decode_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("csrc_digest") != csrc_digest():
        return None
    return d["dram_bytes_per_layer"] * n_layers


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index):
        self.ok = False
        self.samples = []
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = repr(e)
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((mhz, rs))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.ok:
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.err}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [m for m, _ in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= r
        reasons = sorted(n for b, n in self.REASONS.items() if bits & b and n != "gpu_idle")
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(mhz)}


# ------------------------------------------------------------ CPU oracle

def oracle_layer_rate(seconds, layers_wanted=3, seed=0):
    """Time the CPU oracle on (token, layer) evaluations of the stack for about
    `seconds`.  Returns (layer_evals_per_s, evals, threads, sample text)."""
    import oracle
    layers = [synth.make_layer(SHAPE, seed=seed, layer=l) for l in range(layers_wanted)]
    xs = synth.make_tokens(64, SHAPE.H, seed=seed, stream=77)
    threads = oracle.max_threads()
    r = xs[0:1]
    evals, t0 = 0, time.perf_counter()
    while True:
        L = layers[evals % len(layers)]
        xn = oracle.rmsnorm(r)
        _, _, r = oracle.moe_layer(xn, L.router_w, L.router_b, L.codes, L.scales, SHAPE.E,
                                   SHAPE.H, SHAPE.I, SHAPE.top_k, residual=r)
        evals += 1
        dt = time.perf_counter() - t0
        if dt >= seconds:
            break
    sample = (f"{evals} (token, layer) evaluations of the 24B stack (layers 0..{layers_wanted - 1} "
              f"cycled, decode feedback), {dt:.1f} s; tokens/s = evals/s / {N_LAYERS}")
    return evals / dt, evals, threads, sample


def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    import oracle
    layers = [synth.make_layer(SHAPE, seed=args.seed, layer=l) for l in range(2)]
    x = synth.make_tokens(1, SHAPE.H, seed=args.seed, stream=77)
    # one step = one (token, layer) oracle evaluation of the 38-layer stack
    def one(i, r):
        L = layers[i % 2]
        xn = oracle.rmsnorm(r)
        return oracle.moe_layer(xn, L.router_w, L.router_b, L.codes, L.scales, SHAPE.E,
                                SHAPE.H, SHAPE.I, SHAPE.top_k, residual=r)[2]
    r = x
    for i in range(args.warmup):
        r = one(i, r)
    t0 = time.perf_counter()
    for i in range(args.steps):
        r = one(i, r)
    dt = time.perf_counter() - t0
    tok_s = args.steps / N_LAYERS / dt
    cores = oracle.max_threads()
    sample = (f"each step = one (token, layer) evaluation of the 38-layer 24B stack "
              f"(1/38 of a decode token); {args.steps} steps")
    out = {
        "impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "layers": N_LAYERS, "T": 1, "E": SHAPE.E,
                   "H": SHAPE.H, "I": SHAPE.I, "top_k": SHAPE.top_k},
        "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)
    return 0


# ------------------------------------------------------------------ ours

def stack_weights(torch, shape, seed, n_layers, bias=False):
    def gen(l):
        return synth.make_layer(shape, seed=seed, layer=l, bias=bias)

    weights = []
    with ThreadPoolExecutor(4) as ex:
        for L in ex.map(gen, range(n_layers)):
            codes = torch.from_numpy(L.codes).cuda()
            scales = torch.from_numpy(L.scales).cuda()
            rw = torch.from_numpy(L.router_w.view(np.int16)).cuda().view(torch.bfloat16)
            rb = None if L.router_b is None else torch.from_numpy(L.router_b).cuda()
            weights.append((codes, scales, rw, rb))
    return weights


def build_stack(torch, moe, seed, n_layers, persistent=None):
    weights = stack_weights(torch, SHAPE, seed, n_layers)
    return moe.MoEStack(weights, SHAPE.E, SHAPE.H, SHAPE.I, SHAPE.top_k, T=1,
                        persistent=persistent)


def replay_rate(torch, graph, n, stream):
    """Seconds per replay of `graph` over n back-to-back replays (CUDA events
    on `stream`, after two warm replays)."""
    with torch.cuda.stream(stream):
        graph.replay()
        graph.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / 1e3 / n


def nvfp4_stack(torch, moe, st, args, max_steps=8):
    """The same 38-layer decode with NVFP4 experts: each layer reuses the
    MXFP4 layer's codes and router, with E4M3 block scales (a scale per 16,
    positive normal values, exponent fields 1..7) and FP32 multipliers in
    [0.01, 0.02] drawn on the device from a seeded generator.  Timed like
    the main line (graph replays of 64 tokens per step, CUDA events)."""
    gen = torch.Generator(device="cuda")
    gen.manual_seed(args.seed + 7)
    n_sc = 3 * SHAPE.I * SHAPE.H // 16
    weights = []
    for L in st.layers:
        ex = torch.randint(1, 8, (SHAPE.E, n_sc), dtype=torch.uint8, device="cuda", generator=gen)
        man = torch.randint(0, 8, (SHAPE.E, n_sc), dtype=torch.uint8, device="cuda", generator=gen)
        sc = (ex << 3) | man
        gs = torch.rand((SHAPE.E, 2), device="cuda", generator=gen) * 0.01 + 0.01
        weights.append((L.codes, sc, L.router_w, L.router_b, gs))
    nv = moe.MoEStack(weights, SHAPE.E, SHAPE.H, SHAPE.I, SHAPE.top_k, T=1)
    nv.set_tuning(use_pdl=not args.no_pdl, prefetch_down=not args.no_prefetch)
    nv.r.copy_(st.r)
    nv.capture()
    steps = max(1, min(max_steps, args.steps))
    for _ in range(2 * TOKENS_PER_STEP):
        nv.graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stream = torch.cuda.current_stream()
    e0.record(stream)
    for _ in range(steps * TOKENS_PER_STEP):
        nv.graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    t_ms = e0.elapsed_time(e1)
    for L in nv.layers:
        assert L.status() == 0
    ids = nv.ids.cpu().numpy()
    per_expert = 3 * SHAPE.I * SHAPE.H // 2 + 3 * SHAPE.I * SHAPE.H // 16 + 8
    tok_bytes = sum(len(set(ids[l].ravel().tolist())) * per_expert + SHAPE.E * SHAPE.H * 2
                    + 2 * SHAPE.H * 2 for l in range(len(nv.layers)))
    n_tok = steps * TOKENS_PER_STEP
    out = {"workload": f"stack24b with NVFP4 experts ({len(nv.layers)} layers, E4M3 scale per "
                       "16, FP32 multipliers), batch-1 decode",
           "tokens_per_s": n_tok / (t_ms / 1e3), "us_per_token": t_ms * 1e3 / n_tok,
           "bytes_per_token": tok_bytes, "hbm_gbs": tok_bytes * n_tok / (t_ms / 1e3) / 1e9,
           "steps": steps}
    # the grouped path with NVFP4 experts, one layer (mma.sync products at
    # T = 64 and 256, tcgen05 at T = 1024)
    codes, sc, rw, rb, gs = weights[0]
    lay = moe.MoELayer(SHAPE.E, SHAPE.H, SHAPE.I, SHAPE.top_k, codes, sc, rw, rb,
                       max_tokens=1024, gscales=gs)
    grouped = []
    for T in (64, 256, 1024):
        x = torch.from_numpy(synth.make_tokens(T, SHAPE.H, seed=args.seed, stream=T)
                             .view(np.int16)).cuda().view(torch.bfloat16)
        ids_h, w_h = synth.make_routing(T, SHAPE.E, SHAPE.top_k, "uniform",
                                        synth.rng_for(args.seed, 93, T))
        ids, w = torch.from_numpy(ids_h).cuda(), torch.from_numpy(w_h).cuda()
        y = torch.empty_like(x)
        lay.forward(x, ids, w, y=y)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(20):
                lay.forward(x, ids, w, y=y)
        g.replay()
        torch.cuda.synchronize()
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / 20
        del g
        touched = len(set(ids_h.ravel().tolist()))
        tc = T * SHAPE.top_k >= TC_AUTO_GROUP * SHAPE.E
        grouped.append({"T": T, "routing": "uniform", "experts_touched": touched,
                        "products": "tcgen05" if tc else "mma.sync", "us_per_call": us,
                        "hbm_gbs": (touched * per_expert + 2 * T * SHAPE.H * 2) / (us * 1e-6) / 1e9})
    assert lay.status() == 0
    lay.close()
    out["grouped"] = grouped
    nv.close()
    return out


def sym8_stack(torch, moe, st, args, max_steps=4):
    """The same 38-layer decode with sym8 experts (page "LFM2.5-8B-A1B — Core
    AI (.aimodel)", "Provenance": int8 weights, a scale per 32): each layer's
    int8 weights uniform over -127..127 and binary16 block scales (positive
    normal values, exponent fields 2..5, uniform mantissas) drawn on the
    device from a seeded generator, the MXFP4 layer's router reused; one
    route + gate/up + down launch triple per layer, captured in a CUDA graph
    and timed like the NVFP4 line."""
    n_w = 3 * SHAPE.I * SHAPE.H
    weights = draw_sym8_weights(torch, st.layers, args.seed)
    s8 = moe.MoEStack(weights, SHAPE.E, SHAPE.H, SHAPE.I, SHAPE.top_k, T=1, persistent=False)
    s8.r.copy_(st.r)
    s8.capture()
    steps = max(1, min(max_steps, args.steps))
    for _ in range(2 * TOKENS_PER_STEP):
        s8.graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stream = torch.cuda.current_stream()
    e0.record(stream)
    for _ in range(steps * TOKENS_PER_STEP):
        s8.graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    t_ms = e0.elapsed_time(e1)
    assert s8.status() == 0
    ids = s8.ids.cpu().numpy()
    per_expert = n_w + n_w // 16
    tok_bytes = sum(len(set(ids[l].ravel().tolist())) * per_expert + SHAPE.E * SHAPE.H * 2
                    + 2 * SHAPE.H * 2 for l in range(len(s8.layers)))
    n_tok = steps * TOKENS_PER_STEP
    peak, _ = load_peaks()
    out = {"workload": f"stack24b with sym8 experts ({len(s8.layers)} layers, int8 weights, "
                       "binary16 scale per 32), batch-1 decode, per-layer launches",
           "tokens_per_s": n_tok / (t_ms / 1e3), "us_per_token": t_ms * 1e3 / n_tok,
           "bytes_per_token": tok_bytes, "hbm_gbs": tok_bytes * n_tok / (t_ms / 1e3) / 1e9,
           "hbm_frac": tok_bytes * n_tok / (t_ms / 1e3) / 1e9 / peak,
           "gpu_launches_per_token": 3 * len(s8.layers), "steps": steps}
    s8.close()
    out["prefill_s64"] = sym8_prefill_chunk(torch, moe, weights[0], args.seed, peak)
    del weights
    torch.cuda.empty_cache()
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist

    import packed_mxfp4_w4a16_b200 as moe

    rank, local, world = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    if args.only_sym8_prefill:
        st = build_stack(torch, moe, seed=args.seed + rank, n_layers=1, persistent=False)
        weights = draw_sym8_weights(torch, st.layers, args.seed)
        peak, _ = load_peaks()
        row = sym8_prefill_chunk(torch, moe, weights[0], args.seed, peak)
        if rank == 0:
            print(json.dumps({"sym8_prefill_s64": row}), flush=True)
        del weights
        st.close()
        return 0

    if args.only_batched:
        T, dist = args.only_batched.split(":")
        st = build_stack(torch, moe, seed=args.seed + rank, n_layers=1, persistent=False)
        rows = batched_cases(torch, moe, st, args.seed, cases=((int(T), dist),))
        if rank == 0:
            print(json.dumps({"batched": rows}), flush=True)
        st.close()
        return 0

    n_layers = args.layers
    st = build_stack(torch, moe, seed=args.seed + rank, n_layers=n_layers,
                     persistent=False if args.layered else None)
    if not args.layered:
        assert st.stack is not None, "the stack kernel does not take this shape"
    st.set_tuning(use_pdl=not args.no_pdl, prefetch_down=not args.no_prefetch)
    x0 = torch.from_numpy(synth.make_tokens(1, SHAPE.H, seed=args.seed + rank, stream=3)
                          .view(np.int16)).cuda().view(torch.bfloat16)
    st.r.copy_(x0)
    st.capture()
    stream = torch.cuda.current_stream()

    def step():
        for _ in range(TOKENS_PER_STEP):
            st.graph.replay()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # ---- timed region: K steps of 64 graph replays, device-timed ----
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
    t_ms = e0.elapsed_time(e1)
    t_ms = max_over_ranks(t_ms, world, "cuda")
    tok_s = job_throughput(TOKENS_PER_STEP * args.steps, world, t_ms)
    status = st.status()
    assert status == 0, f"device status {status:#x}"

    # bytes per token from the routing of the last replay (distinct experts)
    ids = st.ids.cpu().numpy()
    step_bytes = sum(bytes_per_layer(SHAPE, len(set(ids[l].ravel().tolist())), 1)
                     for l in range(n_layers))
    n_tok = TOKENS_PER_STEP * args.steps
    us_tok = t_ms * 1e3 / n_tok
    gbs = step_bytes * n_tok / (t_ms / 1e3) / 1e9
    peak, peak_kind = load_peaks()

    out = {
        "metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e2m1xbf16->f32", "data": "synthetic",
        "config": {"workload": WORKLOAD if n_layers == N_LAYERS else
                   WORKLOAD.replace(f"{N_LAYERS} MoE layers", f"{n_layers} MoE layers"),
                   "layers": n_layers, "T": 1, "E": SHAPE.E,
                   "H": SHAPE.H, "I": SHAPE.I, "top_k": SHAPE.top_k,
                   "tokens_per_step": TOKENS_PER_STEP, "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2 (12.19 GB resident, 0.77 GB streamed per token "
                         "vs 126 MB L2); no flush",
                   "launch": "layered" if args.layered else "one stack launch per token"},
        "hbm_gbs": gbs, "hbm_frac": gbs / peak, "hbm_peak_gbs": peak,
        "hbm_peak_kind": peak_kind, "bytes_per_token": step_bytes, "us_per_token": us_tok,
        "clocks": clk.summary(),
    }
    if args.layered:
        out["roofline"] = {"bound": "hbm", "kernel": "whole step (3 launches per layer)",
                           "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                           "traffic": None, "bytes_per_launch": None, "peak_kind": peak_kind}
        out["gpu_launches"] = 3 * n_layers * n_tok
    else:
        # the step is one launch of the stack kernel: its duration is the time
        # of one replay (graph launch gaps included, so a lower bound on the
        # kernel's own rate)
        out["roofline"] = {"bound": "hbm", "kernel": "stack_decode_kernel",
                           "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                           "traffic": stored_traffic(n_layers), "bytes_per_launch": step_bytes,
                           "launch_us": us_tok, "peak_kind": peak_kind,
                           "peak_note": "burst copy bandwidth; the kernel is timed in a loop "
                                        "of back-to-back launches"}
        out["gpu_launches"] = n_tok

    if not args.only_main:
        # ---- end to end through the public API with host buffers ----
        out["e2e"] = run_e2e(torch, st, args)
        # ---- the same step one layer at a time (context: the launch structure
        # this kernel replaces) ----
        if not args.layered:
            out["layered"] = layered_rate(torch, moe, st, x0, n_layers, step_bytes)
        if not args.skip_configs:
            out["configs"] = {
                "tiny_layer": config_tiny(torch, moe, args.seed),
                "layer24b": config_layer24b(torch, moe, st, args.seed),
                "stack8b": config_stack8b(torch, moe, args.seed),
            }
        # ---- the grouped path at batch sizes beyond decode (one layer) ----
        out["batched"] = (batched_cases(torch, moe, st, args.seed)
                          if not args.skip_batched else None)
        # ---- the same stack with NVFP4 experts ----
        out["nvfp4"] = nvfp4_stack(torch, moe, st, args) if not args.skip_nvfp4 else None
        # ---- the same stack with sym8 experts ----
        out["sym8"] = sym8_stack(torch, moe, st, args) if not args.skip_sym8 else None

    if rank == 0 and world == 1 and not args.skip_cpu_baseline:
        rate, evals, threads, sample = oracle_layer_rate(12.0)
        out["cpu_baseline"] = {"value": rate / N_LAYERS, "unit": "tokens/s", "cores": threads,
                               "kind": "oracle", "sample": sample}
    if rank == 0:
        print(json.dumps(out), flush=True)
    st.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def layered_rate(torch, moe, st, x0, n_layers, step_bytes):
    """The same decode step with one moe_layer_ex per layer (router, gate/up
    and down launches, programmatic serialization), one CUDA graph per token:
    tokens/s, for comparison with the one-launch stack."""
    lay = moe.MoEStack([(L.codes, L.scales, L.router_w, L.router_b) for L in st.layers],
                       SHAPE.E, SHAPE.H, SHAPE.I, SHAPE.top_k, T=1, persistent=False)
    lay.r.copy_(x0)
    lay.capture()
    sec = replay_rate(torch, lay.graph, 4 * TOKENS_PER_STEP, lay.stream)
    lay.close()
    return {"tokens_per_s": 1.0 / sec, "us_per_token": sec * 1e6,
            "hbm_gbs": step_bytes / sec / 1e9, "launches_per_token": 3 * n_layers}


def config_tiny(torch, moe, seed, reps=200):
    """Tiny single MoE layer (H 512, I 384, E 16, top-4, 4 tokens): route +
    expert FFN + combine (moe_layer_ex, three launches), CUDA graph of `reps`
    calls."""
    shape = synth.TINY
    L = synth.make_layer(shape, seed=seed)
    codes = torch.from_numpy(L.codes).cuda()
    scales = torch.from_numpy(L.scales).cuda()
    rw = torch.from_numpy(L.router_w.view(np.int16)).cuda().view(torch.bfloat16)
    lay = moe.MoELayer(shape.E, shape.H, shape.I, shape.top_k, codes, scales, rw, None,
                       max_tokens=4)
    x = torch.from_numpy(synth.make_tokens(4, shape.H, seed=seed).view(np.int16)).cuda() \
        .view(torch.bfloat16)
    ids = torch.empty(4, shape.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(4, shape.top_k, dtype=torch.float32, device="cuda")
    y = torch.empty_like(x)
    s = torch.cuda.Stream()

    def call():
        moe.moe_layer_ex(lay.handle, x, rw, None, 0, None, None, ids, w, None, y, 0, s)

    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        call()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for _ in range(reps):
            call()
    sec = replay_rate(torch, g, 5, s) / reps
    touched = len(set(ids.cpu().numpy().ravel().tolist()))
    nbytes = bytes_per_layer(shape, touched, 4)
    del g
    lay.close()
    return {"workload": "tiny: one layer H=512, I=384, E=16, top-4, T=4 (route + experts + "
                        "combine, moe_layer_ex)", "us_per_call": sec * 1e6,
            "tokens_per_s": 4 / sec, "hbm_gbs": nbytes / sec / 1e9, "experts_touched": touched}


def config_layer24b(torch, moe, st, seed, calls=1000):
    """One 24B layer at batch-1 decode with fresh routing on every call: the
    stack's 38 layers as 38 one-layer stacks, cycled (1000 calls in a CUDA
    graph, each on its own N(0,1) input token, so every call routes anew and
    the weights read by consecutive calls are different layers' -- 38 x 320
    MB of experts, no L2 reuse).  Each call = one stack-kernel launch of one
    layer (RMSNorm, route, experts, combine, residual).  Also the API path
    moe_route + moe_forward (the four-call boundary), same inputs."""
    n = len(st.layers)
    stacks = []
    for L in st.layers:
        h = moe.moe_stack_create([L.handle], [L.router_w], [L.router_b])
        ws = torch.empty(moe.moe_stack_workspace_bytes(h), dtype=torch.uint8, device="cuda")
        moe.moe_stack_set_workspace(h, ws)
        stacks.append((h, ws))
    xs = torch.from_numpy(synth.make_tokens(calls, SHAPE.H, seed=seed, stream=99)
                          .view(np.int16)).cuda().view(torch.bfloat16)
    ids = torch.zeros(calls, SHAPE.top_k, dtype=torch.int32, device="cuda")
    w = torch.zeros(calls, SHAPE.top_k, dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    r = xs.clone()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for i in range(calls):
            h = stacks[i % n][0]
            moe.moe_stack_decode(h, r[i], topk_ids=ids[i], topk_w=w[i], stream=s)
    with torch.cuda.stream(s):
        r.copy_(xs)
    sec = replay_rate(torch, g, 1, s) / calls
    del g
    ids_h = ids.cpu().numpy()
    touched = float(np.mean([len(set(row.tolist())) for row in ids_h]))
    nbytes = bytes_per_layer(SHAPE, touched, 1)
    for h, _ in stacks:
        moe.moe_stack_destroy(h)
    # the four-call API path: moe_route + moe_forward per call
    y = torch.empty_like(xs)
    g2 = torch.cuda.CUDAGraph()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g2, stream=s):
        for i in range(calls):
            L = st.layers[i % n]
            moe.moe_route(L.handle, xs[i:i + 1], L.router_w, L.router_b, ids[i:i + 1],
                          w[i:i + 1], stream=s)
            moe.moe_forward(L.handle, xs[i:i + 1], ids[i:i + 1], w[i:i + 1], y[i:i + 1],
                            stream=s)
    sec2 = replay_rate(torch, g2, 1, s) / calls
    del g2
    return {"workload": "layer24b: one H=2048, I=1536, E=64, top-4 layer, T=1, fresh input "
                        "and routing per call, 38 distinct layers cycled (no L2 reuse), "
                        f"{calls} calls", "us_per_layer": sec * 1e6,
            "hbm_gbs": nbytes / sec / 1e9, "bytes_per_call": nbytes,
            "launch": "one stack-kernel launch per call (RMSNorm + layer + residual)",
            "api_route_forward_us": sec2 * 1e6, "api_route_forward_gbs": nbytes / sec2 / 1e9}


def config_stack8b(torch, moe, seed, steps=4):
    """8B-A1B-like stack: 22 layers of E=32, H=2048, I=1536, top-4, with a
    per-expert router bias ~N(0,1) skewing popularity; batch-1 decode, one
    stack launch per token, 64 tokens per step.  Bytes per token from the
    actual routing of every timed token (distinct experts per layer)."""
    shape = synth.L8B
    n_layers = 22
    w8 = stack_weights(torch, shape, seed + 8, n_layers, bias=True)
    st = moe.MoEStack(w8, shape.E, shape.H, shape.I, shape.top_k, T=1)
    assert st.stack is not None
    x0 = torch.from_numpy(synth.make_tokens(1, shape.H, seed=seed, stream=8)
                          .view(np.int16)).cuda().view(torch.bfloat16)
    st.r.copy_(x0)
    st.capture()
    n_tok = steps * TOKENS_PER_STEP
    sec = replay_rate(torch, st.graph, n_tok, st.stream)
    # the routing of n_tok consecutive tokens (untimed pass from the same state)
    ids_all = torch.zeros(n_tok, n_layers, shape.top_k, dtype=torch.int32, device="cuda")
    with torch.cuda.stream(st.stream):
        for t in range(n_tok):
            moe.moe_stack_decode(st.stack, st.r, topk_ids=ids_all[t], stream=st.stream)
    torch.cuda.synchronize()
    assert st.status() == 0
    ids_h = ids_all.cpu().numpy()
    per_tok = [sum(bytes_per_layer(shape, len(set(ids_h[t, l].tolist())), 1)
                   for l in range(n_layers)) for t in range(n_tok)]
    tok_bytes = float(np.mean(per_tok))
    # reuse between consecutive tokens: experts a layer already read for the
    # previous token (their bytes may still be in L2)
    same = np.mean([len(set(ids_h[t, l].tolist()) & set(ids_h[t - 1, l].tolist())) / shape.top_k
                    for t in range(1, n_tok) for l in range(n_layers)])
    counts = np.bincount(ids_h.ravel(), minlength=shape.E) / ids_h.size
    st.close()
    return {"workload": "stack8b: 22 layers x (H=2048, I=1536, E=32, top-4), router bias "
                        "N(0,1), batch-1 decode, one stack launch per token",
            "tokens_per_s": 1.0 / sec, "us_per_token": sec * 1e6, "bytes_per_token": tok_bytes,
            "hbm_gbs": tok_bytes / sec / 1e9, "tokens": n_tok,
            "expert_repeat_frac_vs_previous_token": float(same),
            "top_expert_share": float(np.sort(counts)[::-1][:4].sum()),
            "l2_note": "444 MB of experts per token against a 126 MB L2: repeats between "
                       "consecutive tokens can hit L2; GB/s counts every touched expert once "
                       "per token"}


BATCHED_CASES = ((32, "uniform"), (32, "zipf"), (64, "uniform"), (64, "zipf"), (256, "uniform"),
                 (256, "zipf"), (1024, "uniform"), (2048, "uniform"), (2048, "zipf"))
TC_AUTO_GROUP = 40  # the library's tcgen05 products from T k >= 40 E on


def draw_sym8_weights(torch, layers, seed):
    """Per layer of `layers` (their routers are reused): int8 weights uniform
    over -127..127 and binary16 block scales (positive normal values,
    exponent fields 2..5, uniform mantissas), drawn on the device from a
    generator seeded with seed + 11."""
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed + 11)
    n_w = 3 * SHAPE.I * SHAPE.H
    weights = []
    for L in layers:
        q = torch.randint(-127, 128, (SHAPE.E, n_w), dtype=torch.int8, device="cuda",
                          generator=gen)
        ex = torch.randint(2, 6, (SHAPE.E, n_w // 32), dtype=torch.int16, device="cuda",
                           generator=gen)
        man = torch.randint(0, 1024, (SHAPE.E, n_w // 32), dtype=torch.int16, device="cuda",
                            generator=gen)
        weights.append((q, (ex << 10) | man, L.router_w, L.router_b))
    return weights


def sym8_prefill_chunk(torch, moe, lw, seed, peak, T=64, reps=10):
    """One sym8 layer (the first layer's weights of the sym8 stack) at the
    S = 64 prefill chunk with uniform routing: the grouped mma.sync products,
    moe_forward timed in a CUDA graph of `reps` calls.  Bytes: the touched
    experts' int8 codes and binary16 scales + activations."""
    q, sc, rw, rb = lw
    lay = moe.MoELayer(SHAPE.E, SHAPE.H, SHAPE.I, SHAPE.top_k, q, sc, rw, rb, max_tokens=T)
    x = torch.from_numpy(synth.make_tokens(T, SHAPE.H, seed=seed, stream=T)
                         .view(np.int16)).cuda().view(torch.bfloat16)
    ids_h, w_h = synth.make_routing(T, SHAPE.E, SHAPE.top_k, "uniform",
                                    synth.rng_for(seed, 91, T))
    ids, w = torch.from_numpy(ids_h).cuda(), torch.from_numpy(w_h).cuda()
    y = torch.empty_like(x)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        lay.forward(x, ids, w, y=y, stream=s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for _ in range(reps):
            lay.forward(x, ids, w, y=y, stream=s)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / reps
    assert lay.status() == 0
    del g
    lay.close()
    n_w = 3 * SHAPE.I * SHAPE.H
    touched = len(set(ids_h.ravel().tolist()))
    nbytes = touched * (n_w + n_w // 16) + T * SHAPE.H * 2 * 2
    gbs = nbytes / (us * 1e-6) / 1e9
    return {"T": T, "routing": "uniform", "products": "mma.sync (grouped)",
            "experts_touched": touched, "us_per_call": us, "hbm_gbs": gbs,
            "hbm_frac": gbs / peak}


def batched_cases(torch, moe, st, seed, reps=20, cases=BATCHED_CASES):
    """The grouped (token, expert)-sorted path on one 24B layer of the stack at
    batch sizes beyond decode: synthetic routing (k distinct experts per token,
    uniform or Zipf(1.1) popularity), moe_forward timed in a CUDA graph of
    `reps` calls.  Bytes: the touched experts' packed weights + activations.
    Where the library picks the tcgen05 products, the mma.sync tiles are timed
    beside them (FWD_FORCE_MMA)."""
    L = st.layers[0]
    out = []
    expert = 3 * SHAPE.I * SHAPE.H // 2 + 3 * SHAPE.I * SHAPE.H // 32
    tmax = max(t for t, _ in cases)
    lay = moe.MoELayer(SHAPE.E, SHAPE.H, SHAPE.I, SHAPE.top_k, L.codes, L.scales, L.router_w,
                       L.router_b, max_tokens=tmax)
    s = torch.cuda.Stream()
    for T, dist in cases:
        x = torch.from_numpy(synth.make_tokens(T, SHAPE.H, seed=seed, stream=T)
                             .view(np.int16)).cuda().view(torch.bfloat16)
        ids_h, w_h = synth.make_routing(T, SHAPE.E, SHAPE.top_k, dist,
                                        synth.rng_for(seed, 91, T))
        ids, w = torch.from_numpy(ids_h).cuda(), torch.from_numpy(w_h).cuda()
        y = torch.empty_like(x)
        tc = T * SHAPE.top_k >= TC_AUTO_GROUP * SHAPE.E

        def timed(flags):
            s.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(s):
                lay.forward(x, ids, w, y=y, flags=flags, stream=s)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                for _ in range(reps):
                    lay.forward(x, ids, w, y=y, flags=flags, stream=s)
            g.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            del g
            return e0.elapsed_time(e1) * 1e3 / reps

        us = timed(0)
        touched = len(set(ids_h.ravel().tolist()))
        nbytes = touched * expert + T * SHAPE.H * 2 * 2
        row = {"T": T, "routing": dist, "experts_touched": touched,
               "case": "S=64 prefill chunk" if T == 64 else ("decode batch" if T <= 256 else
                                                             "prefill"),
               "products": "tcgen05" if tc else "mma.sync",
               "us_per_call": us, "tokens_per_s": T / (us * 1e-6),
               "hbm_gbs": nbytes / (us * 1e-6) / 1e9}
        if tc:
            row["us_per_call_mma_sync"] = timed(moe.FWD_FORCE_MMA)
        out.append(row)
    lay.close()
    return out


def run_e2e(torch, st, args):
    """Same metric through the public API with host buffers: every token's
    input is copied from pinned host memory and its output read back."""
    T, H = 1, SHAPE.H
    xs = synth.make_tokens(TOKENS_PER_STEP, H, seed=args.seed, stream=11)
    x_host = torch.from_numpy(xs.view(np.int16)).view(torch.bfloat16).pin_memory()
    y_host = torch.empty_like(x_host).pin_memory()
    stream = torch.cuda.current_stream()
    for _ in range(max(1, args.warmup)):
        st.decode_host(x_host, y_host)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        st.decode_host(x_host, y_host)
    e1.record(stream)
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) / 1e3
    return {"value": TOKENS_PER_STEP * args.steps / t, "unit": "tokens/s",
            "h2d_bytes_per_step": TOKENS_PER_STEP * T * H * 2,
            "d2h_bytes_per_step": TOKENS_PER_STEP * T * H * 2}


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
