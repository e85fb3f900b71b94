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
    ap.add_argument("--skip-nvfp4", action="store_true",
                    help="skip the decode measurement of the stack with NVFP4 experts")
    ap.add_argument("--skip-batched", action="store_true",
                    help="skip the grouped-path measurements at batch sizes beyond decode")
    ap.add_argument("--layers", type=int, default=N_LAYERS,
                    help="layers in the stack (fewer: a smaller case for profiling; "
                         "the bench workload is the full stack)")
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


def gateup_bytes(shape, pairs, prefetch_down):
    """Algorithmic DRAM bytes of one gate/up launch: gate + up rows of every
    selected expert, plus the down matrices it stages into L2 when
    prefetching (they are then read from L2 by the down launch)."""
    gu = 2 * (shape.I * shape.H // 2 + shape.I * shape.H // 32)
    dn = shape.I * shape.H // 2 + shape.I * shape.H // 32
    return pairs * (gu + (dn if prefetch_down else 0))


# the translation unit of the decode kernels (gateup_tma_kernel among them)
# and every header it includes: a change to any of them may change the kernel
DECODE_TU = ("decode.cu", "down.cuh", "gemv.cuh", "kernels.cuh", "common.cuh")


def csrc_digest():
    h = hashlib.sha256()
    d = os.path.join(ROOT, "packed_mxfp4_w4a16_b200", "csrc")
    for name in DECODE_TU:
        with open(os.path.join(d, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def stored_traffic():
    """DRAM bytes per gate/up launch from the committed ncu summary, if it was
    taken from the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "gateup_tma_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("csrc_digest") != csrc_digest():
        return None
    return d.get("dram_bytes_per_launch")


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

def build_stack(torch, moe, seed, n_layers):
    def gen(l):
        return synth.make_layer(SHAPE, seed=seed, layer=l)

    weights = []
    with ThreadPoolExecutor(4) as ex:
        for L in ex.map(gen, range(n_layers)):
            codes = torch.from_numpy(L.codes).cuda()
            scales = torch.from_numpy(L.scales).cuda()
            rw = torch.from_numpy(L.router_w.view(np.int16)).cuda().view(torch.bfloat16)
            weights.append((codes, scales, rw, None))
    return moe.MoEStack(weights, SHAPE.E, SHAPE.H, SHAPE.I, SHAPE.top_k, T=1)


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
    nv.close()
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

    n_layers = args.layers
    st = build_stack(torch, moe, seed=args.seed + rank, n_layers=n_layers)
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

    # bytes per token from the routing of the last replay (distinct experts)
    ids = st.ids.cpu().numpy()
    step_bytes = sum(bytes_per_layer(SHAPE, len(set(ids[l].ravel().tolist())), 1)
                     for l in range(n_layers))
    gbs = step_bytes * TOKENS_PER_STEP * args.steps / (t_ms / 1e3) / 1e9
    peak, peak_kind = load_peaks()

    # ---- per-kernel breakdown: graph with external timing events ----
    kern = kernel_breakdown(torch, moe, st, reps=max(8, min(64, args.steps)))
    pf = not args.no_prefetch
    gu_bytes = gateup_bytes(SHAPE, SHAPE.top_k, pf) + SHAPE.H * 2
    gu_gbs = gu_bytes / (kern["gateup_us"] * 1e-6) / 1e9

    # ---- end to end through the public API with host buffers ----
    e2e = run_e2e(torch, st, args)

    # ---- the grouped path at batch sizes beyond decode (one layer) ----
    batched = batched_cases(torch, moe, st, args.seed) if not args.skip_batched else None

    # ---- the same stack with NVFP4 experts ----
    nvfp4 = nvfp4_stack(torch, moe, st, args) if not args.skip_nvfp4 else None

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
                         "vs 126 MB L2); no flush", "pdl": not args.no_pdl,
                   "prefetch_down": pf},
        "hbm_gbs": gbs, "hbm_frac": gbs / peak, "hbm_peak_gbs": peak,
        "hbm_peak_kind": peak_kind, "bytes_per_token": step_bytes,
        "us_per_token": t_ms * 1e3 / (TOKENS_PER_STEP * args.steps),
        "roofline": {"bound": "hbm", "kernel": "gateup_tma_kernel",
                     "achieved": gu_gbs, "peak": peak, "unit": "GB/s",
                     "frac": gu_gbs / peak, "traffic": stored_traffic(),
                     "bytes_per_launch": gu_bytes, "peak_kind": peak_kind},
        "kernels": kern,
        "e2e": e2e,
        "batched": batched,
        "nvfp4": nvfp4,
        "gpu_launches": 3 * n_layers * TOKENS_PER_STEP * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.skip_cpu_baseline:
        import oracle
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


def kernel_breakdown(torch, moe, st, reps):
    """Average launch duration of each decode kernel kind, measured live: for
    each kind a CUDA graph holds that kind's launch of every layer, back to
    back on the stack's stream (programmatic serialization between them, as
    in the decode graph), timed with CUDA events around whole replays.  The
    routing of the last decoded token stays in place, so every launch does
    the work of a real token.  The down-only graph reads its matrices from
    HBM (no gate/up launch before it stages them into L2)."""
    n = len(st.layers)
    s = st.stream
    saved = st.r.clone()

    def route(l, L):
        moe.moe_route_ex(L.handle, st.r, L.router_w, L.router_b, moe.ROUTE_RMSNORM, st.xn, None,
                         st.ids[l], st.w[l], s)

    def gateup(l, L):
        moe.moe_forward_ex(L.handle, st.xn, st.ids[l], st.w[l], st.r, st.r,
                           moe.FWD_PHASE_GATEUP, s)

    def down(l, L):
        moe.moe_forward_ex(L.handle, st.xn, st.ids[l], st.w[l], st.r, st.r,
                           moe.FWD_PHASE_DOWN, s)

    per = {}
    for name, fn in (("route", route), ("gateup", gateup), ("down", down)):
        g = torch.cuda.CUDAGraph()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.graph(g, stream=s):
            for l, L in enumerate(st.layers):
                fn(l, L)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(s):  # replays and events on the stack's stream
            for _ in range(3):
                g.replay()
            torch.cuda.synchronize()
            e0.record(s)
            for _ in range(reps):
                g.replay()
            e1.record(s)
        torch.cuda.synchronize()
        per[name] = e0.elapsed_time(e1) * 1e3 / (reps * n)
        del g
    st.r.copy_(saved)
    total = sum(per.values())
    return {"route_us": per["route"], "gateup_us": per["gateup"], "down_us": per["down"],
            "share": {k: v / total for k, v in per.items()},
            "launches_timed_per_kind": reps * n,
            "method": "per kind: a graph of that kind's launch for every layer, back to back "
                      "with programmatic serialization, CUDA events around the replays"}


BATCHED_CASES = ((32, "uniform"), (32, "zipf"), (64, "uniform"), (256, "uniform"),
                 (256, "zipf"), (1024, "uniform"), (2048, "uniform"), (2048, "zipf"))
TC_AUTO_GROUP = 40  # the library's tcgen05 products from T k >= 40 E on


def batched_cases(torch, moe, st, seed, reps=20):
    """The grouped (token, expert)-sorted path on one 24B layer of the stack at
    batch sizes beyond decode: synthetic routing (k distinct experts per token,
    uniform or Zipf(1.1) popularity), moe_forward timed in a CUDA graph of
    `reps` calls.  Bytes: the touched experts' packed weights + activations.
    Where the library picks the tcgen05 products, the mma.sync tiles are timed
    beside them (FWD_FORCE_MMA)."""
    L = st.layers[0]
    out = []
    expert = 3 * SHAPE.I * SHAPE.H // 2 + 3 * SHAPE.I * SHAPE.H // 32
    tmax = max(t for t, _ in BATCHED_CASES)
    lay = moe.MoELayer(SHAPE.E, SHAPE.H, SHAPE.I, SHAPE.top_k, L.codes, L.scales, L.router_w,
                       L.router_b, max_tokens=tmax)
    s = torch.cuda.Stream()
    for T, dist in BATCHED_CASES:
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
