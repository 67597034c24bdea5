#!/usr/bin/env python
"""Throughput of the fused TileQ MoE-layer forward on B200 (one JSON line).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--batch T]
    python bench.py --impl reference ...      # the fp64 CPU oracle, timed on the host

A step is one full forward (routing, permutation, column projection, gate/up,
down-side projection, row accumulation, down/combine) over one batch of T
synthetic tokens with every input already resident in HBM.  Default workload:
the largest single-GPU configuration, the fine-grained 64-expert layer (8x8
grid, d_model 4096, d_ff 1536, rank 128, 2-bit residual in groups of 128,
top-8) at T=16384 (prefill, tensor-bound).  The default run also times, each
with its own roofline, the Mixtral-8x7B-shaped layer (8 experts on 2x4,
d_model 4096, d_ff 14336, rank 128, top-2) at decode batches of 1, 8, 32 and
64 tokens (HBM-bound) and at a 4096-token prefill (``extra_workloads``).
With N > 1 (torchrun), every rank runs its own batch on its own GPU: weak
scaling, no data-path collective (the forward has no exchange step).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

L2_BYTES = 126 * 2**20
DEFAULT_CONFIG = 4   # the largest single-GPU configuration: 64 experts on 8x8, 16384 tokens
STAGES = ["route", "permute", "zproj", "gateup", "zdown", "shared", "residual", "combine"]


def aggregate(ms_local, world, T, steps, device="cpu"):
    """Whole-job figures of N replicas: the slowest rank's device time (max over
    ranks, one all-reduce) and the tokens all ranks processed in that time."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms_local)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = float(t.item())
    return ms, world * T * steps / (ms / 1000.0)


def rank_seed(seed, rank):
    """Each replica draws its own synthetic batch (same layer weights)."""
    return seed + 1000 * rank


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="tileq", choices=["tileq", "reference"])
    ap.add_argument("--config", type=int, default=DEFAULT_CONFIG)
    ap.add_argument("--batch", type=int, default=None)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-compare", action="store_true", help="skip the unfused / rank-0 comparisons")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the extra decode / Mixtral-prefill workloads of the default run")
    ap.add_argument("--sketch", action="store_true",
                    help="time the Gaussian-sketch global low-rank decomposition of one projection's W_big "
                         "(the configuration's gate projection) instead of the forward")
    ap.add_argument("--place", action="store_true",
                    help="time the expert placement (embeddings, K-Means biclustering, greedy 2D placement) "
                         "of the configuration's gate projection instead of the forward")
    ap.add_argument("--r0", type=int, default=16, help="rank of the per-expert factors for --place")
    ap.add_argument("--bits", type=int, default=2, choices=[2, 3], help="residual code width of the layer")
    return ap.parse_args()


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d["bf16_tflops_sustained"], "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML reads only)
# ---------------------------------------------------------------------------
REASON_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, device_index: int):
        self.samples = []
        self.reasons = 0
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = self._handle(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report no clocks
            self.err = str(e)

    def _handle(self, idx):
        import torch
        nv = self.nv
        try:
            props = torch.cuda.get_device_properties(idx)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(idx)

    def _run(self):
        nv = self.nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= int(get_reasons(self.h))
            except Exception:
                pass
            time.sleep(0.0005)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def report(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        names = [n for b, n in REASON_BITS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": float(self.max_mhz),
                "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# the oracle on the host (CPU baseline and reference arm)
# ---------------------------------------------------------------------------
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def host_cores():
    """Host cores this process may run on (the oracle's BLAS uses them)."""
    return len(os.sched_getaffinity(0))


def blas_on_host_cores():
    """Scope in which the oracle's BLAS runs one thread per host core, whatever
    a launcher set (torchrun sets OMP_NUM_THREADS=1 for every rank; only rank 0
    runs the oracle)."""
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(limits=host_cores(), user_api="blas")
    except Exception:
        import contextlib
        return contextlib.nullcontext()


def oracle_step(layer, x, logits, tok):
    import oracle
    return oracle.forward(layer, x, logits, tokens=[tok])


def cpu_baseline(layer, x, logits, n_tokens=1):
    """The oracle as it stands on a bounded sample: the first n_tokens tokens."""
    with blas_on_host_cores():
        threads = blas_threads()
        t0 = time.perf_counter()
        for t in range(n_tokens):
            oracle_step(layer, x, logits, t)
        dt = time.perf_counter() - t0
    return {"value": n_tokens / dt, "unit": "tokens/s", "cores": host_cores(), "blas_threads": threads,
            "kind": "oracle",
            "sample": f"{n_tokens} token(s) of the batch through the fp64 oracle "
                      f"(dense reconstruction of each routed expert's projections), {dt:.1f} s"}


def run_reference(args, cfg, T):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return  # only rank 0 runs the host oracle
    layer = synth.make_layer(cfg, seed=args.seed)
    logits, x = synth.make_inputs(cfg, T, seed=args.seed)
    with blas_on_host_cores():
        threads = blas_threads()
        for i in range(args.warmup):
            oracle_step(layer, x, logits, i % T)
        t0 = time.perf_counter()
        for i in range(args.steps):
            oracle_step(layer, x, logits, (args.warmup + i) % T)
        dt = time.perf_counter() - t0
    value = args.steps / dt
    line = {
        "impl": "reference", "metric": metric_name(cfg, T), "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(cfg, T, args, "host"),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": host_cores(),
                         "blas_threads": threads,
                         "kind": "oracle",
                         "sample": "each step: one token of the batch through the fp64 oracle"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def metric_name(cfg, T):
    return "TileQ MoE-layer tokens/s"


def workload_config(cfg, T, args, l2):
    return {"workload": f"{cfg.name} T={T}", "experts": cfg.K, "grid": f"{cfg.M}x{cfg.N}",
            "d_model": cfg.d_model, "d_ff": cfg.d_ff, "rank": cfg.rank, "group": cfg.group,
            "top_k": cfg.top_k, "tokens_per_gpu": T, "shared_d_ff": cfg.shared_d_ff,
            "residual_bits": cfg.bits, "parallelism": f"replicas x{args.gpus}", "l2": l2}


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------
def run_sketch(args, cfg):
    """Gaussian-sketch decomposition of the configuration's gate W_big [M*F, N*D] at rank r with
    8 columns of oversampling; synthetic bf16 expert weights and sketch drawn on the device."""
    import ctypes
    import torch
    from tiled_rank_b200 import _lib as L
    if int(os.environ.get("RANK", "0")) != 0:
        return  # one decomposition: replicas would only repeat it
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    K, M, N = cfg.K, cfg.M, cfg.N
    d_out, d_in = cfg.d_ff, cfg.d_model
    r = cfg.rank
    l = r + 8
    gen = torch.Generator(device=dev).manual_seed(args.seed)
    w = (torch.randn((K, d_out, d_in), generator=gen, device=dev) * (d_in ** -0.5)).to(torch.bfloat16)
    om = torch.randn((l, N * d_in), generator=gen, device=dev).to(torch.bfloat16)
    grid = np.arange(K, dtype=np.int32)
    wb = L.tileq_wbig()
    wb.K, wb.M, wb.N, wb.d_out, wb.d_in = K, M, N, d_out, d_in
    wb.w = w.data_ptr()
    wb.grid_assign = grid.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    ws = torch.empty(L.tileq_sketch_workspace_size(wb, l, r), dtype=torch.uint8, device=dev)
    U = torch.empty((M * d_out, r), device=dev)
    S = torch.empty((r,), device=dev)
    V = torch.empty((N * d_in, r), device=dev)
    for _ in range(args.warmup):
        L.tileq_sketch_lowrank(wb, om, l, r, U, S, V, ws)
    torch.cuda.synchronize()
    n0 = L.tileq_launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(0) as clocks:
        e0.record()
        for _ in range(args.steps):
            L.tileq_sketch_lowrank(wb, om, l, r, U, S, V, ws)
        e1.record()
        torch.cuda.synchronize()
    launches = L.tileq_launch_count() - n0
    ms = e0.elapsed_time(e1) / args.steps
    R, C = M * d_out, N * d_in
    flops = 2.0 * 2 * R * C * l  # W_big Omega and Q^T W_big
    peaks = measured_peaks()
    t_roof = flops / (peaks["bf16_tflops"] * 1e12)
    cpu = None
    if not args.no_cpu_baseline:
        from oracle import sketch as osk
        with blas_on_host_cores():
            threads = blas_threads()
            t0 = time.perf_counter()
            w_bits = w.view(torch.int16).cpu().numpy().view(np.uint16)
            big = osk.assemble_wbig(w_bits, grid, M, N)
            omega = osk.widen_bf16(om.view(torch.int16).cpu().numpy().view(np.uint16)).T
            osk.sketch_lowrank(big, omega, r)
            dt = time.perf_counter() - t0
        cpu = {"value": 1.0 / dt, "unit": "sketch/s", "cores": host_cores(), "blas_threads": threads,
               "kind": "oracle",
               "sample": f"the whole decomposition ({R} x {C}, rank {r}, l {l}) through the fp64 oracle, {dt:.1f} s"}
    line = {
        "metric": "TileQ Gaussian-sketch global low-rank decompositions/s", "value": 1000.0 / ms,
        "unit": "sketch/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "replicas only", "vs_baseline": None, "dtype": "bf16/f32/f64",
        "data": "synthetic (Gaussian bf16 expert weights and sketch, seeded)",
        "config": {"workload": f"{cfg.name} gate W_big sketch", "rows": R, "cols": C, "rank": r, "sketch": l,
                   "experts": K, "grid": f"{M}x{N}", "l2": "working set above L2"},
        "roofline": {"bound": "tensor", "achieved": flops / (ms / 1000.0) / 1e12, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": t_roof / (ms / 1000.0), "traffic": None,
                     "note": "large products only; the two l x l Jacobi eigen-decompositions (one CTA, "
                             "latency-bound) take most of the time"},
        "gpu_launches": launches, "clocks": clocks.report(), "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


FP64_TFLOPS = 148 * 64 * 2 * 1.965e9 / 1e12   # SMs x fp64 FMA/clk/SM x 2 x max SM clock


def run_place(args, cfg):
    """Expert placement of the configuration's gate projection: per-expert rank-r0
    factors U_k [d_ff, r0] and V_k [d_model, r0] with a planted grid (synthetic,
    seeded), embeddings + both K-Means + greedy placement per step."""
    import torch
    from tiled_rank_b200 import _lib as L
    if int(os.environ.get("RANK", "0")) != 0:
        return  # one placement: replicas would only repeat it
    if args.warmup < 3:
        raise SystemExit("at least 3 warm-up steps")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    K, M, N, r0 = cfg.K, cfg.M, cfg.N, args.r0
    d_u, d_v = cfg.d_ff, cfg.d_model
    u_np, v_np, _ = synth.planted_factors(K, M, N, d_u, d_v, r0, noise=0.1, seed=args.seed)
    u = torch.from_numpy(u_np).to(dev)
    v = torch.from_numpy(v_np).to(dev)
    pin = L.place_in(u, v, M, N, 100)
    ws = torch.empty(L.tileq_place_workspace_size(pin), dtype=torch.uint8, device=dev)
    grid = torch.empty((K,), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush_buf = torch.empty(256 * 2**20, dtype=torch.uint8, device=dev)   # 2x L2: inputs are smaller
    for _ in range(args.warmup):
        L.tileq_place_experts(pin, grid, ws)
    torch.cuda.synchronize()
    nst = 5
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * args.steps)]
    sevs = [[torch.cuda.Event(enable_timing=True) for _ in range(nst)] for _ in range(args.steps)]
    for sev in sevs:
        for e in sev:
            e.record(stream)
    torch.cuda.synchronize()
    n0 = L.tileq_launch_count()
    with ClockSampler(0) as clocks:
        for i in range(args.steps):
            flush_buf.zero_()
            ev[2 * i].record(stream)
            L.tileq_place_experts(pin, grid, ws)
            ev[2 * i + 1].record(stream)
        torch.cuda.synchronize()
    launches = L.tileq_launch_count() - n0
    # per-stage device times from a second pass of the same steps, with the
    # library's stage-boundary events on (kept out of the timed pass above)
    for i in range(args.steps):
        flush_buf.zero_()
        L.tileq_set_stage_events(sevs[i])
        L.tileq_place_experts(pin, grid, ws)
    torch.cuda.synchronize()
    L.tileq_set_stage_events(None)
    ms = sum(ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(args.steps)) / args.steps
    names = ["sign", "gram", "cluster", "greedy"]
    stage_ms = {n: sum(sevs[i][j].elapsed_time(sevs[i][j + 1]) for i in range(args.steps)) / args.steps
                for j, n in enumerate(names)}
    # end to end through the C ABI: factors from pinned host memory, grid_assign back to the host
    u_h = torch.from_numpy(u_np).pin_memory()
    v_h = torch.from_numpy(v_np).pin_memory()
    g_h = torch.empty((K,), dtype=torch.int32).pin_memory()
    u_d, v_d = torch.empty_like(u), torch.empty_like(v)
    pin_e = L.place_in(u_d, v_d, M, N, 100)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_ms = 0.0
    for i in range(args.warmup + args.steps):
        flush_buf.zero_()
        e0.record(stream)
        u_d.copy_(u_h, non_blocking=True)
        v_d.copy_(v_h, non_blocking=True)
        L.tileq_place_experts(pin_e, grid, ws)
        g_h.copy_(grid, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        if i >= args.warmup:
            e2e_ms += e0.elapsed_time(e1)
    e2e_ms /= args.steps
    D = (d_u + d_v) * r0
    gram_flops = 2.0 * K * (K + 1) / 2 * D        # the symmetric half of E E^T, both sides
    in_bytes = K * D * 4
    cpu = None
    if not args.no_cpu_baseline:
        from oracle import placement as opl
        with blas_on_host_cores():
            threads = blas_threads()
            t0 = time.perf_counter()
            opl.place_experts(u_np, v_np, M, N, 100)
            dt = time.perf_counter() - t0
        cpu = {"value": 1.0 / dt, "unit": "placements/s", "cores": host_cores(), "blas_threads": threads,
               "kind": "oracle", "sample": f"one whole placement ({K} experts, factors {d_u}+{d_v} x {r0}) "
                                           f"through the fp64 oracle, {dt:.2f} s"}
    line = {
        "metric": "TileQ expert placements/s (embeddings + K-Means biclustering + greedy 2D placement)",
        "value": 1000.0 / ms, "unit": "placements/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "replicas only", "vs_baseline": None,
        "dtype": "f32 in, f64", "data": "synthetic (planted-grid orthonormal factors with random column signs, "
                                        "seeded)",
        "config": {"workload": f"{cfg.name} gate-projection expert placement", "experts": K, "grid": f"{M}x{N}",
                   "d_u": d_u, "d_v": d_v, "r0": r0, "l2": "flushed between steps (inputs smaller than L2)"},
        "stages_ms": stage_ms,
        "roofline": {"bound": "alu", "achieved": gram_flops / (stage_ms["gram"] / 1000.0) / 1e12,
                     "peak": FP64_TFLOPS, "unit": "TFLOP/s",
                     "frac": gram_flops / (stage_ms["gram"] / 1000.0) / 1e12 / FP64_TFLOPS, "traffic": None,
                     "kernel": "pl_gram_kernel (fp64 Gram of the embeddings, symmetric half counted)",
                     "hbm_floor_us": in_bytes / (measured_peaks()["hbm_gbs"] * 1e9) * 1e6,
                     "note": "peak derived: 148 SMs x 64 fp64 FMA/clk x 2 x 1965 MHz"},
        "e2e": {"value": 1000.0 / e2e_ms, "unit": "placements/s", "h2d_bytes_per_step": in_bytes,
                "d2h_bytes_per_step": K * 4},
        "gpu_launches": launches, "clocks": clocks.report(), "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def default_batch(cid, cfg):
    return 64 if cid == 1 else cfg.batches[-1]


# Extra workloads timed in the default run, each with its own roofline: the
# Mixtral-shaped decode batches (HBM-bound) and the Mixtral-shaped prefill
# (tensor-bound); the headline is the largest single-GPU configuration.
EXTRAS = [(1, 1), (1, 8), (1, 32), (1, 64), (2, 4096)]


def measure(args, cfg, T, dev, world, rank, e2e=True, compare=True, cpu=True):
    """Time K forwards of one workload; returns the fields of its JSON line."""
    import torch
    import torch.distributed as dist
    import tiled_rank_b200 as tq
    from tiled_rank_b200 import roofline

    local = dev.index
    layer = synth.make_layer(cfg, seed=args.seed)
    logits_np, x_np = synth.make_inputs(cfg, T, seed=rank_seed(args.seed, rank))
    dl = tq.DeviceLayer(layer, dev)
    lg = torch.from_numpy(logits_np).to(dev)
    xt = torch.from_numpy(x_np.view(np.int16)).to(dev).view(torch.bfloat16)
    out = torch.empty((T, dl.d_y), dtype=torch.bfloat16, device=dev)
    ws = dl.workspace(T)
    route = dl.route_buffers(T)
    stream = torch.cuda.current_stream(dev)

    # realised routing -> algorithmic work
    dl.forward(xt, lg, out=out, ws=ws, route=route)
    torch.cuda.synchronize(dev)
    topk = route["topk_idx"].cpu().numpy()
    wk = roofline.work(layer, topk)
    footprint = wk["bytes"]
    flush = footprint < 3 * L2_BYTES
    flush_buf = torch.empty(256 * 2**20, dtype=torch.uint8, device=dev) if flush else None

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        dl.forward(xt, lg, out=out, ws=ws)
    torch.cuda.synchronize(dev)

    # ---------------- timed region: K forwards, inputs resident.  On every
    # SAMPLE-th step the library records one event at every stage boundary on
    # the launching stream (per-kernel device times for the roofline); sampling
    # keeps the events' own cost out of the other steps.
    SAMPLE = 8
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * args.steps)]
    sampled = list(range(0, args.steps, SAMPLE))
    sevs = {i: [torch.cuda.Event(enable_timing=True) for _ in range(len(STAGES) + 1)] for i in sampled}
    for sev in sevs.values():  # create the CUDA events (first record) before the timed region
        for e in sev:
            e.record(stream)
    torch.cuda.synchronize(dev)
    n0 = tq.tileq_launch_count()
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        if flush:
            for i in range(args.steps):
                flush_buf.zero_()
                tq.tileq_set_stage_events(sevs.get(i))
                ev[2 * i].record(stream)
                dl.forward(xt, lg, out=out, ws=ws)
                ev[2 * i + 1].record(stream)
        else:
            ev[0].record(stream)
            for i in range(args.steps):
                tq.tileq_set_stage_events(sevs.get(i))
                dl.forward(xt, lg, out=out, ws=ws)
            ev[1].record(stream)
        torch.cuda.synchronize(dev)
    tq.tileq_set_stage_events(None)
    barrier()
    launches = tq.tileq_launch_count() - n0
    if flush:
        ms = sum(ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(args.steps))
    else:
        ms = ev[0].elapsed_time(ev[1])
    ms, value = aggregate(ms, world, T, args.steps, dev)
    ms_per_step = ms / args.steps

    # ---------------- per-stage device times of the sampled timed steps
    stage_ms = np.zeros(len(STAGES))
    for sev in sevs.values():
        stage_ms += np.array([sev[i].elapsed_time(sev[i + 1]) for i in range(len(STAGES))])
    stage_ms /= len(sevs)
    stage_times = {n: round(float(t), 5) for n, t in zip(STAGES, stage_ms)}

    peaks = measured_peaks()
    dom = max(("gateup", "residual", "zproj", "zdown", "shared"),
              key=lambda n: stage_times.get(n, 0.0) if n in wk["stages"] else -1)
    dw = wk["stages"][dom]
    t_dom = stage_times[dom] / 1000.0
    hbm_s = dw["bytes"] / (peaks["hbm_gbs"] * 1e9)
    tc_s = dw["flops"] / (peaks["bf16_tflops"] * 1e12)
    if hbm_s >= tc_s:
        roof = {"bound": "hbm", "achieved": dw["bytes"] / t_dom / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": dw["flops"] / t_dom / 1e12,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["kernel"] = dom
    roof["kernel_ms"] = stage_times[dom]
    roof["alg_bytes"] = dw["bytes"]
    roof["alg_flops"] = dw["flops"]
    roof["peak_source"] = peaks["source"]
    roof["traffic"] = traffic_for(dom, T, cfg)
    whole = {"alg_bytes": wk["bytes"], "alg_flops": wk["flops"],
             "t_roof_ms": 1000 * max(wk["bytes"] / (peaks["hbm_gbs"] * 1e9),
                                     wk["flops"] / (peaks["bf16_tflops"] * 1e12))}
    whole["frac_of_roofline"] = whole["t_roof_ms"] / ms_per_step
    res = {"ms_per_step": ms_per_step, "value": value, "roofline": roof, "whole_step": whole,
           "stage_ms": stage_times, "gpu_launches": launches, "clocks": clocks.report(),
           "config": workload_config(cfg, T, args,
                                     "L2 flushed (256 MB write) between steps" if flush else
                                     f"working set {footprint / 2**20:.0f} MB > 3x L2, no flush")}

    # ---------------- end to end through the public API with host buffers
    if e2e:
        x_h = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).pin_memory()
        lg_h = torch.from_numpy(logits_np).pin_memory()
        out_h = torch.empty((T, dl.d_y), dtype=torch.bfloat16).pin_memory()
        xd = torch.empty_like(xt)
        lgd = torch.empty_like(lg)
        for _ in range(3):
            xd.copy_(x_h, non_blocking=True)
            lgd.copy_(lg_h, non_blocking=True)
            dl.forward(xd, lgd, out=out, ws=ws)
            out_h.copy_(out, non_blocking=True)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(args.steps):
            xd.copy_(x_h, non_blocking=True)
            lgd.copy_(lg_h, non_blocking=True)
            dl.forward(xd, lgd, out=out, ws=ws)
            out_h.copy_(out, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(e2e_ms, op=dist.ReduceOp.MAX)
        e2e_ms = float(e2e_ms.item())
        res["e2e"] = {"value": world * T * args.steps / (e2e_ms / 1000.0), "unit": "tokens/s",
                      "h2d_bytes_per_step": x_h.numel() * 2 + lg_h.numel() * 4,
                      "d2h_bytes_per_step": out_h.numel() * 2}

    # ---------------- in-run comparisons (rank 0, N = 1)
    if compare and rank == 0 and world == 1 and not args.no_compare:
        res.update(compare_paths(cfg, layer, dl, xt, lg, out, T, args, flush_buf, ms_per_step))
    if cpu and rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(layer, x_np, logits_np, n_tokens=4)
    del dl, ws, route, out, flush_buf
    torch.cuda.empty_cache()
    return res


def main():
    args = parse()
    cid = args.config
    cfg = synth.CONFIGS[cid]
    if args.bits != cfg.bits:
        cfg = dataclasses.replace(cfg, bits=args.bits, name=f"{cfg.name}-{args.bits}bit")
    T = args.batch or default_batch(cid, cfg)
    if args.sketch:
        run_sketch(args, cfg)
        return
    if args.place:
        run_place(args, cfg)
        return
    if args.impl == "reference":
        run_reference(args, cfg, T)
        return
    if args.warmup < 3:
        raise SystemExit("at least 3 warm-up steps")

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    head = measure(args, cfg, T, dev, world, rank)
    extras = {}
    if world == 1 and not args.no_extras and args.batch is None and cid == DEFAULT_CONFIG and args.bits == 2:
        for ec, eT in EXTRAS:
            ecfg = synth.CONFIGS[ec]
            r = measure(args, ecfg, eT, dev, world, rank, e2e=False, compare=False, cpu=False)
            extras[f"{ecfg.name} T={eT}"] = {k: r[k] for k in ("ms_per_step", "value", "roofline", "whole_step",
                                                               "stage_ms", "clocks")}

    if rank == 0:
        line = {
            "metric": metric_name(cfg, T), "value": head["value"], "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
            "data": "synthetic (seeded numpy draws in the stored TileQ format)",
            "config": head["config"], "roofline": head["roofline"], "whole_step": head["whole_step"],
            "stage_ms": head["stage_ms"], "e2e": head["e2e"], "gpu_launches": head["gpu_launches"],
            "cpu_baseline": head.get("cpu_baseline"), "clocks": head["clocks"],
        }
        for k in ("unfused", "rank0"):
            if k in head:
                line[k] = head[k]
        if extras:
            line["extra_workloads"] = extras
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def traffic_for(kernel, T, cfg):
    """DRAM bytes per launch from the committed ncu summary, if it matches the current source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    key = f"{kernel}:{cfg.name}:T={T}"
    ent = d.get(key)
    if not ent or ent.get("source_sha") != source_sha(ent.get("sources")):
        return None
    return ent.get("dram_bytes_per_launch")


def source_sha(files=None):
    """Hash of the CUDA sources: the listed files of tiled_rank_b200/csrc (the
    captured kernel's own file and its headers), or all of them."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "tiled_rank_b200", "csrc")
    names = sorted(files) if files else sorted(f for f in os.listdir(csrc) if f.endswith((".cu", ".cuh")))
    for f in names:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def compare_paths(cfg, layer, dl, xt, lg, out, T, args, flush_buf, fused_ms):
    """Unfused per-expert low-rank path and the rank-0 (residual only) layer, same batch."""
    import torch
    import tiled_rank_b200 as tq
    dev = xt.device
    res = {}

    def time_fn(fn, n):
        for _ in range(3):
            fn()
        torch.cuda.synchronize(dev)
        tot = 0.0
        for _ in range(n):
            if flush_buf is not None:
                flush_buf.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize(dev)
            tot += a.elapsed_time(b)
        return tot / n

    n = max(3, min(args.steps, 20))
    pe = [synth.per_expert_lowrank(layer, p) for p in layer.projs]
    dl.set_per_expert(pe)
    t_unf = time_fn(lambda: dl.forward(xt, lg, out=out, unfused=True), n)
    res["unfused"] = {"ms_per_step": t_unf, "value": T / (t_unf / 1000.0),
                      "fusion_gain": t_unf / fused_ms}
    dl.packed_pe = None
    r0 = tq.DeviceLayer(synth.make_layer(cfg, seed=args.seed, rank=0), dev)
    t_r0 = time_fn(lambda: r0.forward(xt, lg, out=out), n)
    res["rank0"] = {"ms_per_step": t_r0, "lowrank_overhead": fused_ms / t_r0 - 1.0}
    del r0
    return res


if __name__ == "__main__":
    main()
