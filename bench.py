#!/usr/bin/env python
"""MoE-layer forward throughput on B200 (tokens/s) and roofline fractions.

    python bench.py [--gpus N --steps K --warmup W] [--config 2] [--alpha A]
    python bench.py --impl reference ...      (the CPU oracle, timed on host cores)

A step is one pass of the whole path (route, histogram/scan/permute, grouped
SwiGLU, grouped down projection, combine) over one batch of T seeded synthetic
tokens of the Mixtral-8x7B-shaped layer (T=512, H=4096, F=14336, E=8, top-2)
unless --config says otherwise.  Inputs are resident in HBM; L2 is flushed
(a 256 MiB write then a 256 MiB read) between timed steps, outside the timed intervals.  Each step
is timed with CUDA events on the stream the kernels run on, between every
entry point, so the per-kernel times come from the same timed region.

Multi-GPU: the path has no exchange step, so N GPUs run N independent
replicas (one process per GPU, its own token batch); the only collectives are
the barrier and the max-over-ranks of the elapsed time.

Also reported: the end-to-end rate with host copies (pipelined across steps,
and serial), the fp8 layer, every other workload (per_config), the combine
fused into the down GEMM, and the expert-parallel layer with 8 ranks emulated
on one GPU (ep: per-rank kernel times and the bytes of each all-to-all pass).

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "MoE-layer fwd tokens/s at 1 B200; % of roofline (bf16 TC peak or HBM BW)"
FLUSH_BYTES = 256 << 20


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--config", type=int, default=2)
    p.add_argument("--alpha", type=float, default=None)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-per-config", action="store_true",
                   help="time the headline workload only (default: every other workload too, on one GPU)")
    p.add_argument("--per-config-steps", type=int, default=20)
    p.add_argument("--no-fp8", action="store_true", help="skip the fp8 (e4m3) variant of the layer")
    p.add_argument("--no-ep", action="store_true",
                   help="skip the expert-parallel layer (8 ranks emulated on one GPU, decode-shaped workload)")
    p.add_argument("--cpu-budget-s", type=float, default=15.0)
    p.add_argument("--ref-budget-s", type=float, default=150.0)
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def workload(args):
    import synth
    cfg = synth.CONFIGS[args.config]
    if args.alpha is not None:
        cfg = cfg.with_(alpha=args.alpha)
    return cfg


def config_json(cfg, extra=None):
    d = {"workload": cfg.name + ("" if cfg.alpha in (0.0,) else "-alpha%g" % cfg.alpha), "T": cfg.T, "H": cfg.H,
         "F": cfg.F, "E": cfg.E, "k": cfg.k, "C": cfg.C, "alpha": cfg.alpha, "seed": cfg.seed,
         "l2": "flushed between timed steps (256 MiB write, then 256 MiB read); not in the pipelined e2e, "
               "whose per-step inputs (the expert weights) are larger than L2 on every workload but the tiny one",
         "timing": "moe_forward captured once as a CUDA graph, replayed per step, CUDA events around each replay"}
    if extra:
        d.update(extra)
    return d


def dram_traffic(cfg):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    capture, if that capture was taken on this workload and the kernel's
    source has not changed since; else None."""
    import hashlib
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "roofline_traffic.json")))
        src = b"".join(open(os.path.join(ROOT, "grouped_expert_gemm_router_b200", "csrc", f), "rb").read()
                       for f in ("gemm.cu", "common.cuh"))
        if rec["workload"] == cfg.name and rec["source_sha256"] == hashlib.sha256(src).hexdigest():
            return int(rec["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


def routing_stats(counts, C):
    import numpy as np
    n = np.asarray(counts, dtype=np.float64)
    mean = n.mean()
    gini = float(np.abs(n[:, None] - n[None, :]).sum() / (2 * len(n) ** 2 * mean)) if mean > 0 else 0.0
    d = {"counts_min": int(n.min()), "counts_max": int(n.max()), "max_over_mean": float(n.max() / mean),
         "gini": gini, "experts_touched": int((n > 0).sum())}
    if C > 0:
        d["overflow_frac"] = float(np.maximum(n - C, 0).sum() / n.sum())
    return d


def algorithmic_work(cfg, counts):
    """Algorithmic bytes / FLOPs of each kernel from the actual routing.
    Weights count once per touched expert; padded tile rows are not work."""
    T, H, F, k = cfg.T, cfg.H, cfg.F, cfg.k
    R = T * k
    touched = sum(1 for c in counts if c > 0)
    w = {}
    w["swiglu_bytes"] = touched * 2 * H * F * 2 + R * H * 2 + R * F * 2
    w["swiglu_flops"] = 2 * R * H * 2 * F
    w["down_bytes"] = touched * F * H * 2 + R * F * 2 + R * H * 2
    w["down_flops"] = 2 * R * F * H
    w["route_bytes"] = T * H * 2 + H * cfg.E * 4 + T * cfg.E * 4 + T * k * 8
    w["route_flops"] = 2 * T * H * cfg.E
    w["combine_bytes"] = R * H * 2 + T * H * 2 + R * 8
    w["layer_bytes"] = touched * 3 * H * F * 2 + 2 * T * H * 2 + H * cfg.E * 4
    w["layer_flops"] = w["swiglu_flops"] + w["down_flops"] + w["route_flops"]
    return w


class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_id), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def gpu_id_for_smi(torch, dev):
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        return dev


def cpu_baseline(cfg, L, budget_s):
    """The CPU oracle as it stands, single-threaded, on the first S tokens of
    the same batch (route, dispatch, experts, combine), S sized to the budget."""
    import numpy as np

    from oracle import Oracle
    orc = Oracle()

    def run(S):
        x = L.x[:S]
        t0 = time.perf_counter()
        orc.forward(x, L.w_router, L.bias, L.w_gate, L.w_up, L.w_down, cfg.k, C=cfg.C, capped=cfg.C > 0)
        return time.perf_counter() - t0

    t1 = run(1)
    S = int(max(1, min(cfg.T, budget_s / max(t1, 1e-6))))
    dt = run(S) if S > 1 else t1
    return {"value": S / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle", **host_info(),
            "sample": "first %d of the %d tokens of the same seeded batch through the whole oracle forward "
                      "(single-threaded C, fp64 accumulation); %.1f s" % (S, cfg.T, dt)}


def run_reference(args):
    """Reference arm: the CPU oracle timed on the host cores (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import synth
    from oracle import Oracle
    cfg = workload(args)
    L = synth.make_layer(cfg)
    orc = Oracle()

    def step(S):
        t0 = time.perf_counter()
        orc.forward(L.x[:S], L.w_router, L.bias, L.w_gate, L.w_up, L.w_down, cfg.k, C=cfg.C, capped=cfg.C > 0)
        return time.perf_counter() - t0

    t1 = step(1)
    per_step = args.ref_budget_s / max(1, args.steps + args.warmup)
    S = int(max(1, min(cfg.T, per_step / max(t1, 1e-6))))
    for _ in range(args.warmup):
        step(S)
    total = 0.0
    for _ in range(args.steps):
        total += step(S)
    value = S * args.steps / total
    sample = ("first %d of the %d tokens of the seeded batch per step through the whole oracle forward "
              "(single-threaded C, fp64 accumulation)" % (S, cfg.T))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_json(cfg, {"tokens_per_step": S}),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample,
                             **host_info()},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def replica_tokens(cfg, rank, L):
    """The token batch of one replica: rank 0 the seeded batch of the layer,
    rank r the batch drawn with seed offset r (same weights everywhere)."""
    import synth
    return L.x if rank == 0 else synth.x_tokens(cfg, seed_offset=rank)


def max_over_ranks(values, device=None):
    """Element-wise maximum of per-rank timings over every rank of the job
    (the slowest replica sets the job's time); unchanged without a process
    group of more than one rank."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def whole_job_rate(tokens_per_replica_step, steps, world, total_ms):
    """Tokens per second of the whole job: every replica's tokens over the
    slowest replica's time."""
    return tokens_per_replica_step * steps * world / (total_ms * 1e-3)


def forward_launches(cfg):
    """Kernels one moe_forward launches: the router (plus the weight split and
    the tensor-core logits from 2048 tokens on), the histogram and rank
    kernels (only above 4096 routed pairs; below, the router's last CTA builds
    the dispatch), the row copy (unless the SwiGLU GEMM gathers its rows: at
    most 32 routed rows per expert on average), the two grouped GEMMs and the
    combine."""
    router = 3 if cfg.T >= 2048 else 1
    dispatch = 0 if cfg.T * cfg.k <= 4096 else 2
    copy = 0 if cfg.T * cfg.k <= 32 * cfg.E else 1
    return router + dispatch + copy + 3


def host_info():
    """Host cores and CPU model (the CPU baseline's machine)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_nproc": os.cpu_count(), "host_cpu_model": model}


class Bench:
    """One process's device, stream, L2-cleaning buffers and clock sampler."""

    def graph_ms(self, launch, steps):
        """Total device time of `steps` replays of one captured call (L2
        cleaned before each replay, outside the timed interval)."""
        import numpy as np
        torch, dev, stream = self.torch, self.dev, self.stream
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=torch.cuda.Stream(dev)):
            launch()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for _ in range(3):
            self.flush()
            g.replay()
        self.barrier()
        for i in range(steps):
            self.flush()
            ev[i][0].record(stream)
            g.replay()
            ev[i][1].record(stream)
        self.barrier()
        total = float(np.sum([a.elapsed_time(c) for a, c in ev]))
        del g
        return total

    def __init__(self, dev, world, local):
        import torch
        self.torch = torch
        self.dev = dev
        self.world = world
        self.local = local
        self.stream = torch.cuda.current_stream(dev)
        self.flush_w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.flush_r = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def flush(self):
        """Between timed steps: write 256 MiB (evicts everything), then read
        another 256 MiB so the cache holds clean lines and the next step does
        not pay for writing the first buffer back."""
        self.flush_w.zero_()
        self.flush_r.sum()

    def barrier(self):
        import torch.distributed as dist
        if self.world > 1:
            dist.barrier()
        self.torch.cuda.synchronize(self.dev)

    def upload(self, cfg, L, x_rank, flags=0):
        import numpy as np

        import grouped_expert_gemm_router_b200 as moe
        torch, dev = self.torch, self.dev

        def dev_bf16(a):
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

        shape = moe.make_shape(cfg.T, cfg.H, cfg.F, cfg.E, cfg.k, C=cfg.C, capacity=cfg.C > 0, flags=flags)
        b = moe.alloc_buffers(shape, dev)
        b.update(x=dev_bf16(x_rank), w_router=torch.from_numpy(L.w_router).to(dev),
                 bias=None if L.bias is None else torch.from_numpy(L.bias).to(dev),
                 w_gate=dev_bf16(L.w_gate), w_up=dev_bf16(L.w_up), w_down=dev_bf16(L.w_down))
        return shape, b

    def measure(self, cfg, shape, b, steps, warmup):
        """Times one workload: (1) the entry points one by one with CUDA
        events between them (per-kernel times), (2) moe_forward captured once
        as a CUDA graph and replayed per step (the step time).  L2 is cleaned
        before every step, outside the timed intervals."""
        import numpy as np

        import grouped_expert_gemm_router_b200 as moe
        torch, dev, stream = self.torch, self.dev, self.stream
        ws = b["ws"]
        # moe_forward folds the row copy into the SwiGLU GEMM when given no
        # x_perm buffer: the faster choice while the routed rows per expert are few
        gather = cfg.T * cfg.k <= 32 * cfg.E
        fwd_bufs = {**b, "x_perm": None} if gather else b

        def step_events(ev):
            ev[0].record(stream)
            moe.moe_route_dispatch(shape, b["x"], b["w_router"], b["bias"], b["logits"], b["topk_idx"], b["topk_w"],
                                   b["expert_counts"], b["expert_offsets"], b["src_token"], b["dest_row"], ws, stream)
            ev[1].record(stream)
            if not gather:
                moe.moe_gather(shape, b["x"], b["src_token"], b["x_perm"], ws, stream)
            ev[2].record(stream)
            if gather:
                moe.moe_grouped_swiglu_gather(shape, b["x"], b["src_token"], b["w_gate"], b["w_up"], b["h"], ws,
                                              stream)
            else:
                moe.moe_grouped_swiglu(shape, b["x_perm"], b["w_gate"], b["w_up"], b["h"], ws, stream)
            ev[3].record(stream)
            moe.moe_grouped_down(shape, b["h"], b["w_down"], b["y"], ws, stream)
            ev[4].record(stream)
            moe.moe_combine(shape, b["y"], b["dest_row"], b["topk_w"], b["out"], stream)
            ev[5].record(stream)

        wev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
        for _ in range(max(warmup, 3)):
            self.flush()
            step_events(wev)
        torch.cuda.synchronize(dev)
        status = moe.moe_read_status(ws, stream)
        if status & ~moe.MOE_DEV_NAN_LOGIT:
            raise RuntimeError("device status %#x after warm-up (%s)" % (status, cfg.name))

        K = steps
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(K)]
        sampler = ClockSampler(gpu_id_for_smi(torch, self.local))
        self.barrier()
        sampler.start()
        time.sleep(0.15)  # let the sampler take its first reading
        wall0 = time.perf_counter()
        for i in range(K):
            self.flush()
            step_events(evs[i])
        self.barrier()
        seg = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(5)] for i in range(K)])  # ms
        eager_ms = float(seg.sum(axis=1).sum())
        status |= moe.moe_read_status(ws, stream)

        args_c = moe.forward_args(fwd_bufs)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=torch.cuda.Stream(dev)):
            moe.moe_forward(shape, b, ws, args=args_c)
        gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        for i in range(3):
            self.flush()
            g.replay()
        self.barrier()
        for i in range(K):
            self.flush()
            gev[i][0].record(stream)
            g.replay()
            gev[i][1].record(stream)
        self.barrier()
        wall = time.perf_counter() - wall0
        clocks = sampler.stop()
        total_ms = float(np.sum([a.elapsed_time(c) for a, c in gev]))
        del g
        # the same layer with the combine inside the down GEMM's epilogue
        sf = moe.make_shape(shape.T, shape.H, shape.F, shape.E, shape.k, shape.C, flags=shape.flags |
                            moe.MOE_FLAG_FUSED_COMBINE)
        fused_ms = self.graph_ms(lambda: moe.moe_forward(sf, b, ws, args=args_c), K)
        total_ms, eager_ms, fused_ms = max_over_ranks([total_ms, eager_ms, fused_ms], dev)
        status |= moe.moe_read_status(ws, stream)
        return {"total_ms": total_ms, "eager_ms": eager_ms, "kmean_s": seg.mean(axis=0) * 1e-3, "gather": gather,
                "fwd_bufs": fwd_bufs, "clocks": clocks, "status": status, "wall": wall, "fused_ms": fused_ms,
                "counts": b["expert_counts"].cpu().numpy()}

    def measure_fp8(self, cfg, shape, b, steps, warmup):
        """The fp8 (e4m3) layer, same protocol: weights quantized once before
        timing; per step the router/dispatch, the token-row quantization (the
        row copy, or token rows for the row-gathering GEMM), the fp8 SwiGLU
        GEMM, the h quantization, the fp8 down GEMM and the combine."""
        import numpy as np

        import grouped_expert_gemm_router_b200 as moe
        torch, dev, stream = self.torch, self.dev, self.stream
        ws = b["ws"]
        per_token = cfg.T * cfg.k <= 32 * cfg.E
        b.update(moe.alloc_fp8_buffers(shape, per_token=per_token, device=dev))
        moe.quantize_layer_weights_fp8(shape, b, stream)
        src_tok = b["src_token"] if per_token else None

        def step_events(ev):
            ev[0].record(stream)
            moe.moe_route_dispatch(shape, b["x"], b["w_router"], b["bias"], b["logits"], b["topk_idx"], b["topk_w"],
                                   b["expert_counts"], b["expert_offsets"], b["src_token"], b["dest_row"], ws, stream)
            ev[1].record(stream)
            moe.moe_quantize_rows_fp8(shape, moe.MOE_ROWS_TOKENS if per_token else moe.MOE_ROWS_X_PERM, b["x"],
                                      b["src_token"], b["x_q"], b["x_scale"], ws, stream)
            ev[2].record(stream)
            moe.moe_grouped_swiglu_fp8(shape, b["x_q"], b["x_scale"], src_tok, b["wg_q"], b["wg_scale"], b["wu_q"],
                                       b["wu_scale"], b["h"], ws, stream)
            ev[3].record(stream)
            moe.moe_quantize_rows_fp8(shape, moe.MOE_ROWS_H, b["h"], b["src_token"], b["h_q"], b["h_scale"], ws,
                                      stream)
            ev[4].record(stream)
            moe.moe_grouped_down_fp8(shape, b["h_q"], b["h_scale"], b["wd_q"], b["wd_scale"], b["y"], ws, stream)
            ev[5].record(stream)
            moe.moe_combine(shape, b["y"], b["dest_row"], b["topk_w"], b["out"], stream)
            ev[6].record(stream)

        wev = [torch.cuda.Event(enable_timing=True) for _ in range(7)]
        for _ in range(max(warmup, 3)):
            self.flush()
            step_events(wev)
        torch.cuda.synchronize(dev)
        status = moe.moe_read_status(ws, stream)
        if status & ~moe.MOE_DEV_NAN_LOGIT:
            raise RuntimeError("device status %#x after fp8 warm-up (%s)" % (status, cfg.name))
        K = steps
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(K)]
        self.barrier()
        for i in range(K):
            self.flush()
            step_events(evs[i])
        self.barrier()
        seg = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(6)] for i in range(K)])
        args_c = moe.forward_fp8_args(b, per_token)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=torch.cuda.Stream(dev)):
            moe.moe_forward_fp8(shape, b, ws, args=args_c)
        gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        for i in range(3):
            self.flush()
            g.replay()
        self.barrier()
        for i in range(K):
            self.flush()
            gev[i][0].record(stream)
            g.replay()
            gev[i][1].record(stream)
        self.barrier()
        total_ms = float(np.sum([a.elapsed_time(c) for a, c in gev]))
        del g
        sf = moe.make_shape(shape.T, shape.H, shape.F, shape.E, shape.k, shape.C, flags=shape.flags |
                            moe.MOE_FLAG_FUSED_COMBINE)
        fused_ms = self.graph_ms(lambda: moe.moe_forward_fp8(sf, b, ws, args=args_c), K)
        total_ms, fused_ms = max_over_ranks([total_ms, fused_ms], dev)
        status |= moe.moe_read_status(ws, stream)
        return {"total_ms": total_ms, "kmean_s": seg.mean(axis=0) * 1e-3, "per_token": per_token, "status": status,
                "fused_ms": fused_ms, "counts": b["expert_counts"].cpu().numpy()}

    def e2e(self, cfg, shape, b, x_rank, fwd_bufs, steps):
        """The same metric end to end: pinned-host tokens copied in, the layer,
        the output copied back to pinned host memory, every step."""
        import numpy as np

        import grouped_expert_gemm_router_b200 as moe
        torch, dev, stream = self.torch, self.dev, self.stream
        x_host = torch.from_numpy(np.ascontiguousarray(x_rank).view(np.int16)).view(torch.bfloat16).pin_memory()
        out_host = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16).pin_memory()
        args_e = moe.forward_args(fwd_bufs)
        eev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for i in range(-3, steps):
            self.flush()
            if i >= 0:
                eev[i][0].record(stream)
            b["x"].copy_(x_host, non_blocking=True)
            moe.moe_forward(shape, b, b["ws"], stream, args=args_e)
            out_host.copy_(b["out"], non_blocking=True)
            if i >= 0:
                eev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = float(np.sum([a.elapsed_time(c) for a, c in eev]))
        (e2e_ms,) = max_over_ranks([e2e_ms], dev)
        return e2e_ms

    def measure_ep(self, cfg, L, G, steps, warmup):
        """The expert-parallel Cap-and-Spill layer with G ranks held by this
        process on its one GPU: each rank's phases run on its own buffers
        with CUDA events around each, the all-to-alls are carried out as
        device copies (untimed: on G GPUs they cross NVLink).  L2 cleaned
        before every step.  Returns per-phase device times summed over the
        ranks, and each rank's overflow rows."""
        import numpy as np

        import grouped_expert_gemm_router_b200 as moe
        from grouped_expert_gemm_router_b200.ep import CapAndSpillEP, exchange_in_process
        torch, dev, stream = self.torch, self.dev, self.stream

        def dev_bf16(a):
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

        shape = moe.make_shape(cfg.T, cfg.H, cfg.F, cfg.E, cfg.k, C=cfg.C, capacity=True)
        wg, wu, wd = dev_bf16(L.w_gate), dev_bf16(L.w_up), dev_bf16(L.w_down)
        wr = torch.from_numpy(L.w_router).to(dev)
        bias = None if L.bias is None else torch.from_numpy(L.bias).to(dev)
        xs = [dev_bf16(replica_tokens(cfg, r, L)) for r in range(G)]
        ranks = [CapAndSpillEP(shape, G, dev) for _ in range(G)]
        Eg = cfg.E // G
        sl = [slice(r * Eg, (r + 1) * Eg) for r in range(G)]
        phases = ("route_and_pack", "receive", "experts_swiglu", "experts_down", "send_back", "finish")
        calls = {
            "route_and_pack": lambda r: ranks[r].route_and_pack(xs[r], wr, bias, stream),
            "receive": lambda r: ranks[r].receive(stream),
            "experts_swiglu": lambda r: moe.moe_grouped_swiglu(ranks[r].local, ranks[r].x_loc, wg[sl[r]], wu[sl[r]],
                                                               ranks[r].h_loc, ranks[r].ws_loc, stream),
            "experts_down": lambda r: moe.moe_grouped_down(ranks[r].local, ranks[r].h_loc, wd[sl[r]], ranks[r].y_loc,
                                                           ranks[r].ws_loc, stream),
            "send_back": lambda r: ranks[r].send_back(stream),
            "finish": lambda r: ranks[r].finish(stream),
        }

        def step(timed):
            ev = {}
            for ph in phases:
                if ph == "receive":
                    exchange_in_process(ranks, "exchange_in")
                if ph == "finish":
                    exchange_in_process(ranks, "exchange_out")
                for r in range(G):
                    if timed:
                        a, c = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                        a.record(stream)
                        calls[ph](r)
                        c.record(stream)
                        ev[(ph, r)] = (a, c)
                    else:
                        calls[ph](r)
            return ev

        for _ in range(warmup):
            self.flush()
            step(False)
        self.barrier()
        evs = []
        for _ in range(steps):
            self.flush()
            evs.append(step(True))
        self.barrier()
        per_phase = {ph: float(np.mean([sum(e[(ph, r)][0].elapsed_time(e[(ph, r)][1]) for r in range(G))
                                         for e in evs])) * 1e3 for ph in phases}
        lay = moe.moe_workspace_layout(shape)
        spill = [int(ep.ws[lay.total_spill:lay.total_spill + 4].cpu().numpy().view(np.int32)[0]) for ep in ranks]
        status = [moe.moe_read_status(ep.ws) | moe.moe_read_status(ep.ws_loc) for ep in ranks]
        S = ranks[0].S
        # the single-GPU layer on rank 0's tokens, same protocol, for comparison
        shp1, b1 = self.upload(cfg, L, replica_tokens(cfg, 0, L))
        m1 = self.measure(cfg, shp1, b1, steps, warmup)
        del b1, ranks
        return {"G": G, "S": S, "per_phase_us_all_ranks": per_phase, "overflow_rows": spill,
                "device_status": status, "single_gpu_layer_us": m1["total_ms"] / steps * 1e3}

    def measure_ep_direct(self, cfg, L, G, steps, warmup, fp8=False):
        """The peer-store expert-parallel layer with G ranks held by this
        process: peer tables point at the other ranks' own buffers, so the
        stores stay on this GPU (on G GPUs they cross NVLink); the counts
        all-gather is done by copies (untimed).  Per-phase device times summed
        over the ranks, L2 cleaned before every step."""
        import numpy as np

        import grouped_expert_gemm_router_b200 as moe
        from grouped_expert_gemm_router_b200.ep_direct import DirectEP, connect_in_process, gather_counts_in_process
        torch, dev, stream = self.torch, self.dev, self.stream

        def dev_bf16(a):
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

        shape = moe.make_shape(cfg.T, cfg.H, cfg.F, cfg.E, cfg.k)
        wg, wu, wd = dev_bf16(L.w_gate), dev_bf16(L.w_up), dev_bf16(L.w_down)
        wr = torch.from_numpy(L.w_router).to(dev)
        bias = None if L.bias is None else torch.from_numpy(L.bias).to(dev)
        xs = [dev_bf16(replica_tokens(cfg, r, L)) for r in range(G)]
        ranks = [DirectEP(shape, G, r, dev, fp8=fp8) for r in range(G)]
        connect_in_process(ranks)
        Eg = cfg.E // G
        sl = [slice(r * Eg, (r + 1) * Eg) for r in range(G)]
        if fp8:  # the layer's weight codes and scales, sliced per rank below
            wq = {"w_gate": wg, "w_up": wu, "w_down": wd}
            wq.update(moe.alloc_fp8_buffers(shape, device=dev))
            moe.quantize_layer_weights_fp8(shape, wq, stream)
        # The separate launches (plan, dispatch, experts_down, send_back) and
        # their fused forms (plan_dispatch; down_return_fused: the down GEMM
        # storing into the owners' y) all run each step; the totals count one
        # set or the other.
        phases = ("route", "plan", "dispatch", "plan_dispatch", "experts_swiglu", "experts_down", "send_back",
                  "down_return_fused", "finish")
        calls = {
            "route": lambda r: ranks[r].route(xs[r], wr, bias, stream),
            "plan": lambda r: ranks[r].plan(stream),
            "dispatch": lambda r: ranks[r].dispatch(xs[r], stream),
            "plan_dispatch": lambda r: ranks[r].plan_and_dispatch(xs[r], stream),
            "experts_swiglu": lambda r: moe.moe_grouped_swiglu(ranks[r].local, ranks[r].x_loc, wg[sl[r]], wu[sl[r]],
                                                               ranks[r].h_loc, ranks[r].ws_loc, stream),
            "experts_down": lambda r: moe.moe_grouped_down(ranks[r].local, ranks[r].h_loc, wd[sl[r]], ranks[r].y_loc,
                                                           ranks[r].ws_loc, stream),
            "send_back": lambda r: ranks[r].send_back(stream),
            "down_return_fused": lambda r: moe.moe_ep_direct_down_return(shape, G, ranks[r].h_loc, wd[sl[r]],
                                                                         ranks[r].ws_loc, ranks[r].ep_ws, stream),
            "finish": lambda r: ranks[r].finish(stream),
        }

        if fp8:
            L_ = ranks[0].local
            phases = ("route", "plan_dispatch_quantize", "experts_swiglu", "quantize_h", "down_return_fused",
                      "finish")
            calls = {
                "route": lambda r: ranks[r].route(xs[r], wr, bias, stream),
                "plan_dispatch_quantize": lambda r: ranks[r].plan_and_dispatch(xs[r], stream),
                "experts_swiglu": lambda r: moe.moe_grouped_swiglu_fp8(
                    L_, ranks[r].x_loc_q, ranks[r].scale_loc, None, wq["wg_q"][sl[r]], wq["wg_scale"][sl[r]],
                    wq["wu_q"][sl[r]], wq["wu_scale"][sl[r]], ranks[r].h_loc, ranks[r].ws_loc, stream),
                "quantize_h": lambda r: moe.moe_ep_direct_quantize_h(shape, G, ranks[r].h_loc, ranks[r].h_q,
                                                                     ranks[r].h_scale, ranks[r].ep_ws, stream),
                "down_return_fused": lambda r: moe.moe_ep_direct_down_return_fp8(
                    shape, G, ranks[r].h_q, ranks[r].h_scale, wq["wd_q"][sl[r]], wq["wd_scale"][sl[r]],
                    ranks[r].ws_loc, ranks[r].ep_ws, stream),
                "finish": lambda r: ranks[r].finish(stream),
            }

        def step(timed):
            ev = {}
            for ph in phases:
                if ph.startswith("plan"):
                    gather_counts_in_process(ranks)
                for r in range(G):
                    if timed:
                        a, c = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                        a.record(stream)
                        calls[ph](r)
                        c.record(stream)
                        ev[(ph, r)] = (a, c)
                    else:
                        calls[ph](r)
            return ev

        for _ in range(warmup):
            self.flush()
            step(False)
        self.barrier()
        evs = []
        for _ in range(steps):
            self.flush()
            evs.append(step(True))
        self.barrier()
        per_phase = {ph: float(np.mean([sum(e[(ph, r)][0].elapsed_time(e[(ph, r)][1]) for r in range(G))
                                         for e in evs])) * 1e3 for ph in phases}
        status = [moe.moe_read_status(ep.ws) | moe.moe_read_status(ep.ws_loc) for ep in ranks]
        shp1, b1 = self.upload(cfg, L, replica_tokens(cfg, 0, L))
        m1 = self.measure_fp8(cfg, shp1, b1, steps, warmup) if fp8 else self.measure(cfg, shp1, b1, steps, warmup)
        del b1, ranks
        return {"G": G, "fp8": fp8, "per_phase_us_all_ranks": per_phase, "device_status": status,
                "single_gpu_layer_us": m1["total_ms"] / steps * 1e3}

    def e2e_pipelined(self, cfg, shape, b, x_rank, fwd_bufs, steps, warmup):
        """End to end as a serving loop runs it: step i's tokens are copied in
        on one copy stream while step i-1's layer runs, and step i-1's output
        is copied out on another while step i's runs (x and out
        double-buffered on the device).  Timed from the first copy in to the
        last copy out; every step still moves its own tokens and output
        across the host link.  No L2 cleaning between steps (it would sit
        inside the timed interval): the expert weights each step streams are
        larger than L2."""
        import numpy as np

        import grouped_expert_gemm_router_b200 as moe
        torch, dev, comp = self.torch, self.dev, self.stream
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        x_host = torch.from_numpy(np.ascontiguousarray(x_rank).view(np.int16)).view(torch.bfloat16).pin_memory()
        outs_h = [torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        xs = [b["x"], torch.empty_like(b["x"])]
        outs = [fwd_bufs["out"], torch.empty_like(fwd_bufs["out"])]
        bufs = [{**fwd_bufs, "x": xs[j], "out": outs[j]} for j in range(2)]
        # the layer of each buffer set captured once (moe.ForwardGraph), as
        # the headline step is; each replay is one moe_forward
        graphs = [moe.ForwardGraph(shape, bufs[j], b["ws"], comp) for j in range(2)]
        torch.cuda.synchronize(dev)

        def run(n):
            ev_up = [torch.cuda.Event() for _ in range(n)]
            ev_comp = [torch.cuda.Event() for _ in range(n)]
            ev_down = [torch.cuda.Event() for _ in range(n)]
            start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            start.record(up)
            for i in range(n):
                j = i % 2
                if i >= 2:
                    up.wait_event(ev_comp[i - 2])       # the layer of step i-2 has read xs[j]
                with torch.cuda.stream(up):
                    xs[j].copy_(x_host, non_blocking=True)
                ev_up[i].record(up)
                comp.wait_event(ev_up[i])
                if i >= 2:
                    comp.wait_event(ev_down[i - 2])     # outs[j] of step i-2 is on the host
                graphs[j].replay(comp)
                ev_comp[i].record(comp)
                down.wait_event(ev_comp[i])
                with torch.cuda.stream(down):
                    outs_h[j].copy_(outs[j], non_blocking=True)
                ev_down[i].record(down)
            end.record(down)
            return start, end

        run(warmup)
        self.barrier()
        start, end = run(steps)
        self.barrier()
        (ms,) = max_over_ranks([start.elapsed_time(end)], dev)
        return ms


def summarize(cfg, m, steps, world, peaks, peak_src):
    """Throughput, per-kernel times and roofline fractions of one measured
    workload."""
    counts = m["counts"]
    work = algorithmic_work(cfg, counts)
    kmean = m["kmean_s"]
    names = ["route_dispatch", "row_copy", "grouped_swiglu", "grouped_down", "combine"]  # row_copy: 0 if gathered

    def kernel_roof(bytes_, flops, t):
        t_hbm = bytes_ / (peaks["hbm_gbs"] * 1e9)
        t_tc = flops / (peaks["bf16_tflops"] * 1e12)
        if t_hbm >= t_tc:
            a = bytes_ / t / 1e9
            return {"bound": "hbm", "achieved": a, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": a / peaks["hbm_gbs"]}
        a = flops / t / 1e12
        return {"bound": "tensor", "achieved": a, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": a / peaks["bf16_tflops"]}

    # dominant kernel: the fused gate+up SwiGLU grouped GEMM
    roof = kernel_roof(work["swiglu_bytes"], work["swiglu_flops"], kmean[2])
    roof.update({"traffic": dram_traffic(cfg),
                 "kernel": "k_grouped_gemm<0> (moe_grouped_swiglu, or its row-gathering form)",
                 "algorithmic_bytes": work["swiglu_bytes"], "algorithmic_flops": work["swiglu_flops"],
                 "peak_source": peak_src})
    down = kernel_roof(work["down_bytes"], work["down_flops"], kmean[3])
    layer_hbm = work["layer_bytes"] / (peaks["hbm_gbs"] * 1e9)
    layer_tc = work["layer_flops"] / (peaks["bf16_tflops"] * 1e12)
    layer_t = max(layer_hbm, layer_tc)
    kernels = {nm + "_us": t * 1e6 for nm, t in zip(names, kmean)}
    kernels["grouped_swiglu_GBps"] = work["swiglu_bytes"] / kmean[2] / 1e9
    kernels["grouped_swiglu_TFLOPs"] = work["swiglu_flops"] / kmean[2] / 1e12
    kernels["grouped_down_GBps"] = work["down_bytes"] / kmean[3] / 1e9
    kernels["grouped_down_TFLOPs"] = work["down_flops"] / kmean[3] / 1e12
    kernels["grouped_down_roofline"] = {k: down[k] for k in ("bound", "frac", "unit", "achieved")}
    kernels["combine_GBps"] = work["combine_bytes"] / kmean[4] / 1e9
    kernels["combine_hbm_frac"] = kernels["combine_GBps"] / peaks["hbm_gbs"]
    if kmean[1] > 0 and not m["gather"]:
        R = cfg.T * cfg.k
        kernels["row_copy_GBps"] = (cfg.T * cfg.H * 2 + R * cfg.H * 2) / kmean[1] / 1e9
        kernels["row_copy_hbm_frac"] = kernels["row_copy_GBps"] / peaks["hbm_gbs"]
    kernels["swiglu_gathers_rows"] = bool(m["gather"])
    kernels["route_dispatch_TFLOPs_fp32"] = work["route_flops"] / kmean[0] / 1e12
    ms = m["total_ms"] / steps
    return {
        "value": whole_job_rate(cfg.T, steps, world, m["total_ms"]), "ms_per_step": ms,
        "roofline": roof,
        "layer_roofline": {"frac": layer_t / (ms * 1e-3), "roofline_us": layer_t * 1e6,
                           "bound": "hbm" if layer_hbm >= layer_tc else "tensor"},
        "kernels": kernels,
        "eager_entry_points_ms_per_step": m["eager_ms"] / steps,
        "fused_combine": {"value": whole_job_rate(cfg.T, steps, world, m["fused_ms"]),
                          "ms_per_step": m["fused_ms"] / steps,
                          "what": "moe_forward with MOE_FLAG_FUSED_COMBINE (combine in the down GEMM's epilogue)"},
        "clocks": m["clocks"],
        "routing": routing_stats(counts, cfg.C),
        "device_status": m["status"],
        "wall_s_timed_region": m["wall"],
    }


# Peer copy bandwidth per direction between two B200s over NVLink 5, measured
# on this machine type (an exchange model only: no run here had two GPUs).
NVLINK_PEER_GBS = 770.0


def summarize_ep(cfg, e, peaks):
    """The expert-parallel layer per rank: kernel time of each phase, and the
    bytes each rank sends per all-to-all pass (received bytes are the same)."""
    G, S, row = e["G"], e["S"], cfg.H * 2
    Eg = cfg.E // G
    per_rank = {ph: t / G for ph, t in e["per_phase_us_all_ranks"].items()}
    p1, p2, meta = cfg.E * cfg.C * row, G * S * row, G * 2 * Eg * 4
    real = float(sum(e["overflow_rows"])) / G * row
    w_bytes = 3 * Eg * cfg.H * cfg.F * 2
    per_rank["experts"] = per_rank["experts_swiglu"] + per_rank["experts_down"]
    t_exp = per_rank["experts"] * 1e-6
    return {
        "workload": workload_name(cfg), "G": G,
        "ranks": "G ranks emulated on one GPU (each rank's phases on its own buffers); the all-to-alls done as "
                 "device copies and not timed",
        "per_rank_us": per_rank,
        "per_rank_kernels_us": sum(v for k, v in per_rank.items() if k != "experts"),
        "single_gpu_layer_us": e["single_gpu_layer_us"],
        "experts_roofline": {"bound": "hbm", "bytes": w_bytes, "achieved": w_bytes / t_exp / 1e9,
                             "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": w_bytes / t_exp / 1e9 / peaks["hbm_gbs"],
                             "note": "the rank's expert weights over the local SwiGLU + down time",
                             "swiglu_frac": (2 * Eg * cfg.H * cfg.F * 2) / (per_rank["experts_swiglu"] * 1e-6) / 1e9
                             / peaks["hbm_gbs"],
                             "down_frac": (Eg * cfg.H * cfg.F * 2) / (per_rank["experts_down"] * 1e-6) / 1e9
                             / peaks["hbm_gbs"]},
        "exchange_per_rank": {"pass1_bytes": p1, "pass2_bytes": p2, "meta_bytes": meta,
                              "real_overflow_bytes": real, "pass2_padding_frac": 1.0 - real / p2 if p2 else 0.0,
                              "nvlink_model_us": 2 * (p1 + p2 + meta) / (NVLINK_PEER_GBS * 1e9) * 1e6,
                              "nvlink_model": "dispatch and return passes, each rank's sent bytes at %g GB/s per "
                                              "direction (a model, not a measurement)" % NVLINK_PEER_GBS},
        "device_status": e["device_status"],
    }


def experts_roofline(cfg, G, t, peaks, fp8=False):
    """The local grouped GEMMs of one rank (SwiGLU + down, t seconds) against
    the larger of the rank's expert-weight bytes over HBM bandwidth and its
    average rows' (T k) FLOPs over the tensor peak (fp8: one-byte weights,
    twice the bf16 peak)."""
    Eg = cfg.E // G
    w_bytes = 3 * Eg * cfg.H * cfg.F * (1 if fp8 else 2)
    flops = 2.0 * cfg.T * cfg.k * cfg.H * cfg.F * 3
    tc = peaks["bf16_tflops"] * (2 if fp8 else 1)
    if w_bytes / (peaks["hbm_gbs"] * 1e9) >= flops / (tc * 1e12):
        a = w_bytes / t / 1e9
        return {"bound": "hbm", "bytes": w_bytes, "achieved": a, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": a / peaks["hbm_gbs"]}
    a = flops / t / 1e12
    return {"bound": "tensor", "flops": flops, "achieved": a, "peak": tc, "unit": "TFLOP/s", "frac": a / tc}


def summarize_ep_direct(cfg, e, peaks):
    """The peer-store expert-parallel layer per rank: kernel time of each
    phase and the bytes each rank stores into other ranks per direction."""
    G, row = e["G"], cfg.H * 2
    Eg = cfg.E // G
    per_rank = {ph: t / G for ph, t in e["per_phase_us_all_ranks"].items()}
    sent = cfg.T * cfg.k * row  # every routed row once out, its result once back
    out_bytes = cfg.T * cfg.k * (cfg.H + 4) if e.get("fp8") else sent  # fp8: code rows and a scale each
    fp8 = bool(e.get("fp8"))
    down = per_rank["down_return_fused"] if fp8 else per_rank["experts_down"]
    t_exp = (per_rank["experts_swiglu"] + down) * 1e-6
    return {
        "workload": workload_name(cfg) + "-uncapped" + ("-fp8" if fp8 else ""), "G": G,
        "ranks": "G ranks emulated on one GPU: each rank's peer stores go to the other ranks' buffers on the same "
                 "device; the counts all-gather done by copies and not timed",
        "per_rank_us": per_rank,
        # bf16: separate launches (plan, dispatch, down GEMM, return stores)
        # against the fused ones (plan_dispatch, down_return_fused)
        "per_rank_kernels_us": sum(v for k, v in per_rank.items()
                                   if fp8 or k not in ("plan_dispatch", "down_return_fused")),
        "per_rank_kernels_fused_return_us": sum(v for k, v in per_rank.items()
                                                if fp8 or k not in ("plan", "dispatch", "experts_down", "send_back")),
        "single_gpu_layer_us": e["single_gpu_layer_us"],
        "experts_roofline": experts_roofline(cfg, G, t_exp, peaks, fp8),
        "exchange_per_rank": {"dispatch_bytes": out_bytes, "return_bytes": sent, "counts_bytes": G * cfg.E * 4,
                              "nvlink_model_us": (out_bytes + sent) / (NVLINK_PEER_GBS * 1e9) * 1e6,
                              "nvlink_model": "routed rows out and results back at %g GB/s per direction (a "
                                              "model, not a measurement)" % NVLINK_PEER_GBS},
        "device_status": e["device_status"],
    }


def summarize_fp8(cfg, m, steps, world, peaks, peak_src):
    """Throughput and rooflines of the fp8 layer.  Tensor peak for e4m3
    operands: the measured bf16 peak times the nominal fp8/bf16 ratio (2)."""
    counts = m["counts"]
    T, H, F, k = cfg.T, cfg.H, cfg.F, cfg.k
    R = T * k
    touched = sum(1 for c in counts if c > 0)
    kmean = m["kmean_s"]
    names = ["route_dispatch", "quant_x", "grouped_swiglu_fp8", "quant_h", "grouped_down_fp8", "combine"]
    fp8_peak = 2.0 * peaks["bf16_tflops"]

    def roof(bytes_, flops, t):
        t_hbm = bytes_ / (peaks["hbm_gbs"] * 1e9)
        t_tc = flops / (fp8_peak * 1e12)
        if t_hbm >= t_tc:
            a = bytes_ / t / 1e9
            return {"bound": "hbm", "achieved": a, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": a / peaks["hbm_gbs"]}
        a = flops / t / 1e12
        return {"bound": "tensor", "achieved": a, "peak": fp8_peak, "unit": "TFLOP/s", "frac": a / fp8_peak,
                "peak_note": "measured bf16 peak x 2 (nominal e4m3/bf16 ratio)"}

    sw_bytes = touched * 2 * H * F + R * H + R * F * 2
    sw_flops = 4 * R * H * F
    dn_bytes = touched * F * H + R * F + R * H * 2
    dn_flops = 2 * R * F * H
    ms = m["total_ms"] / steps
    layer_bytes = touched * 3 * H * F + 2 * T * H * 2 + H * cfg.E * 4
    layer_flops = sw_flops + dn_flops + 2 * T * H * cfg.E
    layer_t = max(layer_bytes / (peaks["hbm_gbs"] * 1e9), layer_flops / (fp8_peak * 1e12))
    sw = roof(sw_bytes, sw_flops, kmean[2])
    sw.update({"algorithmic_bytes": sw_bytes, "algorithmic_flops": sw_flops, "peak_source": peak_src,
               "kernel": "k_grouped_gemm<0, *, FP8> (moe_grouped_swiglu_fp8)"})
    return {
        "value": whole_job_rate(T, steps, world, m["total_ms"]), "ms_per_step": ms, "dtype": "e4m3 weights and "
        "activations (per-column / per-row power-of-two scales), fp32 accumulate, bf16 h, y, out",
        "kernels": {nm + "_us": t * 1e6 for nm, t in zip(names, kmean)},
        "roofline": sw,
        "grouped_down_roofline": roof(dn_bytes, dn_flops, kmean[4]),
        "layer_roofline": {"frac": layer_t / (ms * 1e-3), "roofline_us": layer_t * 1e6},
        "token_rows_gathered": bool(m["per_token"]), "device_status": m["status"],
        "fused_combine": {"value": whole_job_rate(T, steps, world, m["fused_ms"]), "ms_per_step": m["fused_ms"] / steps},
    }


def per_config_workloads(head):
    """Every workload other than the headline one: configs 1-4 and config 5
    at each skew alpha."""
    import synth
    out = []
    for cid in sorted(synth.CONFIGS):
        alphas = synth.CONFIG5_ALPHAS if cid == 5 else (None,)
        for a in alphas:
            cfg = synth.CONFIGS[cid] if a is None else synth.CONFIGS[cid].with_(alpha=a)
            if (cfg.name, cfg.alpha) != (head.name, head.alpha):
                out.append(cfg)
    return out


def workload_name(cfg):
    return config_json(cfg)["workload"]


def run_ours(args):
    import gc

    import torch
    import torch.distributed as dist

    import grouped_expert_gemm_router_b200 as moe
    import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    cfg = workload(args)
    t0 = time.time()
    L = synth.make_layer(cfg)
    x_rank = replica_tokens(cfg, rank, L)  # each replica its own tokens
    log("rank %d: generated %s in %.1f s" % (rank, cfg.name, time.time() - t0))
    bench = Bench(dev, world, local)
    flags = 0
    shape, b = bench.upload(cfg, L, x_rank, flags)
    K = args.steps
    m = bench.measure(cfg, shape, b, K, args.warmup)
    e2e_ms = bench.e2e(cfg, shape, b, x_rank, m["fwd_bufs"], K)
    e2e_pipe_ms = bench.e2e_pipelined(cfg, shape, b, x_rank, m["fwd_bufs"], K, args.warmup)
    peaks, peak_src = load_peaks()
    m8 = None if args.no_fp8 else bench.measure_fp8(cfg, shape, b, K, args.warmup)

    result = None
    if rank == 0:
        s = summarize(cfg, m, K, world, peaks, peak_src)
        result = {
            "metric": METRIC, "value": s["value"], "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": s["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_json(cfg, {"parallelism": "replicas" if world > 1 else "single-gpu"}),
            "roofline": s["roofline"],
            "layer_roofline": s["layer_roofline"],
            "kernels": s["kernels"],
            "eager_entry_points_ms_per_step": s["eager_entry_points_ms_per_step"],
            "fused_combine": s["fused_combine"],
            "e2e": {"value": whole_job_rate(cfg.T, K, world, e2e_pipe_ms), "unit": "tokens/s",
                    "h2d_bytes_per_step": cfg.T * cfg.H * 2, "d2h_bytes_per_step": cfg.T * cfg.H * 2,
                    "ms_per_step": e2e_pipe_ms / K,
                    "mode": "pipelined: step i's tokens copied in from pinned host memory and step i-1's output "
                            "copied out to pinned host memory on two copy streams while the layer (moe_forward "
                            "replayed from a CUDA graph, moe.ForwardGraph) runs; timed "
                            "from the first copy in to the last copy out; L2 not cleaned between steps (expert "
                            "weights: %.3f GB)" % (3.0 * cfg.E * cfg.H * cfg.F * 2 / 1e9)},
            "e2e_serial": {"value": whole_job_rate(cfg.T, K, world, e2e_ms), "unit": "tokens/s",
                           "h2d_bytes_per_step": cfg.T * cfg.H * 2, "d2h_bytes_per_step": cfg.T * cfg.H * 2,
                           "ms_per_step": e2e_ms / K,
                           "mode": "copy in, moe_forward, copy out on one stream, each step timed alone; "
                                   "L2 cleaned before each step outside the timed interval"},
            "gpu_launches": forward_launches(cfg) * K,
            "clocks": s["clocks"],
            "routing": s["routing"],
            "device_status": s["device_status"],
            "wall_s_timed_region": s["wall_s_timed_region"],
        }
        if m8 is not None:
            result["fp8"] = summarize_fp8(cfg, m8, K, world, peaks, peak_src)
    del b
    gc.collect()
    torch.cuda.empty_cache()

    # every other workload, same protocol (one GPU only: replicas time the
    # headline workload alone)
    per_config = None
    if world == 1 and not args.no_per_config:
        per_config = {}
        for pc in per_config_workloads(cfg):
            t0 = time.time()
            Lp = synth.make_layer(pc)
            shp, bp = bench.upload(pc, Lp, Lp.x, flags)
            kp = min(K, args.per_config_steps)
            mp = bench.measure(pc, shp, bp, kp, min(args.warmup, 5))
            sp = summarize(pc, mp, kp, world, peaks, peak_src)
            sp.update({"steps": kp, "config": config_json(pc), "gpu_launches": forward_launches(pc) * kp})
            if not args.no_fp8 and pc.T * pc.k > 256:  # the tiny layer has nothing to stream
                sp["fp8"] = summarize_fp8(pc, bench.measure_fp8(pc, shp, bp, kp, min(args.warmup, 5)), kp, world,
                                          peaks, peak_src)
            per_config[workload_name(pc)] = sp
            log("per-config %s: %.0f tokens/s (%.1f s)" % (pc.name, sp["value"], time.time() - t0))
            del bp, Lp
            gc.collect()
            torch.cuda.empty_cache()

    # the expert-parallel layer on the decode-shaped workload (C = 16), 8 ranks
    # emulated on this GPU
    ep = None
    if world == 1 and not args.no_ep:
        import synth
        t0 = time.time()
        ce = synth.CONFIGS[4]
        Le = synth.make_layer(ce)
        ep = summarize_ep(ce, bench.measure_ep(ce, Le, 8, min(K, args.per_config_steps), min(args.warmup, 5)), peaks)
        log("expert-parallel %s G=8: %.1f us of kernels per rank (%.1f s)" % (ce.name, ep["per_rank_kernels_us"],
                                                                              time.time() - t0))
        # the same layer by peer stores (uncapped), and the Mixtral-shaped one
        ep["direct"] = summarize_ep_direct(ce, bench.measure_ep_direct(
            ce, Le, 8, min(K, args.per_config_steps), min(args.warmup, 5)), peaks)
        del Le
        gc.collect()
        torch.cuda.empty_cache()
        cm = synth.CONFIGS[2]
        Lm = synth.make_layer(cm)
        ep["direct_mixtral"] = summarize_ep_direct(cm, bench.measure_ep_direct(
            cm, Lm, 8, min(K, args.per_config_steps), min(args.warmup, 5)), peaks)
        ep["direct_fp8"] = summarize_ep_direct(ce, bench.measure_ep_direct(
            ce, synth.make_layer(ce), 8, min(K, args.per_config_steps), min(args.warmup, 5), fp8=True), peaks)
        log("peer-store EP G=8: %.1f / %.1f us of kernels per rank (%.1f s)" % (
            ep["direct"]["per_rank_kernels_us"], ep["direct_mixtral"]["per_rank_kernels_us"], time.time() - t0))
        del Lm
        gc.collect()
        torch.cuda.empty_cache()

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        if per_config is not None:
            result["per_config"] = per_config
        if ep is not None:
            result["ep"] = ep
        if not args.no_cpu_baseline:
            result["cpu_baseline"] = cpu_baseline(cfg, L, args.cpu_budget_s)
        print(json.dumps(result), flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
