#!/usr/bin/env python
"""DCU denoising-step throughput on one B200 (or N independent replicas).

Workload (default): LLaDA-8B-shaped random-init bf16 model (32 layers,
d = 4096, 32 x 128 MHA, SwiGLU 12288, vocab 126464), one sequence of
N = 1024 = 768 prompt + 256 masked positions, B_layer = 32, B_window = 32,
Fréchet commit with delta = 0.1.  A step is one DCU step (layer-0 refresh,
per-layer dynamics / budget / selection / recompute / scatter) plus the commit
(LM head on the masked rows, softmax-max, sort, Fréchet rule), i.e. every row
of the hot path except the dense forward, which fills the caches once before
timing and is reported separately.

Prints one JSON line (rank 0).  ``--impl reference`` times the fp64 CPU
oracle instead, on a bounded sample of the same step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "DCU denoise steps/s & gen tokens/s, LLaDA-8B shape, 1×B200; % of HBM roofline"

WORKLOADS = {
    "llada8b": dict(shape="LLADA_8B", n_prompt=768, n_gen=256, batch=1, B_layer=32, B_window=32, rule=0, param=0.1,
                    desc="LLaDA-8B-shaped DCU step, N=1024 (768 prompt + 256 masked), B_layer=32, B_window=32, "
                         "Frechet delta=0.1"),
    "dream7b": dict(shape="DREAM_7B", n_prompt=768, n_gen=256, batch=1, B_layer=32, B_window=32, rule=2, param=0.9,
                    desc="Dream-7B-shaped DCU step (GQA 28/4), N=1024, B_layer=32, B_window=32, factor f=0.9"),
    "long8k": dict(shape="LLADA_8B", n_prompt=7680, n_gen=512, batch=1, B_layer=96, B_window=64, rule=0,
                   param=0.05, desc="LLaDA-8B shape, N=8192 (7680 prompt + 512 masked), B_layer=96, B_window=64, "
                                    "Frechet delta=0.05"),
    "batch4": dict(shape="LLADA_8B", n_prompt=1536, n_gen=512, batch=4, B_layer=64, B_window=32, rule=1, param=0.9,
                   desc="LLaDA-8B shape, 4 sequences x N=2048 (1536 prompt + 512 masked), B_layer=64, B_window=32, "
                        "threshold tau=0.9"),
    "toy": dict(shape="TOY", n_prompt=192, n_gen=64, batch=1, B_layer=16, B_window=16, rule=0, param=0.1,
                desc="toy fp32 DCU step (4 layers, d=256), N=256 (192 prompt + 64 masked), B_layer=16, B_window=16, "
                     "Frechet delta=0.1"),
}


# ---------------------------------------------------------------- replicas (one per rank, no collective on the data path)

def replica_seed(rank: int) -> int:
    """Seed of the sequences rank `rank` decodes (the model weights are shared)."""
    return 1 + rank


def reduce_over_ranks(x: float, world: int, op: str, device) -> float:
    """max / sum of a per-rank scalar over all ranks (identity for one rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def aggregate_rate(units_per_rank: int, world: int, ms_step_max: float, steps: int) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / (ms_step_max * steps / 1000.0)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


# ---------------------------------------------------------------- clocks sampling

class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons of the GPU
    while running: NVML polled every 2 ms (so a timed region of ~0.1 s still
    gets dozens of samples), else nvidia-smi every 100 ms.  The GPU is found by
    the UUID of the CUDA device, so CUDA_VISIBLE_DEVICES cannot point it at
    another GPU.  Read-only: no setting of the GPU is touched."""

    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, period_s: float = 0.002):
        self.index, self.period = index, period_s
        self.proc = None
        self.thread = None
        self.stop_flag = threading.Event()
        self.samples = []        # (sm_mhz, sm_max_mhz, set of reason names)
        self.source = None

    def _uuid(self):
        try:
            import torch
            u = str(torch.cuda.get_device_properties(self.index).uuid)
            return u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            return None

    def start(self):
        uuid = self._uuid()
        try:
            import pynvml as N
            N.nvmlInit()
            h = N.nvmlDeviceGetHandleByUUID(uuid) if uuid else N.nvmlDeviceGetHandleByIndex(self.index)
            bits = {"hw_slowdown": getattr(N, "nvmlClocksThrottleReasonHwSlowdown", 0x8),
                    "hw_thermal_slowdown": getattr(N, "nvmlClocksThrottleReasonHwThermalSlowdown", 0x40),
                    "sw_thermal_slowdown": getattr(N, "nvmlClocksThrottleReasonSwThermalSlowdown", 0x20),
                    "sw_power_cap": getattr(N, "nvmlClocksThrottleReasonSwPowerCap", 0x4)}
            smax = float(N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM))

            def poll():
                while not self.stop_flag.is_set():
                    try:
                        sm = float(N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM))
                        r = int(N.nvmlDeviceGetCurrentClocksThrottleReasons(h))
                        self.samples.append((sm, smax, {n for n, b in bits.items() if r & b}))
                    except Exception:
                        pass
                    time.sleep(self.period)

            self.source = "nvml"
            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            return
        except Exception:
            pass
        try:
            ident = uuid or str(self.index)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={ident}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi"
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            f = [x.strip() for x in line.strip().split(",")]
            if len(f) < 9:
                continue
            try:
                self.samples.append((float(f[1]), float(f[2]),
                                     {n for n, v in zip(self.NAMES, f[5:9]) if v.lower() == "active"}))
            except ValueError:
                continue

    def stop(self) -> dict:
        self.stop_flag.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"], "samples": 0}
        sm = [x[0] for x in self.samples]
        reasons = set().union(*[x[2] for x in self.samples])
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(x[1] for x in self.samples),
                "sm_mhz_min": min(sm), "reasons": sorted(reasons), "samples": len(sm), "source": self.source}


# ---------------------------------------------------------------- CPU oracle sample

def cpu_sample_step(shape, seed, N, n_prompt, B_layer, B_window, lm_rows=32, vocab_frac=4, target_s=8.0):
    """Times the fp64 oracle on a bounded sample of one DCU step + commit and
    extrapolates to a whole step: one layer's selection + recompute of
    |W| + B_layer rows (x n_layers), and the LM head + softmax-max of `lm_rows`
    masked rows over vocab / vocab_frac entries (scaled to all masked rows and
    the full vocabulary), plus the commit over all masked positions."""
    import numpy as np
    from threadpoolctl import threadpool_info

    import oracle as O
    from dynamic_layer_wise_b200 import inputs as I

    cfg = O.Config(n_layers=shape.n_layers, d_model=shape.d_model, n_heads=shape.n_heads,
                   n_kv_heads=shape.n_kv_heads, head_dim=shape.head_dim, d_ffn=shape.d_ffn, vocab=shape.vocab,
                   dtype=shape.dtype)
    D, Hkv, hd = shape.d_model, shape.n_kv_heads, shape.head_dim
    ones = np.ones(D)
    lw = {"attn_norm": ones, "ffn_norm": ones}
    for n in I.LAYER_TENSORS:
        lw[n] = I.as_f64(I.weight_values(shape, seed, n, 0), shape.dtype)
    H = I.as_f64(I.normal_values(seed, 9001, 0, N * D, 0.5, shape.dtype), shape.dtype).reshape(N, D)
    K = I.as_f64(I.normal_values(seed, 9002, 0, Hkv * N * hd, 1.0, shape.dtype), shape.dtype).reshape(Hkv, N, hd)
    V = I.as_f64(I.normal_values(seed, 9003, 0, Hkv * N * hd, 0.05, shape.dtype), shape.dtype).reshape(Hkv, N, hd)
    d = np.zeros(N, np.float32)
    hot = I.uniform_ints(seed, 9004, 0, 3 * B_layer, N)
    d[hot] = np.abs(I.normal_values(seed, 9005, 0, len(hot), 0.1, "f32")) + 1e-6
    keys = [n_prompt]
    nv = shape.vocab // vocab_frac
    lm = I.as_f64(I.weight_values(shape, seed, "lm_head", rows=np.arange(nv)), shape.dtype)
    n_masked = N - n_prompt
    c_all = np.abs(I.normal_values(seed, 9006, 0, N, 0.001, "f32")) + 1e-5
    masked = np.zeros(N, bool)
    masked[n_prompt:] = True
    t_start = time.perf_counter()
    reps, t_layer = 0, 0.0
    while reps < 32 and (reps == 0 or t_layer < target_s):
        t0 = time.perf_counter()
        U = O.select_rows(d, keys, B_window, B_layer, 0)
        O.layer_rows(lw, cfg, H[U], U, K.copy(), V.copy())
        t_layer += time.perf_counter() - t0
        reps += 1
    t1 = time.perf_counter()
    O.confidence(H[:lm_rows], ones, lm, cfg.rms_eps)
    t2 = time.perf_counter()
    O.commit(c_all, np.zeros(N, np.int64), masked, np.zeros(N, np.int64), O.RULE_FRECHET, 0.1)
    t3 = time.perf_counter()
    step_s = shape.n_layers * (t_layer / reps) + (t2 - t1) * vocab_frac * (n_masked / lm_rows) + (t3 - t2)
    threads = max([x.get("num_threads", 1) for x in threadpool_info()] or [1])
    sample = (f"layer 0 of {shape.n_layers} ({len(U)} recomputed rows, N={N}) timed {reps}x, scaled x{shape.n_layers}; "
              f"LM head + softmax-max of {lm_rows} of {n_masked} masked rows over {nv} of {shape.vocab} vocab "
              f"entries (scaled), commit over {n_masked}; measured {t3 - t_start:.2f} s")
    return step_s, t3 - t_start, threads, sample


# ---------------------------------------------------------------- roofline bookkeeping

def gemm_algorithmic_bytes(shape, rows_per_layer):
    """Weights + bf16 activation in/out bytes of the recompute GEMMs of one step."""
    D, F, H, Hkv, hd = shape.d_model, shape.d_ffn, shape.n_heads, shape.n_kv_heads, shape.head_dim
    es = 2 if shape.dtype == "bf16" else 4
    gemms = [((H + 2 * Hkv) * hd, D), (D, H * hd), (2 * F, D), (D, F)]  # (n_out, K)
    total = 0.0
    for M in rows_per_layer:
        for n_out, K in gemms:
            total += es * (n_out * K + M * K + M * n_out)
    return total, 4 * len(rows_per_layer)


def step_algorithmic_bytes(shape, rows_per_layer, N, batch, n_masked):
    """Roofline bytes of one step: all layer weights once, the LM head once,
    the K/V stream over all N, and the recomputed rows' activations."""
    es = 2 if shape.dtype == "bf16" else 4
    w_layer = sum(o * i for o, i in shape.weight_shapes().values()) * es
    kv = 2 * batch * shape.n_kv_heads * N * shape.head_dim * es
    act = sum(M * shape.d_model * es * 2 for M in rows_per_layer)
    return shape.n_layers * (w_layer + kv) + shape.vocab * shape.d_model * es + act + n_masked * shape.d_model * es


GEMM_SOURCES = ("k_gemm_tc.cu", "tc_ptx.cuh", "gemm_tc.h")


def kernel_source_sha(files) -> str:
    """Hash of the sources a kernel is built from (to tell whether a stored
    ncu figure still describes the current kernel)."""
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "dynamic_layer_wise_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_for(key: str, files, algorithmic_bytes_per_launch: float):
    """DRAM bytes per launch from the committed ncu summary (profiles/traffic.json),
    scaled from the captured launch to the average launch by algorithmic bytes,
    if the capture was taken on the current source of the kernel; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as fh:
        t = json.load(fh)
    e = t.get(key)
    if not e or e.get("source_sha") != kernel_source_sha(files):
        return None
    return e["dram_bytes"] / e["algorithmic_bytes"] * algorithmic_bytes_per_launch


# ---------------------------------------------------------------- profiling cases

def profile_case_gemm(shape, reps):
    """The QKV recompute GEMM alone (M = 65 selected rows, K = d_model,
    N = (H + 2 H_kv) hd): for ncu captures of the tcgen05 kernel."""
    import torch
    from dynamic_layer_wise_b200 import dcu
    from dynamic_layer_wise_b200 import inputs as I
    n_out = (shape.n_heads + 2 * shape.n_kv_heads) * shape.head_dim
    W = I.device_normal_(torch.empty((n_out, shape.d_model), dtype=torch.bfloat16, device="cuda"), 0, 1, 0.02)
    X = I.device_normal_(torch.empty((65, shape.d_model), dtype=torch.bfloat16, device="cuda"), 0, 2, 1.0)
    for _ in range(max(1, reps)):
        dcu.dcu_linear(X, W)
    torch.cuda.synchronize()
    print(json.dumps({"case": "gemm", "M": 65, "K": shape.d_model, "N": n_out, "reps": reps}))
    return 0


# ---------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="dcu", choices=["dcu", "reference"])
    ap.add_argument("--workload", default="llada8b", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graphs", action="store_true", help="launch every kernel directly (no CUDA graphs)")
    ap.add_argument("--fused", type=int, default=None,
                    help="DCU_OPT_FUSED_EPILOGUE (1: epilogues inside the layer GEMMs); default: the library's")
    ap.add_argument("--l2-prefetch", type=int, default=None,
                    help="DCU_OPT_L2_PREFETCH (next-GEMM weight units per CTA into L2); default: the library's")
    ap.add_argument("--gemm-smem-kb", type=int, default=None,
                    help="DCU_OPT_GEMM_SMEM_KB (layer GEMM shared memory per CTA); default: the library's")
    ap.add_argument("--gemm-pass-sweep", type=int, choices=[0, 1], default=None,
                    help="DCU_OPT_GEMM_PASS_SWEEP (token passes sharing each weight tile); default: the library's")
    ap.add_argument("--attention", choices=["tcgen05", "mma_sync"], default=None,
                    help="attention implementation (DCU_OPT_ATTENTION; default: the library's)")
    ap.add_argument("--layers", type=int, default=0,
                    help="profiling only: override the number of layers (the JSON line is then not a bench value)")
    ap.add_argument("--case", default="", choices=["", "gemm"],
                    help="profiling only: run one kernel on a small case instead of the step (gemm: QKV shape, "
                         "M = 65 rows, 100 MB of weights)")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    wl = WORKLOADS[args.workload]

    from dynamic_layer_wise_b200 import inputs as I
    shape = getattr(I, wl["shape"])
    if args.layers:
        import dataclasses
        shape = dataclasses.replace(shape, n_layers=args.layers)
    if args.case == "gemm":
        return profile_case_gemm(shape, args.steps)
    N = wl["n_prompt"] + wl["n_gen"]
    B = wl["batch"]
    config = {"workload": wl["desc"], "batch": B, "seq_len": N, "B_layer": wl["B_layer"], "B_window": wl["B_window"],
              "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
              "l2": "inputs larger than L2: every step streams all layer weights (~15 GB) and the LM head"}

    if args.impl == "reference":
        if rank != 0:
            return 0
        times = []
        info = None
        for i in range(args.warmup + args.steps):
            step_s, measured, threads, sample = cpu_sample_step(shape, 0, N, wl["n_prompt"], wl["B_layer"],
                                                                wl["B_window"])
            if i >= args.warmup:
                times.append(step_s)
            info = (threads, sample)
        ms = 1000.0 * statistics.mean(times)
        v = 1000.0 / ms
        print(json.dumps({"impl": "reference", "metric": METRIC, "value": v, "unit": "steps/s", "n_gpus": args.gpus,
                          "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                          "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                          "config": config,
                          "cpu_baseline": {"value": v, "unit": "steps/s", "cores": info[0], "kind": "oracle",
                                           "sample": info[1]},
                          "e2e": {"value": v, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))
        return 0

    import torch
    import torch.distributed as dist
    from dynamic_layer_wise_b200 import dcu

    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=600))

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x: float) -> float:
        return reduce_over_ranks(x, world, "max", "cuda")

    def sum_over_ranks(x: float) -> float:
        return reduce_over_ranks(x, world, "sum", "cuda")

    stream = torch.cuda.current_stream()
    W = I.device_weights(shape, 0)
    ctx = dcu.dcu_create(W, I.cfg_dict(shape, B, N))
    dcu.dcu_set_graphs(ctx, not args.no_graphs)
    if args.fused is not None:
        dcu.dcu_set_option(ctx, dcu.DCU_OPT_FUSED_EPILOGUE, args.fused)
    if args.l2_prefetch is not None:
        dcu.dcu_set_option(ctx, dcu.DCU_OPT_L2_PREFETCH, args.l2_prefetch)
    if args.gemm_smem_kb is not None:
        dcu.dcu_set_option(ctx, dcu.DCU_OPT_GEMM_SMEM_KB, args.gemm_smem_kb)
        config["gemm_smem_kb"] = args.gemm_smem_kb
    if args.gemm_pass_sweep is not None:
        dcu.dcu_set_option(ctx, dcu.DCU_OPT_GEMM_PASS_SWEEP, args.gemm_pass_sweep)
        config["gemm_pass_sweep"] = args.gemm_pass_sweep
    if args.attention is not None:
        dcu.dcu_set_option(ctx, dcu.DCU_OPT_ATTENTION,
                           dcu.DCU_ATTN_TCGEN05 if args.attention == "tcgen05" else dcu.DCU_ATTN_MMA_SYNC)
        config["attention"] = args.attention
    seq_seed = replica_seed(rank)                         # each replica decodes its own sequences
    ids_h = torch.stack([torch.tensor(I.sequence_ids(seq_seed, b, wl["n_prompt"], wl["n_gen"], shape.vocab),
                                      dtype=torch.int32) for b in range(B)])
    ids = ids_h.cuda()
    masked = (ids == shape.mask_id).to(torch.uint8)
    pos = torch.zeros((B, N), dtype=torch.int32, device="cuda")
    cnt = torch.zeros(B, dtype=torch.int32, device="cuda")

    def new_generation():
        """Every timed pass starts from the same state: the prompt and an all-masked
        generated tail, the dense forward, the first commit (none of it timed), so
        the passes decode the same steps of a generation (the LM head of the commit
        covers the still-masked rows, which shrink as the generation proceeds)."""
        ids.copy_(ids_h)
        masked.copy_((ids == shape.mask_id).to(torch.uint8))
        pos.zero_()
        cnt.zero_()
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        dcu.dcu_full_forward(ctx, ids)
        g1.record(stream)
        torch.cuda.synchronize()
        dcu.commit_select(ctx, wl["rule"], wl["param"], masked, ids, pos, cnt)
        return g0.elapsed_time(g1)

    def step():
        dcu.dcu_step(ctx, ids, pos, cnt, wl["B_layer"], wl["B_window"])
        dcu.commit_select(ctx, wl["rule"], wl["param"], masked, ids, pos, cnt)

    full_ms = new_generation()

    # (1) the headline: K steps with nothing but the step's own kernels in the
    # graph (event-record nodes would split it and cut the programmatic edges
    # between consecutive kernels)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if dcu.dcu_status(ctx) != 0:
        raise RuntimeError("device status word set during warm-up")
    masked_before = int(masked.sum().item())
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    launches0 = dcu.dcu_launch_count(ctx)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks.start()                                        # samples span the timed region only
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier()
    ms_total = t0.elapsed_time(t1)
    launches = dcu.dcu_launch_count(ctx) - launches0
    masked_after = int(masked.sum().item())
    committed = masked_before - masked_after
    config["masked_rows_first_last_step"] = [masked_before, masked_after]
    ms_step = max_over_ranks(ms_total / args.steps)
    steps_all = args.steps * world
    value = aggregate_rate(args.steps, world, ms_step, args.steps)
    tokens_per_s = sum_over_ranks(committed) / (ms_step * args.steps / 1000.0)

    # (2) per kernel class: a second timed pass of K steps whose graphs carry an
    # event pair around every launch (captured during its own warm-up)
    per_step_launches_guess = 2 + shape.n_layers * 12 + 6
    # event slots for launches outside graphs (with graphs on, the captured
    # graphs carry their own event nodes)
    slots = (args.steps + args.warmup) if args.no_graphs else 2
    dcu.dcu_profile_enable(ctx, slots * per_step_launches_guess)
    new_generation()
    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize()
    for k in range(dcu.DCU_K_COUNT):
        dcu.dcu_profile_read(ctx, k, reset=True)
    barrier()
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    for _ in range(args.steps):
        step()
    p1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_prof_total = p0.elapsed_time(p1)
    per_kernel = {}
    for k in range(dcu.DCU_K_COUNT):
        ms_k, n_k = dcu.dcu_profile_read(ctx, k)
        per_kernel[dcu.dcu_kernel_class_name(k)] = {"ms_per_step": ms_k / args.steps,
                                                    "launches_per_step": n_k / args.steps,
                                                    "share": ms_k / ms_prof_total if ms_prof_total > 0 else None}
    dcu.dcu_profile_enable(ctx, 0)
    rows = [int(dcu.dcu_get_tensor(ctx, dcu.DCU_T_SEL_COUNT, l).sum().item()) for l in range(shape.n_layers)]
    gemm_bytes, gemm_launches = gemm_algorithmic_bytes(shape, rows)
    gemm_ms_step = per_kernel["gemm"]["ms_per_step"]
    hbm, tflops, peak_src = measured_peaks()
    achieved = gemm_bytes / (gemm_ms_step / 1000.0) / 1e9 if gemm_ms_step > 0 else None
    step_bytes = step_algorithmic_bytes(shape, rows, N, B, int(masked.sum().item()) + 1)
    roofline = {"bound": "hbm", "kernel": "gemm (recompute projections + FFN)", "achieved": achieved,
                "peak": hbm, "unit": "GB/s", "frac": (achieved / hbm) if achieved else None,
                "traffic": traffic_for("k_gemm_tc", GEMM_SOURCES, gemm_bytes / gemm_launches),
                "peak_source": peak_src,
                "algorithmic_bytes_per_launch": gemm_bytes / gemm_launches,
                "step_bytes": step_bytes, "step_roofline_ms": step_bytes / (hbm * 1e9) * 1e3,
                "step_frac_of_measured": (step_bytes / (hbm * 1e9) * 1e3) / ms_step,
                "step_frac_of_8TBps": (step_bytes / 8e12 * 1e3) / ms_step}

    e2e = None
    if not args.no_e2e:
        # through the C ABI with host buffers: ids/keys in from pinned memory, result out, every step
        new_generation()
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        h_ids = ids.cpu().pin_memory()
        h_pos = pos.cpu().pin_memory()
        h_cnt = cnt.cpu().pin_memory()
        h_out = torch.empty((B, N), dtype=torch.int32).pin_memory()
        h_oc = torch.empty(B, dtype=torch.int32).pin_memory()
        barrier()
        torch.cuda.synchronize()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(args.steps):
            ids.copy_(h_ids, non_blocking=True)
            pos.copy_(h_pos, non_blocking=True)
            cnt.copy_(h_cnt, non_blocking=True)
            step()
            h_out.copy_(pos, non_blocking=True)
            h_oc.copy_(cnt, non_blocking=True)
            h_ids.copy_(ids, non_blocking=True)
            stream.synchronize()
            h_pos.copy_(h_out)
            h_cnt.copy_(h_oc)
        a1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks(a0.elapsed_time(a1) / args.steps)
        e2e = {"value": steps_all / (e2e_ms * args.steps / 1000.0), "unit": "steps/s",
               "h2d_bytes_per_step": 4 * (2 * B * N + B), "d2h_bytes_per_step": 4 * (2 * B * N + B),
               "ms_per_step": e2e_ms}

    cpu_base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        step_s, measured, threads, sample = cpu_sample_step(shape, 0, N, wl["n_prompt"], wl["B_layer"],
                                                            wl["B_window"])
        cpu_base = {"value": 1.0 / step_s, "unit": "steps/s", "cores": threads, "kind": "oracle", "sample": sample}

    if rank == 0:
        out = {"metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world, "steps": args.steps,
               "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
               "vs_baseline": None, "dtype": "bf16" if shape.dtype == "bf16" else "f32", "data": "synthetic",
               "config": config, "gen_tokens_per_s": tokens_per_s, "full_forward_ms": full_ms,
               "per_kernel": per_kernel, "profiled_ms_per_step": ms_prof_total / args.steps, "rows_per_layer_last_step": rows, "roofline": roofline,
               "cpu_baseline": cpu_base, "e2e": e2e, "clocks": clk, "gpu_launches": launches,
               "graphs": not args.no_graphs}
        if args.layers:
            out["profiling_only"] = f"n_layers overridden to {args.layers}: not a bench value"
        print(json.dumps(out))
    ctx.close()
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
