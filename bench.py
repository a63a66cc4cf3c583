#!/usr/bin/env python
"""Throughput of the smoothed-INT8-QK / FP8-PV attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload llm_prefill]
    python bench.py --impl reference ...        # the fp64 CPU oracle on the host cores

One step = one pass of the whole hot path over one batch of synthetic input
already resident in HBM, through the public C-ABI call sage_attn_fwd: the
smoothing/quantization pre-pass of Q, K and V, the dS product, and the fused
attention kernel.  A second timed loop runs the attention kernel alone
(sage_attn_fwd_prequant on the same workspace) for its roofline figure.  With
--fuse-q the step is sage_attn_fwd_qfused_gqa instead (K / V pre-pass, then the
attention kernel that quantizes its own Q tiles and forms dS itself), and the second
loop times that kernel (the same entry without v).  Metric: attention TOPS
= 4 B H N_q N_kv d / t (halved when causal), summed over all ranks.  With N > 1 the
ranks compute disjoint slices of one seeded global problem, split by heads (each head's
K mean, delta_V, dS and O depend on that head alone, so no data-path collective is
needed): by default the global problem holds N batch blocks of the workload and rank r
computes block r (weak scaling); --scaling strong splits the workload's own heads into
N contiguous ranges.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention TOPS (4*B*H*Nq*Nkv*d/t, causal /2) and % of B200 dense INT8/FP8 peak"
UNIT = "TOPS"
SPEC_INT8_TOPS = 4500.0          # B200 dense INT8 / FP8 datasheet figure
FALLBACK_BF16_TFLOPS = 1590.0    # pool measurement used when MEASURED_PEAKS.json is absent
# library kernels per step of sage_attn_fwd: kv_stats, kv_finalize, quant_q, quant_k,
# quant_v, ds_gemm, attn_fwd_kernel; with --fuse-q: kv_stats, kv_finalize, quant_k,
# quant_v, attn_fwd_kernel
LAUNCHES_PER_STEP = 7
LAUNCHES_PER_STEP_FUSE_Q = 5
KERNEL_SOURCES = ["quantized_attention_fine_b200/csrc/attn_fwd.cu", "quantized_attention_fine_b200/csrc/attn_mma.cuh",
                  "quantized_attention_fine_b200/csrc/sage_device.cuh"]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llm_prefill")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="oracle time budget of the CPU baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--pv", default="fp8", choices=["fp8", "fp16"],
                    help="PV precision: fp8 (the method's default) or fp16 (the qk_int8_pv_fp16 mode)")
    ap.add_argument("--fuse-q", action="store_true",
                    help="quantize Q inside the attention kernel (sage_attn_fwd_qfused_gqa) instead of the pre-pass")
    ap.add_argument("--qk", default="int8", choices=["int8", "fp4"],
                    help="Q / K precision: int8 (grouped INT8, the default) or fp4 (the 4-bit mode: block-scaled "
                         "E2M1 on tcgen05.mma kind::mxf4nvf4; d = 64 workloads)")
    ap.add_argument("--graph", action="store_true",
                    help="time the step as a replay of a CUDA graph that captured one sage_attn_fwd call")
    ap.add_argument("--scaling", default="weak", choices=["weak", "strong"],
                    help="N > 1: weak = N batch blocks of the workload, one per rank; strong = the workload's "
                         "heads split across the ranks")
    ap.add_argument("--no-probe", action="store_true", help="skip the tcgen05.mma rate probe (second denominator)")
    ap.add_argument("--lib-peaks", action="store_true",
                    help="diagnostic: library INT8 / FP8 / BF16 GEMM rates (torch._int_mm, torch._scaled_mm, "
                         "torch.matmul; 8192^3, best of 10 and a sustained loop)")
    ap.add_argument("--mma-rates", action="store_true",
                    help="print the tensor-core rate of each tcgen05.mma form (diagnostic) and exit")
    args = ap.parse_args()
    if args.fuse_q and args.qk == "fp4":
        ap.error("--fuse-q: the 4-bit mode quantizes Q in the pre-pass (no in-kernel form)")
    return args


def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("LOCAL_RANK", "0"))


# ---------------------------------------------------------------------------
# Multi-rank host logic: every rank computes a disjoint slice of one seeded global
# problem, split by heads; no data-path collective.  Tested with gloo ranks on the CPU.
#
# The unit of work is one key/value head group: key/value head (b, h_kv) with its
# H / H_kv query heads (one head under multi-head attention).  Units are independent:
# a head's K mean, delta_V, Q blocks, dS and O use no other head.
#   weak   the global problem is `world` batch blocks of the workload (B_g = world * B);
#          block r is drawn from seed + 7919 r, and rank r computes block r.
#   strong the global problem is the workload; its B * H_kv units are split into
#          `world` contiguous ranges (world must divide B * H_kv).
# ---------------------------------------------------------------------------
def rank_workload(w, rank: int):
    """Batch block `rank` of the weak-scaling global problem: the workload drawn from
    the block's own seed (block 0 is the workload itself)."""
    from quantized_attention_fine_b200 import workloads as wl
    return wl.Workload(w.name, w.B, w.H, w.N_q, w.N_kv, w.d, w.causal, w.dtype, w.seed + 7919 * rank, w.recipe,
                       H_kv=w.H_kv)


def unit_range(n_units: int, world: int, rank: int):
    """Contiguous share [u0, u1) of n_units units for rank of world (world divides n_units)."""
    if world < 1 or n_units % world:
        raise ValueError("%d ranks cannot split %d key/value head groups evenly" % (world, n_units))
    per = n_units // world
    return rank * per, (rank + 1) * per


def global_inputs(w, world: int, scaling: str):
    """The seeded global problem (q, k, v) of a world-rank run, as one [B_g, H, N, d] batch."""
    from quantized_attention_fine_b200 import workloads as wl
    import torch
    if scaling == "strong":
        return wl.generate(w)
    blocks = [wl.generate(rank_workload(w, r)) for r in range(world)]
    return tuple(torch.cat([b[i] for b in blocks], dim=0) for i in range(3))


def rank_inputs(w, world: int, rank: int, scaling: str):
    """(sub-workload, q, k, v) of rank: its slice of the global problem, drawn without
    drawing the rest under weak scaling.  Under strong scaling the slice is units
    [u0, u1) of the workload, returned as one batch of (u1 - u0) * group query heads
    over (u1 - u0) key/value heads (HND tensors, contiguous)."""
    from quantized_attention_fine_b200 import workloads as wl
    if scaling == "weak":
        wr = rank_workload(w, rank)
        return (wr,) + tuple(wl.generate(wr))
    q, k, v = wl.generate(w)
    group = w.H // w.Hk
    u0, u1 = unit_range(w.B * w.Hk, world, rank)
    qs = q.reshape(w.B * w.Hk, group, w.N_q, w.d)[u0:u1].reshape(1, (u1 - u0) * group, w.N_q, w.d).contiguous()
    ks = k.reshape(w.B * w.Hk, w.N_kv, w.d)[u0:u1].unsqueeze(0).contiguous()
    vs = v.reshape(w.B * w.Hk, w.N_kv, w.d)[u0:u1].unsqueeze(0).contiguous()
    sub = wl.Workload(w.name, 1, (u1 - u0) * group, w.N_q, w.N_kv, w.d, w.causal, w.dtype, w.seed, w.recipe,
                      H_kv=(u1 - u0) if group > 1 else 0)
    return sub, qs, ks, vs


def parallelism_label(w, world: int, scaling: str) -> str:
    if world == 1:
        return "one GPU: the whole workload (%d heads)" % (w.B * w.H)
    if scaling == "weak":
        return ("heads split, weak: global problem of %d batch blocks (%d heads); rank r computes block r "
                "(%d heads); no data-path collective" % (world, world * w.B * w.H, w.B * w.H))
    return ("heads split, strong: the workload's %d heads in %d contiguous ranges of %d; no data-path collective"
            % (w.B * w.H, world, w.B * w.H // world))


def max_over_ranks(values, device="cpu"):
    """Element-wise max of per-rank timings (ms) over the process group, if any."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x) for x in values], device=device, dtype=torch.float64)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def whole_job_tops(world: int, ops_per_rank_step: float, ms_per_step: float) -> float:
    """Aggregate throughput: the units every rank processed over the slowest rank's time."""
    return world * ops_per_rank_step / (ms_per_step * 1e-3) / 1e12


# ---------------------------------------------------------------------------
# CPU oracle sample (baseline arm and cpu_baseline key)
# ---------------------------------------------------------------------------
_HEAD_CACHE = {}


def oracle_sample(w, seconds: float, quant=(1, 1, 1)):
    """Time the fp64 oracle on a bounded sample of workload w: head (0, 0) of the seeded
    inputs, its pre-pass, then Q blocks in a seeded order until `seconds` have passed.
    quant: the oracle's (QK, P, V) mode of the run.  Returns (ops_done, time_s,
    description, threads)."""
    import numpy as np
    import oracle
    from quantized_attention_fine_b200 import workloads as wl
    if w.name not in _HEAD_CACHE:  # the seeded inputs are drawn once per process
        q, k, v = wl.generate(w)
        _HEAD_CACHE[w.name] = tuple(x[0, 0].double().numpy() for x in (q, k, v))
        del q, k, v
    qh, kh, vh = _HEAD_CACHE[w.name]
    t0 = time.perf_counter()
    pre = oracle.prepass_head(qh, kh, vh, quant=quant)
    t_pre = time.perf_counter() - t0
    tq = -(-w.N_q // 128)
    order = np.random.default_rng(w.seed).permutation(tq)
    off = w.N_kv - w.N_q
    ops, t_blocks, done = 0.0, 0.0, []
    for t in order:
        t1 = time.perf_counter()
        oracle.attn_head(pre, causal=w.causal, qblocks=[int(t)])
        t_blocks += time.perf_counter() - t1
        rows = np.arange(t * 128, min(t * 128 + 128, w.N_q))
        keys = np.clip(rows + off + 1, 0, w.N_kv) if w.causal else np.full(rows.shape, w.N_kv)
        ops += 4.0 * w.d * float(keys.sum())
        done.append(int(t))
        if t_blocks + t_pre >= seconds:
            break
    t_total = t_blocks + t_pre * len(done) / tq   # the head's pre-pass, charged pro rata
    desc = ("head (b0,h0) of %s: its pre-pass (%.2fs, charged %d/%d) + %d of %d Q blocks (seeded order) over the "
            "full KV range" % (w.name, t_pre, len(done), tq, len(done), tq))
    return ops, t_total, desc, oracle.num_threads()


def reference_arm(args, w):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    per_step = max(2.0, min(args.cpu_seconds, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(w, per_step)
    ops, secs, desc = 0.0, 0.0, ""
    threads = 1
    for _ in range(args.steps):
        o, s, desc, threads = oracle_sample(w, per_step)
        ops += o
        secs += s
    value = ops / secs / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(w.describe(), parallelism="oracle on host cores, rank 0 only"),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc,
                             "host": host_cpu(), "pair_updates_per_s": ops / secs / (4.0 * w.d),
                             "extrapolated_step_s": w.ops() / (ops / secs)},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# Clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, enabled: bool = True):
        self.proc = None
        self.idx = device_index
        self.path = None
        if not enabled:
            return
        try:
            # the raw samples go to a temporary file (or to $SAGE_BENCH_LOG_DIR, kept)
            log_dir = os.environ.get("SAGE_BENCH_LOG_DIR")
            if log_dir:
                os.makedirs(log_dir, exist_ok=True)
                self.path, self.keep = os.path.join(log_dir, "clocks_rank%d.csv" % device_index), True
            else:
                fd, self.path = tempfile.mkstemp(prefix="sage_clocks_rank%d_" % device_index, suffix=".csv")
                os.close(fd)
                self.keep = False
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(device_index), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.fh,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in open(self.path):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not self.keep:
            os.remove(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    return FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def library_gemm_peaks(n: int = 8192, sustained_s: float = 4.0) -> dict:
    """Dense GEMM rates of the vendor library on this GPU (context for the roofline's
    denominator): INT8 (torch._int_mm, int32 out), FP8 E4M3 (torch._scaled_mm, bf16 out)
    and BF16 (torch.matmul), n^3 each; the best of 10 single launches and the mean over a
    loop of about sustained_s seconds, with the SM clock sampled during the loops."""
    import torch
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(1)
    a8 = torch.randint(-127, 128, (n, n), generator=g, device=dev, dtype=torch.int8)
    b8 = torch.randint(-127, 128, (n, n), generator=g, device=dev, dtype=torch.int8)
    af = torch.randn(n, n, generator=g, device=dev).to(torch.float8_e4m3fn)
    bf = torch.randn(n, n, generator=g, device=dev).to(torch.float8_e4m3fn).t()   # column-major operand
    one = torch.ones((), device=dev)
    ab = torch.randn(n, n, generator=g, device=dev, dtype=torch.bfloat16)
    bb = torch.randn(n, n, generator=g, device=dev, dtype=torch.bfloat16)
    ops = {"int8": lambda: torch._int_mm(a8, b8),
           "fp8": lambda: torch._scaled_mm(af, bf, scale_a=one, scale_b=one, out_dtype=torch.bfloat16),
           "bf16": lambda: torch.matmul(ab, bb)}
    work = 2.0 * n ** 3
    clocks = ClockSampler(0, enabled=True)
    out = {}
    for name, fn in ops.items():
        for _ in range(3):
            fn()
        torch.cuda.synchronize(dev)
        best = float("inf")
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize(dev)
            best = min(best, e0.elapsed_time(e1) * 1e-3)
        reps = max(10, int(sustained_s / best))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize(dev)
        mean = e0.elapsed_time(e1) * 1e-3 / reps
        out[name] = {"burst": work / best / 1e12, "sustained": work / mean / 1e12}
    return {"lib_gemm_peaks": out, "unit": "TOPS (int8) / TFLOP/s", "shape": "%d^3" % n, "clocks": clocks.stop()}


def host_cpu() -> dict:
    """The host the CPU baseline ran on: its processor model and logical core count."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu": model, "nproc": os.cpu_count()}


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        h.update(open(os.path.join(ROOT, rel), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch of the attention kernel from the committed ncu summary, if it was
    taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "attn_fwd_traffic.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path))
    entry = d.get(workload)
    if not entry or entry.get("kernel_source_hash") != kernel_source_hash():
        return None
    return entry.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
def main():
    args = parse_args()
    from quantized_attention_fine_b200 import workloads as wl
    try:
        w = wl.by_name(args.workload)
    except KeyError as e:
        raise SystemExit("%s (choices: %s, or sweep_n<N>_d<64|128>_<causal|full>)" % (e, ", ".join(wl.WORKLOADS)))
    if args.impl == "reference":
        return reference_arm(args, w)
    if args.lib_peaks:
        print(json.dumps(library_gemm_peaks()), flush=True)
        return 0
    if args.mma_rates:
        import quantized_attention_fine_b200 as sage
        rates = {k: sage.debug_mma_rate(k) for k in sage.MMA_KINDS}
        print(json.dumps({"mma_rates": rates, "unit": "TFLOP/s (TOPS for s8_s32)", "shape": "M128 N256, one CTA per SM"}),
              flush=True)
        return 0

    import torch
    import torch.distributed as dist
    import quantized_attention_fine_b200 as sage
    from datetime import timedelta

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    sage.load_library()

    # this rank's slice of the seeded global problem
    wr, q_cpu, k_cpu, v_cpu = rank_inputs(w, world, rank, args.scaling)
    q, k, v = q_cpu.to(dev), k_cpu.to(dev), v_cpu.to(dev)
    B, H, nq, nk, d = wr.B, wr.H, wr.N_q, wr.N_kv, wr.d
    pv16 = args.pv == "fp16"
    fp4 = args.qk == "fp4"
    gran = "fp4" if fp4 else "per_threadgroup"
    ws = sage.make_workspace(B, H, nq, nk, d, device=dev, H_kv=wr.Hk, pv_fp16=pv16, qk_fp4=fp4)
    out = torch.empty_like(q)
    mode = sage.QuantMode.make(gran, pv=args.pv)
    stream = torch.cuda.current_stream(dev)

    fuse_q = bool(args.fuse_q)

    def step_eager():
        sage.attn_fwd(q, k, v, causal=w.causal, out=out, workspace=ws, pv=args.pv, granularity=gran, fuse_q=fuse_q)

    step = step_eager
    graph = None
    if args.graph:  # one captured call, replayed each step (no host launch cost)
        step_eager()
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step_eager()
        step = graph.replay

    def attn_only():   # the attention kernel of the step, on the workspace the step filled
        if fuse_q:
            sage.attn_fwd_qfused(q, k, ws, causal=w.causal, mode=mode, out=out)
        else:
            sage.attn_fwd_prequant(ws, dtype=q.dtype, causal=w.causal, mode=mode, out=out)

    def prepass_only():   # the step's pre-pass launches alone (the Q-fused form has no separate entry)
        sage.quant_qk(q, k, mode=mode, workspace=ws)
        sage.quant_v(v, n_q=nq, H=H, mode=mode, workspace=ws)

    for _ in range(args.warmup):
        step()
        attn_only()
        if not fuse_q:
            prepass_only()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    clocks = ClockSampler(local, enabled=not args.no_clocks)
    if clocks.proc is not None:
        time.sleep(0.3)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step()
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    # the attention kernel alone, each launch bracketed by events on its stream
    for i in range(args.steps):
        ev[i][0].record(stream)
        attn_only()
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    # the pre-pass alone, the same way (it refills the workspace with the same codes)
    evp = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    if not fuse_q:
        for i in range(args.steps):
            evp[i][0].record(stream)
            prepass_only()
            evp[i][1].record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clk = clocks.stop()

    total_ms = t_start.elapsed_time(t_end)
    attn_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(args.steps)]
    pre_ms = [evp[i][0].elapsed_time(evp[i][1]) for i in range(args.steps)] if not fuse_q else [0.0]
    total_ms, attn_avg_ms, attn_med_ms, pre_meas_ms = max_over_ranks(
        [total_ms, statistics.mean(attn_ms), statistics.median(attn_ms), statistics.mean(pre_ms)], device=dev)
    ms_per_step = total_ms / args.steps
    # with Q quantized in the attention kernel there is no pre-pass call of its own to time
    pre_avg_ms = (ms_per_step - attn_avg_ms) if fuse_q else pre_meas_ms
    ops_step = wr.ops()     # this rank's slice; every rank's slice has the same size
    value = whole_job_tops(world, ops_step, ms_per_step)
    attn_tops = ops_step / (attn_avg_ms * 1e-3) / 1e12

    # end to end through the public call with host buffers: H2D of Q, K, V from pinned memory,
    # sage_attn_fwd, D2H of O, every step
    e2e = None
    if not args.no_e2e:
        # Every step copies its Q, K, V in from pinned host memory, runs sage_attn_fwd and
        # copies O back.  Steps are pipelined over three streams, with two device buffer
        # sets: step i + 1's inputs travel while step i computes and step i - 1's output
        # travels back.  The timed region runs from the first input copy to the last
        # output copy.
        qh, kh, vh = q_cpu.pin_memory(), k_cpu.pin_memory(), v_cpu.pin_memory()
        oh = torch.empty_like(q_cpu).pin_memory()
        dbuf = [(torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(q)) for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def e2e_run(n_steps):
            ev_in = [torch.cuda.Event() for _ in range(n_steps)]
            ev_comp = [torch.cuda.Event() for _ in range(n_steps)]
            ev_out = [torch.cuda.Event() for _ in range(n_steps)]
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(s_in)
            for i in range(n_steps):
                qd, kd, vd, od = dbuf[i % 2]
                if i >= 2:
                    s_in.wait_event(ev_comp[i - 2])      # this buffer set's inputs are consumed
                with torch.cuda.stream(s_in):
                    qd.copy_(qh, non_blocking=True)
                    kd.copy_(kh, non_blocking=True)
                    vd.copy_(vh, non_blocking=True)
                ev_in[i].record(s_in)
                stream.wait_event(ev_in[i])
                if i >= 2:
                    stream.wait_event(ev_out[i - 2])     # and its output has been copied out
                sage.attn_fwd(qd, kd, vd, causal=w.causal, out=od, workspace=ws, stream=stream, pv=args.pv,
                              granularity=gran, fuse_q=fuse_q)
                ev_comp[i].record(stream)
                s_out.wait_event(ev_comp[i])
                with torch.cuda.stream(s_out):
                    oh.copy_(od, non_blocking=True)
                ev_out[i].record(s_out)
            t1.record(s_out)
            torch.cuda.synchronize(dev)
            return t0.elapsed_time(t1)

        e2e_run(2)
        if world > 1:
            dist.barrier()
        e_ms = max_over_ranks([e2e_run(args.e2e_steps) / args.e2e_steps], device=dev)[0]
        qbytes, kvbytes = q.numel() * q.element_size(), k.numel() * k.element_size()
        e2e = {"value": whole_job_tops(world, ops_step, e_ms), "unit": UNIT, "ms_per_step": e_ms,
               "h2d_bytes_per_step": qbytes + 2 * kvbytes, "d2h_bytes_per_step": qbytes,
               "call": "sage_attn_fwd with pinned-host Q/K/V copied in and O copied out each step; "
                       "copies and compute of neighbouring steps overlap on three streams"}

    code, site = sage.get_device_status(ws)
    if code != 0:
        raise SystemExit("device status %d at site %d" % (code, site))
    if graph is not None:
        del graph

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    bf16_burst, bf16_sust, peak_src = measured_peaks()
    peak = 2.0 * bf16_burst   # dense INT8 / FP8 = 2x dense BF16 (nominal 4.5 vs 2.25 PFLOP/s)
    peak_note = "%s bf16 burst %.1f x 2 (dense int8/fp8 = 2x bf16)" % (peak_src, bf16_burst)
    if fp4:   # QK^T at the FP4 rate (nominal 2x FP8), PV at the FP8 rate, equal work: the harmonic mean
        peak = 2.0 / (1.0 / (4.0 * bf16_burst) + 1.0 / (2.0 * bf16_burst))
        peak_note = ("%s bf16 burst %.1f: FP4 QK at 4x (nominal 2x FP8), FP8 PV at 2x, equal work: harmonic mean"
                     % (peak_src, bf16_burst))
    if pv16:  # half the work at the INT8 rate, half at the FP16 rate: the harmonic mean
        peak = 2.0 / (1.0 / (2.0 * bf16_burst) + 1.0 / bf16_burst)
        peak_note = ("%s bf16 burst %.1f: INT8 QK at 2x, FP16 PV at 1x, equal work: harmonic mean"
                     % (peak_src, bf16_burst))
    # the tensor cores' own rate on this GPU (tcgen05.mma probe, one CTA per SM), the
    # second denominator: QK^T at the S8 rate and PV at the E4M3 (or BF16) rate, equal
    # work, so their harmonic mean
    probe = None
    if not args.no_probe:
        # the 4-bit QK^T rate is taken as twice the probe's E4M3 rate (the nominal ratio)
        r_qk = 2.0 * sage.debug_mma_rate("e4m3_f32") if fp4 else sage.debug_mma_rate("s8_s32")
        r_pv = sage.debug_mma_rate("bf16_f32" if pv16 else "e4m3_f32")
        probe = 2.0 / (1.0 / r_qk + 1.0 / r_pv)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        ops_s, secs, desc, threads = oracle_sample(w, args.cpu_seconds,
                                                   quant=(2 if fp4 else 1, 2 if pv16 else 1, 2 if pv16 else 1))
        cpu = {"value": ops_s / secs / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc,
               "host": host_cpu(), "pair_updates_per_s": ops_s / secs / (4.0 * w.d),
               "extrapolated_step_s": ops_step / (ops_s / secs)}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": args.scaling if world > 1 else "weak",
        "vs_baseline": None, "dtype": ("e2m1" if fp4 else "int8") + ("+fp16" if pv16 else "+e4m3"),
        "data": "synthetic",
        "config": dict(w.describe(), parallelism=parallelism_label(w, world, args.scaling),
                       l2="inputs (%.0f MiB) larger than L2 (126 MB); no flush" % ((2 * q.numel() + 2 * k.numel()) * 2 / 2 ** 20),
                       granularity=("fp4 (E2M1, E4M3 scale per 16 channels, fp32 scale per 128-row tile)" if fp4
                                    else "per_threadgroup (g_q=32, g_k=16)"),
                       **({"pv": "fp16 (qk_int8_pv_fp16)"} if pv16 else {"pv": "fp8", "pr": 448, "vr": 448})),
        "attn_kernel_tops": attn_tops, "attn_kernel_ms": attn_avg_ms, "attn_kernel_ms_median": attn_med_ms,
        "prepass_ms": pre_avg_ms, "step_minus_attn_ms": ms_per_step - attn_avg_ms,
        "step_call": (("sage_attn_fwd_qfused_gqa (K / V pre-pass + attention with Q quantization and dS in the kernel)"
                       if fuse_q else "sage_attn_fwd (pre-pass + dS + attention)")
                      + (", replayed from a CUDA graph" if args.graph else "")
                      + ("; prepass_ms = ms_per_step - attn_kernel_ms" if fuse_q else
                         "; prepass_ms: sage_quant_qk_gqa + sage_quant_v_gqa timed alone with CUDA events (the "
                         "step's pre-pass kernels, with the K and the V statistics in two launches instead of one)")),
        "attn_frac_of_spec_4500": attn_tops / SPEC_INT8_TOPS,
        "roofline": {"bound": "tensor", "achieved": attn_tops, "peak": peak, "unit": "TFLOP/s",
                     "frac": attn_tops / peak, "traffic": None if (pv16 or fp4 or fuse_q) else recorded_traffic(w.name),
                     "frac_of_tcgen05_probe": (attn_tops / probe) if probe else None,
                     "tcgen05_probe_peak": probe,
                     "peak_source": peak_note,
                     "kernel": "attn_fwd_kernel<%d>%s" % (d, " (4-bit QK)" if fp4 else
                                                          (" (Q quantized in the kernel)" if fuse_q else ""))},
        "cpu_baseline": cpu, "e2e": e2e, "clocks": clk,
        "gpu_launches": args.steps * (LAUNCHES_PER_STEP_FUSE_Q if fuse_q else LAUNCHES_PER_STEP),
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
