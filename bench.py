"""Benchmark of the fused MoE layer forward on B200: MoE-layer tokens/s and TFLOP/s, with the
dominant kernel's fraction of the HBM (or tensor) roofline.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mine|reference]
                  [--workload flashmoe_prefill] [--no-cpu-baseline] [--e2e-steps M]

One step = one whole layer forward (router projection, gating, align, row gather, expert
GEMMs with the fused SwiGLU and router weighting, and the combine) over one batch of seeded synthetic input already resident
in HBM. The default workload is the FlashMoE-shaped prefill layer (T=4096, H=2048, D=2048,
E=64, top-2, capacity factor 1.0); its 1.6 GB of expert weights exceed the 126 MB L2, so no
L2 flush is needed between steps. With N > 1 (torchrun) every rank runs an independent
replica on its own GPU (no collective on the data path; weak scaling); rank 0 prints one
JSON line. `--impl reference` times the CPU oracle instead, on a bounded sample of the same
workload.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from mixture_experts_layer_block_b200 import configs, inputs as gen  # noqa: E402

METRIC = "MoE layer tokens/s and TFLOP/s on 1 B200; % of bf16/HBM roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one expert-GEMM launch, from
# the ncu captures summarised under profiles/, with the hash of the kernel sources it was taken
# on. A different hash (the kernel changed since) reports null.
KERNEL_SOURCES = ["mixture_experts_layer_block_b200/csrc/moe_gemm.cu",
                  "mixture_experts_layer_block_b200/csrc/common.cuh",
                  "mixture_experts_layer_block_b200/csrc/ptx.cuh",
                  "mixture_experts_layer_block_b200/csrc/launch.h"]
MEASURED_TRAFFIC = {
    "flashmoe_prefill": ("8e58c2e2d8dae369", 1.677245e9 + 0.061002e9, "one full-size launch"),
    "decode": ("8e58c2e2d8dae369", 0.337762e9 + 0.004001e9, "one full-size launch"),
    # full DSV3 holds 22.6 GB of weights, too large for a multi-pass capture: the T=512, E=32
    # case of the same layer (the same per-expert load, 1/8 of the experts and tokens) scaled
    # by the 8x more units of a full launch
    "dsv3": ("8e58c2e2d8dae369", 8 * (3.063093e9 + 0.115249e9), "T=512, E=32 capture x 8"),
}


def kernel_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(workload: str):
    rec = MEASURED_TRAFFIC.get(workload)
    if rec is None or rec[0] != kernel_source_hash():
        return None
    return rec[1]


def measured_traffic_note(workload: str):
    rec = MEASURED_TRAFFIC.get(workload)
    return rec[2] if rec is not None and rec[0] == kernel_source_hash() else None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------------------------------
# workload arithmetic (reporting only)
# ------------------------------------------------------------------------------------------

def algorithmic_bytes_gemm(w, hit_experts: int, mxfp8: bool = False) -> float:
    """Bytes the expert-GEMM kernel must move at least once: the weights of the experts that
    receive tokens, the shared expert's weights, x and out (fp32). Weights and x are bf16, or
    with MXFP8 experts one byte per element plus one scale byte per 32 elements."""
    e = (1.0 + 1.0 / 32.0) if mxfp8 else 2.0
    b = 3.0 * hit_experts * w.D * w.H * e
    b += 3.0 * w.D_shared * w.H * e
    b += w.T * w.H * e + w.T * w.H * 4
    return b


def sm_busy_fraction(records: np.ndarray, n_ctas: int) -> dict:
    """SM-busy fraction of one traced forward of the expert-GEMM kernel: per CTA the union of
    its tasks' [claim, done] intervals, summed, over n_ctas x (last done - first claim)."""
    if records.size == 0:
        return {"sm_busy": None}
    r = records[(records[:, 2] > 0) & (records[:, 3] >= records[:, 2])]
    t0, t1 = r[:, 2].min(), r[:, 3].max()
    busy = 0
    for cta in np.unique(r[:, 0]):
        iv = r[r[:, 0] == cta][:, 2:4]
        iv = iv[np.argsort(iv[:, 0])]
        cur_s, cur_e = iv[0]
        for s_, e_ in iv[1:]:
            if s_ > cur_e:
                busy += cur_e - cur_s
                cur_s, cur_e = s_, e_
            else:
                cur_e = max(cur_e, e_)
        busy += cur_e - cur_s
    return {"sm_busy": float(busy / (n_ctas * (t1 - t0))), "makespan_us": float((t1 - t0) / 1e3),
            "tasks": int(r.shape[0])}


def tile_flags(args) -> int:
    from mixture_experts_layer_block_b200 import native
    f = {"auto": 0, "pair": native.MOE_FLAG_PAIR_TILES, "single": native.MOE_FLAG_SINGLE_TILES}[
        getattr(args, "tiles", "auto")]
    if getattr(args, "sched", "dynamic") == "static":
        f |= native.MOE_FLAG_STATIC_QUOTA
    return f


def run_forward(layer, x, wts, out, wq=None):
    """One layer forward: bf16 experts, or MXFP8 experts when `wq` holds their quantisation."""
    if wq is None:
        layer.forward(x, wts, out)
    else:
        layer.forward_mxfp8(x, wts["W_router"], wts.get("bias"), wq, out)


def traced_forward(w, wts, x, out, extra_flags=0, wq=None):
    """One extra forward with per-task tracing (outside the timed region)."""
    from mixture_experts_layer_block_b200.native import MOE_FLAG_TRACE, MoELayer
    layer = MoELayer.for_workload(w, flags=MOE_FLAG_TRACE | extra_flags)
    for _ in range(2):
        run_forward(layer, x, wts, out, wq)
    torch.cuda.synchronize()
    rec = layer.trace(1 << 20)
    n_ctas = layer.query(1)
    layer.close()
    return sm_busy_fraction(rec, n_ctas)


def routing_stats(layer, w, dev):
    dbg = layer.debug_outputs(w.T, w.top_k, dev)
    torch.cuda.synchronize()
    S = w.T * w.top_k
    P = int(dbg["num_post_padded"].item())
    body = dbg["sorted_ids"][:P]
    kept_ids = dbg["topk_ids"].reshape(-1)[body[body < S].long()]
    counts = torch.bincount(kept_ids, minlength=w.E).cpu().numpy()
    return {"kept_slots": int(counts.sum()), "hit_experts": int((counts > 0).sum()),
            "max_over_mean_load": float(counts.max() / max(counts.mean(), 1e-9)),
            "empty_experts_frac": float((counts == 0).mean())}


# ------------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.15)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
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
        loaded = [s for s in sm if s > 0.5 * max(sm)]
        return {"sm_mhz": float(np.median(loaded)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------------------------
# CPU oracle timing (the reported baseline, and the reference arm)
# ------------------------------------------------------------------------------------------

def oracle_sample_time(w, wts_host, x_host, n_tokens, mxfp8=False):
    from oracle import oracle
    sub = w.replace(T=n_tokens)
    inp = dict(wts_host, x=x_host[:n_tokens])
    t0 = time.perf_counter()
    oracle.forward(inp, sub.top_k, sub.block_m, sub.capacity_factor, mxfp8=mxfp8)
    return time.perf_counter() - t0


def cpu_baseline(w, wts_dev, x_dev, budget_s=12.0, mxfp8=False):
    """Time the oracle, as it stands, on the first n tokens of the batch (a smaller batch of
    the same layer), n sized for about `budget_s` of CPU work."""
    from oracle import oracle
    wts_host = {k: (v.cpu() if v is not None else None) for k, v in wts_dev.items()}
    x_host = x_dev.cpu()
    n = min(w.T, 4 if mxfp8 else 16)
    dt = oracle_sample_time(w, wts_host, x_host, n, mxfp8)
    n2 = int(min(w.T, max(n, n * budget_s / max(dt, 1e-3))))
    if n2 > n:
        n = n2
        dt = oracle_sample_time(w, wts_host, x_host, n, mxfp8)
    return {"value": n / dt, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"oracle forward (fp64 C, OpenMP) on the first {n} tokens of the {w.name} batch "
                      f"as a batch of its own ({dt:.1f} s)"}


# ------------------------------------------------------------------------------------------
# main
# ------------------------------------------------------------------------------------------

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def max_over_ranks(value: float, world: int) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


REF_BUDGET_S = 150.0  # CPU seconds of the reference arm's timed steps, whatever --steps is


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    w = workload_of(args)
    wts = gen.make_weights(w, "cpu")
    x = gen.make_x(w, "cpu")
    from oracle import oracle
    mx = getattr(args, "precision", "bf16") == "mxfp8"
    # each step is a bounded sample: at most --ref-tokens tokens, and few enough that the K
    # timed steps take about REF_BUDGET_S in all (sized from a probe that is also the warm-up)
    n_max = min(w.T, args.ref_tokens)
    n_probe = min(n_max, 8)
    t_probe = oracle_sample_time(w, wts, x, n_probe, mx)
    per_step = REF_BUDGET_S / max(args.steps, 1)
    n = int(min(n_max, max(1, n_probe * per_step / max(t_probe, 1e-6))))
    times = [oracle_sample_time(w, wts, x, n, mx) for _ in range(args.steps)]
    per_tok = float(np.mean(times)) / n
    value = 1.0 / per_tok
    ms_step = per_tok * w.T * 1e3
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": w.name, **w.describe(),
                                            "precision": getattr(args, "precision", "bf16")},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": f"each step: oracle forward on the first {n} tokens of the batch"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["mine", "reference"], default="mine")
    ap.add_argument("--workload", default="flashmoe_prefill", choices=sorted(configs.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-trace", action="store_true", help="skip the traced forward (SM-busy)")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--ref-tokens", type=int, default=256)
    ap.add_argument("--T", type=int, default=None, help="override the workload's token count (profiling)")
    ap.add_argument("--E", type=int, default=None, help="override the workload's expert count (profiling)")
    ap.add_argument("--tiles", choices=["auto", "pair", "single"], default="auto",
                    help="expert-GEMM shape: the library's choice, 256-row tiles on SM pairs, or "
                         "128-row tiles on single SMs")
    ap.add_argument("--sched", choices=["dynamic", "static"], default="dynamic",
                    help="task scheduling of the expert GEMMs: the atomic queue, or the static "
                         "per-expert SM quota baseline (ablation)")
    ap.add_argument("--precision", choices=["bf16", "mxfp8"], default="bf16",
                    help="expert weights and activations in bf16, or MXFP8 (E4M3, 32-element blocks)")
    ap.add_argument("--traffic-bytes", type=float, default=None,
                    help="ncu dram bytes per launch of the expert-GEMM kernel, if captured")
    args = ap.parse_args()
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            return run_reference(args, world, rank)
        return run_mine(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


def workload_of(args):
    w = configs.WORKLOADS[args.workload]
    if args.T is not None:
        w = w.replace(T=args.T)
    if args.E is not None:
        w = w.replace(E=args.E)
    return w


def run_mine(args, world, rank, local):
    from mixture_experts_layer_block_b200.native import (MOE_FLAG_HOST_STAGING, MOE_FLAG_MXFP8,
                                                         MOE_FLAG_STAGE_TIMING, MoELayer)
    w = workload_of(args)
    mx = args.precision == "mxfp8"
    prec_flags = MOE_FLAG_MXFP8 if mx else 0
    dev = torch.device("cuda", local)
    wts = gen.make_weights(w, dev)
    x = gen.make_x(w.replace(seed=w.seed + 1000 * rank) if rank else w, dev)  # each replica its own tokens
    out = torch.empty((w.T, w.H), dtype=torch.float32, device=dev)
    layer = MoELayer.for_workload(w, flags=MOE_FLAG_HOST_STAGING | prec_flags | tile_flags(args))
    stream = torch.cuda.current_stream(dev)
    # MXFP8 experts: the weights are quantised once, before any timing (a model stores them so)
    wq = layer.quantize_experts_mxfp8(wts) if mx else None

    for _ in range(args.warmup):
        run_forward(layer, x, wts, out, wq)
    torch.cuda.synchronize()
    rc, st = layer.status()
    assert rc == 0 and st == 0, (rc, st)
    gemm_shape = {"tile_m": layer.query(6), "workers": layer.query(1), "shape": layer.query(8),
                  "scheduler": getattr(args, "sched", "dynamic"),
                  "kind": "SM pairs (2-CTA clusters)" if layer.query(6) == 256 else "single SMs"}
    stats = routing_stats(layer, w, dev)

    # headline: K whole forwards back to back, nothing recorded between the kernels
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            run_forward(layer, x, wts, out, wq)
        e1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms = e0.elapsed_time(e1) / args.steps
    ms = max_over_ranks(ms, world)
    rc, st = layer.status()
    assert rc == 0 and st == 0, (rc, st)

    tokens_per_s = world * w.T / (ms * 1e-3)
    flops = configs.useful_flops(w, stats["kept_slots"])
    tflops = flops / (ms * 1e-3) / 1e12

    # end to end through the C ABI with host buffers: every step copies x from pinned host memory
    # to the device and the step's out back. Pipelined: moe_forward_host_async overlaps step
    # i+1's upload and step i-1's download with step i's forward; the events bracket all steps
    # and the final join. Also the synchronous moe_forward_host (upload, forward, download, wait).
    x_pin = x.cpu().pin_memory()
    out_pin = torch.empty((w.T, w.H), dtype=torch.float32).pin_memory()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if not mx:
        for _ in range(3):
            layer.forward_host(x_pin, wts, out_pin)
        barrier(world)
        torch.cuda.synchronize()
        f0.record(stream)
        for _ in range(args.e2e_steps):
            layer.forward_host_async(x_pin, wts, out_pin, stream=stream)
        layer.forward_host_join(stream=stream, block=False)
        f1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(f0.elapsed_time(f1) / args.e2e_steps, world)
    # synchronous: upload, forward, download, wait (for MXFP8 experts, which have no host-buffer
    # entry point, the caller's own copies around moe_forward_mxfp8)
    x_dev = torch.empty_like(x)

    def host_step():
        if mx:
            x_dev.copy_(x_pin, non_blocking=True)
            run_forward(layer, x_dev, wts, out, wq)
            out_pin.copy_(out, non_blocking=True)
            stream.synchronize()
        else:
            layer.forward_host(x_pin, wts, out_pin)
    for _ in range(3):
        host_step()
    barrier(world)
    torch.cuda.synchronize()
    f0.record(stream)
    for _ in range(args.e2e_steps):
        host_step()
    f1.record(stream)
    torch.cuda.synchronize()
    e2e_sync_ms = max_over_ranks(f0.elapsed_time(f1) / args.e2e_steps, world)
    if mx:
        e2e_ms = e2e_sync_ms
    layer.close()

    # per-kernel durations: a second timed pass whose handle records CUDA events around every
    # kernel on the launching stream (events between kernels stop them from overlapping, so
    # this pass is kept apart from the headline one)
    layer_t = MoELayer.for_workload(w, flags=MOE_FLAG_STAGE_TIMING | prec_flags | tile_flags(args))
    for _ in range(3):
        run_forward(layer_t, x, wts, out, wq)
    torch.cuda.synchronize()
    layer_t.stage_times()  # drop the warm-up window
    barrier(world)
    for _ in range(min(args.steps, 256)):
        run_forward(layer_t, x, wts, out, wq)
    stage_ms = layer_t.stage_times()
    rc, st = layer_t.status()
    assert rc == 0 and st == 0, (rc, st)
    layer_t.close()

    peaks, peak_src = load_peaks()
    gemm_ms = stage_ms[4]
    gbytes = algorithmic_bytes_gemm(w, stats["hit_experts"], mx)
    gemm_flops = flops - 2.0 * w.T * w.H * w.E
    # The GEMM is timed inside a loop of forwards. When that loop keeps the tensor cores busy for
    # a second or more the 1 kW power cap sets the clock, and the sustained GEMM peak (a cuBLAS
    # loop of seconds) is the fair denominator; a shorter pass is compared with the burst peak.
    timed_pass_s = min(args.steps, 256) * ms * 1e-3
    tc_kind = "sustained" if timed_pass_s >= 1.0 else "burst"
    tc_peak = peaks["bf16_tflops_sustained"] if tc_kind == "sustained" else peaks["bf16_tflops"]
    # MXFP8 MMAs: the measured bf16 peak times the nominal fp8 / bf16 ratio (4.5 / 2.25 PFLOP/s)
    tc_ratio = 2.0 if mx else 1.0
    tc_peak *= tc_ratio
    hbm_t = gbytes / (peaks["hbm_gbs"] * 1e9)
    tc_t = gemm_flops / (tc_peak * 1e12)
    if hbm_t >= tc_t:
        achieved = gbytes / (gemm_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"]}
    else:
        achieved = gemm_flops / (gemm_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tc_peak, "unit": "TFLOP/s",
                "frac": achieved / tc_peak, "peak_kind": tc_kind,
                "timed_pass_s": timed_pass_s, "frac_of_burst_peak": achieved / (tc_ratio * peaks["bf16_tflops"])}
        if mx:
            roof["peak_dtype"] = "mxfp8: measured bf16 peak x 2 (nominal 4.5 / 2.25 PFLOP/s)"
    traffic = args.traffic_bytes if args.traffic_bytes is not None else (None if mx else measured_traffic(w.name))
    roof.update({"traffic": traffic, "traffic_source": measured_traffic_note(w.name) if args.traffic_bytes is None
                 else "--traffic-bytes", "kernel": "moe_gemm_mx_kernel" if mx else "moe_gemm_kernel",
                 "algorithmic_bytes": gbytes, "kernel_ms": gemm_ms, "peak_source": peak_src,
                 "kernel_timing": f"CUDA events around the kernel over {min(args.steps, 256)} timed forwards "
                                  "of a second pass"})

    line = {"metric": METRIC, "value": tokens_per_s, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "mxfp8-e4m3 experts, bf16 router" if mx else "bf16",
            "data": "synthetic",
            "config": {"workload": w.name, "T": w.T, "H": w.H, "D": w.D, "E": w.E, "top_k": w.top_k,
                       "block_m": w.block_m, "D_shared": w.D_shared, "capacity_factor": w.capacity_factor,
                       "precision": args.precision,
                       "parallelism": f"replicas{world}",
                       "l2": "inputs larger than L2 (expert weights read each step exceed 126 MB)"},
            "tflops": tflops, "tflops_frac_of_bf16_peak": tflops / peaks["bf16_tflops"],
            "stage_ms": dict(zip(MoELayer.STAGES, stage_ms)),
            "routing": stats, "roofline": roof,
            "e2e": {"value": world * w.T / (e2e_ms * 1e-3), "unit": UNIT,
                    "h2d_bytes_per_step": w.T * w.H * 2, "d2h_bytes_per_step": w.T * w.H * 4,
                    "api": ("moe_forward_mxfp8 between the caller's pinned-host copies of x and out, "
                            "synchronised every step") if mx else
                           ("moe_forward_host_async, steps pipelined (copies overlap the previous "
                            "and next forwards), joined inside the timed region"),
                    "synchronous": {"value": world * w.T / (e2e_sync_ms * 1e-3),
                                    "api": "as above" if mx else "moe_forward_host"}},
            "gpu_launches": len(MoELayer.STAGES) * args.steps,
            "gemm_shape": gemm_shape,
            "clocks": clk.summary()}
    if not args.no_trace:
        line["scheduler"] = traced_forward(w, wts, x, out, tile_flags(args) | prec_flags, wq)
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, wts, x, mxfp8=mx)
    if rank == 0:
        print(json.dumps(line))
    return 0


if __name__ == "__main__":
    sys.exit(main())
