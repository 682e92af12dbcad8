"""Benchmark of the fused MoE layer forward on B200: MoE-layer tokens/s and TFLOP/s, with the
dominant kernel's fraction of the HBM (or tensor) roofline.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mine|reference]
                  [--workload dsv3] [--no-per-config] [--no-cpu-baseline] [--e2e-steps M]

One step = one whole layer forward (router projection, gating, align, row gather, expert
GEMMs with the fused SwiGLU and router weighting, and the combine) over one batch of seeded
synthetic input already resident in HBM. The headline workload is the largest single-GPU
layer, the DeepSeek-V3-style one (T=4096, H=7168, 256 routed experts top-8 plus a shared
expert, 22.6 GB of expert weights, far larger than the 126 MB L2). The line also carries a
`per_config` object: every other workload (the FlashMoE-shaped prefill, decode on seeds 0, 1
and 2, the skewed router and the same router without its bias, and the tiny layer), the
static per-expert-quota ablation and the MXFP8 experts, each with its own timing, roofline
fractions and SM-busy fraction, plus the skew overhead. Every timing is given twice: K
forwards back to back (the headline), and K forwards each after a write of a buffer twice the
L2 size (outside the timed events).

With N > 1 (torchrun) every rank runs an independent replica on its own GPU (no collective on
the data path; weak scaling); rank 0 prints one JSON line. `--impl reference` times the CPU
oracle instead, on a bounded token sample of the same workload.
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
L2_BYTES = 126 * 1024 * 1024


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one expert-GEMM launch, from
# the ncu captures summarised under profiles/, with the hash of the kernel sources it was taken
# on. A different hash (the kernel changed since) reports null.
KERNEL_SOURCES = ["mixture_experts_layer_block_b200/csrc/moe_gemm.cu",
                  "mixture_experts_layer_block_b200/csrc/front.cuh",
                  "mixture_experts_layer_block_b200/csrc/route.cuh",
                  "mixture_experts_layer_block_b200/csrc/mx.cuh",
                  "mixture_experts_layer_block_b200/csrc/common.cuh",
                  "mixture_experts_layer_block_b200/csrc/ptx.cuh",
                  "mixture_experts_layer_block_b200/csrc/launch.h"]
MEASURED_TRAFFIC = {
    "flashmoe_prefill": ("f7bab268de21caa7", 1.679793e9 + 0.059929e9, "one full-size launch"),
    # at most 16 tokens the forward is one launch: its traffic covers the router, gather and combine
    "decode": ("f7bab268de21caa7", 0.338417e9 + 0.004369e9, "one full-size launch of the fused forward"),
    # full DSV3 holds 22.6 GB of weights, too large for a multi-pass capture: the T=512, E=32
    # case of the same layer (the same per-expert load, 1/8 of the experts and tokens) scaled
    # by the 8x more units of a full launch
    "dsv3": ("f7bab268de21caa7", 8 * (3.035066e9 + 0.113653e9), "T=512, E=32 capture x 8"),
}


def kernel_source_hash() -> str:
    """SHA-256 (first 16 hex digits) of the kernel sources with their comments and blank lines
    left out: a comment edit keeps the measured traffic, a code edit drops it."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        code = "\n".join(line.rstrip() for line in text.splitlines() if line.strip())
        h.update(code.encode("utf-8"))
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


def algorithmic_bytes_layer(w, hit_experts: int, mxfp8: bool = False) -> float:
    """The whole layer's algorithmic bytes: the expert GEMMs' (hit experts' and shared weights,
    x and out) plus the router weights (bf16 [E][H])."""
    return algorithmic_bytes_gemm(w, hit_experts, mxfp8) + 2.0 * w.E * w.H


def config_of(w, precision: str, world: int) -> dict:
    """The `config` object of the JSON line: the workload only, identical in both arms."""
    return {"workload": w.name, "T": w.T, "H": w.H, "D": w.D, "E": w.E, "top_k": w.top_k,
            "block_m": w.block_m, "D_shared": w.D_shared, "capacity_factor": w.capacity_factor,
            "seed": w.seed, "precision": precision, "parallelism": f"replicas{world}",
            "l2": "inputs larger than L2 (the expert weights read each step exceed 126 MB); "
                  "L2-flushed timings reported beside"}


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


def roofline(w, peaks, gemm_ms, kept, hit, mx, timed_pass_s):
    """Roofline of the dominant kernel (the expert GEMMs): HBM- or tensor-bound, whichever
    roofline time is longer; achieved = algorithmic bytes (or useful FLOPs) / kernel time."""
    flops = configs.useful_flops(w, kept)
    gemm_flops = flops - 2.0 * w.T * w.H * w.E
    gbytes = algorithmic_bytes_gemm(w, hit, mx)
    # A GEMM timed inside a loop that keeps the tensor cores busy for a second or more runs at
    # the clock the 1 kW power cap allows: the sustained GEMM peak (a cuBLAS loop of seconds) is
    # then the fair denominator; a shorter pass is compared with the burst peak.
    tc_kind = "sustained" if timed_pass_s >= 1.0 else "burst"
    tc_peak = peaks["bf16_tflops_sustained"] if tc_kind == "sustained" else peaks["bf16_tflops"]
    tc_ratio = 2.0 if mx else 1.0  # MXFP8 MMAs: the measured bf16 peak x nominal fp8/bf16 (4.5/2.25)
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
                "frac": achieved / tc_peak, "peak_kind": tc_kind, "timed_pass_s": timed_pass_s,
                "frac_of_burst_peak": achieved / (tc_ratio * peaks["bf16_tflops"])}
        if mx:
            roof["peak_dtype"] = "mxfp8: measured bf16 peak x 2 (nominal 4.5 / 2.25 PFLOP/s)"
    roof["algorithmic_bytes"] = gbytes
    roof["kernel_ms"] = gemm_ms
    return roof


def layer_fraction(w, peaks, ms, kept, hit, mx):
    """The whole step against its own roofline: max(useful FLOPs / tensor peak, algorithmic
    bytes / HBM peak) over the measured step time (the burst tensor peak)."""
    flops = configs.useful_flops(w, kept)
    b = algorithmic_bytes_layer(w, hit, mx)
    t_hbm = b / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / ((2.0 if mx else 1.0) * peaks["bf16_tflops"] * 1e12)
    return {"bound": "hbm" if t_hbm >= t_tc else "tensor", "frac": max(t_hbm, t_tc) / (ms * 1e-3),
            "algorithmic_bytes": b, "useful_flops": flops}


# handle options the command line sets once for every layer bench.py builds
LAYER_KW = {}


def tile_flags(args) -> int:
    from mixture_experts_layer_block_b200 import native
    f = {"auto": 0, "pair": native.MOE_FLAG_PAIR_TILES, "single": native.MOE_FLAG_SINGLE_TILES,
         "two": native.MOE_FLAG_TWO_TILES, "tail": native.MOE_FLAG_TAIL_TILES,
         "general": native.MOE_FLAG_NO_TAIL_TILES}[getattr(args, "tiles", "auto")]
    if getattr(args, "sched", "dynamic") == "static":
        f |= native.MOE_FLAG_STATIC_QUOTA
    if getattr(args, "unfused_small", False):
        f |= native.MOE_FLAG_UNFUSED_SMALL
    return f


def run_forward(layer, x, wts, out, wq=None):
    """One layer forward: bf16 experts, or MXFP8 experts when `wq` holds their quantisation."""
    if wq is None:
        layer.forward(x, wts, out)
    else:
        layer.forward_mxfp8(x, wts["W_router"], wts.get("bias"), wq, out)


def traced_forward(w, wts, x, out, extra_flags=0, wq=None):
    """One extra forward with per-task tracing (outside the timed region)."""
    from mixture_experts_layer_block_b200.native import MOE_FLAG_MXFP8, MOE_FLAG_TRACE, MoELayer
    layer = MoELayer.for_workload(w, flags=MOE_FLAG_TRACE | extra_flags | (MOE_FLAG_MXFP8 if wq else 0), **LAYER_KW)
    for _ in range(2):
        run_forward(layer, x, wts, out, wq)
    torch.cuda.synchronize()
    rec = layer.trace(1 << 20)
    n_ctas = layer.query(1)
    res = sm_busy_fraction(rec, n_ctas)
    if layer.query(8) != 3:  # every expert-GEMM kernel but the SM-pair one keeps wait accounting
        res["waits"] = wait_fractions(layer.trace_waits(), MoELayer.WAITS)
    layer.close()
    return res


def wait_fractions(w: np.ndarray, names) -> dict:
    """Where each role's issuing thread spent its loop, summed over the CTAs: the fraction of
    the MMA lane's loop spent waiting for operands, for a free accumulator, for tasks (the rest
    is issuing MMAs), and likewise for the producer and the epilogue."""
    if w.size == 0:
        return {}
    tot = w.sum(axis=0).astype(np.float64)
    col = {n: tot[i] for i, n in enumerate(names)}
    f = lambda a, b: float(col[a] / col[b]) if col[b] > 0 else None
    return {"mma": {"operands": f("mma_full", "mma_loop"), "accumulator": f("mma_acc", "mma_loop"),
                    "task": f("mma_task", "mma_loop")},
            "producer": {"free_stage": f("prod_empty", "prod_loop"), "dependency": f("prod_dep", "prod_loop"),
                         "ring": f("prod_ring", "prod_loop"), "claim_decode": f("prod_claim", "prod_loop")},
            "epilogue": {"task": f("epi_task", "epi_loop"), "accumulator": f("epi_acc", "epi_loop")},
            **({"front_us": front_timeline(w, names)} if col["front_to_end"] > 0 else {})}


def front_timeline(w: np.ndarray, names) -> dict:
    """The fused small-batch forward's front in microseconds: the median CTA's router slice and
    gather; the arrival plus the schedule in CTA 0 (which also writes the align outputs; its steps
    are `schedule_steps`) and the median over the other CTAs; the median time from the front's
    start to the end of the epilogue loop; the column-block counting and combines."""
    c = {n: w[:, i] for i, n in enumerate(names)}
    last = c["front_last"] == 1
    med = lambda v: float(np.median(v) / 1e3) if v.size else None
    steps = {n[6:]: med(c[n][last]) for n in names if n.startswith("sched_")}
    comb = c["combine_run"] > 0
    return {"router": med(c["front_router"]), "schedule_compute": med(c["front_schedule"][last]),
            "schedule_steps": steps, "schedule_wait": med(c["front_schedule"][~last]),
            "gather": med(c["front_gather"]), "front_to_end": med(c["front_to_end"]),
            "max_front_to_end": float(c["front_to_end"].max() / 1e3),
            # per CTA: the column-block counting after its down tasks, and its combines
            "combine_count": med(c["combine_count"]), "combine_run": med(c["combine_run"][comb]),
            "combining_ctas": int(comb.sum())}


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

def host_inputs(w, device):
    """The workload's seeded inputs drawn on `device` (the same values the timed GPU arm uses
    when that is the GPU) and copied to host memory for the oracle."""
    wts = gen.make_weights(w, device)
    x = gen.make_x(w, device)
    wts = {k: (v.cpu() if v is not None else None) for k, v in wts.items()}
    return wts, x.cpu()


def oracle_sample_time(w, wts_host, x_host, n_tokens, mxfp8=False):
    """Seconds of one oracle forward (router, gating, align, experts, combine) on the first
    n_tokens tokens as a batch of their own."""
    from oracle import oracle
    sub = w.replace(T=n_tokens)
    inp = dict(wts_host, x=x_host[:n_tokens])
    t0 = time.perf_counter()
    oracle.forward(inp, sub.top_k, sub.block_m, sub.capacity_factor, mxfp8=mxfp8)
    return time.perf_counter() - t0


def cpu_baseline(w, wts_host, x_host, budget_s=12.0, mxfp8=False):
    """Time the oracle, as it stands, on the first n tokens of the batch (a smaller batch of
    the same layer), n sized for about `budget_s` of CPU work."""
    from oracle import oracle
    n = min(w.T, 16)
    dt = oracle_sample_time(w, wts_host, x_host, n, mxfp8)
    n2 = int(min(w.T, max(n, n * budget_s / max(dt, 1e-3))))
    if n2 > n:
        n = n2
        dt = oracle_sample_time(w, wts_host, x_host, n, mxfp8)
    return {"value": n / dt, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"oracle forward (fp64 C, OpenMP) on the first {n} tokens of the {w.name} batch "
                      f"as a batch of their own ({dt:.1f} s)"}


# ------------------------------------------------------------------------------------------
# process plumbing
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
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=300))
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


REF_BUDGET_S = 60.0  # CPU seconds of the reference arm's timed steps, whatever --steps is


def run_reference(args, world, rank):
    """The reference arm: the CPU oracle, as it stands, on the host cores, on the same
    workload and config as the GPU arm. Each timed step runs the oracle's whole forward on the
    first n tokens of the batch, n sized so that the K steps take about REF_BUDGET_S; the line
    reports the measured seconds per step and the sampled tokens per second."""
    if rank != 0:
        return 0
    w = workload_of(args)
    from oracle import oracle
    mx = getattr(args, "precision", "bf16") == "mxfp8"
    wts, x = host_inputs(w, "cuda" if torch.cuda.is_available() else "cpu")
    n_max = min(w.T, args.ref_tokens)
    n_probe = min(n_max, 8)
    oracle_sample_time(w, wts, x, n_probe, mx)  # warm-up (also loads the oracle)
    t_probe = oracle_sample_time(w, wts, x, n_probe, mx)
    per_step = REF_BUDGET_S / max(args.steps, 1)
    n = int(min(n_max, max(1, n_probe * per_step / max(t_probe, 1e-6))))
    for _ in range(max(0, min(args.warmup, 1))):
        oracle_sample_time(w, wts, x, n, mx)
    times = [oracle_sample_time(w, wts, x, n, mx) for _ in range(args.steps)]
    step_s = float(np.mean(times))
    value = n / step_s
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(w, getattr(args, "precision", "bf16"), world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": f"each step: the oracle's forward on the first {n} of the batch's "
                                       f"{w.T} tokens (a batch of their own); ms_per_step is that step's "
                                       f"measured time"},
            "tokens_per_step": n,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def workload_of(args, name=None):
    w = configs.WORKLOADS[name or args.workload]
    if getattr(args, "T", None) is not None:
        w = w.replace(T=args.T)
    if getattr(args, "E", None) is not None:
        w = w.replace(E=args.E)
    return w


# ------------------------------------------------------------------------------------------
# the GPU arm
# ------------------------------------------------------------------------------------------

class Flusher:
    """Writes a buffer of twice the L2 size, so that nothing of the previous step stays in L2."""

    def __init__(self, dev):
        try:
            l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        except (AttributeError, RuntimeError):
            l2 = L2_BYTES
        self.buf = torch.empty(2 * max(l2, L2_BYTES) // 4, dtype=torch.float32, device=dev)

    def __call__(self):
        self.buf.fill_(1.0)


def timed_steps(layer, x, wts, out, wq, steps, stream, world, flusher=None):
    """Device time per step (ms), max over ranks. Without `flusher`: K forwards back to back
    between two events. With it: each forward between its own pair of events, after an L2 flush
    outside them; the per-step times are summed."""
    barrier(world)
    torch.cuda.synchronize()
    if flusher is None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            run_forward(layer, x, wts, out, wq)
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / steps
    else:
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for a, b in evs:
            flusher()
            a.record(stream)
            run_forward(layer, x, wts, out, wq)
            b.record(stream)
        torch.cuda.synchronize()
        ms = sum(a.elapsed_time(b) for a, b in evs) / steps
    barrier(world)
    return max_over_ranks(ms, world)


def measure(w, dev, world, rank, steps, warmup, peaks, flusher, mx=False, flags=0, trace=True,
            keep=False, sched="dynamic"):
    """One workload: warm-up, K steps back to back (clocks sampled), K steps with L2 flushes,
    a per-kernel timing pass, a traced forward (SM-busy); the roofline of the expert GEMMs and
    of the whole step. With `keep`, also returns the layer and inputs (for the e2e legs)."""
    from mixture_experts_layer_block_b200.native import (MOE_FLAG_HOST_STAGING, MOE_FLAG_MXFP8,
                                                         MOE_FLAG_STAGE_TIMING, MoELayer)
    prec = MOE_FLAG_MXFP8 if mx else 0
    wts = gen.make_weights(w, dev)
    x = gen.make_x(w.replace(seed=w.seed + 1000 * rank) if rank else w, dev)  # each replica its own tokens
    out = torch.empty((w.T, w.H), dtype=torch.float32, device=dev)
    layer = MoELayer.for_workload(w, flags=(MOE_FLAG_HOST_STAGING if keep else 0) | prec | flags, **LAYER_KW)
    stream = torch.cuda.current_stream(dev)
    wq = layer.quantize_experts_mxfp8(wts) if mx else None  # weights are stored quantised
    for _ in range(warmup):
        run_forward(layer, x, wts, out, wq)
    torch.cuda.synchronize()
    rc, st = layer.status()
    assert rc == 0 and st == 0, (w.name, rc, st)
    stats = routing_stats(layer, w, dev)
    shape = {"tile_m": layer.query(6), "workers": layer.query(1), "shape": layer.query(8), "scheduler": sched,
             "kernels_per_forward": layer.query(11), "claim_batch": max(1, LAYER_KW.get("claim_batch", 1))}
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        ms = timed_steps(layer, x, wts, out, wq, steps, stream, world)
    ms_flushed = timed_steps(layer, x, wts, out, wq, steps, stream, world, flusher)
    rc, st = layer.status()
    assert rc == 0 and st == 0, (w.name, rc, st)

    # per-kernel durations: a separate pass whose handle records CUDA events around every kernel
    # on the launching stream (events between kernels stop them from overlapping)
    lt = MoELayer.for_workload(w, flags=MOE_FLAG_STAGE_TIMING | prec | flags, **LAYER_KW)
    for _ in range(3):
        run_forward(lt, x, wts, out, wq)
    torch.cuda.synchronize()
    lt.stage_times()  # drop the warm-up window
    barrier(world)
    n_stage = min(steps, 256)
    for _ in range(n_stage):
        run_forward(lt, x, wts, out, wq)
    stage_ms = lt.stage_times()
    rc, st = lt.status()
    assert rc == 0 and st == 0, (w.name, rc, st)
    lt.close()
    stage_ms = [max_over_ranks(v, world) for v in stage_ms]

    kept, hit = stats["kept_slots"], stats["hit_experts"]
    flops = configs.useful_flops(w, kept)
    roof = roofline(w, peaks, stage_ms[4], kept, hit, mx, n_stage * ms * 1e-3)
    res = {"workload": w.name, "seed": w.seed, "precision": "mxfp8" if mx else "bf16", "steps": steps,
           "warmup": warmup, "ms_per_step": ms, "ms_per_step_l2_flushed": ms_flushed,
           "tokens_per_s": world * w.T / (ms * 1e-3), "tflops": flops / (ms * 1e-3) / 1e12,
           "stage_ms": dict(zip(MoELayer.STAGES, stage_ms)), "routing": stats, "gemm_shape": shape,
           "roofline": roof, "layer_roofline": layer_fraction(w, peaks, ms, kept, hit, mx),
           "layer_roofline_l2_flushed": layer_fraction(w, peaks, ms_flushed, kept, hit, mx),
           "clocks": clk.summary(), "kernel_timing": f"CUDA events around each kernel, {n_stage} forwards"}
    if trace:
        res["scheduler"] = traced_forward(w, wts, x, out, flags, wq)
    if keep:
        return res, (layer, x, wts, out, wq, stream)
    layer.close()
    del wts, x, out, wq
    torch.cuda.empty_cache()
    return res


def e2e_legs(w, layer, x, wts, out, wq, stream, world, steps, mx):
    """End to end through the C ABI with host buffers: every step copies x from pinned host
    memory to the device and the step's out back. Pipelined: moe_forward_host_async overlaps step
    i+1's upload and step i-1's download with step i's forward; the events bracket all steps and
    the final join. Also the synchronous moe_forward_host (upload, forward, download, wait)."""
    x_pin = x.cpu().pin_memory()
    out_pin = torch.empty((w.T, w.H), dtype=torch.float32).pin_memory()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_ms = None
    if not mx:
        for _ in range(3):
            layer.forward_host(x_pin, wts, out_pin)
        barrier(world)
        torch.cuda.synchronize()
        f0.record(stream)
        for _ in range(steps):
            layer.forward_host_async(x_pin, wts, out_pin, stream=stream)
        layer.forward_host_join(stream=stream, block=False)
        f1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(f0.elapsed_time(f1) / steps, world)
    x_dev = torch.empty_like(x)

    def host_step():
        if mx:  # MXFP8 experts have no host-buffer entry point: the caller's own copies
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
    for _ in range(steps):
        host_step()
    f1.record(stream)
    torch.cuda.synchronize()
    sync_ms = max_over_ranks(f0.elapsed_time(f1) / steps, world)
    if mx:
        e2e_ms = sync_ms
    return {"value": world * w.T / (e2e_ms * 1e-3), "unit": UNIT,
            "h2d_bytes_per_step": w.T * w.H * 2, "d2h_bytes_per_step": w.T * w.H * 4,
            "api": ("moe_forward_mxfp8 between the caller's pinned-host copies of x and out, synchronised every "
                    "step") if mx else
                   ("moe_forward_host_async, steps pipelined (copies overlap the previous and next forwards), "
                    "joined inside the timed region"),
            "synchronous": {"value": world * w.T / (sync_ms * 1e-3), "api": "as above" if mx else "moe_forward_host"}}


# per_config entries: (key, workload name, seed, precision, extra flags, scheduler)
def per_config_plan():
    from mixture_experts_layer_block_b200.native import MOE_FLAG_STATIC_QUOTA as SQ
    return [
        ("tiny", "tiny", 0, "bf16", 0, "dynamic"),
        ("flashmoe_prefill", "flashmoe_prefill", 0, "bf16", 0, "dynamic"),
        ("decode", "decode", 0, "bf16", 0, "dynamic"),
        ("decode_seed1", "decode", 1, "bf16", 0, "dynamic"),
        ("decode_seed2", "decode", 2, "bf16", 0, "dynamic"),
        ("skew", "skew", 0, "bf16", 0, "dynamic"),
        ("skew_uniform", "skew_uniform", 0, "bf16", 0, "dynamic"),
        # the static per-expert SM quota baseline (Weave blog, section 1.2) on the same layers
        ("static_quota/skew", "skew", 0, "bf16", SQ, "static"),
        ("static_quota/skew_uniform", "skew_uniform", 0, "bf16", SQ, "static"),
        ("static_quota/dsv3", "dsv3", 0, "bf16", SQ, "static"),
        ("static_quota/flashmoe_prefill", "flashmoe_prefill", 0, "bf16", SQ, "static"),
        ("static_quota/decode", "decode", 0, "bf16", SQ, "static"),
        # MXFP8 experts
        ("mxfp8/dsv3", "dsv3", 0, "mxfp8", 0, "dynamic"),
        ("mxfp8/flashmoe_prefill", "flashmoe_prefill", 0, "mxfp8", 0, "dynamic"),
        ("mxfp8/decode", "decode", 0, "mxfp8", 0, "dynamic"),
        ("mxfp8/skew", "skew", 0, "mxfp8", 0, "dynamic"),
    ]


def compact(entry):
    """A per_config entry without the bulky parts."""
    keep = ("workload", "seed", "precision", "steps", "ms_per_step", "ms_per_step_l2_flushed", "tokens_per_s",
            "tflops", "stage_ms", "routing", "gemm_shape", "scheduler", "clocks")
    d = {k: entry[k] for k in keep if k in entry}
    r = entry["roofline"]
    d["gemm_roofline"] = {k: r[k] for k in ("bound", "achieved", "unit", "peak", "frac", "peak_kind",
                                            "frac_of_burst_peak", "kernel_ms") if k in r}
    d["layer_roofline"] = {"bound": entry["layer_roofline"]["bound"], "frac": entry["layer_roofline"]["frac"],
                           "frac_l2_flushed": entry["layer_roofline_l2_flushed"]["frac"]}
    return d


def run_profile(args, local):
    """--profile: the workload's warm-up and K timed forwards and nothing else (no flushed pass,
    no per-kernel timing pass, no host-buffer legs, no traced forward), for profiler captures."""
    from mixture_experts_layer_block_b200.native import MOE_FLAG_MXFP8, MoELayer
    dev = torch.device("cuda", local)
    w = workload_of(args)
    mx = args.precision == "mxfp8"
    wts = gen.make_weights(w, dev)
    x = gen.make_x(w, dev)
    out = torch.empty((w.T, w.H), dtype=torch.float32, device=dev)
    layer = MoELayer.for_workload(w, flags=(MOE_FLAG_MXFP8 if mx else 0) | tile_flags(args), **LAYER_KW)
    wq = layer.quantize_experts_mxfp8(wts) if mx else None
    for _ in range(args.warmup):
        run_forward(layer, x, wts, out, wq)
    torch.cuda.synchronize()
    ms = timed_steps(layer, x, wts, out, wq, args.steps, torch.cuda.current_stream(dev), 1)
    rc, st = layer.status()
    assert rc == 0 and st == 0, (rc, st)
    print(json.dumps({"profile": True, "workload": w.name, "T": w.T, "E": w.E, "precision": args.precision,
                      "ms_per_step": ms, "kernels_per_forward": layer.query(11)}))
    layer.close()
    return 0


def run_mine(args, world, rank, local):
    dev = torch.device("cuda", local)
    peaks, peak_src = load_peaks()
    flusher = Flusher(dev)
    w = workload_of(args)
    mx = args.precision == "mxfp8"
    head, (layer, x, wts, out, wq, stream) = measure(
        w, dev, world, rank, args.steps, args.warmup, peaks, flusher, mx, tile_flags(args),
        trace=not args.no_trace, keep=True, sched=args.sched)
    e2e = e2e_legs(w, layer, x, wts, out, wq, stream, world, args.e2e_steps, mx)
    layer.close()
    cpu = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        wts_h = {k: (v.cpu() if v is not None else None) for k, v in wts.items()}
        x_h = x.cpu()
        del layer, x, wts, out, wq
        torch.cuda.empty_cache()
        cpu = cpu_baseline(w, wts_h, x_h, mxfp8=mx)
        del wts_h, x_h
    else:
        del layer, x, wts, out, wq
        torch.cuda.empty_cache()

    roof = dict(head["roofline"])
    traffic = args.traffic_bytes if args.traffic_bytes is not None else (None if mx else measured_traffic(w.name))
    roof.update({"traffic": traffic,
                 "traffic_source": (measured_traffic_note(w.name) if args.traffic_bytes is None else "--traffic-bytes"),
                 "kernel": "moe_gemm_mx_kernel" if mx else "moe_gemm_kernel", "peak_source": peak_src,
                 "kernel_timing": head["kernel_timing"] + " of a second pass"})
    line = {"metric": METRIC, "value": head["tokens_per_s"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "mxfp8-e4m3 experts, bf16 router" if mx else "bf16", "data": "synthetic",
            "config": config_of(w, args.precision, world),
            "ms_per_step_l2_flushed": head["ms_per_step_l2_flushed"],
            "tflops": head["tflops"], "tflops_frac_of_bf16_peak": head["tflops"] / peaks["bf16_tflops"],
            "stage_ms": head["stage_ms"], "routing": head["routing"], "roofline": roof,
            "layer_roofline": head["layer_roofline"], "layer_roofline_l2_flushed": head["layer_roofline_l2_flushed"],
            "e2e": e2e, "gpu_launches": head["gemm_shape"]["kernels_per_forward"] * args.steps,
            "gemm_shape": head["gemm_shape"],
            "clocks": head["clocks"]}
    if "scheduler" in head:
        line["scheduler"] = head["scheduler"]
    if cpu is not None:
        line["cpu_baseline"] = cpu

    if not args.no_per_config:
        pc = {}
        for key, name, seed, prec, flags, sched in per_config_plan():
            if name == w.name and seed == w.seed and prec == args.precision and flags == tile_flags(args):
                continue  # the headline itself
            wk = configs.WORKLOADS[name].replace(seed=seed)
            slow = sched == "static"
            e = measure(wk, dev, world, rank, max(5, args.steps // 2) if slow else args.steps,
                        min(args.warmup, 3) if slow else args.warmup, peaks, flusher, prec == "mxfp8", flags,
                        trace=not args.no_trace, sched=sched)
            pc[key] = compact(e)
        pc[w.name if not mx else f"mxfp8/{w.name}"] = compact(head)
        line["per_config"] = pc
        if "skew" in pc and "skew_uniform" in pc:
            s, u = pc["skew"], pc["skew_uniform"]
            line["skew_overhead"] = {
                "layer": s["ms_per_step"] / u["ms_per_step"] - 1.0,
                "layer_l2_flushed": s["ms_per_step_l2_flushed"] / u["ms_per_step_l2_flushed"] - 1.0,
                "expert_gemm": s["stage_ms"]["expert_gemm"] / u["stage_ms"]["expert_gemm"] - 1.0,
                "useful_flops_ratio": (configs.useful_flops(configs.SKEW, s["routing"]["kept_slots"]) /
                                       configs.useful_flops(configs.SKEW_UNIFORM, u["routing"]["kept_slots"])),
                "sm_busy": {"skew": s.get("scheduler", {}).get("sm_busy"),
                            "uniform": u.get("scheduler", {}).get("sm_busy")},
                "target": "<= 0.15 (time under skewed routing over uniform routing at equal useful FLOPs, minus 1)"}
    if rank == 0:
        print(json.dumps(line))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["mine", "reference"], default="mine")
    ap.add_argument("--workload", default="dsv3", choices=sorted(configs.WORKLOADS))
    ap.add_argument("--no-per-config", action="store_true", help="time only the headline workload")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-trace", action="store_true", help="skip the traced forwards (SM-busy)")
    ap.add_argument("--e2e-steps", type=int, default=30)
    ap.add_argument("--ref-tokens", type=int, default=256)
    ap.add_argument("--T", type=int, default=None, help="override the workload's token count (profiling)")
    ap.add_argument("--E", type=int, default=None, help="override the workload's expert count (profiling)")
    ap.add_argument("--tiles", choices=["auto", "pair", "single", "two", "tail", "general"], default="auto",
                    help="expert-GEMM shape: the library's choice, 256-row tiles on SM pairs, "
                         "128-row tiles on single SMs (the library's merge choice), two 128-row tiles "
                         "per task, tails of <= 32 rows merged into the previous tile, or no merging")
    ap.add_argument("--sched", choices=["dynamic", "static"], default="dynamic",
                    help="task scheduling of the expert GEMMs: the atomic queue, or the static "
                         "per-expert SM quota baseline (ablation)")
    ap.add_argument("--unfused-small", action="store_true",
                    help="run batches of at most 16 tokens as six kernels instead of one fused launch")
    ap.add_argument("--precision", choices=["bf16", "mxfp8"], default="bf16",
                    help="expert weights and activations in bf16, or MXFP8 (E4M3, 32-element blocks)")
    ap.add_argument("--traffic-bytes", type=float, default=None,
                    help="ncu dram bytes per launch of the expert-GEMM kernel, if captured")
    ap.add_argument("--profile", action="store_true",
                    help="only the warm-up and the K timed forwards of --workload (for profiler captures)")
    ap.add_argument("--claim-batch", type=int, default=0,
                    help="expert-GEMM task ids a CTA takes per claim on the shared counter (0 = 1)")
    args = ap.parse_args()
    if args.claim_batch:
        LAYER_KW["claim_batch"] = args.claim_batch
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            return run_reference(args, world, rank)
        if args.profile:
            return run_profile(args, local)
        return run_mine(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
