"""The benchmark's roofline arithmetic against the per-layer figures worked out by hand for the
workloads (useful FLOPs per kept slot 6*H*D plus router and shared expert; algorithmic bytes =
the weights of the experts actually hit, plus x and out), so the reported fractions rest on
checked numbers (no GPU needed)."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from mixture_experts_layer_block_b200 import configs  # noqa: E402


def test_prefill_figures():
    w = configs.FLASHMOE_PREFILL
    kept = w.T * w.top_k  # the upper bound: no slot dropped by the capacity limit
    flops = configs.useful_flops(w, kept)
    assert flops - 2.0 * w.T * w.H * w.E == pytest.approx(206.2e9, rel=1e-3)
    assert 2.0 * w.T * w.H * w.E == pytest.approx(1.07e9, rel=1e-2)
    weights = 3.0 * w.E * w.D * w.H * 2
    assert weights == pytest.approx(1.611e9, rel=1e-3)
    assert bench.algorithmic_bytes_gemm(w, w.E) == pytest.approx(weights + w.T * w.H * 6, rel=1e-12)


def test_dsv3_figures():
    w = configs.DSV3
    flops = configs.useful_flops(w, w.T * w.top_k)
    routed = 6.0 * w.T * w.top_k * w.H * w.D
    shared = 6.0 * w.T * w.H * w.D_shared
    assert routed == pytest.approx(2.886e12, rel=1e-3)
    assert shared == pytest.approx(0.361e12, rel=1e-3)
    assert flops == pytest.approx(2.886e12 + 0.361e12 + 0.015e12, rel=2e-3)
    per_expert = 3.0 * w.D * w.H * 2
    assert per_expert == pytest.approx(88.08e6, rel=1e-3)
    b = bench.algorithmic_bytes_gemm(w, w.E)
    assert b - w.T * w.H * 6 == pytest.approx(257 * per_expert, rel=1e-12)
    assert 257 * per_expert == pytest.approx(22.64e9, rel=1e-3)


def test_mxfp8_bytes_are_one_byte_plus_a_scale_per_32():
    w = configs.FLASHMOE_PREFILL
    b16 = bench.algorithmic_bytes_gemm(w, 10)
    b8 = bench.algorithmic_bytes_gemm(w, 10, mxfp8=True)
    out = w.T * w.H * 4
    assert (b8 - out) == pytest.approx((b16 - out) * (1 + 1 / 32) / 2, rel=1e-12)


def test_skew_is_tensor_bound_and_prefill_hbm_bound():
    peaks = {"hbm_gbs": 6459.3, "bf16_tflops": 1653.5}
    for name, bound in (("skew", "tensor"), ("flashmoe_prefill", "hbm"), ("dsv3", "hbm")):
        w = configs.WORKLOADS[name]
        flops = configs.useful_flops(w, w.T * w.top_k) - 2.0 * w.T * w.H * w.E
        t_tc = flops / (peaks["bf16_tflops"] * 1e12)
        t_hbm = bench.algorithmic_bytes_gemm(w, w.E) / (peaks["hbm_gbs"] * 1e9)
        assert (t_tc > t_hbm) == (bound == "tensor"), name


def test_layer_fraction_adds_the_router_weights():
    peaks = {"hbm_gbs": 6459.3, "bf16_tflops": 1653.5}
    w = configs.DECODE
    b = bench.algorithmic_bytes_layer(w, 53)
    assert b == pytest.approx(bench.algorithmic_bytes_gemm(w, 53) + 2.0 * w.E * w.H, rel=1e-12)
    # 53 hit experts of 6.29 MB, the router weights, x and out: about 334.6 MB
    assert b == pytest.approx(334.6e6, rel=2e-3)
    f = bench.layer_fraction(w, peaks, 0.074, w.T * w.top_k, 53, False)
    assert f["bound"] == "hbm" and f["frac"] == pytest.approx(b / 6459.3e9 / 0.074e-3, rel=1e-12)
    assert f["frac"] == pytest.approx(0.70, abs=0.005)


def test_config_object_is_the_same_in_both_arms():
    """The reference arm and the GPU arm print the same config object for the same workload."""
    w = configs.DSV3
    a = bench.config_of(w, "bf16", 1)
    assert a == bench.config_of(configs.WORKLOADS["dsv3"], "bf16", 1)
    assert a["workload"] == "dsv3" and a["T"] == 4096 and a["E"] == 256 and a["D_shared"] == 2048
    assert bench.config_of(w, "bf16", 2)["parallelism"] == "replicas2"


def test_per_config_plan_covers_every_workload_and_the_decode_seeds():
    names = {(n, s) for _, n, s, p, f, _ in bench.per_config_plan() if p == "bf16" and f == 0}
    for n in ("tiny", "flashmoe_prefill", "skew", "skew_uniform"):
        assert (n, 0) in names
    assert {("decode", 0), ("decode", 1), ("decode", 2)} <= names
    keys = [k for k, *_ in bench.per_config_plan()]
    assert len(keys) == len(set(keys))
    assert any(k.startswith("static_quota/") for k in keys) and any(k.startswith("mxfp8/") for k in keys)


def test_wait_fractions_and_front_timeline():
    """The traced forward's per-CTA wait totals become fractions of each role's loop, and the
    fused front's timeline medians (the scheduling CTA's steps apart)."""
    import numpy as np
    names = ("prod_empty", "prod_dep", "prod_ring", "prod_claim", "mma_full", "mma_acc", "mma_task",
             "epi_task", "epi_acc", "prod_loop", "mma_loop", "epi_loop", "front_router", "front_schedule",
             "front_gather", "front_last", "front_to_end", "sched_arrive", "sched_logits", "sched_gating",
             "sched_tables", "sched_writes", "sched_publish", "combine_count", "combine_run")
    w = np.zeros((4, len(names)), dtype=np.int64)
    col = {n: i for i, n in enumerate(names)}
    w[:, col["mma_loop"]] = 1000
    w[:, col["mma_full"]] = [600, 700, 500, 200]
    w[:, col["prod_loop"]] = 1000
    w[:, col["prod_empty"]] = 250
    w[:, col["epi_loop"]] = 1000
    w[:, col["front_router"]] = [3000, 4000, 5000, 6000]
    w[:, col["front_schedule"]] = [10000, 12000, 14000, 9000]
    w[:, col["front_last"]] = [0, 0, 0, 1]
    w[:, col["front_to_end"]] = [80000, 81000, 82000, 90000]
    w[3, col["sched_gating"]] = 4000
    w[:, col["combine_count"]] = [1000, 2000, 3000, 4000]
    w[:, col["combine_run"]] = [0, 5000, 7000, 0]
    f = bench.wait_fractions(w, names)
    assert f["mma"]["operands"] == pytest.approx(2000 / 4000)
    assert f["producer"]["free_stage"] == pytest.approx(0.25)
    fr = f["front_us"]
    assert fr["schedule_compute"] == pytest.approx(9.0) and fr["schedule_wait"] == pytest.approx(12.0)
    assert fr["router"] == pytest.approx(4.5) and fr["max_front_to_end"] == pytest.approx(90.0)
    assert fr["schedule_steps"]["gating"] == pytest.approx(4.0)
    assert fr["combine_count"] == pytest.approx(2.5) and fr["combine_run"] == pytest.approx(6.0)
    assert fr["combining_ctas"] == 2


def test_kernel_source_hash_ignores_comments_only(tmp_path, monkeypatch):
    """The traffic figures stay tied to the kernel code: a comment edit keeps the hash, a code edit
    changes it (and bench.py then reports the traffic as null)."""
    import shutil
    for f in bench.KERNEL_SOURCES:
        dst = tmp_path / f
        dst.parent.mkdir(parents=True, exist_ok=True)
        shutil.copy(os.path.join(bench.ROOT, f), dst)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    base = bench.kernel_source_hash()
    target = tmp_path / bench.KERNEL_SOURCES[0]
    text = target.read_text()
    target.write_text(text + "\n// a note\n/* a block\n   comment */\n\n")
    assert bench.kernel_source_hash() == base
    target.write_text(text + "\nstatic int moe_extra_symbol = 1;\n")
    assert bench.kernel_source_hash() != base
    for w, rec in bench.MEASURED_TRAFFIC.items():
        assert bench.measured_traffic(w) is None
