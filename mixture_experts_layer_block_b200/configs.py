"""The five synthetic MoE-layer workloads, as shapes and input distributions only.

Nothing here computes any part of the layer: it is the shared description that the
seeded input generator, the tests and the benchmark read. Sizes follow the workloads
described on the pages (FlashMoE review, "experimental setup": H=2048, D=2048, top-2,
capacity factor 1.0; Mixture-of-Kittens blog, "Overlapping compute and communication in
MoE": a DeepSeek-V3-style layer with one shared expert and many routed experts; vLLM
execution analysis, "Per-decode-step kernel launches": 256 experts, top-8 decode with
BLOCK_SIZE_M 16).
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass


@dataclass(frozen=True)
class MoEWorkload:
    name: str
    T: int                      # tokens in the batch
    H: int                      # hidden (model) dimension
    D: int                      # routed-expert intermediate dimension
    E: int                      # routed experts
    top_k: int
    block_m: int                # align block size (segment padding granularity)
    D_shared: int = 0           # shared-expert intermediate dimension, 0 = no shared expert
    capacity_factor: float = 0.0  # 0 = dropless
    sigma_x: float = 1.0        # x ~ N(0, sigma_x), rounded to bf16
    sigma_w: float = 0.02       # expert and shared weights ~ N(0, sigma_w), rounded to bf16
    sigma_router: float = 0.02  # router weights ~ N(0, sigma_router), rounded to bf16
    bias: str = "none"          # per-expert router-logit bias: none | gaussian | zipf
    seed: int = 0

    def replace(self, **kw) -> "MoEWorkload":
        return dataclasses.replace(self, **kw)

    @property
    def slots(self) -> int:
        return self.T * self.top_k

    def describe(self) -> dict:
        return {k: v for k, v in dataclasses.asdict(self).items()}


TINY = MoEWorkload("tiny", T=64, H=256, D=128, E=8, top_k=2, block_m=16)

# Capacity factor 1.0 with overflow slots dropped in token order. The align block for this
# shape is not stated; 128 (the tensor-core tile height) is the reading taken.
FLASHMOE_PREFILL = MoEWorkload("flashmoe_prefill", T=4096, H=2048, D=2048, E=64, top_k=2,
                               block_m=128, capacity_factor=1.0)

DSV3 = MoEWorkload("dsv3", T=4096, H=7168, D=2048, E=256, top_k=8, block_m=128,
                   D_shared=2048, sigma_w=0.006, sigma_router=0.006)

DECODE = MoEWorkload("decode", T=16, H=2048, D=512, E=256, top_k=8, block_m=16,
                     bias="gaussian")

# Router bias 2*log(1/rank) with rank = e+1. The skew-overhead comparison runs the same
# router without the bias (SKEW_UNIFORM).
SKEW = MoEWorkload("skew", T=16384, H=4096, D=1536, E=128, top_k=8, block_m=128,
                   bias="zipf")
SKEW_UNIFORM = SKEW.replace(name="skew_uniform", bias="none")

WORKLOADS = {w.name: w for w in (TINY, FLASHMOE_PREFILL, DSV3, DECODE, SKEW, SKEW_UNIFORM)}


def useful_flops(w: MoEWorkload, kept_slots: int) -> float:
    """Useful FLOPs of one layer forward: router projection, plus 3 GEMMs of 2*H*D per kept
    slot, plus the shared expert over every token. Padding rows are not counted."""
    f = 2.0 * w.T * w.H * w.E
    f += 6.0 * kept_slots * w.H * w.D
    f += 6.0 * w.T * w.H * w.D_shared
    return f
