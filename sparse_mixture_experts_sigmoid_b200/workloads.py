"""The layer shapes this library is measured and checked on.

Each workload is a top-k routed MoE SwiGLU FFN layer shape with the input
recipe used to synthesise it (all inputs are seeded and synthetic; no model
weights or datasets are read).  The shapes stand in for the models that the
source pages discuss:

* ``tiny`` -- a small fp32 case that the float64 oracle checks in full.
* ``gemma_upcycle`` -- Gemma-3-270M drop-upcycled to 256 experts, top-4,
  softmax over the four kept scores ("Small models, sparse experts", section
  "How it works", steps 1-3).
* ``olmoe_zipf`` -- OLMoE-like fine-grained layer, 64 experts, top-8, no
  renormalisation, router skewed so expert loads follow a Zipf(1.1) spread
  ("Small MoE Architecture, in depth", section "How small MoEs are actually
  shaped").
* ``qwen_shared`` -- Qwen-style layer, 60 experts top-4 plus an always-on
  shared SwiGLU expert gated by sigmoid(w_s . x) (same section).
* ``mixtral_prefill`` / ``mixtral_decode`` -- Mixtral-like coarse layer, 8
  experts of width 14336, top-2 renormalised; decode is one token, for which
  only the two chosen experts' weights are read ("Small MoE Architecture, in
  depth", section "Why small changes the MoE trade-off").
"""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    E: int
    h: int
    k: int
    score: str = "softmax"          # "softmax" | "sigmoid"
    norm_topk: bool = True
    h_shared: int = 0
    dtype: str = "bf16"             # "bf16" | "f32"
    recipe: str = "normal"          # "normal" | "upcycle" | "zipf"
    x_std: float = 1.0
    router_std: float = 0.02
    weight_std: float = 0.02
    seed: int = 1
    # drop-upcycle recipe
    up_slices: int = 4
    up_copies: int = 64
    up_redraw: float = 0.10
    up_scale: float = 4.0           # 64 ** (1/3), exactly 4
    # Zipf router skew
    zipf_a: float = 1.1

    @property
    def R(self) -> int:
        """Number of (token, expert) assignments, T * k."""
        return self.T * self.k

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    # ---- algorithmic work (padding and tile waste excluded) ----
    def flops(self) -> float:
        f = 2.0 * self.T * self.k * 3 * self.d * self.h + 2.0 * self.T * self.E * self.d
        if self.h_shared:
            f += 2.0 * self.T * 3 * self.d * self.h_shared + 2.0 * self.T * self.d
        return f

    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2


WORKLOADS: dict[str, Workload] = {
    "tiny": Workload("tiny", T=64, d=64, E=8, h=128, k=2, dtype="f32", seed=1),
    "gemma_upcycle": Workload("gemma_upcycle", T=2048, d=640, E=256, h=512, k=4,
                              recipe="upcycle", router_std=0.01, seed=2),
    "olmoe_zipf": Workload("olmoe_zipf", T=8192, d=2048, E=64, h=1024, k=8, norm_topk=False,
                           recipe="zipf", seed=3),
    "qwen_shared": Workload("qwen_shared", T=4096, d=2048, E=60, h=1408, k=4, norm_topk=False,
                            h_shared=5632, seed=4),
    "mixtral_prefill": Workload("mixtral_prefill", T=4096, d=4096, E=8, h=14336, k=2, seed=5),
    "mixtral_decode": Workload("mixtral_decode", T=1, d=4096, E=8, h=14336, k=2, seed=5),
    # small case of the Mixtral-like expert shape (2 experts, 0.7 GB of weights) for
    # full profiler captures, which must stay a few GB on the device
    "mixtral_e2_profile": Workload("mixtral_e2_profile", T=2048, d=4096, E=2, h=14336, k=2, seed=6),
    # small case of the OLMoE-like expert shape (a quarter of the tokens, half the
    # experts: 0.4 GB of weights) for full profiler
    # captures of the training step's kernels
    "olmoe_profile": Workload("olmoe_profile", T=2048, d=2048, E=32, h=1024, k=8, norm_topk=False, seed=7),
}

# The workload that the headline benchmark line is quoted on: the largest
# layer that fits one GPU (the Mixtral-like prefill, 22.5 GB of expert weights).
HEADLINE = "mixtral_prefill"

# The layer shapes reported side by side in every benchmark line.
REPORTED = ("tiny", "gemma_upcycle", "olmoe_zipf", "qwen_shared", "mixtral_prefill", "mixtral_decode")
