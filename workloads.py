"""Named S2-Attn workloads (synthetic stand-ins for the pages' LLaMA2 long-context runs).

Each entry gives the shape, dtype, RoPE/PI settings and the input recipe: q, k, v iid
N(0,1) * scale and dO iid N(0,1), drawn by ``synth`` with seed = the workload's seed.
The LLaMA2 shapes follow the pages' context-extension settings (7B at 8k, 32k and ~100k
tokens, 70B at 32k; group size G = N/4; PI scale s = N / 4096).
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    N: int
    Hq: int
    Hkv: int
    d: int
    G: int
    pi_scale: float
    dtype: str          # "bf16" or "f32"
    in_scale: float     # q, k, v = N(0,1) * in_scale
    backward: bool      # the workload includes the backward pass
    seed: int
    causal: bool = True
    rope_base: float = 10000.0
    shift: str = "half"  # shifted heads: "half", "alternate" (odd kv heads) or "none"


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny_fp32", 1, 256, 4, 4, 64, 64, 2.0, "f32", 1.0, True, 0),
        Workload("llama2_7b_8k_fwd", 1, 8192, 32, 32, 128, 2048, 2.0, "bf16", 0.5, False, 1),
        Workload("llama2_7b_32k", 1, 32768, 32, 32, 128, 8192, 8.0, "bf16", 0.5, True, 2),
        Workload("llama2_7b_100k", 1, 102400, 32, 32, 128, 25600, 25.0, "bf16", 0.5, True, 3),
        Workload("llama2_70b_gqa_32k", 1, 32768, 64, 8, 128, 8192, 8.0, "bf16", 0.5, True, 4),
        # a smaller case of the same shape family for ncu captures (q is 134 MB > L2)
        Workload("llama2_7b_16k", 1, 16384, 32, 32, 128, 4096, 4.0, "bf16", 0.5, True, 5),
        # variants of the 7B-32k step: no mask inside the groups (the full-group reading);
        # odd kv heads shifted instead of the second half; RoPE base scaled by the extension
        # ratio instead of interpolated positions (base 10000 * 8, s = 1)
        Workload("llama2_7b_32k_noncausal", 1, 32768, 32, 32, 128, 8192, 8.0, "bf16", 0.5,
                 True, 6, causal=False),
        Workload("llama2_7b_32k_alternate", 1, 32768, 32, 32, 128, 8192, 8.0, "bf16", 0.5,
                 True, 7, shift="alternate"),
        Workload("llama2_7b_32k_base_scaled", 1, 32768, 32, 32, 128, 8192, 1.0, "bf16", 0.5,
                 True, 8, rope_base=80000.0),
        # inference at the extended length: one group of all 32k tokens, no shift, i.e.
        # dense causal attention, forward only
        Workload("llama2_7b_32k_dense_infer", 1, 32768, 32, 32, 128, 32768, 8.0, "bf16", 0.5,
                 False, 9, shift="none"),
    ]
}

# The workload the headline throughput is measured on.
HEADLINE = "llama2_7b_32k"
