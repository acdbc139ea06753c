"""Seeded synthetic inputs for S²-Attn.

This module only draws random numbers and names workload shapes. It holds none of
the method's arithmetic, so both the CUDA path and the CPU oracle can be fed from it.

Workloads are Llama2 attention-layer shapes (7B: 32 heads of dim 128; 70B: 64 query
heads over 8 key/value heads) at the context lengths and group sizes LongLoRA trains
with (group size G = N/4, the default in the LongLoRA summary page, §3.4 "Group size
ablation" / Table 7). The pages train on RedPajama and evaluate on PG19; neither the
datasets nor Llama2 weights are used here: Q, K, V and dO are i.i.d. N(0, 1) samples
rounded to bf16, standing in for projected activations.

Recipe: ``torch.Generator('cpu').manual_seed(seed)``, then ``randn`` fp32 for Q, K, V,
dO in that order, each rounded to bf16 (round-to-nearest-even). ``q_gain`` multiplies
Q before rounding (a "peaky" variant that stresses the running-max rescale).
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    G: int
    d: int
    seed: int

    @property
    def scale(self) -> float:
        return 1.0 / float(self.d) ** 0.5

    def describe(self) -> str:
        return (f"B={self.B} Hq={self.Hq} Hkv={self.Hkv} N={self.N} G={self.G} d={self.d}")


# The five workloads the path is checked and measured on.
WORKLOADS = {
    "small_h4_n256_g64_d64": Workload("small_h4_n256_g64_d64", 1, 4, 4, 256, 64, 64, 1000),
    "llama7b_n8192_g2048": Workload("llama7b_n8192_g2048", 1, 32, 32, 8192, 2048, 128, 1001),
    "llama7b_n32768_g8192": Workload("llama7b_n32768_g8192", 1, 32, 32, 32768, 8192, 128, 1002),
    "llama7b_b4_n8192_g2048": Workload("llama7b_b4_n8192_g2048", 4, 32, 32, 8192, 2048, 128, 1005),
    "llama7b_n102400_g25600": Workload("llama7b_n102400_g25600", 1, 32, 32, 102400, 25600, 128, 1003),
    "llama70b_gqa_n32768_g8192": Workload("llama70b_gqa_n32768_g8192", 1, 64, 8, 32768, 8192, 128, 1004),
}

# Workload the throughput metric is quoted on (Llama2-7B layer, N=8192, G=2048).
METRIC_WORKLOAD = "llama7b_n8192_g2048"


def make_inputs(B: int, Hq: int, Hkv: int, N: int, d: int, seed: int, q_gain: float = 1.0):
    """Return bf16 CPU tensors q [B,N,Hq,d], k [B,N,Hkv,d], v [B,N,Hkv,d], do [B,N,Hq,d]."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    q = torch.randn((B, N, Hq, d), generator=gen, dtype=torch.float32)
    k = torch.randn((B, N, Hkv, d), generator=gen, dtype=torch.float32)
    v = torch.randn((B, N, Hkv, d), generator=gen, dtype=torch.float32)
    do = torch.randn((B, N, Hq, d), generator=gen, dtype=torch.float32)
    if q_gain != 1.0:
        q = q * q_gain
    return (q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16),
            do.to(torch.bfloat16))


def make_workload_inputs(w: Workload, q_gain: float = 1.0):
    return make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed, q_gain)


def to_f64(x: torch.Tensor):
    """Widen a bf16 tensor to a float64 numpy array (exact)."""
    return x.to(torch.float64).numpy()
