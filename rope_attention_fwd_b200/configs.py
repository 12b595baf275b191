"""The five synthetic RoPE-attention workloads, as plain data.

Each workload fixes the shape [B, H, n, d], the storage dtype, the causal flag,
the RoPE base b, the distribution of Q, K, V, E and the distribution of the
LeRoPE log-frequency offsets alpha (one per band, d/2 of them, shared by all
heads).  Nothing here computes any part of the attention; the draw itself is
in :mod:`rope_attention_fwd_b200.inputs`.

Shapes echo the pages' own setting where they give one: head dimension 64 and
sequence length 2048 come from the LeRoPE paper's experimental setup
("LeRoPE: learnable RoPE frequencies", Experimental configuration); base
10000 is the standard RoPE baseline named there.  The public corpora the pages
train on (C4, StarCoder-Python) are replaced by seeded Gaussian / uniform
tensors of the same shapes.
"""
from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    n: int
    d: int
    dtype: str          # "f32" or "bf16": storage and MMA operand type
    causal: bool
    base: float
    qkve: str           # "normal" -> N(0,1); "uniform" -> U[lo, hi]
    lo: float = -1.0
    hi: float = 1.0
    alpha: str = "zero"  # "zero" | "normal" | "uniform"
    alpha_a: float = 0.0  # normal: std; uniform: low end
    alpha_b: float = 0.0  # uniform: high end
    seed: int = 1000

    @property
    def M(self) -> int:
        return self.d // 2

    def flops_fwd(self) -> float:
        """4 n^2 d per (b, h); half when causal."""
        f = 4.0 * self.B * self.H * self.n * self.n * self.d
        return f / 2 if self.causal else f

    def flops_bwd(self) -> float:
        """10 n^2 d per (b, h) (S, dP, dV, dK, dQ); half when causal."""
        f = 10.0 * self.B * self.H * self.n * self.n * self.d
        return f / 2 if self.causal else f

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    1: Workload("tiny exact 1x1x256x64 fp32 non-causal", 1, 1, 256, 64, "f32", False, 1e4,
                "uniform", -1.0, 1.0, "zero", seed=1001),
    2: Workload("4x16x2048x64 bf16 causal", 4, 16, 2048, 64, "bf16", True, 1e4,
                "normal", alpha="normal", alpha_a=0.5, seed=1002),
    3: Workload("2x32x8192x128 bf16 causal", 2, 32, 8192, 128, "bf16", True, 1e4,
                "normal", alpha="normal", alpha_a=0.3, seed=1003),
    4: Workload("bounded-entry 1x8x32768x128 bf16 non-causal", 1, 8, 32768, 128, "bf16", False, 5e5,
                "uniform", -3.0, 3.0, "zero", seed=1004),
    5: Workload("spread-frequency 8x16x4096x128 bf16 causal", 8, 16, 4096, 128, "bf16", True, 5e5,
                "normal", alpha="uniform", alpha_a=-6.907755278982137, alpha_b=1.3862943611198906,
                seed=1005),
}

HEADLINE = 3
