"""Seeded synthetic attention workloads (shapes, seeds and input draws only).

This module holds no attention arithmetic.  It is the one piece shared by the
tests, the benchmark and the oracle-side checks: it only draws inputs.

Recipe (fixed so that every machine draws the same tensors): a CPU
``torch.Generator`` seeded with the workload's seed draws ``torch.randn``
float32 tensors of shape [B, H, N, d] in the order Q, K, V, dO; workloads with
``qk_std != 1`` multiply Q and K by it; all four are then rounded to bf16.
The oracle reads the same bf16 values upcast exactly to float64.
"""

from dataclasses import dataclass
import math

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    p_drop: float
    seed: int
    qk_std: float = 1.0
    backward: bool = True
    sample_rows: int = 0  # >0: check this many seeded query rows per head

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def fwd_flops(self) -> float:
        """4*B*H*N^2*d, halved when causal."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f

    def bwd_flops(self) -> float:
        return 2.5 * self.fwd_flops()

    def describe(self) -> str:
        return (f"B={self.B} H={self.H} N={self.N} d={self.d} "
                f"{'causal' if self.causal else 'non-causal'} p={self.p_drop} seed={self.seed}")


# The five synthetic workloads: single tile; short causal; d=128 causal with
# dropout; wide logit spread (Q, K ~ N(0, 4^2)); long context with dropout.
WORKLOADS = [
    Workload("single_tile_N128_d64", 1, 1, 128, 64, False, 0.0, 0, backward=False),
    Workload("causal_N1024_d64", 2, 8, 1024, 64, True, 0.0, 1),
    Workload("causal_dropout_N4096_d128", 4, 16, 4096, 128, True, 0.1, 2),
    Workload("causal_widelogits_N16384_d64", 2, 32, 16384, 64, True, 0.0, 3, qk_std=4.0),
    Workload("causal_dropout_N32768_d128", 1, 32, 32768, 128, True, 0.1, 4, sample_rows=256),
]

BY_NAME = {w.name: w for w in WORKLOADS}


def draw_inputs(w: Workload, B=None, H=None, N=None, dtype=torch.bfloat16):
    """(Q, K, V, dO) as CPU tensors [B, H, N, d] drawn by the recipe above,
    rounded to ``dtype`` (bf16 unless asked for fp16).

    B, H, N may be overridden to draw a reduced case with the same recipe.
    """
    B = w.B if B is None else B
    H = w.H if H is None else H
    N = w.N if N is None else N
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    shape = (B, H, N, w.d)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    do = torch.randn(shape, generator=g, dtype=torch.float32)
    if w.qk_std != 1.0:
        q = q * w.qk_std
        k = k * w.qk_std
    return tuple(x.to(dtype) for x in (q, k, v, do))


def sample_rows(w: Workload, n_rows=None, B=None, H=None, N=None):
    """Seeded query-row sample per (b, h): list indexed [b][h] of int64 index tensors (sorted)."""
    B = w.B if B is None else B
    H = w.H if H is None else H
    N = w.N if N is None else N
    n_rows = w.sample_rows if n_rows is None else n_rows
    g = torch.Generator(device="cpu").manual_seed(w.seed + 1000)
    out = []
    for _b in range(B):
        row = []
        for _h in range(H):
            idx = torch.randperm(N, generator=g)[:n_rows]
            row.append(torch.sort(idx).values)
        out.append(row)
    return out


def to_f64(x: torch.Tensor):
    """Exact upcast of a bf16 tensor to a float64 NumPy array."""
    return x.to(torch.float64).numpy()
