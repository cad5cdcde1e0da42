"""The five synthetic decode workloads, by name.

Each stands in for a setting the pages discuss (the sparse decode kernel's 50x
and 500x sparsity points, HyLRA's layer reuse, 128-token blocks with a per-layer
full/sparse route); the pages' own evaluation suites are not used.  Shapes only:
tensors come from :mod:`inputs`.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

# route codes (also the C-ABI's mode values)
FULL, SELECT, REUSE = 0, 1, 2


@dataclass
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    Ncap: int
    d: int = 128
    k: int | None = None  # fixed k (tokens or blocks) per sequence
    k_div: int | None = None  # k_b = ceil(len_b / k_div) when k is None
    lens: tuple | None = None  # (lo, hi) ragged lengths, else every len = Ncap
    plant_frac: float = 0.0
    layers: int = 1
    route: tuple = (SELECT,)  # per layer
    reuse_from: tuple = (-1,)  # per layer: source layer of a REUSE layer
    block: int = 1  # 1 = token mode, 128 = block mode
    q_drift: float = 0.0  # q_{l+1} = bf16(q_l + q_drift * N(0,1)); 0 = fresh Q per layer
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def k_per_seq(self, lens) -> list:
        out = []
        for n in lens:
            if self.k is not None:
                out.append(int(self.k))
            else:
                out.append(int(math.ceil(int(n) / self.k_div)))
        return out


TINY = Workload("tiny sparse decode (B=1, 8/2 heads, N=4096, k=128)", B=1, Hq=8, Hkv=2, Ncap=4096,
                k=128, plant_frac=0.01)

LLAMA8B = Workload("Llama-3.1-8B-shaped decode layer (B=8, 32/8 heads, N=32768, k=655)", B=8, Hq=32,
                   Hkv=8, Ncap=32768, k=655, plant_frac=0.01)

REUSE128K = Workload("long-context index reuse (B=1, 32/8 heads, N=131072, k=2621, 4 layers)", B=1,
                     Hq=32, Hkv=8, Ncap=131072, k=2621, layers=4,
                     route=(SELECT, REUSE, REUSE, REUSE), reuse_from=(-1, 0, 0, 0), q_drift=0.3)

LARGE_BATCH = Workload("large-batch 500x sparsity (B=64, 64/8 heads, ragged N in [8192,32768])", B=64,
                       Hq=64, Hkv=8, Ncap=32768, k_div=500, lens=(8192, 32768), plant_frac=0.002)

HYBRID = Workload("hybrid routed block stack (B=2, 8 layers, 32/8 heads, N=262144, top 32 blocks)",
                  B=2, Hq=32, Hkv=8, Ncap=262144, k=32, plant_frac=0.01, layers=8, block=128,
                  route=(FULL, FULL, SELECT, REUSE, SELECT, REUSE, SELECT, REUSE),
                  reuse_from=(-1, -1, -1, 2, -1, 4, -1, 6))

ALL = {"tiny": TINY, "llama8b": LLAMA8B, "reuse128k": REUSE128K, "large_batch": LARGE_BATCH,
       "hybrid": HYBRID}
