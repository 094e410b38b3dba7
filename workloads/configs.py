"""The five synthetic indexer workloads, as plain data.

Each workload is a decode (or prefill-chunk) step of one 4-layer LatentIndex
group.  Shapes follow the LatentIndex paper (arXiv 2610.04635): G = 4 layers
per group (Sec. 4.1 "Experimental setup"), up to 2048 selected tokens per query
(Sec. 4.1), an HS candidate budget B (Sec. 3.2 "Training-free LatentIndex",
Sec. C.4 "Hierarchical selection and decode indexer timing"), and the
DeepSeek-V3.2-like indexer width (64 heads of dimension 128, a 192-wide latent
= 128 NoPE + 64 RoPE, Sec. C.3 and Sec. D.2).

This module holds numbers only: no arithmetic of the method.
"""
from dataclasses import dataclass, field
from typing import Optional, Tuple


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    batch: int
    capacity: int            # cache rows per sequence
    length_range: Tuple[int, int]   # inclusive range of valid lengths (equal ends = fixed)
    group: int               # layers per group (G)
    heads: int               # indexer heads H
    d_k: int                 # indexer head dim
    d_c: int                 # shared latent dim
    k: int                   # final per-layer budget
    B: Optional[int]         # HS candidate budget (None: no HS in this workload)
    cache_dtype: str         # "f32" | "bf16" | "e4m3"
    seed: int
    planted_frac: float      # fraction of tokens planted with high affinity
    outlier_channels: int = 0     # latent channels multiplied by outlier_mult
    outlier_mult: float = 1.0
    layer_specific_frac: float = 0.0   # per layer, tokens planted along a direction only that layer favours
    d_model: int = 7168      # hidden width used for latent / key construction
    latent_from_hidden: bool = False   # True: c = W_down h is built by the append step
    queries: int = 1         # query tokens per sequence (1 = decode)
    paths: Tuple[str, ...] = ("full", "hs", "dsa")

    @property
    def decode(self) -> bool:
        return self.queries == 1

    def query_positions(self, length: int):
        """Causal positions of the query tokens: the last `queries` positions."""
        return list(range(length - self.queries, length))


WORKLOADS = [
    Workload(name="tiny-f32-n512", index=0, batch=1, capacity=512, length_range=(512, 512),
             group=4, heads=8, d_k=32, d_c=48, k=64, B=128, cache_dtype="f32", seed=0,
             planted_frac=0.02, d_model=96, latent_from_hidden=True),
    Workload(name="v32-decode-bf16-n8k", index=1, batch=1, capacity=8192,
             length_range=(8192, 8192), group=4, heads=64, d_k=128, d_c=192, k=2048, B=4096,
             cache_dtype="bf16", seed=1, planted_frac=0.01),
    Workload(name="batched-ragged-bf16-n32k", index=2, batch=8, capacity=32768,
             length_range=(16384, 32768), group=4, heads=64, d_k=128, d_c=192, k=2048, B=8192,
             cache_dtype="bf16", seed=2, planted_frac=0.01),
    Workload(name="long-e4m3-n128k", index=3, batch=4, capacity=131072,
             length_range=(131072, 131072), group=4, heads=64, d_k=128, d_c=192, k=2048,
             B=8192, cache_dtype="e4m3", seed=3, planted_frac=0.01, outlier_channels=1,
             outlier_mult=8.0),
    Workload(name="prefill-chunk-bf16-n64k", index=4, batch=1, capacity=65536,
             length_range=(65536, 65536), group=4, heads=32, d_k=128, d_c=256, k=2048, B=None,
             cache_dtype="bf16", seed=4, planted_frac=0.0, queries=1024, paths=("full",)),
]


def workload(i: int) -> Workload:
    return WORKLOADS[i]
