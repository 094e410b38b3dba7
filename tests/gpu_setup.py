"""Put a generated workload on the GPU through the library's own entry points,
and compute the oracle's reference for it.  Used by the GPU tests and smoke()."""
import numpy as np
import torch

import cross_layer_latent_b200 as li
from oracle import indexer
from workloads import Inputs

DTYPE = {"f32": li.LI_F32, "bf16": li.LI_BF16, "e4m3": li.LI_E4M3}


def build_group(ctx, inp: Inputs, dsa: bool = True, device="cuda:0") -> li.GroupIndexer:
    wl = inp.wl
    g = li.GroupIndexer(ctx, batch=wl.batch, capacity=wl.capacity, d_c=wl.d_c, H=wl.heads, d_k=wl.d_k, G=wl.group,
                        dtype=DTYPE[wl.cache_dtype], k=wl.k, B=wl.B, T=wl.queries, dsa=dsa, device=device)
    g.load(inp.lengths, inp.W_K, inp.q, inp.w, latent=inp.latent, hidden=inp.hidden, W_down=inp.W_down,
           q_pos=inp.q_pos)
    torch.cuda.synchronize()
    return g


def ref_latent(inp: Inputs) -> np.ndarray:
    if inp.hidden is not None:
        return indexer.latent(inp.hidden, inp.W_down)
    return inp.latent.astype(np.float64)


class Reference:
    """Oracle scores and error scales of one layer for one (sequence, query) row."""

    def __init__(self, inp: Inputs, c64: np.ndarray, layer: int, b: int, t: int = 0):
        self.n = indexer.valid_length(inp.lengths[b], None if inp.q_pos is None else inp.q_pos[b, t])
        qt, _ = indexer.absorb(inp.q[layer][b, t], inp.W_K[layer])
        w = inp.w[layer][b, t]
        rows = c64[b, : self.n]
        self.qt = qt
        self.scores = indexer.score(rows, qt, w)
        self.M = indexer.error_scale(rows, qt, w)
        self.dsa_scores = indexer.dsa_score(rows, inp.W_K[layer], inp.q[layer][b, t], w)
        keys = rows @ inp.W_K[layer].astype(np.float64).T
        self.dsa_M = indexer.error_scale(keys, inp.q[layer][b, t], w)
