"""Selection-quality metrics and the IndexCache comparator, in plain float64.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Sources (LatentIndex, paperlayer summary of arXiv 2610.04635):

* Sec. 4.1 and Table 1: selectors are compared by attention-mass recall.
* Sec. D.3: Recall@2048 is the attention mass a selection captures relative
  to each head's own top-K set, K = min(2048, N) for a causal prefix of N
  positions, from each layer's dense attention distribution; Sec. C.2: it is
  averaged over heads.
* Sec. C.3: mean-attention recall asks whether one shared token set keeps the
  head-averaged attention mass, relative to the best shared set of size K.
* Sec. 1, Sec. 2 and Sec. D.3: IndexCache lets a follower reuse the anchor's
  top-k indices instead of selecting its own.

A selection is an int array of positions, -1 padded (the library's output).
Attention probabilities are [H, N] per query row, each head's row summing to
1 over the valid prefix.
"""
import numpy as np

F64 = np.float64


def _positions(sel) -> np.ndarray:
    sel = np.asarray(sel)
    return sel[sel >= 0]


def top_mass(p: np.ndarray, K: int) -> np.ndarray:
    """Sum of the K largest entries of each row of p [..., N] (K capped at N):
    the mass of the best size-K set for that row."""
    p = np.asarray(p, F64)
    K = min(K, p.shape[-1])
    if K <= 0:
        return np.zeros(p.shape[:-1])
    return -np.sort(-p, axis=-1)[..., :K].sum(axis=-1)


def head_mass_recall(p: np.ndarray, sel, K: int) -> np.ndarray:
    """Per-head recall [H] of a selection against attention p [H, N]: the
    selected mass of head h over the mass of head h's own top-K set."""
    p = np.asarray(p, F64)
    pos = _positions(sel)
    got = p[:, pos].sum(axis=1)
    best = top_mass(p, K)
    return np.where(best > 0, got / np.where(best > 0, best, 1.0), 0.0)


def mean_attention_recall(p: np.ndarray, sel, K: int) -> float:
    """Recall of a selection against the head-averaged attention of p [H, N],
    relative to the best shared set of size K for that average."""
    pbar = np.asarray(p, F64).mean(axis=0)
    best = top_mass(pbar, K)
    got = pbar[_positions(sel)].sum()
    return float(got / best) if best > 0 else 0.0


def index_cache_follower(anchor_sel) -> np.ndarray:
    """IndexCache: the follower's selection is the anchor's, unchanged."""
    return np.array(anchor_sel, copy=True)


def attention(logits: np.ndarray, n: int) -> np.ndarray:
    """Softmax over the first n positions of logits [H, >= n] (one row per
    head); the rest of the row gets probability 0."""
    x = np.asarray(logits, F64)[:, :n]
    x = x - x.max(axis=1, keepdims=True)
    e = np.exp(x)
    out = np.zeros(np.shape(logits), F64)
    out[:, :n] = e / e.sum(axis=1, keepdims=True)
    return out
