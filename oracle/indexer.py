"""Plain float64 definition of what the LatentIndex decode indexer computes.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Sources (LatentIndex: Cross-Layer Sharing with Layer-Specific Selection for
Sparse Attention, paperlayer summary of arXiv 2610.04635):

* Sec. 3.1 "Shared key representations with layer-specific indexers": each
  group's anchor builds one shared latent c_s from its hidden state; every
  layer l of the group decodes it with its own decoder; at inference the
  decoder is absorbed into the query, which is exact in exact arithmetic.
* Sec. 3.2 "Training-free LatentIndex" and Sec. C.4 "Hierarchical selection
  and decode indexer timing": in HS the anchor scores the whole prefix and
  proposes the top-B candidates; each follower rescores only those and picks
  its own top-k; budgets are capped by the valid prefix length.
* Sec. A.3 "Joint NoPE regression": decoders may carry output biases.
* The head-weighted ReLU scoring form is not printed on the pages; this build
  fixes it as score(t, s) = sum_h w_{t,h} * max(0, qt_{t,h} . c_s (+ beta_{t,h}))
  with qt_{t,h} = W_K^T q_{t,h}, the DSA-style form of the workload definition.

Conventions: a decoder W_K is stored [d_k, d_c] (key = W_K c); queries are
[..., H, d_k]; a selection is the k_eff = min(k, n) best positions by
(score descending, position ascending), returned in ascending position order
and padded with -1.
"""
import numpy as np

F64 = np.float64


# ------------------------------------------------------------------ construction (a1)

def latent(h: np.ndarray, W_down: np.ndarray) -> np.ndarray:
    """c = W_down h for every token: h [..., d_model], W_down [d_c, d_model]."""
    return np.asarray(h, F64) @ np.asarray(W_down, F64).T


# ------------------------------------------------------------------ absorption (a2)

def absorb(q: np.ndarray, W_K: np.ndarray, b_K: np.ndarray = None):
    """Absorbed query qt = W_K^T q and bias term beta = q . b_K.

    q [..., H, d_k]; W_K [d_k, d_c] shared by all heads or [H, d_k, d_c] per
    head; b_K None, [d_k] or [H, d_k].  Returns (qt [..., H, d_c], beta [..., H]
    or None)."""
    q = np.asarray(q, F64)
    W = np.asarray(W_K, F64)
    if W.ndim == 2:
        qt = np.einsum("...hk,kc->...hc", q, W)
    else:
        qt = np.einsum("...hk,hkc->...hc", q, W)
    beta = None
    if b_K is not None:
        b = np.asarray(b_K, F64)
        beta = np.einsum("...hk,k->...h", q, b) if b.ndim == 1 else np.einsum("...hk,hk->...h", q, b)
    return qt, beta


# ------------------------------------------------------------------ scoring (a3, a7)

def score(c_rows: np.ndarray, qt: np.ndarray, w: np.ndarray, beta: np.ndarray = None) -> np.ndarray:
    """score[s] = sum_h w_h * max(0, qt_h . c_s + beta_h) for the rows c_rows [n, d]."""
    pre = np.asarray(c_rows, F64) @ np.asarray(qt, F64).T          # [n, H]
    if beta is not None:
        pre = pre + np.asarray(beta, F64)[None, :]
    return np.maximum(pre, 0.0) @ np.asarray(w, F64)


def error_scale(c_rows: np.ndarray, qt: np.ndarray, w: np.ndarray) -> np.ndarray:
    """M_s = sum_h |w_h| sum_i |qt_{h,i}| |c_{s,i}|: the a-priori magnitude of the
    rounding error of a sum of products (Higham), used to normalise score errors."""
    return (np.abs(np.asarray(c_rows, F64)) @ np.abs(np.asarray(qt, F64)).T) @ np.abs(np.asarray(w, F64))


def dsa_score(c_rows: np.ndarray, W_K: np.ndarray, q: np.ndarray, w: np.ndarray) -> np.ndarray:
    """DSA-style per-layer path: reconstruct every key k_s = W_K c_s explicitly,
    then score[s] = sum_h w_h * max(0, q_h . k_s)."""
    keys = np.asarray(c_rows, F64) @ np.asarray(W_K, F64).T          # [n, d_k]
    return np.maximum(keys @ np.asarray(q, F64).T, 0.0) @ np.asarray(w, F64)


def dsa_score_keys(key_rows: np.ndarray, q: np.ndarray, w: np.ndarray) -> np.ndarray:
    """DSA-style scoring of already-materialised keys [n, d_k]."""
    return np.maximum(np.asarray(key_rows, F64) @ np.asarray(q, F64).T, 0.0) @ np.asarray(w, F64)


# ------------------------------------------------------------------ selection (a4)

def valid_length(length: int, q_pos: int = None) -> int:
    """Positions a query may attend: [0, length) in decode (the current token is
    appended before scoring), [0, q_pos] for a prefill query at position q_pos."""
    return int(length) if q_pos is None else min(int(length), int(q_pos) + 1)


def topk(scores: np.ndarray, k: int, n: int = None):
    """Top k_eff = min(k, n) of scores[:n] by (score desc, position asc).

    Returns (idx int32 [k] ascending then -1, vals [k] matching, -inf pad)."""
    s = np.asarray(scores)[: (len(scores) if n is None else n)]
    assert not np.any(np.isnan(s)), "NaN scores are invalid input"
    n = len(s)
    keff = min(int(k), n)
    order = np.lexsort((np.arange(n), -s.astype(F64)))
    sel = np.sort(order[:keff])
    idx = np.full(k, -1, dtype=np.int32)
    idx[:keff] = sel
    vals = np.full(k, -np.inf, dtype=F64)
    vals[:keff] = s[sel]
    return idx, vals


def kth_score(scores: np.ndarray, k: int, n: int = None) -> float:
    """The k_eff-th best score of scores[:n] (the selection boundary)."""
    s = np.asarray(scores, F64)[: (len(scores) if n is None else n)]
    keff = min(int(k), len(s))
    if keff == 0:
        return np.inf
    return float(np.sort(s)[::-1][keff - 1])


# ------------------------------------------------------------------ hierarchical selection (a5, a6)

def hs_anchor(scores: np.ndarray, B: int, k: int, n: int = None):
    """Anchor step: candidates = top-min(B, n) of the full prefix; the anchor's
    own selection = top-min(k, n) of the same scores.

    Returns (cand int32 [B] ascending, -1 pad; cand_n; anchor_idx [k])."""
    n = len(scores) if n is None else n
    cand, _ = topk(scores, B, n)
    anchor_idx, _ = topk(scores, k, n)
    return cand, min(int(B), int(n)), anchor_idx


def hs_follower(cand_scores: np.ndarray, cand: np.ndarray, cand_n: int, k: int):
    """Follower step: scores of the candidates only (cand_scores[j] belongs to
    token cand[j], cand ascending); select top-min(k, cand_n) by (score desc,
    token asc) and return token indices ascending, -1 padded."""
    pos, vals = topk(np.asarray(cand_scores)[:cand_n], k, cand_n)
    out = np.full(k, -1, dtype=np.int32)
    m = pos >= 0
    out[m] = np.asarray(cand)[pos[m]]
    return out, vals
