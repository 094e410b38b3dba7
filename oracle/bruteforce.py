"""Pure-Python brute force of the indexer for tiny inputs.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

It takes the long way on purpose, so that it shares no arithmetic route with
oracle/indexer.py: every layer's key is reconstructed explicitly from the
shared latent with the layer's decoder (k_s = W_K c_s + b, LatentIndex summary,
Sec. 3.1 and Sec. A.3), scores are explicit dot products of the raw query with
that key, and selection is a full ``sorted`` of (-score, position) pairs.
Inputs are nested Python lists (or anything indexable) of floats.
"""


def reconstruct_key(W_K, c, b=None):
    d_k, d_c = len(W_K), len(W_K[0])
    out = []
    for j in range(d_k):
        acc = 0.0
        for i in range(d_c):
            acc += float(W_K[j][i]) * float(c[i])
        if b is not None:
            acc += float(b[j])
        out.append(acc)
    return out


def head_score(q_heads, w, key):
    """sum_h w_h * max(0, q_h . key)."""
    total = 0.0
    for h in range(len(q_heads)):
        dot = 0.0
        for j in range(len(key)):
            dot += float(q_heads[h][j]) * float(key[j])
        total += float(w[h]) * (dot if dot > 0.0 else 0.0)
    return total


def layer_scores(latent_rows, W_K, q_heads, w, b=None):
    """Scores of one layer over the rows, by explicit key reconstruction."""
    return [head_score(q_heads, w, reconstruct_key(W_K, c, b)) for c in latent_rows]


def select(scores, k):
    """Top-min(k, n) by (score desc, position asc), ascending positions, -1 pad."""
    n = len(scores)
    ranked = sorted(range(n), key=lambda s: (-scores[s], s))
    keep = sorted(ranked[: min(k, n)])
    return keep + [-1] * (k - len(keep))


def hs(latent_rows, layers, B, k):
    """Hierarchical selection for one group.  layers = [(W_K, q_heads, w), ...];
    the first entry is the anchor.  Returns (candidates, [selection per layer])."""
    W0, q0, w0 = layers[0]
    s0 = layer_scores(latent_rows, W0, q0, w0)
    cand = [c for c in select(s0, B) if c >= 0]
    sels = [select(s0, k)]
    for W, q, w in layers[1:]:
        cs = [head_score(q, w, reconstruct_key(W, latent_rows[t])) for t in cand]
        pos = [p for p in select(cs, k) if p >= 0]
        toks = sorted(cand[p] for p in pos)
        sels.append(toks + [-1] * (k - len(toks)))
    return cand + [-1] * (B - len(cand)), sels
