"""Closed-form counters of the LatentIndex summary.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

* Positions scored per query (Sec. 3.4 "Storage and computation", Sec. B.3
  "Computation with and without hierarchical selection"): a group of m layers
  scores m*L positions with full-prefix scoring and L + (m - 1) * min(B, L)
  with hierarchical selection.
* Logical indexer-cache bytes per token (Sec. B.1 "Cache storage and fixed
  parameters"): one fp8 key of d_k bytes plus a 4-byte fp32 scale per layer
  for native DSA; for LatentIndex one row per group, an fp8 latent of d_c bytes
  plus two 4-byte scales (one per NoPE / RoPE segment), with the independent
  first layer keeping a native key.
"""


def positions_scored_group(L: int, m: int, B: int = None) -> int:
    if B is None:
        return m * L
    return L + (m - 1) * min(B, L)


def positions_scored_model(L: int, groups, B: int = None, independent_layers: int = 1) -> int:
    """groups: list of group sizes; independent layers score the full prefix."""
    return independent_layers * L + sum(positions_scored_group(L, m, B) for m in groups)


def dsa_key_bytes(d_k: int = 128, scale_bytes: int = 4) -> int:
    return d_k + scale_bytes


def latent_row_bytes(d_c: int = 192, segments: int = 2, scale_bytes: int = 4) -> int:
    return d_c + segments * scale_bytes


def cache_bytes_per_token_dsa(layers: int, d_k: int = 128) -> int:
    return layers * dsa_key_bytes(d_k)


def cache_bytes_per_token_latent(groups: int, independent_layers: int = 1, d_k: int = 128,
                                 d_c: int = 192) -> int:
    return independent_layers * dsa_key_bytes(d_k) + groups * latent_row_bytes(d_c)
