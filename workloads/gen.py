"""Seeded synthetic inputs for the indexer workloads.

Both the CUDA path (through the tests and the bench) and the CPU oracle read
their inputs from here, so this module does data synthesis only: Gaussian
draws, a rank-one "affinity" spike that makes a few tokens score high, and the
outlier channel of the fp8 workload.  It performs no scoring, absorption,
quantisation or selection.

Recipe (all draws from ``numpy.random.default_rng(seed)``, float32):

* sigma_c = 1/sqrt(d_model): the spread a latent c = W_down h has when h and
  W_down are N(0, 1/sqrt(d_model)) (std).  Workloads with
  ``latent_from_hidden`` draw h [b, cap, d_model] and W_down [d_c, d_model]
  instead and let the append step build c.
* Decoders W_K[l] = (G_l + sqrt(d_c) * v_l u^T) / sqrt(d_k), G_l ~ N(0, 1):
  Gaussian plus a rank-one spike that maps the latent direction u onto the
  key direction v_l.
* Optional layer-specific relevance (``layer_specific_frac``): each layer's
  decoder gains a second spike from its own direction u_l (orthogonal to u)
  to the key direction that u already reaches, and that fraction of each
  sequence's tokens is planted along u_l, relevant to layer l only.
* Head weights w[l] ~ N(0, 1/sqrt(H)) (std); queries
  q[l] = (g + 2 sign(w[l]) v_l) / sqrt(d_k), g ~ N(0, 1), so heads with
  positive weight lean toward +v_l and heads with negative weight toward -v_l.
* Planted tokens: ceil(p * len) positions per sequence, sampled without
  replacement, get c += 3 sigma_c sqrt(d_c) u (or h += 3 sigma_h sqrt(d_model)
  * unit(W_down^T u) when the latent is built from h).
* Outlier channels: ``outlier_channels`` latent channels, chosen by the seed,
  are multiplied by ``outlier_mult`` for every token (before any quantisation).
* Ragged lengths: integers uniform in ``length_range`` (inclusive).
* Prefill queries sit at the last ``queries`` positions of each sequence.
"""
from dataclasses import dataclass, replace
import math
from typing import List, Optional

import numpy as np

from .configs import Workload, workload


@dataclass
class Inputs:
    wl: Workload
    lengths: np.ndarray            # int32 [b]
    latent: Optional[np.ndarray]   # float32 [b, cap, d_c] (None when built from h)
    hidden: Optional[np.ndarray]   # float32 [b, cap, d_model] (latent_from_hidden only)
    W_down: Optional[np.ndarray]   # float32 [d_c, d_model]
    W_K: List[np.ndarray]          # per layer float32 [d_k, d_c]
    q: List[np.ndarray]            # per layer float32 [b, T, H, d_k]
    w: List[np.ndarray]            # per layer float32 [b, T, H]
    q_pos: Optional[np.ndarray]    # int32 [b, T] for prefill, None for decode
    planted: List[np.ndarray]      # per sequence int64 positions
    outlier_channels: np.ndarray   # int64 channel ids


def shrunk(wl: Workload, capacity: int, batch: Optional[int] = None,
           length_range=None, queries: Optional[int] = None) -> Workload:
    """Same distributions, smaller sizes (for oracle-sized parity cases)."""
    lr = length_range if length_range is not None else (
        (capacity, capacity) if wl.length_range[0] == wl.length_range[1]
        else (max(1, capacity // 2), capacity))
    return replace(wl, capacity=capacity, batch=batch or wl.batch, length_range=lr,
                   queries=queries or wl.queries,
                   k=min(wl.k, capacity), B=None if wl.B is None else min(wl.B, capacity))


def _unit(x: np.ndarray) -> np.ndarray:
    return (x / np.linalg.norm(x)).astype(np.float32)


def generate(wl, seed: Optional[int] = None) -> Inputs:
    if isinstance(wl, int):
        wl = workload(wl)
    rng = np.random.default_rng(wl.seed if seed is None else seed)
    b, cap, G, H, dk, dc, T = wl.batch, wl.capacity, wl.group, wl.heads, wl.d_k, wl.d_c, wl.queries
    lo, hi = wl.length_range
    if lo == hi:
        lengths = np.full(b, lo, dtype=np.int32)
    else:
        lengths = rng.integers(lo, hi + 1, size=b).astype(np.int32)

    u = _unit(rng.standard_normal(dc, dtype=np.float32))
    W_K, q, w = [], [], []
    for _ in range(G):
        v = _unit(rng.standard_normal(dk, dtype=np.float32))
        Gl = rng.standard_normal((dk, dc), dtype=np.float32)
        W_K.append(((Gl + math.sqrt(dc) * np.outer(v, u)) / math.sqrt(dk)).astype(np.float32))
        wl_ = (rng.standard_normal((b, T, H), dtype=np.float32) / math.sqrt(H)).astype(np.float32)
        g = rng.standard_normal((b, T, H, dk), dtype=np.float32)
        ql = (g + 2.0 * np.sign(wl_)[..., None] * v) / math.sqrt(dk)
        q.append(ql.astype(np.float32))
        w.append(wl_)

    planted = []
    for i in range(b):
        n_p = int(math.ceil(wl.planted_frac * int(lengths[i])))
        planted.append(np.sort(rng.choice(int(lengths[i]), size=n_p, replace=False)) if n_p else
                       np.zeros(0, dtype=np.int64))

    hidden = W_down = latent = None
    if wl.latent_from_hidden:
        dm = wl.d_model
        s = 1.0 / math.sqrt(dm)
        W_down = (rng.standard_normal((dc, dm), dtype=np.float32) * s).astype(np.float32)
        hidden = (rng.standard_normal((b, cap, dm), dtype=np.float32) * s).astype(np.float32)
        # unit(W_down^T u): the hidden-space direction that W_down maps closest to u.
        dirn = _unit(W_down.T.astype(np.float64) @ u.astype(np.float64))
        for i in range(b):
            hidden[i, planted[i], :] += np.float32(3.0 * s * math.sqrt(dm)) * dirn
    else:
        s = 1.0 / math.sqrt(wl.d_model)
        latent = rng.standard_normal((b, cap, dc), dtype=np.float32)
        latent *= np.float32(s)
        for i in range(b):
            latent[i, planted[i], :] += np.float32(3.0 * s * math.sqrt(dc)) * u

    outl = np.sort(rng.choice(dc, size=wl.outlier_channels, replace=False)) if wl.outlier_channels \
        else np.zeros(0, dtype=np.int64)
    if len(outl):
        if latent is not None:
            latent[:, :, outl] *= np.float32(wl.outlier_mult)
        # (workloads built from h carry no outlier channels)

    if wl.layer_specific_frac > 0 and latent is not None:
        # Layer-specific relevance: layer l's decoder also maps a direction
        # u_l (orthogonal to u) onto its key direction v_l, and a fraction of
        # tokens per sequence is planted along u_l, so they matter to layer l
        # only.  A separate stream keeps the other draws unchanged.
        rl = np.random.default_rng(wl.seed + 3000)
        s = 1.0 / math.sqrt(wl.d_model)
        for l in range(G):
            ul = rl.standard_normal(dc)
            ul = _unit(ul - (ul @ u) * u)
            # the key direction u already reaches (the queries lean toward it)
            v = _unit(W_K[l].astype(np.float64) @ u.astype(np.float64))
            W_K[l] = (W_K[l] + math.sqrt(dc) * np.outer(v, ul) / math.sqrt(dk)).astype(np.float32)
            for i in range(b):
                n_l = int(math.ceil(wl.layer_specific_frac * int(lengths[i])))
                idx = rl.choice(int(lengths[i]), size=n_l, replace=False)
                latent[i, idx, :] += np.float32(3.0 * s * math.sqrt(dc)) * ul

    q_pos = None
    if T > 1:
        q_pos = np.stack([np.arange(int(L) - T, int(L), dtype=np.int32) for L in lengths])
    return Inputs(wl=wl, lengths=lengths, latent=latent, hidden=hidden, W_down=W_down,
                  W_K=W_K, q=q, w=w, q_pos=q_pos, planted=planted, outlier_channels=outl)


def construction_inputs(wl: Workload, seed: Optional[int] = None):
    """Weights and one new hidden state per sequence for the per-step key /
    latent construction (decode step "with construction"): h_new [b, 1, d_model],
    W_down [d_c, d_model] and one DSA key projection W_k[l] [d_k, d_model] per
    layer, all N(0, 1/sqrt(d_model)) (std)."""
    rng = np.random.default_rng((wl.seed if seed is None else seed) + 1000)
    s = 1.0 / math.sqrt(wl.d_model)
    h_new = (rng.standard_normal((wl.batch, 1, wl.d_model), dtype=np.float32) * s)
    W_down = (rng.standard_normal((wl.d_c, wl.d_model), dtype=np.float32) * s)
    W_k = [(rng.standard_normal((wl.d_k, wl.d_model), dtype=np.float32) * s)
           for _ in range(wl.group)]
    return h_new.astype(np.float32), W_down.astype(np.float32), [x.astype(np.float32) for x in W_k]


@dataclass
class RopeInputs:
    """Parameters of a two-branch (RoPE + NoPE) latent and of layer decoders
    that are frequency-wise complex on the rotary branch.

    Layout (this build's reading of "RoPE64/NoPE128"): the latent row is
    [rotary rope_dim | NoPE norm_dim]; a layer's native key is
    [rotary 2F | NoPE d_k - 2F] with F = rope_dim / (2 sources) frequencies.
    Recipe: inv_freq[f] = base^(-f / F) with base 10000 (float32); LayerNorm
    gamma = 1 + 0.1 N(0, 1), beta = 0.1 N(0, 1), eps 1e-6; complex decoder
    coefficients d[l][f, j] with real and imaginary parts
    N(0, sqrt(d_model / (2 sources))) (std), which gives rotary key
    components of unit variance from latents of std 1/sqrt(d_model); NoPE
    decoders W_nope[l] ~ N(0, 1/sqrt(norm_dim)), biases b_nope[l] ~ 0.1 N(0, 1).
    The queries of the workload serve as post-RoPE queries."""
    rope_offset: int
    rope_dim: int
    sources: int
    inv_freq: np.ndarray          # float32 [F]
    norm_offset: int
    norm_dim: int
    gamma: np.ndarray             # float32 [norm_dim]
    beta: np.ndarray              # float32 [norm_dim]
    eps: float
    d_re: List[np.ndarray]        # per layer float32 [F, sources]
    d_im: List[np.ndarray]
    W_nope: List[np.ndarray]      # per layer float32 [d_k - 2F, norm_dim]
    b_nope: List[np.ndarray]      # per layer float32 [d_k - 2F]


def rope_inputs(wl: Workload, sources: int = 1, rope_dim: int = 64, seed: Optional[int] = None) -> RopeInputs:
    rng = np.random.default_rng((wl.seed if seed is None else seed) + 2000 + sources)
    F = rope_dim // (2 * sources)
    norm_dim = wl.d_c - rope_dim
    d_nope = wl.d_k - 2 * F
    inv_freq = (10000.0 ** (-np.arange(F, dtype=np.float64) / F)).astype(np.float32)
    gamma = (1.0 + 0.1 * rng.standard_normal(norm_dim)).astype(np.float32)
    beta = (0.1 * rng.standard_normal(norm_dim)).astype(np.float32)
    sd = math.sqrt(wl.d_model / (2.0 * sources))
    d_re, d_im, W_nope, b_nope = [], [], [], []
    for _ in range(wl.group):
        d_re.append((rng.standard_normal((F, sources)) * sd).astype(np.float32))
        d_im.append((rng.standard_normal((F, sources)) * sd).astype(np.float32))
        W_nope.append((rng.standard_normal((d_nope, norm_dim)) / math.sqrt(norm_dim)).astype(np.float32))
        b_nope.append((0.1 * rng.standard_normal(d_nope)).astype(np.float32))
    return RopeInputs(rope_offset=0, rope_dim=rope_dim, sources=sources, inv_freq=inv_freq,
                      norm_offset=rope_dim, norm_dim=norm_dim, gamma=gamma, beta=beta, eps=1e-6,
                      d_re=d_re, d_im=d_im, W_nope=W_nope, b_nope=b_nope)
