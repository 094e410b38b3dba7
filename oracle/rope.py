"""The RoPE-compatible two-branch latent, in plain float64.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Sources (LatentIndex, paperlayer summary of arXiv 2610.04635):

* Sec. 3.1: the anchor's hidden state gives a shared RoPE branch and a NoPE
  branch, concatenated and cached once per group; every layer reaches its
  effective key through its own decoder.
* Sec. A.2 "RoPE-compatible decoders": the rotary sources of each frequency
  share the native rotary phase, so the latent is rotated before caching
  and each layer's decoder is absorbed into its post-RoPE query.
* Sec. A.4 "Frequency-wise complex RoPE regression": each rotary frequency
  has its own complex sources (one per frequency, or two in GLM-5) and each
  layer a complex decoder coefficient per (frequency, source).
* Sec. A.3: NoPE decoders carry output biases.
* Sec. D.2: LayerNorm applies to the NoPE latent only; the RoPE part is used
  as it is.

Conventions of this build (the pages fix none of them): a rotary slot is a
pair of adjacent reals (x[2p], x[2p+1]) read as the complex number
x[2p] + i x[2p+1]; slot p of a segment with r sources per frequency belongs
to frequency p // r; a token at cache row s sits at position s and its slots
turn by the angle s * inv_freq[f] (multiplication by exp(i s inv_freq[f])).
LayerNorm uses the biased variance and eps inside the square root.
"""
from dataclasses import dataclass
from typing import Optional

import numpy as np

F64 = np.float64


def as_slots(x: np.ndarray) -> np.ndarray:
    """Adjacent real pairs of the last axis as complex numbers: [..., 2P] -> [..., P]."""
    x = np.asarray(x, F64)
    return x[..., 0::2] + 1j * x[..., 1::2]


def from_slots(z: np.ndarray) -> np.ndarray:
    """Inverse of as_slots: [..., P] complex -> [..., 2P] real."""
    out = np.empty(z.shape[:-1] + (2 * z.shape[-1],), F64)
    out[..., 0::2] = z.real
    out[..., 1::2] = z.imag
    return out


def rotate(x: np.ndarray, pos, inv_freq: np.ndarray, sources: int = 1) -> np.ndarray:
    """Rotary rotation of a segment: x [..., 2P] at positions pos (scalar, or
    one per leading row); slot p turns by pos * inv_freq[p // sources]."""
    z = as_slots(x)
    P = z.shape[-1]
    freq = np.asarray(inv_freq, F64)[np.arange(P) // sources]
    pos = np.asarray(pos, F64)
    angle = pos[..., None] * freq if pos.ndim else pos * freq
    return from_slots(z * np.exp(1j * angle))


def layer_norm(x: np.ndarray, gamma: Optional[np.ndarray] = None, beta: Optional[np.ndarray] = None,
               eps: float = 1e-6) -> np.ndarray:
    """(x - mean) / sqrt(var + eps) * gamma + beta over the last axis (biased var)."""
    x = np.asarray(x, F64)
    mean = x.mean(axis=-1, keepdims=True)
    var = ((x - mean) ** 2).mean(axis=-1, keepdims=True)
    y = (x - mean) / np.sqrt(var + eps)
    if gamma is not None:
        y = y * np.asarray(gamma, F64)
    if beta is not None:
        y = y + np.asarray(beta, F64)
    return y


@dataclass
class LatentFormat:
    """Where the two branches sit in a latent row of d_c elements."""
    rope_offset: int = 0
    rope_dim: int = 0                 # 0: no rotary branch
    sources: int = 1                  # complex sources per frequency
    inv_freq: Optional[np.ndarray] = None   # [rope_dim // (2 sources)] rad per position
    norm_offset: int = 0
    norm_dim: int = 0                 # 0: no LayerNorm
    gamma: Optional[np.ndarray] = None
    beta: Optional[np.ndarray] = None
    eps: float = 1e-6


def cache_rows(c: np.ndarray, positions: np.ndarray, fmt: LatentFormat) -> np.ndarray:
    """What the cache holds for latent rows c [n, d_c] at positions [n],
    before quantisation: the NoPE branch layer-normed, the RoPE branch
    rotated at each row's position, every other element as it is."""
    out = np.array(c, F64, copy=True)
    if fmt.norm_dim:
        a, b = fmt.norm_offset, fmt.norm_offset + fmt.norm_dim
        out[..., a:b] = layer_norm(out[..., a:b], fmt.gamma, fmt.beta, fmt.eps)
    if fmt.rope_dim:
        a, b = fmt.rope_offset, fmt.rope_offset + fmt.rope_dim
        out[..., a:b] = rotate(out[..., a:b], positions, fmt.inv_freq, fmt.sources)
    return out


def native_keys(c: np.ndarray, positions: np.ndarray, fmt: LatentFormat, d: np.ndarray,
                W_nope: np.ndarray, b_nope: Optional[np.ndarray]) -> np.ndarray:
    """A layer's own indexer keys, built the native way from the UNROTATED
    latent rows c [n, d_c]: per frequency f the complex decoder gives
    k_f = sum_j d[f, j] * z[f, j] from that frequency's sources z, and the key
    is then rotated at its position; the NoPE part is
    W_nope @ LayerNorm(c_nope) + b_nope.  Returns [n, 2F + d_nope] with the
    rotary part first, in the same adjacent-pair layout."""
    d = np.asarray(d, np.complex128)                    # [F, r]
    F, r = d.shape
    a = fmt.rope_offset
    z = as_slots(np.asarray(c, F64)[..., a:a + fmt.rope_dim]).reshape(c.shape[:-1] + (F, r))
    k_rope = from_slots((z * d).sum(axis=-1))
    k_rope = rotate(k_rope, positions, fmt.inv_freq, 1)
    nope = np.asarray(c, F64)[..., fmt.norm_offset:fmt.norm_offset + fmt.norm_dim]
    if fmt.norm_dim:
        nope = layer_norm(nope, fmt.gamma, fmt.beta, fmt.eps)
    k_nope = nope @ np.asarray(W_nope, F64).T
    if b_nope is not None:
        k_nope = k_nope + np.asarray(b_nope, F64)
    return np.concatenate([k_rope, k_nope], axis=-1)
