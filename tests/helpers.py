"""Comparison rules shared by the parity tests.

Score tolerance: a GPU score s_hat of token s passes when
    |s_hat - s_ref| <= rtol * M_s,   M_s = sum_h |w_h| sum_i |qt_{h,i}| |c_{s,i}|
(the a-priori error magnitude of a sum of products).  rtol = 2e-3 for bf16
and fp32 (tf32 tensor cores) caches, 3e-2 for e4m3 caches.

Selection rule: both selections hold k_eff = min(k, n) positions; every
position in their symmetric difference must have an oracle score within
rtol * max(M_s, M_kth) of the oracle's k_eff-th score.
"""
import numpy as np

from oracle import indexer

RTOL = {"f32": 2e-3, "bf16": 2e-3, "e4m3": 3e-2}


def score_errors(gpu: np.ndarray, ref: np.ndarray, M: np.ndarray):
    """Normalised errors |gpu - ref| / M (M > 0)."""
    return np.abs(gpu.astype(np.float64) - ref) / np.maximum(M, 1e-300)


def assert_scores_close(gpu, ref, M, rtol, what=""):
    err = score_errors(gpu, ref, M)
    worst = int(np.argmax(err)) if err.size else 0
    assert err.size == 0 or err.max() <= rtol, (
        f"{what}: max normalised error {err.max():.3e} > {rtol} at {worst} "
        f"(gpu {gpu[worst]!r}, ref {ref[worst]!r}, M {M[worst]!r})")
    return float(err.max()) if err.size else 0.0


def assert_selection_close(gpu_idx, ref_scores, M, k, n, rtol, what=""):
    """gpu_idx: [k] int32 ascending, -1 padded.  ref_scores / M: oracle scores
    and error scales over the n valid positions."""
    keff = min(k, n)
    gpu_idx = np.asarray(gpu_idx)
    sel = gpu_idx[gpu_idx >= 0]
    assert len(sel) == keff, f"{what}: {len(sel)} selected, expected {keff}"
    assert np.all(gpu_idx[keff:] == -1), f"{what}: padding is not -1"
    assert np.all(np.diff(sel) > 0), f"{what}: output not strictly ascending"
    assert sel.min(initial=0) >= 0 and (len(sel) == 0 or sel.max() < n), f"{what}: index out of range"
    ref_idx, _ = indexer.topk(ref_scores, k, n)
    ref_sel = ref_idx[ref_idx >= 0]
    diff = np.setxor1d(sel, ref_sel)
    if len(diff) == 0:
        return 0
    kth = indexer.kth_score(ref_scores, k, n)
    kth_pos = ref_sel[np.argmin(ref_scores[ref_sel])] if len(ref_sel) else 0
    tol = rtol * np.maximum(M[diff], M[kth_pos])
    gap = np.abs(ref_scores[diff] - kth)
    bad = diff[gap > tol]
    assert len(bad) == 0, (f"{what}: {len(bad)} of {len(diff)} differing positions are not near the boundary; "
                           f"first {bad[:5]}, gap {gap[gap > tol][:5]}, tol {tol[gap > tol][:5]}")
    return len(diff)


# ------------------------------------------------------------------ two-branch (RoPE + NoPE) latent

def latent_format(ri):
    """The oracle's LatentFormat for generated RopeInputs."""
    from oracle.rope import LatentFormat
    return LatentFormat(rope_offset=ri.rope_offset, rope_dim=ri.rope_dim, sources=ri.sources,
                        inv_freq=ri.inv_freq, norm_offset=ri.norm_offset, norm_dim=ri.norm_dim,
                        gamma=ri.gamma, beta=ri.beta, eps=ri.eps)


def rope_decoder_matrix(ri, layer: int, d_k: int, d_c: int):
    """Layer `layer`'s decoder as one real matrix W [d_k, d_c] (key = W c) plus
    its bias [d_k], the form the absorption entry point takes.  Native key
    slot f (reals 2f, 2f+1) gets sum_j d[f, j] * latent slot (f, j): the
    complex product (a + ib)(x + iy) is the real block [[a, -b], [b, a]]
    acting on (x, y).  The NoPE rows take W_nope on the NoPE columns."""
    F, r = ri.d_re[layer].shape
    W = np.zeros((d_k, d_c), np.float32)
    for f in range(F):
        for j in range(r):
            a, b = ri.d_re[layer][f, j], ri.d_im[layer][f, j]
            col = ri.rope_offset + 2 * (f * r + j)
            W[2 * f, col], W[2 * f, col + 1] = a, -b
            W[2 * f + 1, col], W[2 * f + 1, col + 1] = b, a
    d_nope = d_k - 2 * F
    W[2 * F:, ri.norm_offset:ri.norm_offset + ri.norm_dim] = ri.W_nope[layer]
    bias = np.zeros(d_k, np.float32)
    bias[2 * F:] = ri.b_nope[layer]
    assert ri.W_nope[layer].shape == (d_nope, ri.norm_dim)
    return W, bias
