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
