"""The pins must catch a plausible mistake in the oracle: each case plants one
mistake (in the oracle, on the CPU) and checks that some pin then fails."""
import numpy as np
import pytest

import oracle.indexer as ix
from tests import test_oracle as pins


def _dropped_relu(c_rows, qt, w, beta=None):
    pre = np.asarray(c_rows, float) @ np.asarray(qt, float).T
    if beta is not None:
        pre = pre + beta
    return pre @ np.asarray(w, float)


def _relu_after_weight(c_rows, qt, w, beta=None):
    pre = np.asarray(c_rows, float) @ np.asarray(qt, float).T
    if beta is not None:
        pre = pre + beta
    return np.maximum(pre * np.asarray(w, float), 0).sum(axis=1)


def _absorb_wrong_operand(q, W_K, b_K=None):
    q = np.asarray(q, float)
    W = np.asarray(W_K, float)
    # a plausible slip: use the decoder's rows as the absorbed query directly
    qt = np.einsum("...hk,kc->...hc", q, np.abs(W))
    beta = None if b_K is None else np.einsum("...hk,k->...h", q, np.asarray(b_K, float))
    return qt, beta


def _topk_high_index_ties(scores, k, n=None):
    s = np.asarray(scores)[: (len(scores) if n is None else n)]
    n = len(s)
    keff = min(k, n)
    order = np.lexsort((-np.arange(n), -s.astype(float)))
    sel = np.sort(order[:keff])
    idx = np.full(k, -1, np.int32)
    idx[:keff] = sel
    vals = np.full(k, -np.inf)
    vals[:keff] = s[sel]
    return idx, vals


def _topk_unsorted_output(scores, k, n=None):
    s = np.asarray(scores)[: (len(scores) if n is None else n)]
    n = len(s)
    keff = min(k, n)
    order = np.lexsort((np.arange(n), -s.astype(float)))[:keff]
    idx = np.full(k, -1, np.int32)
    idx[:keff] = order
    vals = np.full(k, -np.inf)
    vals[:keff] = s[order]
    return idx, vals


def _kth_off_by_one(scores, k, n=None):
    s = np.asarray(scores, float)[: (len(scores) if n is None else n)]
    keff = min(int(k), len(s))
    if keff == 0:
        return np.inf
    return float(np.sort(s)[::-1][min(keff, len(s) - 1)])


def _kth_distinct_values(scores, k, n=None):
    # a slip: the k-th best distinct value (ties counted once)
    s = np.asarray(scores, float)[: (len(scores) if n is None else n)]
    u = np.unique(s)[::-1]
    return np.inf if len(s) == 0 else float(u[min(int(k), len(u)) - 1])


PIN_SETS = [pins.test_hand_example_scores_and_selection, pins.test_hand_example_hs,
            pins.test_hand_example_bias, pins.test_hand_example_kth_score,
            lambda: pins.test_kth_score_counts(0),
            lambda: pins.test_absorbed_scoring_equals_explicit_keys(0),
            lambda: pins.test_topk_matches_sorted(5)]


@pytest.mark.parametrize("name,attr,bad", [
    ("dropped ReLU", "score", _dropped_relu),
    ("ReLU after weighting", "score", _relu_after_weight),
    ("wrong absorbed operand", "absorb", _absorb_wrong_operand),
    ("ties to the higher index", "topk", _topk_high_index_ties),
    ("selection not in position order", "topk", _topk_unsorted_output),
    ("k-th score off by one", "kth_score", _kth_off_by_one),
    ("k-th score over distinct values", "kth_score", _kth_distinct_values),
])
def test_planted_mistake_is_caught(monkeypatch, name, attr, bad):
    monkeypatch.setattr(ix, attr, bad)
    failures = 0
    for pin in PIN_SETS:
        try:
            pin()
        except AssertionError:
            failures += 1
    assert failures > 0, f"no pin caught: {name}"


# ------------------------------------------------------------------ two-branch latent (oracle/rope.py)

import oracle.rope as rp  # noqa: E402
from tests import test_oracle_rope as rope_pins  # noqa: E402

_rotate = rp.rotate


def _rotate_wrong_sign(x, pos, inv_freq, sources=1):
    return _rotate(x, -np.asarray(pos), inv_freq, sources)


def _rotate_slot_frequency(x, pos, inv_freq, sources=1):
    # a slip: slot p takes frequency p instead of p // sources
    z = rp.as_slots(x)
    P = z.shape[-1]
    freq = np.resize(np.asarray(inv_freq, float), P)
    pos = np.asarray(pos, float)
    angle = pos[..., None] * freq if pos.ndim else pos * freq
    return rp.from_slots(z * np.exp(1j * angle))


def _layer_norm_unbiased(x, gamma=None, beta=None, eps=1e-6):
    x = np.asarray(x, float)
    y = (x - x.mean(axis=-1, keepdims=True)) / np.sqrt(x.var(axis=-1, ddof=1, keepdims=True) + eps)
    if gamma is not None:
        y = y * gamma
    return y if beta is None else y + beta


ROPE_PINS = [rope_pins.test_quarter_turn_of_a_unit_pair, rope_pins.test_rotation_laws,
             rope_pins.test_sources_of_one_frequency_share_its_phase, rope_pins.test_layer_norm_matches_torch,
             lambda: rope_pins.test_absorbed_scoring_of_rotated_latent_equals_native_rotated_keys(2)]


@pytest.mark.parametrize("name,attr,bad", [
    ("rotation the wrong way", "rotate", _rotate_wrong_sign),
    ("slot frequency ignores the sources", "rotate", _rotate_slot_frequency),
    ("LayerNorm with the unbiased variance", "layer_norm", _layer_norm_unbiased),
])
def test_planted_rope_mistake_is_caught(monkeypatch, name, attr, bad):
    monkeypatch.setattr(rp, attr, bad)
    failures = 0
    for pin in ROPE_PINS:
        try:
            pin()
        except AssertionError:
            failures += 1
    assert failures > 0, f"no pin caught: {name}"
