"""Pins of the oracle's selection-quality metrics (oracle/recall.py): a
hand-computed example, a brute force over all size-K sets, the range and
special cases of the recall, and scipy's softmax."""
import itertools
import json
import os

import numpy as np
import pytest
from scipy.special import softmax

from oracle import recall

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_hand_example():
    g = json.load(open(os.path.join(GOLDEN, "recall_example.json")))
    p = np.array(g["p"])
    np.testing.assert_allclose(recall.head_mass_recall(p, g["sel"], g["K"]), g["head_recall"], rtol=1e-14)
    assert recall.mean_attention_recall(p, g["sel"], g["K"]) == pytest.approx(g["mean_recall"], rel=1e-14)


def test_top_mass_is_the_best_subset_by_brute_force():
    rng = np.random.default_rng(0)
    p = rng.dirichlet(np.ones(7), size=3)
    for K in (1, 2, 3, 7, 9):
        kk = min(K, 7)
        brute = [max(sum(row[list(c)]) for c in itertools.combinations(range(7), kk)) for row in p]
        np.testing.assert_allclose(recall.top_mass(p, K), brute, rtol=1e-14)


def test_recall_range_and_special_cases():
    rng = np.random.default_rng(1)
    H, N, K = 4, 50, 8
    p = rng.dirichlet(np.full(N, 0.3), size=H)
    for _ in range(20):
        sel = np.sort(rng.choice(N, size=K, replace=False))
        r = recall.head_mass_recall(p, sel, K)
        assert np.all((r >= 0) & (r <= 1 + 1e-12))
        assert 0 <= recall.mean_attention_recall(p, sel, K) <= 1 + 1e-12
    # a head's own top-K set scores 1 for that head; nothing selected scores 0
    best0 = np.sort(np.argsort(-p[0])[:K])
    assert recall.head_mass_recall(p, best0, K)[0] == pytest.approx(1.0, rel=1e-14)
    assert np.all(recall.head_mass_recall(p, np.full(K, -1), K) == 0)
    # with identical heads the mean-attention recall is the head recall
    same = np.repeat(p[:1], 3, axis=0)
    sel = np.sort(rng.choice(N, size=K, replace=False))
    assert recall.mean_attention_recall(same, sel, K) == pytest.approx(recall.head_mass_recall(same, sel, K)[0])
    # K past the prefix is capped: selecting the whole prefix recalls everything
    assert np.allclose(recall.head_mass_recall(p, np.arange(N), 4 * N), 1.0)


def test_index_cache_follower_reuses_the_anchor_selection():
    a = np.array([3, 9, 17, -1], np.int32)
    f = recall.index_cache_follower(a)
    assert np.array_equal(f, a) and f is not a


def test_attention_is_softmax_over_the_prefix():
    rng = np.random.default_rng(2)
    logits = rng.standard_normal((3, 20)) * 4
    p = recall.attention(logits, 12)
    np.testing.assert_allclose(p[:, :12], softmax(logits[:, :12], axis=1), rtol=1e-13)
    assert np.all(p[:, 12:] == 0)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=1e-14)
