"""Pins of the CPU oracle against facts that do not come from the oracle itself:
hand arithmetic, numbers printed in the LatentIndex summary, an independent
pure-Python brute force, invariants of the method, and library codecs."""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import bruteforce, codecs, counters, indexer

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ------------------------------------------------------------------ worked example (hand arithmetic)

def test_hand_example_scores_and_selection():
    g = _golden("hand_example.json")
    c = np.array(g["latent"], float)
    a = g["anchor"]
    qt, beta = indexer.absorb(np.array(a["q"], float), np.array(a["W_K"], float))
    assert beta is None
    np.testing.assert_array_equal(qt, np.array(a["absorbed"], float))
    s = indexer.score(c, qt, np.array(a["w"]))
    np.testing.assert_array_equal(s, np.array(a["scores"]))
    assert indexer.topk(s, 2)[0].tolist() == a["top2"]
    assert indexer.topk(s, 3)[0].tolist() == a["top3"]
    assert indexer.topk(s, 8)[0].tolist() == a["top8"]
    # the same through explicit keys
    assert indexer.dsa_score(c, np.array(a["W_K"], float), np.array(a["q"], float),
                             np.array(a["w"])).tolist() == a["scores"]


def test_hand_example_kth_score():
    """The selection boundary used by the tolerance rule: the k_eff-th best
    score, worked by hand on the example's scores (ties and k past n)."""
    a = _golden("hand_example.json")["anchor"]
    s = np.array(a["scores"])
    for k, v in a["kth"].items():
        assert indexer.kth_score(s, int(k)) == v
    for k, v in a["kth_n2"].items():
        assert indexer.kth_score(s, int(k), n=2) == v
    assert indexer.kth_score(s, 3, n=0) == np.inf


@pytest.mark.parametrize("seed", range(3))
def test_kth_score_counts(seed):
    """Pure-Python characterisation without sorting: v is the k_eff-th best
    score iff v is one of the scores, fewer than k_eff scores exceed it and
    at least k_eff reach it; it is also the lowest score the top-k keeps."""
    rng = np.random.default_rng(40 + seed)
    for row in _adversarial_rows(rng):
        vals = row.astype(float).tolist()
        for k in (1, 2, 7, len(vals), len(vals) + 3):
            for n in (len(vals), len(vals) // 2):
                v = indexer.kth_score(row, k, n)
                pre = vals[:n]
                keff = min(k, n)
                if keff == 0:
                    assert v == np.inf
                    continue
                assert v in pre
                assert sum(1 for x in pre if x > v) < keff <= sum(1 for x in pre if x >= v)
                idx, kept = indexer.topk(row, k, n)
                assert kept[idx >= 0].min() == v


def test_hand_example_bias():
    g = _golden("hand_example.json")
    c = np.array(g["latent"], float)
    a = g["anchor"]
    qt, beta = indexer.absorb(np.array(a["q"], float), np.array(a["W_K"], float),
                              np.array(a["bias"], float))
    np.testing.assert_array_equal(beta, np.array(a["beta"]))
    s = indexer.score(c, qt, np.array(a["w"]), beta)
    np.testing.assert_array_equal(s, np.array(a["scores_bias"]))


def test_hand_example_hs():
    g = _golden("hand_example.json")
    c = np.array(g["latent"], float)
    a, f, hs = g["anchor"], g["follower"], g["hs"]
    qa, _ = indexer.absorb(np.array(a["q"], float), np.array(a["W_K"], float))
    sa = indexer.score(c, qa, np.array(a["w"]))
    cand, cand_n, anchor_idx = indexer.hs_anchor(sa, hs["B"], hs["k"])
    assert cand.tolist() == hs["candidates"] and cand_n == 3
    assert anchor_idx.tolist() == hs["anchor_top2"]
    qf, _ = indexer.absorb(np.array(f["q"], float), np.array(f["W_K"], float))
    sf = indexer.score(c, qf, np.array(f["w"]))
    np.testing.assert_array_equal(sf, np.array(f["scores"]))
    fol, _ = indexer.hs_follower(sf[cand[:cand_n]], cand, cand_n, hs["k"])
    assert fol.tolist() == hs["follower_top2"]
    assert indexer.topk(sf, 2)[0].tolist() == f["full_top2"]


# ------------------------------------------------------------------ printed numbers (closed forms)

def test_cache_bytes_match_printed_numbers():
    g = _golden("printed_numbers.json")["cache_bytes_per_token"]
    dsa = counters.cache_bytes_per_token_dsa(g["indexed_layers"])
    li = counters.cache_bytes_per_token_latent(g["groups_g4"], g["independent_layers"])
    assert dsa == g["dsa"]
    assert li == g["latentindex_g4"]
    assert round(100.0 * (1 - li / dsa), 1) == g["reduction_percent_1dp"]


def test_positions_scored_match_printed_formula():
    g = _golden("printed_numbers.json")["positions_scored"]
    B = g["B"]
    for L in (8193, 16384, 65536, 131072):
        hs = counters.positions_scored_model(L, [4] * 15, B)
        dsa = counters.positions_scored_model(L, [4] * 15, None)
        assert hs == g["hs_linear_coeff"] * L + g["hs_constant_blocks"] * B
        assert dsa == g["dsa_linear_coeff"] * L
    # below the budget HS scores everything (min(B, L) = L)
    assert counters.positions_scored_group(4096, 4, 8192) == 4 * 4096


# ------------------------------------------------------------------ brute force (explicit keys, sorted)

def _tiny(rng, n=23, H=3, dk=5, dc=7):
    c = rng.standard_normal((n, dc))
    W = rng.standard_normal((dk, dc))
    q = rng.standard_normal((H, dk))
    w = rng.standard_normal(H)
    b = rng.standard_normal(dk)
    return c, W, q, w, b


@pytest.mark.parametrize("seed", range(6))
def test_absorbed_scoring_equals_explicit_keys(seed):
    """Absorption is exact in exact arithmetic (Sec. 3.1): absorbed scoring
    equals explicit key reconstruction followed by dot products."""
    rng = np.random.default_rng(seed)
    c, W, q, w, b = _tiny(rng)
    qt, beta = indexer.absorb(q, W, b)
    ours = indexer.score(c, qt, w, beta)
    brute = bruteforce.layer_scores(c.tolist(), W.tolist(), q.tolist(), w.tolist(), b.tolist())
    M = indexer.error_scale(c, qt, w) + np.abs(beta).sum()
    assert np.all(np.abs(ours - np.array(brute)) <= 1e-12 * (M + 1))
    ours_nb = indexer.score(c, indexer.absorb(q, W)[0], w)
    brute_nb = bruteforce.layer_scores(c.tolist(), W.tolist(), q.tolist(), w.tolist())
    assert np.allclose(ours_nb, brute_nb, rtol=0, atol=1e-12 * (M.max() + 1))


def test_per_head_decoders():
    rng = np.random.default_rng(7)
    c, _, q, w, _ = _tiny(rng)
    Wh = rng.standard_normal((3, 5, 7))
    qt, _ = indexer.absorb(q, Wh)
    for h in range(3):
        brute = bruteforce.layer_scores(c.tolist(), Wh[h].tolist(), [q[h].tolist()], [w[h]])
        np.testing.assert_allclose(indexer.score(c, qt[h:h + 1], w[h:h + 1]), brute,
                                   rtol=1e-12, atol=1e-12)


def test_dsa_score_matches_brute_force():
    rng = np.random.default_rng(11)
    c, W, q, w, _ = _tiny(rng)
    np.testing.assert_allclose(indexer.dsa_score(c, W, q, w),
                               bruteforce.layer_scores(c.tolist(), W.tolist(), q.tolist(), w.tolist()),
                               rtol=1e-12, atol=1e-12)


def test_latent_matches_brute_force():
    rng = np.random.default_rng(12)
    h = rng.standard_normal((9, 6))
    Wd = rng.standard_normal((4, 6))
    c = indexer.latent(h, Wd)
    for s in range(9):
        np.testing.assert_allclose(c[s], bruteforce.reconstruct_key(Wd.tolist(), h[s].tolist()),
                                   rtol=1e-12, atol=1e-12)
    # identity projection returns the input
    np.testing.assert_array_equal(indexer.latent(h, np.eye(6)), h)


def _adversarial_rows(rng):
    rows = [
        rng.standard_normal(50),
        np.zeros(40),                                     # all ties
        np.array([0.0, -0.0, 0.0, -0.0, 1.0, -1.0, -0.0]),  # signed zeros tie
        np.round(rng.standard_normal(64) * 2) / 2,          # many ties at the boundary
        -np.abs(rng.standard_normal(30)),                   # all negative
        np.array([np.inf, -np.inf, 1.0, np.inf, 0.0]),
        rng.standard_normal(3),                             # fewer than k
        np.zeros(0),
    ]
    return [r.astype(np.float32) for r in rows]


@pytest.mark.parametrize("k", [1, 2, 5, 16, 100])
def test_topk_matches_sorted(k):
    rng = np.random.default_rng(3)
    for row in _adversarial_rows(rng):
        idx, vals = indexer.topk(row, k)
        assert idx.tolist() == bruteforce.select(row.astype(float).tolist(), k)
        keep = idx >= 0
        np.testing.assert_array_equal(vals[keep], row[idx[keep]])
        assert np.all(np.isneginf(vals[~keep]))


def test_topk_respects_valid_length():
    row = np.array([5, 4, 3, 9, 9, 9], np.float32)
    assert indexer.topk(row, 2, n=3)[0].tolist() == [0, 1]
    assert indexer.topk(row, 5, n=3)[0].tolist() == [0, 1, 2, -1, -1]
    assert indexer.valid_length(100) == 100
    assert indexer.valid_length(100, q_pos=41) == 42


@pytest.mark.parametrize("seed", range(4))
def test_hs_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    n, H, dk, dc, B, k = 31, 2, 4, 6, 9, 4
    c = rng.standard_normal((n, dc))
    layers = [(rng.standard_normal((dk, dc)), rng.standard_normal((H, dk)), rng.standard_normal(H))
              for _ in range(4)]
    cand_b, sels_b = bruteforce.hs(c.tolist(), [(W.tolist(), q.tolist(), w.tolist())
                                                for W, q, w in layers], B, k)
    s0 = indexer.score(c, indexer.absorb(layers[0][1], layers[0][0])[0], layers[0][2])
    cand, cand_n, a_idx = indexer.hs_anchor(s0, B, k)
    assert cand.tolist() == cand_b and a_idx.tolist() == sels_b[0]
    for li in range(1, 4):
        W, q, w = layers[li]
        s = indexer.score(c, indexer.absorb(q, W)[0], w)
        fol, _ = indexer.hs_follower(s[cand[:cand_n]], cand, cand_n, k)
        assert fol.tolist() == sels_b[li]
        assert set(fol[fol >= 0]) <= set(cand[:cand_n])


# ------------------------------------------------------------------ invariants of the method

@pytest.mark.parametrize("seed", range(3))
def test_hs_with_budget_covering_prefix_equals_full(seed):
    """B >= L makes HS score every position (min(B, L) = L, Sec. 3.4), so HS
    equals full-prefix LatentIndex."""
    rng = np.random.default_rng(200 + seed)
    n, H, dc, k = 64, 4, 8, 10
    c = rng.standard_normal((n, dc))
    qts = [rng.standard_normal((H, dc)) for _ in range(4)]
    ws = [rng.standard_normal(H) for _ in range(4)]
    s0 = indexer.score(c, qts[0], ws[0])
    for B in (n, n + 5, 4 * n):
        cand, cand_n, a_idx = indexer.hs_anchor(s0, B, k)
        assert cand_n == n and cand[:n].tolist() == list(range(n))
        assert a_idx.tolist() == indexer.topk(s0, k)[0].tolist()
        for l in range(1, 4):
            s = indexer.score(c, qts[l], ws[l])
            fol, _ = indexer.hs_follower(s[cand[:cand_n]], cand, cand_n, k)
            assert fol.tolist() == indexer.topk(s, k)[0].tolist()


def test_group_of_one_with_identity_decoder_is_dsa():
    """G = 1 with identity decoders: the latent is the key, and absorbed scoring
    reduces to DSA-style scoring of that key."""
    rng = np.random.default_rng(5)
    n, H, d = 40, 6, 16
    keys = rng.standard_normal((n, d))
    q = rng.standard_normal((H, d))
    w = rng.standard_normal(H)
    qt, _ = indexer.absorb(q, np.eye(d))
    np.testing.assert_array_equal(qt, q)
    np.testing.assert_array_equal(indexer.score(keys, qt, w), indexer.dsa_score_keys(keys, q, w))
    np.testing.assert_array_equal(indexer.score(keys, qt, w), indexer.dsa_score(keys, np.eye(d), q, w))


def test_relu_positive_homogeneity_and_weight_sign():
    """Scaling a latent row by a > 0 scales its score by a; flipping every head
    weight flips every score."""
    rng = np.random.default_rng(9)
    c, W, q, w, _ = _tiny(rng)
    qt, _ = indexer.absorb(q, W)
    s = indexer.score(c, qt, w)
    np.testing.assert_allclose(indexer.score(3.5 * c, qt, w), 3.5 * s, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(indexer.score(c, qt, -w), -s, rtol=1e-12, atol=1e-12)


def test_error_scale_bounds_score():
    rng = np.random.default_rng(10)
    c, W, q, w, _ = _tiny(rng)
    qt, _ = indexer.absorb(q, W)
    assert np.all(np.abs(indexer.score(c, qt, w)) <= indexer.error_scale(c, qt, w) * (1 + 1e-12))


# ------------------------------------------------------------------ codecs vs library conversions

def test_bf16_decode_all_codes_match_torch():
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = codecs.bf16_decode(codes)
    ref = torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).float().numpy()
    same = (ours.view(np.uint32) == ref.view(np.uint32)) | (np.isnan(ours) & np.isnan(ref))
    assert same.all()


def test_bf16_encode_matches_torch_rne():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 30, 200000).astype(np.float32),
        # exact midpoints between neighbouring bf16 values (ties)
        (np.arange(1, 4000, dtype=np.uint32) << 16 | np.uint32(0x8000)).view(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0, np.inf, -np.inf, 3.4e38, -3.4e38, 1e-40, -1e-40], np.float32),
    ]).astype(np.float32)
    x = x[np.isfinite(x) | np.isinf(x)]
    ours = codecs.bf16_encode(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_e4m3_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = codecs.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    same = (ours == ref) | (np.isnan(ours) & np.isnan(ref))
    assert same.all() and np.sum(np.isnan(ours)) == 2
    assert codecs.E4M3_TABLE[0x7E] == 448.0 and codecs.E4M3_TABLE[0x01] == 2.0 ** -9


def test_e4m3_encode_matches_bruteforce_and_torch():
    rng = np.random.default_rng(1)
    finite = codecs.E4M3_TABLE[:0x7F]
    mids = (finite[:-1] + finite[1:]) / 2
    x = np.concatenate([finite, mids, -mids, rng.standard_normal(3000) * 50,
                        rng.standard_normal(2000) * 0.01, [500.0, -1e6, 460.0, 1e-5, -1e-5]]).astype(np.float32)
    ours = codecs.e4m3_encode(x)
    assert np.array_equal(ours, codecs.e4m3_encode_bruteforce(x))
    inrange = np.abs(x) < 464.0          # torch's cast does not saturate beyond the last midpoint
    ref = torch.from_numpy(x[inrange]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours[inrange], ref)
    assert codecs.e4m3_encode(np.array([1e9, -1e9], np.float32)).tolist() == [0x7E, 0xFE]


def test_e4m3_row_quantisation_properties():
    rng = np.random.default_rng(2)
    c = rng.standard_normal((64, 192)).astype(np.float32)
    c[:, 5] *= 8
    c[3] = 0
    codes, scale = codecs.e4m3_quantize_rows(c)
    assert scale[3] == 1.0 and np.all(codes[3] == 0)
    dq = codecs.e4m3_dequantize_rows(codes, scale)
    # the largest element maps to (about) +-448; every element within half a
    # spacing of e4m3 (relative 2^-4, absolute 2^-10 in the subnormal range)
    amax_codes = np.max(np.abs(codecs.e4m3_decode(codes)), axis=1)
    assert np.all((amax_codes[np.arange(64) != 3] >= 416) & (amax_codes[np.arange(64) != 3] <= 448))
    err = np.abs(dq - c)
    bound = np.maximum(np.abs(c) * 2.0 ** -4, 2.0 ** -10 * scale[:, None]) * (1 + 1e-6)
    assert np.all(err <= bound)


def test_segmented_e4m3_keeps_each_branch_range():
    """Segmented fp8: the small-range branch keeps its resolution next to a
    large-range one; scaling one segment by a power of two scales its scale
    exactly and changes no code; each element decodes within half an e4m3
    spacing of its own segment; torch's float8_e4m3fn gives the same codes."""
    rng = np.random.default_rng(3)
    c = rng.standard_normal((32, 192)).astype(np.float32)
    c[:, :64] *= 2e-6                          # a rotary branch far smaller than the NoPE branch
    codes, scale = codecs.e4m3_quantize_rows_segmented(c, 64)
    assert codes.shape == (32, 192) and scale.shape == (32, 2)
    dq = codecs.e4m3_dequantize_rows_segmented(codes, scale, 64)
    for a, b, k in ((0, 64, 0), (64, 192, 1)):
        bound = np.maximum(np.abs(c[:, a:b]) * 2.0 ** -4, 2.0 ** -10 * scale[:, k:k + 1]) * (1 + 1e-6)
        assert np.all(np.abs(dq[:, a:b] - c[:, a:b]) <= bound)
        ref = (torch.from_numpy(c[:, a:b]) / torch.from_numpy(scale[:, k:k + 1])).to(torch.float8_e4m3fn)
        assert np.array_equal(codes[:, a:b], ref.view(torch.uint8).numpy())
    # one scale per row would lose the small branch: most of its codes flush to zero
    one, _ = codecs.e4m3_quantize_rows(c)
    assert np.mean((one[:, :64] & 0x7F) == 0) > 0.9 and np.mean((codes[:, :64] & 0x7F) == 0) < 0.05
    c2 = c.copy()
    c2[:, 64:] *= 4
    codes2, scale2 = codecs.e4m3_quantize_rows_segmented(c2, 64)
    assert np.array_equal(codes2, codes)
    assert np.array_equal(scale2[:, 0], scale[:, 0]) and np.array_equal(scale2[:, 1], 4 * scale[:, 1])
