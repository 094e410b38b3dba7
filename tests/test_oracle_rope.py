"""Pins of the oracle's two-branch latent (oracle/rope.py): the rotary
rotation against plane geometry and its group laws, LayerNorm against
torch's float64 layer_norm, and the central claim of the RoPE-compatible
decoders (LatentIndex summary, Sec. 3.1 and Sec. A.2): with frequency-wise
complex decoders, scoring the rotated latent with absorbed post-RoPE queries
equals scoring each layer's natively built and rotated keys."""
import math

import numpy as np
import pytest
import torch

from oracle import indexer, rope
from tests.helpers import latent_format, rope_decoder_matrix
from workloads import generate, rope_inputs, shrunk, workload


def test_quarter_turn_of_a_unit_pair():
    # one slot, frequency pi/2 per position: (1, 0) -> (0, 1) -> (-1, 0)
    f = np.array([math.pi / 2])
    np.testing.assert_allclose(rope.rotate([1.0, 0.0], 1, f), [0.0, 1.0], atol=1e-15)
    np.testing.assert_allclose(rope.rotate([1.0, 0.0], 2, f), [-1.0, 0.0], atol=1e-15)
    # (x, y) turned by theta: (x cos - y sin, x sin + y cos)
    th = 0.3
    np.testing.assert_allclose(rope.rotate([2.0, 5.0], 1, np.array([th])),
                               [2 * math.cos(th) - 5 * math.sin(th), 2 * math.sin(th) + 5 * math.cos(th)],
                               rtol=1e-15)


def test_rotation_laws():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((7, 16))
    f = rng.uniform(0, 1, 8)
    pos = rng.integers(0, 100000, 7)
    np.testing.assert_array_equal(rope.rotate(x, 0, f), x)
    y = rope.rotate(x, pos, f)
    np.testing.assert_allclose(np.hypot(y[:, 0::2], y[:, 1::2]), np.hypot(x[:, 0::2], x[:, 1::2]), rtol=1e-12)
    np.testing.assert_allclose(rope.rotate(rope.rotate(x, 3, f), pos, f), rope.rotate(x, pos + 3, f),
                               rtol=1e-9, atol=1e-9)
    # relative position: <R_m q, R_n k> = <q, R_{n-m} k>
    q, k = rng.standard_normal(16), rng.standard_normal(16)
    for m, n in ((5, 17), (1000, 3), (0, 0)):
        assert rope.rotate(q, m, f) @ rope.rotate(k, n, f) == pytest.approx(q @ rope.rotate(k, n - m, f), rel=1e-9)


def test_sources_of_one_frequency_share_its_phase():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(12)                    # 6 slots: 3 frequencies x 2 sources
    f = np.array([0.1, 0.7, 2.3])
    y = rope.rotate(x, 5, f, sources=2)
    turned = np.angle(rope.as_slots(y) / rope.as_slots(x))
    want = np.angle(np.exp(1j * 5 * f[[0, 0, 1, 1, 2, 2]]))
    np.testing.assert_allclose(turned, want, atol=1e-12)


def test_layer_norm_matches_torch():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 128)) * 3 + 1
    g, b = rng.standard_normal(128), rng.standard_normal(128)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(x), (128,), torch.from_numpy(g), torch.from_numpy(b), 1e-6)
    np.testing.assert_allclose(rope.layer_norm(x, g, b, 1e-6), ref.numpy(), rtol=1e-12, atol=1e-12)
    y = rope.layer_norm(x, eps=0.0)
    np.testing.assert_allclose(y.mean(axis=1), 0, atol=1e-12)
    np.testing.assert_allclose((y ** 2).mean(axis=1), 1, rtol=1e-12)
    np.testing.assert_array_equal(rope.layer_norm(np.full(8, 4.0), None, np.arange(8.0)), np.arange(8.0))


@pytest.mark.parametrize("sources", [1, 2])
def test_absorbed_scoring_of_rotated_latent_equals_native_rotated_keys(sources):
    wl = shrunk(workload(1), capacity=300)
    inp = generate(wl)
    ri = rope_inputs(wl, sources=sources)
    fmt = latent_format(ri)
    pos = np.arange(300) + 70000                   # far positions: large angles
    c = inp.latent[0].astype(np.float64)
    rows = rope.cache_rows(c, pos, fmt)
    for l in range(wl.group):
        W, bias = rope_decoder_matrix(ri, l, wl.d_k, wl.d_c)
        q, w = inp.q[l][0, 0], inp.w[l][0, 0]
        qt, beta = indexer.absorb(q, W, bias)
        absorbed = indexer.score(rows, qt, w, beta)
        d = ri.d_re[l].astype(np.float64) + 1j * ri.d_im[l]
        keys = rope.native_keys(c, pos, fmt, d, ri.W_nope[l], ri.b_nope[l])
        native = indexer.dsa_score_keys(keys, q, w)
        M = indexer.error_scale(keys, q, w)
        assert np.max(np.abs(absorbed - native) / M) < 1e-12
        # the rotation matters: scoring unrotated rows does not reproduce it
        plain = indexer.score(rope.cache_rows(c, 0 * pos, fmt), qt, w, beta)
        assert np.max(np.abs(plain - native) / M) > 1e-3
