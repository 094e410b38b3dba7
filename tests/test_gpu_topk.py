"""li_topk on identical fp32 arrays must match the oracle's sort bit for bit."""
import zlib

import numpy as np
import pytest
import torch

from oracle import indexer

pytestmark = pytest.mark.gpu
li = pytest.importorskip("cross_layer_latent_b200")

DEV = "cuda:0"


@pytest.fixture(scope="module")
def ctx():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    c = li.Context(0)
    yield c
    c.close()


def _seed(*parts):
    """A seed that is the same in every process (str hashes are salted)."""
    return zlib.crc32(repr(parts).encode())


def _rows(kind, rows, n, rng):
    if kind == "gauss":
        return rng.standard_normal((rows, n)).astype(np.float32)
    if kind == "ties":        # few distinct values: many ties at the boundary
        return (rng.integers(-3, 4, (rows, n)) * 0.5).astype(np.float32)
    if kind == "zeros":       # +0 and -0 everywhere
        return np.where(rng.random((rows, n)) < 0.5, np.float32(0.0), np.float32(-0.0)).astype(np.float32)
    if kind == "const":
        return np.full((rows, n), 1.25, np.float32)
    if kind == "wide":        # magnitudes across the whole exponent range, both signs, infinities
        x = rng.standard_normal((rows, n)) * 10.0 ** rng.integers(-30, 30, (rows, n))
        x[:, ::97] = np.inf
        x[:, 5::101] = -np.inf
        return x.astype(np.float32)
    if kind == "neg":
        return -np.abs(rng.standard_normal((rows, n))).astype(np.float32)
    raise ValueError(kind)


def _check(ctx, x, k, lengths=None):
    rows, n = x.shape
    xd = torch.from_numpy(x).to(DEV)
    idx = torch.full((rows, k), -7, dtype=torch.int32, device=DEV)
    val = torch.zeros(rows, k, device=DEV)
    ws = li.workspace(ctx, rows, 1, n, 1, k)
    ld = None if lengths is None else torch.from_numpy(lengths.astype(np.int32)).to(DEV)
    li.li_topk(ctx, xd, k, idx, val, ws, lengths=ld)
    torch.cuda.synchronize()
    gi, gv = idx.cpu().numpy(), val.cpu().numpy()
    for r in range(rows):
        nr = n if lengths is None else int(np.clip(lengths[r], 0, n))
        ei, ev = indexer.topk(x[r], k, nr)
        assert np.array_equal(gi[r], ei), f"row {r}: first difference at {np.argmax(gi[r] != ei)}"
        keep = ei >= 0
        # selected scores are the inputs bit for bit, except that -0.0 may
        # come back as +0.0, the value it is ranked as
        want = x[r][ei[keep]]
        want = np.where(want == 0, np.float32(0), want)
        got = gv[r][keep]
        got = np.where(got == 0, np.float32(0), got)
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
        assert np.all(np.isneginf(gv[r][~keep]))


@pytest.mark.parametrize("kind", ["gauss", "ties", "zeros", "const", "wide", "neg"])
@pytest.mark.parametrize("rows,n,k", [(1, 8192, 2048), (4, 131072, 2048), (3, 1000, 64), (5, 4097, 4097),
                                      (64, 5000, 100)])
def test_topk_bit_exact(ctx, kind, rows, n, k):
    rng = np.random.default_rng(_seed(kind, rows, n, k))
    _check(ctx, _rows(kind, rows, n, rng), k)


def test_topk_ragged_lengths_and_short_rows(ctx):
    rng = np.random.default_rng(1)
    x = _rows("ties", 9, 20000, rng)
    lengths = np.array([0, 1, 5, 63, 64, 65, 4096, 12345, 20000])
    _check(ctx, x, 64, lengths)
    _check(ctx, x, 2048, lengths)


@pytest.mark.parametrize("kind", ["gauss", "ties", "const"])
def test_topk_ragged_rows_in_the_widest_clusters(ctx, kind):
    """Rows of 131072 positions take 16-CTA clusters; valid prefixes that end
    inside one CTA, leave 15 CTAs of the cluster empty, or are empty."""
    rng = np.random.default_rng(7)
    x = _rows(kind, 4, 131072, rng)
    _check(ctx, x, 2048, np.array([70001, 131072, 3, 0]))
    _check(ctx, x, 2048, np.array([8191, 8192, 8193, 131071]))


def _launched_keys_per_thread(ctx, fn, rows, n):
    """Run fn with the launch profile on; the keys a thread of the one
    cluster selection it launched holds (4, 8, 16 or 32)."""
    li.li_profile_enable(ctx, True)
    li.li_profile_reset(ctx)
    fn()
    torch.cuda.synchronize()
    recs = li.li_profile_read(ctx)
    li.li_profile_enable(ctx, False)
    li.li_profile_reset(ctx)
    sel = [r for r in recs if r["kernel"].startswith("topk")]
    assert len(sel) == 1 and sel[0]["kernel"] == "topk_cluster", [r["kernel"] for r in recs]
    cs = sel[0]["grid"] // rows
    per = -(-n // (cs * 512))
    return next(p for p in (4, 8, 16, 32) if per <= p)


@pytest.mark.parametrize("kind", ["gauss", "ties", "zeros"])
@pytest.mark.parametrize("rows,n", [(1024, 65536), (400, 20000)])
def test_topk_many_rows_take_the_throughput_selection(ctx, kind, rows, n):
    """Many rows (a prefill chunk's queries) fill the GPU many times over and
    take the selection sized for throughput, 32 keys a thread; it must stay
    bit-exact, with ragged valid prefixes (empty, ending inside a CTA, full)."""
    rng = np.random.default_rng(_seed(kind, rows, n, 32))
    x = _rows(kind, rows, n, rng)
    lengths = rng.integers(0, n + 1, rows)
    lengths[:4] = [0, 1, n, n - 1]
    k = 2048
    xd = torch.from_numpy(x).to(DEV)
    ld = torch.from_numpy(lengths.astype(np.int32)).to(DEV)
    idx = torch.full((rows, k), -7, dtype=torch.int32, device=DEV)
    val = torch.zeros(rows, k, device=DEV)
    ws = li.workspace(ctx, rows, 1, n, 1, k)
    pt = _launched_keys_per_thread(ctx, lambda: li.li_topk(ctx, xd, k, idx, val, ws, lengths=ld), rows, n)
    assert pt == 32, f"launched the {pt}-keys-a-thread selection"
    gi, gv = idx.cpu().numpy(), val.cpu().numpy()
    for r in range(rows):
        ei, _ = indexer.topk(x[r], k, int(lengths[r]))
        assert np.array_equal(gi[r], ei), f"row {r} (length {lengths[r]}): first difference at {np.argmax(gi[r] != ei)}"
        keep = ei >= 0
        want = np.where(x[r][ei[keep]] == 0, np.float32(0), x[r][ei[keep]])
        got = np.where(gv[r][keep] == 0, np.float32(0), gv[r][keep])
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
