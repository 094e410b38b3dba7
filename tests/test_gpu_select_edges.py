"""Selection after the decode scans, the HS anchor and the followers (one
query row per sequence), on the rows that stress it.

Every layer keeps its own top-k (LatentIndex summary, Sec. 3.1), the anchor
its top-B candidates and its top-k, the followers their top-k among the
candidates (Sec. 3.2, Sec. C.4).  The selections must equal the oracle's
top-k of the GPU's own fp32 scores bit for bit, also when
  * every score is equal (a zero head weight vector: only the position
    tie-break decides),
  * a few distinct scores cover the whole row (the boundary bin of the first
    radix digit holds most of the row),
  * valid lengths are 0, 1, k - 1, k, k + 1 and full within one batch,
  * the candidate budget exceeds the valid prefix,
and repeated calls on one workspace give identical results."""
from dataclasses import replace

import numpy as np
import pytest
import torch

import cross_layer_latent_b200 as li
from oracle import indexer
from tests.gpu_setup import build_group
from workloads import generate, shrunk, workload

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def ctx():
    c = li.Context(0)
    yield c
    c.close()


def _np(t):
    return t.detach().cpu().numpy()


def _check_rows(d, idx, sc, lengths, k, what):
    for b, n in enumerate(lengths):
        n = int(n)
        e, ev = indexer.topk(d[b, 0, :n], k, n)
        assert np.array_equal(idx[b, 0], e), f"{what} seq {b} (length {n})"
        if sc is not None:
            keep = e >= 0
            got = np.where(sc[b, 0][keep] == 0, np.float32(0), sc[b, 0][keep])
            want = np.where(ev[keep] == 0, 0.0, ev[keep]).astype(np.float32)
            assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), f"{what} seq {b}: scores"
            assert np.all(np.isneginf(sc[b, 0][~keep]))


def _group(ctx, batch, capacity, lengths, kind="bf16", k=64, B=256, latent_fn=None, seed=0):
    wl = shrunk(workload(1 if kind == "bf16" else 3), capacity=capacity, batch=batch)
    wl = replace(wl, k=k, B=B)
    inp = generate(wl, seed=seed)
    inp.lengths = np.asarray(lengths, np.int32)
    if latent_fn is not None:
        inp.latent = latent_fn(inp.latent)
    return wl, inp, build_group(ctx, inp, dsa=True)


@pytest.mark.parametrize("kind", ["bf16", "e4m3"])
def test_ragged_lengths_around_the_budget(ctx, kind):
    k = 64
    lengths = [0, 1, k - 1, k, k + 1, 777, 4999, 5000]
    wl, inp, g = _group(ctx, len(lengths), 5000, lengths, kind, k=k, B=300)
    dump = torch.full((wl.batch, 1, wl.capacity), float("nan"), device=DEV)
    g.score_topk(0, dump=dump)
    torch.cuda.synchronize()
    assert li.li_device_status(ctx, g.ws) == "LI_OK"
    _check_rows(_np(dump), _np(g.idx[0]), _np(g.score[0]), lengths, k, f"{kind} full")
    g.dsa_score_topk(1, dump=dump)
    torch.cuda.synchronize()
    assert li.li_device_status(ctx, g.ws) == "LI_OK"
    _check_rows(_np(dump), _np(g.idx[1]), _np(g.score[1]), lengths, k, f"{kind} dsa")
    # HS: candidates (B = 300, above some lengths), the anchor's top-k, followers
    g.hs_anchor(0, dump=dump)
    torch.cuda.synchronize()
    assert li.li_device_status(ctx, g.ws) == "LI_OK"
    d, cand, cand_n = _np(dump), _np(g.cand), _np(g.cand_n)
    for b, n in enumerate(lengths):
        ec, _ = indexer.topk(d[b, 0, :n], wl.B, n)
        assert np.array_equal(cand[b, 0], ec) and cand_n[b, 0] == min(wl.B, n), f"{kind} candidates seq {b}"
    _check_rows(d, _np(g.idx[0]), _np(g.score[0]), lengths, k, f"{kind} anchor")
    fd = torch.full((wl.batch, 1, wl.B), float("nan"), device=DEV)
    g.hs_follower(2, dump=fd)
    torch.cuda.synchronize()
    assert li.li_device_status(ctx, g.ws) == "LI_OK"
    fdn, fidx = _np(fd), _np(g.idx[2])
    for b, n in enumerate(lengths):
        cn = int(cand_n[b, 0])
        ef, _ = indexer.hs_follower(fdn[b, 0, :cn], cand[b, 0], cn, k)
        assert np.array_equal(fidx[b, 0], ef), f"{kind} follower seq {b}"


def test_all_scores_equal(ctx):
    """w = 0: every score is 0, so the selection is the first k positions."""
    lengths = [3000, 2048, 100]
    wl, inp, g = _group(ctx, 3, 3000, lengths, k=2048, B=2500)
    for l in range(wl.group):
        g.w[l].zero_()
    dump = torch.full((wl.batch, 1, wl.capacity), float("nan"), device=DEV)
    g.score_topk(1, dump=dump)
    g.hs_anchor(0)
    torch.cuda.synchronize()
    assert li.li_device_status(ctx, g.ws) == "LI_OK"
    assert np.all(_np(dump)[0, 0] == 0)
    _check_rows(_np(dump), _np(g.idx[1]), _np(g.score[1]), lengths, wl.k, "equal scores")
    cand, cand_n, a_idx = _np(g.cand), _np(g.cand_n), _np(g.idx[0])
    for b, n in enumerate(lengths):
        m = min(wl.B, n)
        assert cand_n[b, 0] == m and np.array_equal(cand[b, 0, :m], np.arange(m)) and np.all(cand[b, 0, m:] == -1)
        kk = min(wl.k, n)
        assert np.array_equal(a_idx[b, 0, :kk], np.arange(kk)) and np.all(a_idx[b, 0, kk:] == -1)


def test_few_distinct_scores(ctx):
    """Every latent row is one of three vectors: three distinct scores over
    the whole row, ties at the boundary decided by position."""
    rng = np.random.default_rng(3)

    def three_rows(lat):
        pick = rng.integers(0, 3, lat.shape[:2])
        base = lat[0, :3].copy()
        return base[pick].astype(np.float32)

    lengths = [6000, 5000]
    wl, inp, g = _group(ctx, 2, 6000, lengths, k=1000, B=3000, latent_fn=three_rows)
    dump = torch.full((wl.batch, 1, wl.capacity), float("nan"), device=DEV)
    g.score_topk(2, dump=dump)
    torch.cuda.synchronize()
    assert li.li_device_status(ctx, g.ws) == "LI_OK"
    d = _np(dump)
    assert len(np.unique(d[0, 0, :6000])) <= 3
    _check_rows(d, _np(g.idx[2]), _np(g.score[2]), lengths, wl.k, "three values")
    g.hs_anchor(0, dump=dump)
    fd = torch.full((wl.batch, 1, wl.B), float("nan"), device=DEV)
    g.hs_follower(1, dump=fd)
    torch.cuda.synchronize()
    assert li.li_device_status(ctx, g.ws) == "LI_OK"
    d, cand, cand_n, fdn, fidx = _np(dump), _np(g.cand), _np(g.cand_n), _np(fd), _np(g.idx[1])
    for b, n in enumerate(lengths):
        ec, _ = indexer.topk(d[b, 0, :n], wl.B, n)
        assert np.array_equal(cand[b, 0], ec)
        cn = int(cand_n[b, 0])
        ef, _ = indexer.hs_follower(fdn[b, 0, :cn], cand[b, 0], cn, wl.k)
        assert np.array_equal(fidx[b, 0], ef)


def test_repeated_calls_on_one_workspace(ctx):
    """Ten calls in a row on one workspace (interleaved with anchor and
    follower calls) select the same."""
    wl = shrunk(workload(3), capacity=8192, batch=4)
    inp = generate(wl)
    g = build_group(ctx, inp, dsa=False)
    g.score_topk(1)
    torch.cuda.synchronize()
    first = _np(g.idx[1]).copy()
    for _ in range(10):
        g.score_topk(1)
        g.hs_anchor(0)
        g.hs_follower(3)
    torch.cuda.synchronize()
    assert li.li_device_status(ctx, g.ws) == "LI_OK"
    assert np.array_equal(_np(g.idx[1]), first)
