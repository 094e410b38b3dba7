"""Parity at the full decode sizes, in the launch configuration the benchmark
times: every selection is checked bit-exactly against the oracle's top-k of
the GPU's own scores, and the scores themselves against the oracle on a
sample of positions (random positions plus the neighbourhood of the k-th and
B-th scores), computed one by one in fp64."""
import numpy as np
import pytest
import torch

import cross_layer_latent_b200 as li
from oracle import indexer
from tests.gpu_setup import build_group
from tests.helpers import RTOL, assert_scores_close, assert_selection_close
from workloads import generate, workload

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def ctx():
    c = li.Context(0)
    yield c
    c.close()


def _np(t):
    return t.detach().cpu().numpy()


def _sample(rng, scores, n, budgets, size=1024):
    """Random valid positions plus the 64 positions ranked around each budget."""
    pos = set(rng.choice(n, size=min(size, n), replace=False).tolist())
    ranked = np.lexsort((np.arange(n), -scores[:n].astype(np.float64)))
    for k in budgets:
        lo, hi = max(0, min(k, n) - 32), min(n, min(k, n) + 32)
        pos.update(ranked[lo:hi].tolist())
    return np.array(sorted(pos), dtype=np.int64)


@pytest.mark.parametrize("index", [1, 2, 3])
def test_full_size_hs_and_dsa(ctx, index):
    wl = workload(index)
    inp = generate(wl)
    g = build_group(ctx, inp)
    rtol = RTOL[wl.cache_dtype]
    rng = np.random.default_rng(100 + index)

    # a5: anchor scan over the full prefix, candidates and its own top-k
    dump = torch.full((wl.batch, 1, wl.capacity), float("nan"), device=DEV)
    g.hs_anchor(0, dump=dump)
    torch.cuda.synchronize()
    assert li.li_device_status(ctx, g.ws) == "LI_OK"
    d, cand, cand_n, a_idx = _np(dump), _np(g.cand), _np(g.cand_n), _np(g.idx[0])
    for b in range(wl.batch):
        n = int(inp.lengths[b])
        ec, _ = indexer.topk(d[b, 0, :n], wl.B, n)
        assert np.array_equal(cand[b, 0], ec) and cand_n[b, 0] == min(wl.B, n), f"{wl.name} seq {b}: candidates"
        ea, _ = indexer.topk(d[b, 0, :n], wl.k, n)
        assert np.array_equal(a_idx[b, 0], ea), f"{wl.name} seq {b}: anchor top-k"
        pos = _sample(rng, d[b, 0], n, (wl.k, wl.B))
        c = inp.latent[b, pos].astype(np.float64)
        qt, _ = indexer.absorb(inp.q[0][b, 0], inp.W_K[0])
        ref = indexer.score(c, qt, inp.w[0][b, 0])
        M = indexer.error_scale(c, qt, inp.w[0][b, 0])
        assert_scores_close(d[b, 0, pos], ref, M, rtol, f"{wl.name} anchor seq {b}")

    # a6: every follower on the GPU's candidate lists
    fdump = torch.full((wl.batch, 1, wl.B), float("nan"), device=DEV)
    for l in range(1, wl.group):
        g.hs_follower(l, dump=fdump)
        torch.cuda.synchronize()
        assert li.li_device_status(ctx, g.ws) == "LI_OK"
        fd, fidx = _np(fdump), _np(g.idx[l])
        for b in range(wl.batch):
            cn = int(cand_n[b, 0])
            ef, _ = indexer.hs_follower(fd[b, 0, :cn], cand[b, 0], cn, wl.k)
            assert np.array_equal(fidx[b, 0], ef), f"{wl.name} follower {l} seq {b}"
            js = rng.choice(cn, size=min(512, cn), replace=False)
            toks = cand[b, 0, js]
            c = inp.latent[b, toks].astype(np.float64)
            qt, _ = indexer.absorb(inp.q[l][b, 0], inp.W_K[l])
            ref = indexer.score(c, qt, inp.w[l][b, 0])
            M = indexer.error_scale(c, qt, inp.w[l][b, 0])
            assert_scores_close(fd[b, 0, js], ref, M, rtol, f"{wl.name} follower {l} seq {b}")

    # a7: the DSA-style path of layer 0 (its key cache was built by the append kernel)
    g.dsa_score_topk(0, dump=dump)
    torch.cuda.synchronize()
    assert li.li_device_status(ctx, g.ws) == "LI_OK"
    d, idx = _np(dump), _np(g.idx[0])
    for b in range(wl.batch):
        n = int(inp.lengths[b])
        e, _ = indexer.topk(d[b, 0, :n], wl.k, n)
        assert np.array_equal(idx[b, 0], e), f"{wl.name} DSA seq {b}"
        pos = _sample(rng, d[b, 0], n, (wl.k,))
        keys = inp.latent[b, pos].astype(np.float64) @ inp.W_K[0].astype(np.float64).T
        ref = indexer.dsa_score_keys(keys, inp.q[0][b, 0], inp.w[0][b, 0])
        M = indexer.error_scale(keys, inp.q[0][b, 0], inp.w[0][b, 0])
        assert_scores_close(d[b, 0, pos], ref, M, rtol, f"{wl.name} DSA seq {b}")


def test_full_size_prefill_chunk(ctx):
    """The whole prefill chunk: 1024 queries at positions 64512..65535 against
    their causal prefixes of the 65536-row bf16 latent (H 32, d_c 256, k 2048;
    each layer keeps its own top-k, up to 2048 per query: LatentIndex summary,
    Sec. 3.1 and Sec. 4.1), through li_score_topk in the configuration the
    benchmark times.  A seeded sample of 32 query rows (the first and the last
    among them) in two layers is compared with the oracle element by element;
    every selection of those rows is bit-exact against the oracle's top-k of
    the dumped row and within the selection rule of the oracle's own scores.
    The launch must take the many-rows selection (32 keys a thread)."""
    wl = workload(4)
    inp = generate(wl)
    g = build_group(ctx, inp, dsa=False)
    rtol = RTOL[wl.cache_dtype]
    rng = np.random.default_rng(404)
    rows = np.unique(np.concatenate([[0, wl.queries - 1], rng.choice(wl.queries, 30, replace=False)]))
    dump = torch.full((1, wl.queries, wl.capacity), float("nan"), device=DEV)
    c64 = inp.latent[0].astype(np.float64)
    for l in range(2):
        li.li_profile_enable(ctx, True)
        li.li_profile_reset(ctx)
        g.score_topk(l, dump=dump)
        torch.cuda.synchronize()
        recs = li.li_profile_read(ctx)
        li.li_profile_enable(ctx, False)
        li.li_profile_reset(ctx)
        assert li.li_device_status(ctx, g.ws) == "LI_OK"
        sel = [r for r in recs if r["kernel"].startswith("topk")]
        assert len(sel) == 1 and sel[0]["kernel"] == "topk_cluster", [r["kernel"] for r in recs]
        cs = sel[0]["grid"] // wl.queries
        assert -(-wl.capacity // (cs * 512)) == 32, f"selection took {cs} CTAs a row, not 32 keys a thread"
        d, idx, sc = _np(dump), _np(g.idx[l]), _np(g.score[l])
        qt_all, _ = indexer.absorb(inp.q[l][0], inp.W_K[l])
        for t in rows:
            n = indexer.valid_length(inp.lengths[0], inp.q_pos[0, t])
            assert n == int(inp.q_pos[0, t]) + 1
            assert np.all(np.isnan(d[0, t, n:])), f"layer {l} query {t}: scores past its causal prefix"
            ref = indexer.score(c64[:n], qt_all[t], inp.w[l][0, t])
            M = indexer.error_scale(c64[:n], qt_all[t], inp.w[l][0, t])
            assert_scores_close(d[0, t, :n], ref, M, rtol, f"prefill layer {l} query {t}")
            e, ev = indexer.topk(d[0, t, :n], wl.k, n)
            assert np.array_equal(idx[0, t], e), f"prefill layer {l} query {t}: selection"
            keep = e >= 0
            got = np.where(sc[0, t][keep] == 0, np.float32(0), sc[0, t][keep])
            want = np.where(ev[keep] == 0, 0.0, ev[keep]).astype(np.float32)
            assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
            assert_selection_close(idx[0, t], ref, M, wl.k, n, rtol, f"prefill layer {l} query {t}")
