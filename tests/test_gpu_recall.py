"""Selection quality on the GPU (li_attention_recall) against the oracle:
per-head attention-mass recall and mean-attention recall (LatentIndex
summary, Sec. 4.1, Sec. C.2, Sec. C.3, Sec. D.3), for random selections on
ragged prefixes and for the library's own selections (full LatentIndex,
hierarchical selection, and the IndexCache comparator, whose followers reuse
the anchor's selection) on a synthetic dense attention."""
import numpy as np
import pytest
import torch

import cross_layer_latent_b200 as li
from oracle import indexer, recall
from tests.gpu_setup import build_group, ref_latent
from workloads import generate, shrunk, workload

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
RTOL = 5e-5          # fp32 sums of up to K probabilities against fp64


@pytest.fixture(scope="module")
def ctx():
    c = li.Context(0)
    yield c
    c.close()


@pytest.mark.parametrize("rows,H,N,k,K", [(3, 8, 3000, 256, 256), (2, 4, 70000, 2048, 2048), (1, 2, 500, 64, 1000)])
def test_recall_matches_oracle(ctx, rows, H, N, k, K):
    rng = np.random.default_rng(rows * 100 + H)
    lengths = rng.integers(N // 2, N + 1, size=rows).astype(np.int32)
    lengths[0] = N
    p = np.zeros((rows, H, N), np.float32)
    for r in range(rows):
        p[r, :, :lengths[r]] = rng.dirichlet(np.full(lengths[r], 0.05), size=H).astype(np.float32)
    sel = np.full((rows, k), -1, np.int32)
    for r in range(rows):
        m = min(k, int(lengths[r])) - 3
        s = np.sort(rng.choice(int(lengths[r]), size=m, replace=False))
        sel[r, :m] = s
        sel[r, m] = N + 5                       # out of range: ignored
    rec, mrec = li.li_attention_recall(ctx, torch.from_numpy(p).to(DEV), torch.from_numpy(sel).to(DEV), K,
                                       lengths=torch.from_numpy(lengths).to(DEV))
    torch.cuda.synchronize()
    rec, mrec = rec.cpu().numpy(), mrec.cpu().numpy()
    for r in range(rows):
        n = int(lengths[r])
        pr = p[r, :, :n].astype(np.float64)
        want = recall.head_mass_recall(pr, sel[r][sel[r] < n], K)
        np.testing.assert_allclose(rec[r], want, rtol=RTOL, atol=1e-7)
        assert mrec[r] == pytest.approx(recall.mean_attention_recall(pr, sel[r][sel[r] < n], K), rel=RTOL)


def _synthetic_attention(inp, c64, l, b, beta=2.5):
    """Layer l's dense attention for sequence b: per head, the native logits
    q_h . k_s (keys k = W_K c) standardised over the prefix and sharpened by
    beta before the softmax."""
    n = int(inp.lengths[b])
    keys = c64[b, :n] @ inp.W_K[l].astype(np.float64).T
    logits = inp.q[l][b, 0].astype(np.float64) @ keys.T          # [H, n]
    z = (logits - logits.mean(axis=1, keepdims=True)) / logits.std(axis=1, keepdims=True)
    return recall.attention(beta * z, n)


def test_recall_of_the_library_selections(ctx):
    """Full LatentIndex, HS and IndexCache selections of a bf16 group, scored
    on the GPU against a synthetic attention, equal the oracle's recall of the
    same selections; full LatentIndex recalls what the DSA-style selection
    does (absorption is exact), and every recall lies in [0, 1]."""
    wl = shrunk(workload(1), capacity=6000)
    inp = generate(wl)
    g = build_group(ctx, inp)
    c64 = ref_latent(inp)
    K = wl.k
    sels = {"full": [], "dsa": [], "hs": [], "index_cache": []}
    for l in range(wl.group):
        g.score_topk(l)
        sels["full"].append(g.idx[l].clone())
        g.dsa_score_topk(l)
        sels["dsa"].append(g.idx[l].clone())
    g.hs_anchor(0)
    anchor = g.idx[0].clone()
    sels["hs"].append(anchor)
    sels["index_cache"].append(anchor)
    for l in range(1, wl.group):
        g.hs_follower(l)
        sels["hs"].append(g.idx[l].clone())
        sels["index_cache"].append(anchor)
    torch.cuda.synchronize()
    means = {m: [] for m in sels}
    for l in range(wl.group):
        p = np.stack([_synthetic_attention(inp, c64, l, b) for b in range(wl.batch)]).astype(np.float32)
        pd = torch.from_numpy(p).to(DEV)
        for m, ss in sels.items():
            rec, mrec = li.li_attention_recall(ctx, pd, ss[l][:, 0].contiguous(), K)
            torch.cuda.synchronize()
            rec, mrec = rec.cpu().numpy(), mrec.cpu().numpy()
            sel = ss[l][:, 0].cpu().numpy()
            for b in range(wl.batch):
                pr = p[b].astype(np.float64)
                np.testing.assert_allclose(rec[b], recall.head_mass_recall(pr, sel[b], K), rtol=RTOL, atol=1e-7)
                assert mrec[b] == pytest.approx(recall.mean_attention_recall(pr, sel[b], K), rel=RTOL)
                assert np.all((rec[b] >= 0) & (rec[b] <= 1 + 1e-5))
            means[m].append(float(rec.mean()))
    np.testing.assert_allclose(means["full"], means["dsa"], rtol=2e-3)


def test_recall_rejects_bad_arguments(ctx):
    p = torch.zeros(2, 4, 100, device=DEV)
    sel = torch.zeros(2, 8, dtype=torch.int32, device=DEV)
    with pytest.raises(li.LiError):                      # K below 1
        li.li_attention_recall(ctx, p, sel, 0)
    small = torch.zeros(16, dtype=torch.uint8, device=DEV)
    with pytest.raises(li.LiError):                      # workspace too small
        rec = torch.empty(2, 4, device=DEV)
        ctx.check(li._binding._lib.li_attention_recall(ctx.handle, li._binding._ptr(p), 2, 4, 100, None,
                                                       li._binding._ptr(sel), 8, 8, li._binding._ptr(rec), None,
                                                       li._binding._ptr(small), small.numel(), None))
