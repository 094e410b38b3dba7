"""Fused group scan (the training-aware instantiation's full LatentIndex):
the G layers' absorbed decode queries stacked as G query rows, one scan of
the shared latent for the whole group.  Every layer's scores and selection
must equal those of its own per-layer scan (each output column of the
contraction is computed the same way whatever the number of columns), and
match the oracle within the score tolerance."""
from dataclasses import replace

import numpy as np
import pytest
import torch

import cross_layer_latent_b200 as li
from oracle import indexer
from tests.gpu_setup import Reference, build_group, ref_latent
from tests.helpers import RTOL, assert_scores_close
from workloads import generate, shrunk, workload

pytestmark = pytest.mark.gpu
DEV = "cuda:0"

CASES = {
    "tiny-f32": lambda: workload(0),
    "v32-bf16-n3000": lambda: shrunk(workload(1), capacity=3000, queries=1),
    "long-e4m3-n5000": lambda: shrunk(workload(3), capacity=5000, batch=2),
    # G = 8 at H = 64: 512 query columns, two passes of 4 layers each
    "g8-e4m3-n4100": lambda: replace(shrunk(workload(3), capacity=4100, batch=2), group=8),
}


@pytest.fixture(scope="module")
def ctx():
    c = li.Context(0)
    yield c
    c.close()


@pytest.mark.parametrize("name", list(CASES))
def test_fused_group_scan_equals_per_layer_scans(ctx, name):
    wl = CASES[name]()
    inp = generate(wl)
    g = build_group(ctx, inp, dsa=False)
    c64 = ref_latent(inp)
    per_layer = []
    for l in range(wl.group):
        dump = torch.full((wl.batch, 1, wl.capacity), float("nan"), device=DEV)
        g.score_topk(l, dump=dump)
        torch.cuda.synchronize()
        per_layer.append((dump.cpu().numpy()[:, 0], g.idx[l].cpu().numpy()[:, 0]))
    # the group's queries stacked [batch, G, H, d_k], absorbed in one launch
    q_stack = torch.from_numpy(np.ascontiguousarray(np.stack([inp.q[l][:, 0] for l in range(wl.group)], axis=1)))
    w_stack = torch.from_numpy(np.ascontiguousarray(np.stack([inp.w[l][:, 0] for l in range(wl.group)], axis=1)))
    W_K = [torch.from_numpy(inp.W_K[l]).to(DEV).contiguous() for l in range(wl.group)]
    g.set_group_queries(q_stack.to(DEV), W_K, w_stack.to(DEV))
    gdump = torch.full((wl.batch, wl.group, wl.capacity), float("nan"), device=DEV)
    g.fused_group_score_topk(dump=gdump)
    # the group absorb writes the per-layer absorb's values, stacked
    for l in range(wl.group):
        assert torch.equal(g.q_group[:, l], g.q_abs[l][:, 0]), f"{name} layer {l}: absorbed queries differ"
        if g.q_group_scale is not None:
            assert torch.equal(g.q_group_scale[:, l], g.q_abs_scale[l][:, 0])
    torch.cuda.synchronize()
    assert li.li_device_status(ctx, g.ws_group) == "LI_OK"
    gd, gidx = gdump.cpu().numpy(), g.idx_group.cpu().numpy()
    for l in range(wl.group):
        d, idx = per_layer[l]
        for b in range(wl.batch):
            n = int(inp.lengths[b])
            assert np.array_equal(gd[b, l, :n], d[b, :n]), f"{name} layer {l} seq {b}: scores differ"
            assert np.array_equal(gidx[b, l], idx[b]), f"{name} layer {l} seq {b}: selection differs"
            e, _ = indexer.topk(gd[b, l, :n], wl.k, n)
            assert np.array_equal(gidx[b, l], e)
            ref = Reference(inp, c64, l, b)
            assert_scores_close(gd[b, l, :n], ref.scores, ref.M, RTOL[wl.cache_dtype], f"{name} fused layer {l}")


def test_group_absorb_rejects_bad_arguments(ctx):
    q = torch.zeros(2, 9, 16, 32, device=DEV)
    W = [torch.zeros(32, 64, device=DEV) for _ in range(9)]
    out = torch.zeros(2, 9, 16, 64, device=DEV)
    with pytest.raises(li.LiError):                      # more than 8 layers
        li.li_absorb_query_group(ctx, q, W, 64, li.LI_F32, out)
    q4 = q[:, :4].contiguous()
    out4 = out[:, :4].contiguous()
    with pytest.raises(li.LiError):                      # a decoder off 16-byte alignment
        li.li_absorb_query_group(ctx, q4, [W[0], W[1], W[2], W[3].view(-1)[1:].view(-1)[:32 * 64 - 1]], 64,
                                 li.LI_F32, out4)
    with pytest.raises(li.LiError):                      # e4m3 output without scales
        li.li_absorb_query_group(ctx, q4, W[:4], 64, li.LI_E4M3, out4.to(torch.uint8))
    torch.cuda.synchronize()
    assert not out4.any()
