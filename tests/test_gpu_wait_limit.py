"""Bounded waits: with a wait limit of 0 every wait of the scan that is not
already satisfied gives up (the first wait for copied data always is not);
the kernel records LI_ERR_DEVICE_TIMEOUT, lets its own copies land, frees
its tensor memory and returns, and the context stays usable."""
import numpy as np
import pytest
import torch

import cross_layer_latent_b200 as li
from oracle import indexer
from tests.gpu_setup import build_group
from workloads import generate, shrunk, workload

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def test_wait_that_runs_out_is_reported_and_the_context_recovers():
    ctx = li.Context(0)
    try:
        wl = shrunk(workload(1), capacity=3000, queries=1)
        inp = generate(wl)
        g = build_group(ctx, inp, dsa=False)
        assert li.li_device_status(ctx, g.ws) == "LI_OK"
        li.li_set_wait_limit(ctx, 0)
        try:
            g.score_topk(0)
            st = li.li_device_status(ctx, g.ws)
        finally:
            li.li_set_wait_limit(ctx, 2_000_000_000)
        assert st == "LI_ERR_DEVICE_TIMEOUT"
        dump = torch.full((wl.batch, 1, wl.capacity), float("nan"), device=DEV)
        g.score_topk(0, dump=dump)
        assert li.li_device_status(ctx, g.ws) == "LI_OK"
        d, idx = dump.cpu().numpy(), g.idx[0].cpu().numpy()
        n = int(inp.lengths[0])
        e, _ = indexer.topk(d[0, 0, :n], wl.k, n)
        assert np.array_equal(idx[0, 0], e)
        assert np.isfinite(d[0, 0, :n]).all()
    finally:
        ctx.close()


def test_follower_gather_wait_that_runs_out_is_reported_and_the_context_recovers():
    """The same for the row-gather scan, whose two loader warps hand each
    stage over through a barrier of their own."""
    ctx = li.Context(0)
    try:
        wl = shrunk(workload(1), capacity=3000, queries=1)
        inp = generate(wl)
        g = build_group(ctx, inp, dsa=False)
        g.hs_anchor(0)
        torch.cuda.synchronize()
        assert li.li_device_status(ctx, g.ws) == "LI_OK"
        li.li_set_wait_limit(ctx, 0)
        try:
            g.hs_follower(1)
            st = li.li_device_status(ctx, g.ws)
        finally:
            li.li_set_wait_limit(ctx, 2_000_000_000)
        assert st == "LI_ERR_DEVICE_TIMEOUT"
        g.hs_anchor(0)                     # fresh candidates (li_device_status cleared the status)
        fdump = torch.full((wl.batch, 1, wl.B), float("nan"), device=DEV)
        g.hs_follower(1, dump=fdump)
        assert li.li_device_status(ctx, g.ws) == "LI_OK"
        fd, fidx = fdump.cpu().numpy(), g.idx[1].cpu().numpy()
        cand, cand_n = g.cand.cpu().numpy(), g.cand_n.cpu().numpy()
        cn = int(cand_n[0, 0])
        ef, _ = indexer.hs_follower(fd[0, 0, :cn], cand[0, 0], cn, wl.k)
        assert np.array_equal(fidx[0, 0], ef)
        assert np.isfinite(fd[0, 0, :cn]).all()
    finally:
        ctx.close()
