"""The benchmark's step issues the HS path's query absorptions on a second
stream, beside the anchor's append.  The selections it produces must be the
ones the same calls give in plain stream order, eagerly and from the captured
step graph (bit-exact: the same kernels on the same inputs)."""
import pytest
import torch

import bench
import cross_layer_latent_b200 as li
from workloads import shrunk, workload

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _serial_hs(step):
    g, wl = step.g, step.wl
    g.idx = step.hs_idx
    g.append(step.h_anchor, step.W_down)
    for l in range(wl.group):
        li.li_absorb_query(step.ctx, step.q[l], step.W_K[l], wl.d_c, g.dtype, g.q_abs[l], g.q_abs_scale[l])
    g.hs_anchor(0)
    for l in range(1, wl.group):
        g.hs_follower(l)


@pytest.mark.parametrize("idx,n", [(2, 6000), (3, 9000)])
def test_step_paths_match_plain_order(idx, n):
    ctx = li.Context(0)
    try:
        wl = shrunk(workload(idx), capacity=n, length_range=(n // 2, n))
        step = bench.Step(li, ctx, wl, 0, DEV)
        step.reset()
        _serial_hs(step)
        step.dsa_path()
        torch.cuda.synchronize()
        want = step.out_dev.clone()
        step.out_dev.fill_(-7)

        step.reset()
        step.hs_path()
        step.dsa_path()
        torch.cuda.synchronize()
        assert torch.equal(step.out_dev, want), "eager step with the absorptions aside"
        step.status("eager step")

        step.out_dev.fill_(-7)
        step.capture()
        for _ in range(2):
            step.reset()
            step.graphs[0].replay()
            step.graphs[1].replay()
        torch.cuda.synchronize()
        assert torch.equal(step.out_dev, want), "replayed step graphs"
        step.status("replayed step")
        step.graphs = None
    finally:
        ctx.close()
