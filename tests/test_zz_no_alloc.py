"""The allocation-free scan-and-select entry point (li_score_topk_static),
called through the C ABI, against li_score_topk with a caller workspace on
the same inputs: two calls in a row must both reproduce it.  This file sorts
last so that it also runs after every other GPU test in the same process."""
import numpy as np
import pytest
import torch

import cross_layer_latent_b200 as li
from tests.gpu_setup import build_group
from workloads import generate, shrunk, workload

pytestmark = pytest.mark.gpu
DEV = "cuda:0"

CASES = {
    "v32-bf16-n3000": lambda: shrunk(workload(1), capacity=3000, queries=1),
    "long-e4m3-n5000": lambda: shrunk(workload(3), capacity=5000, batch=2),
    # 64 query rows of a prefill chunk: enough rows for the many-rows selection
    "prefill-bf16-64x20000": lambda: shrunk(workload(4), capacity=20000, queries=64),
}


@pytest.fixture(scope="module")
def ctx():
    c = li.Context(0)
    yield c
    c.close()


@pytest.mark.parametrize("name", list(CASES))
def test_static_scratch_matches_workspace_entry_point(ctx, name):
    wl = CASES[name]()
    inp = generate(wl)
    g = build_group(ctx, inp, dsa=False)
    rows = (wl.batch, wl.queries, wl.k)
    ref_idx = torch.empty(rows, dtype=torch.int32, device=DEV)
    ref_score = torch.empty(rows, device=DEV)
    li.li_score_topk(ctx, g.latent, g.query(0), wl.k, ref_idx, ref_score, None, g.ws)
    torch.cuda.synchronize()
    for call in range(2):
        idx = torch.full(rows, -7, dtype=torch.int32, device=DEV)
        score = torch.full(rows, float("nan"), device=DEV)
        status = torch.full((1,), -1, dtype=torch.int32, device=DEV)
        li.li_score_topk_static(ctx, g.latent, g.query(0), wl.k, idx, score, status)
        torch.cuda.synchronize()
        # the same kernels on the same inputs: identical bits
        assert torch.equal(idx, ref_idx), f"{name}: call {call} selected different tokens"
        assert torch.equal(score.view(torch.int32), ref_score.view(torch.int32)), f"{name}: call {call} scores"
        assert int(status.item()) == 0, f"{name}: call {call} device status {int(status.item())}"


def test_static_scratch_refuses_requests_beyond_its_size(ctx):
    # 16 sequences x 131072 positions of fp32 scores exceed the 8 MiB scratch;
    # the request is refused on the host before anything touches the data,
    # so the views below need no memory of their own
    base = torch.zeros(1, 1, 32, dtype=torch.bfloat16, device=DEV)
    cache = li.Cache(data=base.expand(16, 131072, 32), lengths=torch.zeros(16, dtype=torch.int32, device=DEV))
    q = li.Query(q=torch.zeros(16, 1, 16, 32, dtype=torch.bfloat16, device=DEV),
                 w=torch.zeros(16, 1, 16, device=DEV))
    out = torch.full((16, 1, 64), -5, dtype=torch.int32, device=DEV)
    with pytest.raises(li.LiError) as err:
        li.li_score_topk_static(ctx, cache, q, 64, out)
    assert "LI_ERR_WORKSPACE" in str(err.value) and "static" in str(err.value)
    torch.cuda.synchronize()
    assert np.all(out.cpu().numpy() == -5)          # nothing was enqueued
