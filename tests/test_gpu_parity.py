"""Parity of the CUDA path (through the C ABI) with the CPU oracle."""
from dataclasses import replace

import numpy as np
import pytest
import torch

from oracle import codecs, indexer
from tests.helpers import RTOL, assert_scores_close, assert_selection_close
from workloads import generate, shrunk, workload

pytestmark = pytest.mark.gpu

li = pytest.importorskip("cross_layer_latent_b200")
from tests.gpu_setup import Reference, build_group, ref_latent  # noqa: E402

DEV = "cuda:0"


@pytest.fixture(scope="module")
def ctx():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    c = li.Context(0)
    yield c
    c.close()


def _np(t):
    if t.dtype == torch.bfloat16:
        return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)
    return t.detach().cpu().numpy()


# ------------------------------------------------------------------ a1: append (codecs bit-exact)

@pytest.mark.parametrize("dtype", ["bf16", "e4m3", "f32"])
def test_append_matches_codec_bit_exactly(ctx, dtype):
    rng = np.random.default_rng(5)
    b, cap, T, d = 3, 650, 300, 192
    c = (rng.standard_normal((b, T, d)) * 0.05).astype(np.float32)
    c[:, :, 7] *= 8
    c[1, 5] = 0.0
    cache = li.GroupIndexer(ctx, batch=b, capacity=cap, d_c=d, H=16, d_k=32, dtype={"bf16": li.LI_BF16,
                            "e4m3": li.LI_E4M3, "f32": li.LI_F32}[dtype], k=16).latent
    ws = li.workspace(ctx, b, 1, cap, 16, 16)
    cache.lengths.copy_(torch.tensor([0, 10, 400], dtype=torch.int32))
    li.li_append_latent(ctx, cache, torch.from_numpy(c).to(DEV), None, T, ws)
    torch.cuda.synchronize()
    assert _np(cache.lengths).tolist() == [300, 310, 400]      # the last one would overflow: unchanged
    assert li.li_device_status(ctx, ws) == "LI_ERR_CAPACITY"
    data = _np(cache.data)
    for i, start in ((0, 0), (1, 10)):
        rows = data[i, start:start + T]
        if dtype == "bf16":
            assert np.array_equal(rows.view(np.uint16), codecs.bf16_encode(c[i]))
        elif dtype == "e4m3":
            codes, scale = codecs.e4m3_quantize_rows(c[i])
            assert np.array_equal(rows, codes)
            assert np.array_equal(_np(cache.scale)[i, start:start + T], scale)
        else:
            assert np.array_equal(rows, c[i])
    assert not data[2].any()          # nothing written for the overflowing sequence


@pytest.mark.parametrize("b,T", [(2, 5), (4, 1), (8, 1), (1, 3)])
def test_append_with_projection(ctx, b, T):
    """Multi-token appends (GEMV, then a store launch) and decode-sized ones
    (one launch: the last block reduces the splits and stores)."""
    rng = np.random.default_rng(6 + 10 * b + T)
    cap, dm, d = 64, 7168, 192
    h = (rng.standard_normal((b, T, dm)) / np.sqrt(dm)).astype(np.float32)
    W = (rng.standard_normal((d, dm)) / np.sqrt(dm)).astype(np.float32)
    g32 = li.GroupIndexer(ctx, batch=b, capacity=cap, d_c=d, H=16, d_k=32, dtype=li.LI_F32, k=8)
    g16 = li.GroupIndexer(ctx, batch=b, capacity=cap, d_c=d, H=16, d_k=32, dtype=li.LI_BF16, k=8)
    g8 = li.GroupIndexer(ctx, batch=b, capacity=cap, d_c=d, H=16, d_k=32, dtype=li.LI_E4M3, k=8)
    for g in (g32, g16, g8):
        g.append(torch.from_numpy(h).to(DEV), torch.from_numpy(W).to(DEV))
    torch.cuda.synchronize()
    c_gpu = _np(g32.latent.data)[:, :T]
    c_ref = indexer.latent(h, W)
    bound = np.abs(h) @ np.abs(W).T.astype(np.float64)
    assert np.all(np.abs(c_gpu - c_ref) <= 1e-5 * bound + 1e-30)
    # the bf16 / e4m3 caches hold the codec of the same fp32 rows
    assert np.array_equal(_np(g16.latent.data)[:, :T].view(np.uint16), codecs.bf16_encode(c_gpu))
    codes, scale = codecs.e4m3_quantize_rows(c_gpu)
    assert np.array_equal(_np(g8.latent.data)[:, :T], codes)
    assert np.array_equal(_np(g8.latent.scale)[:, :T], scale)
    assert _np(g32.latent.lengths).tolist() == [T] * b


# ------------------------------------------------------------------ a2: absorption

def test_absorb_matches_oracle_and_codecs(ctx):
    rng = np.random.default_rng(7)
    n, H, dk, dc = 5, 64, 128, 192
    q = (rng.standard_normal((n, H, dk)) / np.sqrt(dk)).astype(np.float32)
    W = (rng.standard_normal((dk, dc)) / np.sqrt(dk)).astype(np.float32)
    bK = rng.standard_normal(dk).astype(np.float32)
    qd, Wd = torch.from_numpy(q).to(DEV), torch.from_numpy(W).to(DEV)
    out32 = torch.empty(n, H, dc, device=DEV)
    beta = torch.empty(n, H, device=DEV)
    li.li_absorb_query(ctx, qd, Wd, dc, li.LI_F32, out32, b_K=torch.from_numpy(bK).to(DEV), beta=beta)
    out16 = torch.empty(n, H, dc, dtype=torch.bfloat16, device=DEV)
    li.li_absorb_query(ctx, qd, Wd, dc, li.LI_BF16, out16)
    out8 = torch.empty(n, H, dc, dtype=torch.uint8, device=DEV)
    sc8 = torch.empty(n, H, device=DEV)
    li.li_absorb_query(ctx, qd, Wd, dc, li.LI_E4M3, out8, sc8)
    torch.cuda.synchronize()
    ref, bref = indexer.absorb(q, W, bK)
    bound = np.einsum("nhk,kc->nhc", np.abs(q), np.abs(W).astype(np.float64))
    assert np.all(np.abs(_np(out32) - ref) <= 1e-5 * bound + 1e-30)
    assert np.all(np.abs(_np(beta) - bref) <= 1e-5 * (np.abs(q) @ np.abs(bK)) + 1e-30)
    g32 = _np(out32)
    assert np.array_equal(_np(out16), codecs.bf16_encode(g32))
    codes, scale = codecs.e4m3_quantize_rows(g32)
    assert np.array_equal(_np(out8), codes) and np.array_equal(_np(sc8), scale)
    # the per-head kernel, given the shared decoder once per head, gives identical bits
    Wt = np.ascontiguousarray(np.broadcast_to(W, (H, dk, dc)))
    outt = torch.empty(n, H, dc, device=DEV)
    li.li_absorb_query(ctx, qd, torch.from_numpy(Wt).to(DEV), dc, li.LI_F32, outt, W_K_head_stride=dk * dc)
    torch.cuda.synchronize()
    assert np.array_equal(_np(outt), g32)
    # per-head decoders through the head stride
    Wh = (rng.standard_normal((H, dk, dc)) / np.sqrt(dk)).astype(np.float32)
    outh = torch.empty(n, H, dc, device=DEV)
    li.li_absorb_query(ctx, qd, torch.from_numpy(Wh).to(DEV), dc, li.LI_F32, outh, W_K_head_stride=dk * dc)
    torch.cuda.synchronize()
    refh, _ = indexer.absorb(q, Wh)
    boundh = np.einsum("nhk,hkc->nhc", np.abs(q), np.abs(Wh).astype(np.float64))
    assert np.all(np.abs(_np(outh) - refh) <= 1e-5 * boundh + 1e-30)


@pytest.mark.parametrize("n,H,dk,dc", [(4, 64, 128, 192), (1, 8, 32, 48), (40, 32, 128, 256)])
def test_absorb_bf16_inputs(ctx, n, H, dk, dc):
    """bf16 queries and decoder (the decode path's inputs) against the oracle
    on the decoded bf16 values, for decode, tiny and prefill-like shapes."""
    rng = np.random.default_rng(8 + n)
    q = torch.from_numpy((rng.standard_normal((n, H, dk)) / np.sqrt(dk)).astype(np.float32)).to(torch.bfloat16)
    W = torch.from_numpy((rng.standard_normal((dk, dc)) / np.sqrt(dk)).astype(np.float32)).to(torch.bfloat16)
    out = torch.empty(n, H, dc, device=DEV)
    li.li_absorb_query(ctx, q.to(DEV), W.to(DEV), dc, li.LI_F32, out)
    torch.cuda.synchronize()
    qf, Wf = q.float().numpy(), W.float().numpy()
    ref, _ = indexer.absorb(qf, Wf)
    bound = np.einsum("nhk,kc->nhc", np.abs(qf), np.abs(Wf).astype(np.float64))
    assert np.all(np.abs(_np(out) - ref) <= 1e-5 * bound + 1e-30)


# ------------------------------------------------------------------ a3 + a4, a5 + a6, a7 on workloads

CASES = {
    "tiny-f32": lambda: workload(0),
    "v32-bf16-n3000": lambda: shrunk(workload(1), capacity=3000, queries=1),
    "ragged-bf16": lambda: shrunk(workload(2), capacity=2500, batch=3, length_range=(700, 2500)),
    "long-e4m3-n5000": lambda: shrunk(workload(3), capacity=5000, batch=2),
    "long-e4m3-n70k": lambda: shrunk(workload(3), capacity=70000, batch=2, length_range=(66000, 70000)),
    # past 131072 positions the selections take the chunked multi-kernel path,
    # and the anchor selects its candidates and then its own top-k from the
    # candidates' scores in a second selection
    "long-e4m3-n140k": lambda: shrunk(workload(3), capacity=140000, batch=1),
}


@pytest.fixture(scope="module", params=list(CASES))
def case(request, ctx):
    wl = CASES[request.param]()
    inp = generate(wl)
    g = build_group(ctx, inp)
    return request.param, inp, g, ref_latent(inp)


def test_score_topk_parity(ctx, case):
    name, inp, g, c64 = case
    wl = inp.wl
    rtol = RTOL[wl.cache_dtype]
    dump = torch.full((wl.batch, 1, wl.capacity), float("nan"), device=DEV)
    for l in range(wl.group):
        g.score_topk(l, dump=dump)
        torch.cuda.synchronize()
        d = _np(dump)
        idx = _np(g.idx[l])
        sc = _np(g.score[l])
        for b in range(wl.batch):
            ref = Reference(inp, c64, l, b)
            n = ref.n
            assert_scores_close(d[b, 0, :n], ref.scores, ref.M, rtol, f"{name} layer {l} seq {b} scores")
            # selection on the dumped fp32 scores is exact
            exact_idx, exact_val = indexer.topk(d[b, 0, :n], wl.k, n)
            assert np.array_equal(idx[b, 0], exact_idx), f"{name} layer {l} seq {b}: top-k differs"
            keep = exact_idx >= 0
            assert np.array_equal(sc[b, 0][keep], d[b, 0, exact_idx[keep]])
            assert_selection_close(idx[b, 0], ref.scores, ref.M, wl.k, n, rtol, f"{name} layer {l} seq {b}")


def test_hs_parity(ctx, case):
    name, inp, g, c64 = case
    wl = inp.wl
    rtol = RTOL[wl.cache_dtype]
    dump = torch.full((wl.batch, 1, wl.capacity), float("nan"), device=DEV)
    g.hs_anchor(0, dump=dump)
    torch.cuda.synchronize()
    d = _np(dump)
    cand, cand_n = _np(g.cand), _np(g.cand_n)
    a_idx = _np(g.idx[0])
    for b in range(wl.batch):
        n = int(inp.lengths[b])
        ec, _ = indexer.topk(d[b, 0, :n], wl.B, n)
        assert np.array_equal(cand[b, 0], ec) and cand_n[b, 0] == min(wl.B, n)
        ea, _ = indexer.topk(d[b, 0, :n], wl.k, n)
        assert np.array_equal(a_idx[b, 0], ea)
        ref = Reference(inp, c64, 0, b)
        assert_selection_close(cand[b, 0], ref.scores, ref.M, wl.B, n, rtol, f"{name} candidates seq {b}")
    fdump = torch.full((wl.batch, 1, wl.B), float("nan"), device=DEV)
    for l in range(1, wl.group):
        g.hs_follower(l, dump=fdump)
        torch.cuda.synchronize()
        fd, fidx = _np(fdump), _np(g.idx[l])
        for b in range(wl.batch):
            cn = int(cand_n[b, 0])
            toks = cand[b, 0, :cn]
            ref = Reference(inp, c64, l, b)
            assert_scores_close(fd[b, 0, :cn], ref.scores[toks], ref.M[toks], rtol, f"{name} follower {l}")
            ef, _ = indexer.hs_follower(fd[b, 0, :cn], cand[b, 0], cn, wl.k)
            assert np.array_equal(fidx[b, 0], ef), f"{name} follower {l} seq {b}: selection differs"
            assert set(fidx[b, 0][fidx[b, 0] >= 0]) <= set(toks)


def test_dsa_parity(ctx, case):
    name, inp, g, c64 = case
    wl = inp.wl
    rtol = RTOL[wl.cache_dtype]
    dump = torch.full((wl.batch, 1, wl.capacity), float("nan"), device=DEV)
    for l in range(wl.group):
        g.dsa_score_topk(l, dump=dump)
        torch.cuda.synchronize()
        d, idx = _np(dump), _np(g.idx[l])
        for b in range(wl.batch):
            ref = Reference(inp, c64, l, b)
            n = ref.n
            assert_scores_close(d[b, 0, :n], ref.dsa_scores, ref.dsa_M, rtol, f"{name} DSA layer {l}")
            e, _ = indexer.topk(d[b, 0, :n], wl.k, n)
            assert np.array_equal(idx[b, 0], e)
            assert_selection_close(idx[b, 0], ref.dsa_scores, ref.dsa_M, wl.k, n, rtol, f"{name} DSA layer {l}")


# ------------------------------------------------------------------ invariants on the GPU (bit-exact)

def test_hs_with_full_budget_equals_full_scan(ctx):
    wl = shrunk(workload(1), capacity=1500)
    wl = replace(wl, B=1536, k=300)
    inp = generate(wl)
    g = build_group(ctx, inp, dsa=False)
    dump = torch.zeros(1, 1, wl.capacity, device=DEV)
    full = []
    for l in range(wl.group):
        g.score_topk(l, dump=dump)
        torch.cuda.synchronize()
        full.append((_np(g.idx[l]).copy(), _np(dump).copy()))
    g.hs_anchor(0)
    torch.cuda.synchronize()
    assert _np(g.cand_n)[0, 0] == 1500 and np.array_equal(_np(g.cand)[0, 0, :1500], np.arange(1500))
    assert np.array_equal(_np(g.idx[0]), full[0][0])
    fdump = torch.zeros(1, 1, wl.B, device=DEV)
    for l in range(1, wl.group):
        g.hs_follower(l, dump=fdump)
        torch.cuda.synchronize()
        assert np.array_equal(_np(g.idx[l]), full[l][0]), f"layer {l}"
        assert np.array_equal(_np(fdump)[0, 0, :1500].view(np.uint32), full[l][1][0, 0, :1500].view(np.uint32))


@pytest.mark.parametrize("dtype", ["bf16", "e4m3", "f32"])
def test_identity_decoder_reduces_to_dsa(ctx, dtype):
    wl = shrunk(workload(1), capacity=2000)
    wl = replace(wl, d_c=128, cache_dtype=dtype, group=1, k=100)
    inp = generate(wl)
    inp.W_K = [np.eye(128, dtype=np.float32)]
    g = build_group(ctx, inp)
    d1 = torch.zeros(1, 1, wl.capacity, device=DEV)
    d2 = torch.zeros(1, 1, wl.capacity, device=DEV)
    g.score_topk(0, dump=d1)
    i1 = _np(g.idx[0]).copy()
    g.dsa_score_topk(0, dump=d2)
    torch.cuda.synchronize()
    assert np.array_equal(i1, _np(g.idx[0]))
    assert np.array_equal(_np(d1)[0, 0, :2000].view(np.uint32), _np(d2)[0, 0, :2000].view(np.uint32))


# ------------------------------------------------------------------ a8: prefill-chunk scoring

def test_prefill_chunk_parity(ctx):
    wl = shrunk(workload(4), capacity=1500, queries=96)
    wl = replace(wl, k=200)
    inp = generate(wl)
    g = build_group(ctx, inp, dsa=False)
    dump = torch.full((1, wl.queries, wl.capacity), float("nan"), device=DEV)
    c64 = ref_latent(inp)
    for l in range(2):
        g.score_topk(l, dump=dump)
        torch.cuda.synchronize()
        d, idx = _np(dump), _np(g.idx[l])
        for t in range(0, wl.queries, 7):
            ref = Reference(inp, c64, l, 0, t)
            n = ref.n
            assert n == inp.q_pos[0, t] + 1
            assert_scores_close(d[0, t, :n], ref.scores, ref.M, RTOL["bf16"], f"prefill layer {l} query {t}")
            e, _ = indexer.topk(d[0, t, :n], wl.k, n)
            assert np.array_equal(idx[0, t], e)
            assert_selection_close(idx[0, t], ref.scores, ref.M, wl.k, n, RTOL["bf16"], f"prefill q{t}")
