"""The RoPE-compatible two-branch latent and segmented fp8 on the GPU.

* Append with the row transforms (LatentIndex summary, Sec. 3.1, Sec. A.2,
  Sec. D.2): an fp32 cache holds the transformed rows (checked against the
  oracle), and the bf16 / e4m3 / segmented-e4m3 caches hold exactly the
  codec of those fp32 rows, for the store path, the one-launch decode path
  and the multi-token GEMV path, at positions up to 131071.
* Scoring the rotated latent with absorbed post-RoPE queries reproduces each
  layer's native rotated keys (frequency-wise complex decoders, Sec. A.4):
  GPU scores against the oracle's native-key scores, selections bit-exact on
  the GPU's own scores.
* Segmented fp8 (Sec. B.2): the scan and the follower gather combine the two
  per-branch scales; scores match each layer's native rotated keys within
  the fp8 tolerance (the scan arithmetic on oracle-encoded segmented
  operands is pinned to 2e-5 M in test_gpu_stored_operands.py).
"""
import numpy as np
import pytest
import torch

import cross_layer_latent_b200 as li
from oracle import codecs, indexer, rope
from tests.helpers import RTOL, assert_scores_close, assert_selection_close, latent_format, rope_decoder_matrix
from workloads import generate, rope_inputs, shrunk, workload

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
SPLIT = 64          # the rotary branch [0, 64) gets the first scale, the NoPE branch the second


@pytest.fixture(scope="module")
def ctx():
    c = li.Context(0)
    yield c
    c.close()


def _np(t):
    if t.dtype == torch.bfloat16:
        return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)
    return t.detach().cpu().numpy()


def _transform(ri):
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(DEV)  # noqa: E731
    return li.LatentTransform(rope_offset=ri.rope_offset, rope_dim=ri.rope_dim, rope_sources=ri.sources,
                              inv_freq=t(ri.inv_freq), norm_offset=ri.norm_offset, norm_dim=ri.norm_dim,
                              gamma=t(ri.gamma), beta=t(ri.beta), eps=ri.eps)


def _caches(ctx, b, cap, d, starts, tf):
    out = {}
    for name, dt, split in (("f32", li.LI_F32, 0), ("bf16", li.LI_BF16, 0), ("e4m3", li.LI_E4M3, 0),
                            ("seg", li.LI_E4M3, SPLIT)):
        g = li.GroupIndexer(ctx, batch=b, capacity=cap, d_c=d, H=16, d_k=32, dtype=dt, k=8, transform=tf,
                            scale_split=split)
        g.latent.lengths.copy_(torch.tensor(starts, dtype=torch.int32))
        out[name] = g
    return out


def _tol(ref, ri):
    """fp32 transform error allowance: 2e-6 of each element plus the RMS of
    its own branch (the two branches differ in scale by orders of magnitude)."""
    rms = np.empty_like(ref)
    for a, b in ((ri.rope_offset, ri.rope_offset + ri.rope_dim), (ri.norm_offset, ri.norm_offset + ri.norm_dim)):
        rms[..., a:b] = np.sqrt(np.mean(ref[..., a:b] ** 2, axis=-1, keepdims=True))
    return 2e-6 * (np.abs(ref) + rms)


def _check_codecs(gs, rows_of, T):
    """Every quantised cache holds the codec of the fp32 cache's rows."""
    f32 = rows_of(gs["f32"].latent.data)
    assert np.array_equal(rows_of(gs["bf16"].latent.data).view(np.uint16), codecs.bf16_encode(f32))
    codes, scale = codecs.e4m3_quantize_rows(f32)
    assert np.array_equal(rows_of(gs["e4m3"].latent.data), codes)
    assert np.array_equal(rows_of(gs["e4m3"].latent.scale), scale)
    codes, scale = codecs.e4m3_quantize_rows_segmented(f32, SPLIT)
    assert np.array_equal(rows_of(gs["seg"].latent.data), codes)
    assert np.array_equal(rows_of(gs["seg"].latent.scale), scale)
    return f32


@pytest.mark.parametrize("sources", [1, 2])
def test_append_transform_store_path(ctx, sources):
    wl = workload(1)
    ri = rope_inputs(wl, sources=sources)
    fmt = latent_format(ri)
    rng = np.random.default_rng(40 + sources)
    b, T, d = 3, 40, wl.d_c
    starts = [0, 1000, 131072 - T]
    cap = 131072
    c = (rng.standard_normal((b, T, d)) / np.sqrt(wl.d_model)).astype(np.float32)
    c[1, 7] = 0.0                                 # a zero row: LayerNorm of a constant is its beta
    gs = _caches(ctx, b, cap, d, starts, _transform(ri))
    for g in gs.values():
        g.append(torch.from_numpy(c).to(DEV))
    torch.cuda.synchronize()
    rows_of = lambda t: np.stack([_np(t[i, starts[i]:starts[i] + T]) for i in range(b)])  # noqa: E731
    f32 = _check_codecs(gs, rows_of, T)
    for i in range(b):
        ref = rope.cache_rows(c[i].astype(np.float64), np.arange(starts[i], starts[i] + T), fmt)
        assert np.all(np.abs(f32[i] - ref) <= _tol(ref, ri)), f"seq {i}: max err {np.max(np.abs(f32[i] - ref))}"
    assert _np(gs["f32"].latent.lengths).tolist() == [s + T for s in starts]


@pytest.mark.parametrize("b,T", [(4, 1), (1, 1), (2, 5)])
def test_append_transform_projection_paths(ctx, b, T):
    """Decode (one launch) and multi-token (GEMV + store) appends from h:
    the transform of the GPU's own projection, checked against the oracle's
    transform of the same fp32 rows (taken from an untransformed append)."""
    wl = workload(3)
    ri = rope_inputs(wl)
    fmt = latent_format(ri)
    rng = np.random.default_rng(50 + b + 10 * T)
    cap, dm, d = 131072, wl.d_model, wl.d_c
    starts = [131071 - T - 3 * i for i in range(b)]
    h = (rng.standard_normal((b, T, dm)) / np.sqrt(dm)).astype(np.float32)
    W = (rng.standard_normal((d, dm)) / np.sqrt(dm)).astype(np.float32)
    gs = _caches(ctx, b, cap, d, starts, _transform(ri))
    plain = li.GroupIndexer(ctx, batch=b, capacity=cap, d_c=d, H=16, d_k=32, dtype=li.LI_F32, k=8)
    plain.latent.lengths.copy_(torch.tensor(starts, dtype=torch.int32))
    hd, Wd = torch.from_numpy(h).to(DEV), torch.from_numpy(W).to(DEV)
    for g in list(gs.values()) + [plain]:
        g.append(hd, Wd)
    torch.cuda.synchronize()
    rows_of = lambda t: np.stack([_np(t[i, starts[i]:starts[i] + T]) for i in range(b)])  # noqa: E731
    f32 = _check_codecs(gs, rows_of, T)
    c_gpu = rows_of(plain.latent.data)
    bound = np.abs(h) @ np.abs(W).T.astype(np.float64)
    assert np.all(np.abs(c_gpu - indexer.latent(h, W)) <= 1e-5 * bound + 1e-30)
    for i in range(b):
        ref = rope.cache_rows(c_gpu[i].astype(np.float64), np.arange(starts[i], starts[i] + T), fmt)
        assert np.all(np.abs(f32[i] - ref) <= _tol(ref, ri))


def test_append_transform_rejects_bad_ranges(ctx):
    g = li.GroupIndexer(ctx, batch=1, capacity=64, d_c=192, H=16, d_k=32, dtype=li.LI_BF16, k=8)
    inv = torch.ones(32, device=DEV)
    c = torch.zeros(1, 1, 192, device=DEV)
    bad = [li.LatentTransform(rope_offset=1, rope_dim=64, inv_freq=inv),          # odd start
           li.LatentTransform(rope_offset=160, rope_dim=64, inv_freq=inv),        # past the row
           li.LatentTransform(rope_dim=64, rope_sources=3, inv_freq=inv),         # partial frequency
           li.LatentTransform(rope_dim=64, inv_freq=None),
           li.LatentTransform(rope_dim=64, inv_freq=inv, norm_offset=32, norm_dim=64),   # overlap
           li.LatentTransform(norm_offset=64, norm_dim=128, eps=float("nan"))]
    for tf in bad:
        with pytest.raises(li.LiError):
            li.li_append_latent_ex(ctx, g.latent, c, None, 1, tf, g.ws)
    torch.cuda.synchronize()
    assert int(g.latent.lengths.item()) == 0


CASES = {
    "bf16-n3000": (lambda: shrunk(workload(1), capacity=3000), li.LI_BF16, 0, 1),
    "bf16-2src-n3000": (lambda: shrunk(workload(1), capacity=3000), li.LI_BF16, 0, 2),
    "e4m3-n4096x2": (lambda: shrunk(workload(3), capacity=4096, batch=2), li.LI_E4M3, 0, 1),
    "seg-e4m3-n4096x2": (lambda: shrunk(workload(3), capacity=4096, batch=2), li.LI_E4M3, SPLIT, 1),
}


def _two_branch_group(ctx, name):
    mk, dt, split, sources = CASES[name]
    wl = mk()
    inp = generate(wl)
    ri = rope_inputs(wl, sources=sources)
    g = li.GroupIndexer(ctx, batch=wl.batch, capacity=wl.capacity, d_c=wl.d_c, H=wl.heads, d_k=wl.d_k,
                        G=wl.group, dtype=dt, k=wl.k, B=wl.B, transform=_transform(ri), scale_split=split)
    maxlen = int(inp.lengths.max())
    g.append(torch.from_numpy(inp.latent[:, :maxlen]).to(DEV))
    g.set_lengths(torch.from_numpy(inp.lengths).to(DEV))
    Ws = []
    for l in range(wl.group):
        W, bias = rope_decoder_matrix(ri, l, wl.d_k, wl.d_c)
        Ws.append((W, bias))
        g.set_queries(l, torch.from_numpy(inp.q[l]).to(DEV), torch.from_numpy(W).to(DEV),
                      torch.from_numpy(inp.w[l]).to(DEV), b_K=torch.from_numpy(bias).to(DEV))
    torch.cuda.synchronize()
    return wl, inp, ri, g, Ws, split


@pytest.mark.parametrize("name", list(CASES))
def test_two_branch_scoring_reproduces_native_rotated_keys(ctx, name):
    wl, inp, ri, g, Ws, split = _two_branch_group(ctx, name)
    fmt = latent_format(ri)
    cdt = "bf16" if g.dtype == li.LI_BF16 else "e4m3"
    for l in range(wl.group):
        dump = torch.full((wl.batch, 1, wl.capacity), float("nan"), device=DEV)
        g.score_topk(l, dump=dump)
        torch.cuda.synchronize()
        assert li.li_device_status(ctx, g.ws) == "LI_OK"
        d, idx = _np(dump), _np(g.idx[l])
        d_coef = ri.d_re[l].astype(np.float64) + 1j * ri.d_im[l]
        for b in range(wl.batch):
            n = int(inp.lengths[b])
            pos = np.arange(n)
            c = inp.latent[b, :n].astype(np.float64)
            q, w = inp.q[l][b, 0], inp.w[l][b, 0]
            keys = rope.native_keys(c, pos, fmt, d_coef, ri.W_nope[l], ri.b_nope[l])
            native = indexer.dsa_score_keys(keys, q, w)
            qt, beta = indexer.absorb(q, *Ws[l])
            M = indexer.error_scale(rope.cache_rows(c, pos, fmt), qt, w)
            assert_scores_close(d[b, 0, :n], native, M, RTOL[cdt], f"{name} layer {l} seq {b} vs native keys")
            e, _ = indexer.topk(d[b, 0, :n], wl.k, n)
            assert np.array_equal(idx[b, 0], e), f"{name} layer {l} seq {b}: selection"
            assert_selection_close(idx[b, 0], native, M, wl.k, n, RTOL[cdt], f"{name} layer {l} seq {b}")


@pytest.mark.parametrize("name", ["bf16-n3000", "seg-e4m3-n4096x2"])
def test_two_branch_hs_path(ctx, name):
    """HS on the two-branch latent: the anchor's candidates and the
    followers' rescoring (row gathers; with segmented fp8 the two scales
    arrive by 8-byte copies and the split falls inside a gathered chunk)."""
    wl, inp, ri, g, Ws, split = _two_branch_group(ctx, name)
    fmt = latent_format(ri)
    cdt = "bf16" if g.dtype == li.LI_BF16 else "e4m3"
    dump = torch.full((wl.batch, 1, wl.capacity), float("nan"), device=DEV)
    g.hs_anchor(0, dump=dump)
    torch.cuda.synchronize()
    assert li.li_device_status(ctx, g.ws) == "LI_OK"
    cand, cand_n = _np(g.cand), _np(g.cand_n)
    d = _np(dump)
    for b in range(wl.batch):
        n = int(inp.lengths[b])
        ec, _ = indexer.topk(d[b, 0, :n], wl.B, n)
        assert np.array_equal(cand[b, 0], ec)
    fdump = torch.full((wl.batch, 1, wl.B), float("nan"), device=DEV)
    for l in range(1, wl.group):
        g.hs_follower(l, dump=fdump)
        torch.cuda.synchronize()
        assert li.li_device_status(ctx, g.ws) == "LI_OK"
        fd, fidx = _np(fdump), _np(g.idx[l])
        for b in range(wl.batch):
            cn = int(cand_n[b, 0])
            ef, _ = indexer.hs_follower(fd[b, 0, :cn], cand[b, 0], cn, wl.k)
            assert np.array_equal(fidx[b, 0], ef), f"{name} follower {l} seq {b}"
            toks = cand[b, 0, :cn]
            n = int(inp.lengths[b])
            c = inp.latent[b, :n].astype(np.float64)
            q, w = inp.q[l][b, 0], inp.w[l][b, 0]
            keys = rope.native_keys(c, np.arange(n), fmt, ri.d_re[l].astype(np.float64) + 1j * ri.d_im[l],
                                    ri.W_nope[l], ri.b_nope[l])
            native = indexer.dsa_score_keys(keys[toks], q, w)
            qt, _ = indexer.absorb(q, *Ws[l])
            M = indexer.error_scale(rope.cache_rows(c, np.arange(n), fmt)[toks], qt, w)
            assert_scores_close(fd[b, 0, :cn], native, M, RTOL[cdt], f"{name} follower {l} seq {b} vs native keys")
