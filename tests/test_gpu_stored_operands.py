"""Scan arithmetic on operands the oracle encodes itself.

The parity tests compare the GPU's scores with the oracle on the unquantised
latent, so they can only be as tight as the bf16 / e4m3 rounding of the
cache (rtol 2e-3 / 3e-2 of the error scale M).  A fault that moves a score by
less than that -- one head or one K slice dropped from a 64-head, 192-wide
contraction changes a score by about 1e-3 M -- would pass them.  Here every
operand of the scan is made on the CPU by the oracle's codecs: the cache rows
(bf16 codes, e4m3 codes with their per-token scale, segmented e4m3 with two
scales), the absorbed or raw queries (codes and per-head scales) and, for the
follower, the candidate list.  They are written straight into the library's
buffers, so the scan, the row gather and the prefill epilogue are the only
GPU steps.  The oracle then scores the decoded operands in fp64, and the GPU
must agree within 2e-5 M: fp32 accumulation over K <= 256 products and
H <= 256 heads, with margin, and 50x tighter than the effect of a dropped
head.  The fp32 cache is not in this test: its tensor-core path rounds both
operands to tf32 inside the MMA, a step the oracle does not model.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

import cross_layer_latent_b200 as li
from oracle import codecs, indexer
from tests.helpers import assert_scores_close
from workloads import generate, shrunk, workload

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TOL = 2e-5
SPLIT = 64


@pytest.fixture(scope="module")
def ctx():
    c = li.Context(0)
    yield c
    c.close()


def _bf16_tensor(codes: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(codes).view(np.int16)).view(torch.bfloat16).to(DEV)


def _encode(x32: np.ndarray, kind: str):
    """Oracle codes of float32 rows [..., d] and the decoded fp64 values."""
    if kind == "bf16":
        codes = codecs.bf16_encode(x32)
        return _bf16_tensor(codes), None, codecs.bf16_decode(codes).astype(np.float64)
    if kind == "seg":
        codes, scale = codecs.e4m3_quantize_rows_segmented(x32, SPLIT)
        dec = codecs.e4m3_dequantize_rows_segmented(codes, scale, SPLIT)
    else:
        codes, scale = codecs.e4m3_quantize_rows(x32)
        dec = codecs.e4m3_dequantize_rows(codes, scale)
    return torch.from_numpy(codes).to(DEV), torch.from_numpy(scale).to(DEV), dec


class Stored:
    """A group whose cache and queries hold oracle-encoded operands."""

    def __init__(self, ctx, wl, kind, dsa_layer=None):
        self.wl, self.kind = wl, kind
        self.inp = inp = generate(wl)
        dt = li.LI_BF16 if kind == "bf16" else li.LI_E4M3
        self.g = g = li.GroupIndexer(ctx, batch=wl.batch, capacity=wl.capacity, d_c=wl.d_c, H=wl.heads,
                                     d_k=wl.d_k, G=wl.group, dtype=dt, k=wl.k, B=wl.B, T=wl.queries,
                                     dsa=dsa_layer is not None, scale_split=SPLIT if kind == "seg" else 0)
        lat = inp.latent.astype(np.float32)
        data, scale, self.rows = _encode(lat, kind)
        g.latent.data.copy_(data.view(g.latent.data.dtype).reshape(g.latent.data.shape))
        if scale is not None:
            g.latent.scale.copy_(scale.reshape(g.latent.scale.shape))
        g.set_lengths(torch.from_numpy(inp.lengths).to(DEV))
        if inp.q_pos is not None:
            g.q_pos = torch.from_numpy(inp.q_pos.astype(np.int32)).to(DEV)
        qkind = "e4m3" if kind == "seg" else kind
        self.q = []
        for l in range(wl.group):
            qt, _ = indexer.absorb(inp.q[l], inp.W_K[l])             # fp64 [b, T, H, d_c]
            qd, qs, qdec = _encode(qt.astype(np.float32), qkind)
            g.q_abs[l].copy_(qd.view(g.q_abs[l].dtype).reshape(g.q_abs[l].shape))
            if qs is not None:
                g.q_abs_scale[l].copy_(qs.reshape(g.q_abs_scale[l].shape))
            g.w[l].copy_(torch.from_numpy(inp.w[l]).to(DEV))
            self.q.append(qdec)
        if dsa_layer is not None:
            l = dsa_layer
            keys = (inp.latent.astype(np.float64) @ inp.W_K[l].astype(np.float64).T).astype(np.float32)
            kd, ks, self.keys = _encode(keys, qkind)
            kc = g.keys[l]
            kc.data.copy_(kd.view(kc.data.dtype).reshape(kc.data.shape))
            if ks is not None:
                kc.scale.copy_(ks.reshape(kc.scale.shape))
            qd, qs, self.q_raw = _encode(inp.q[l].astype(np.float32), qkind)
            g.q_raw[l].copy_(qd.view(g.q_raw[l].dtype).reshape(g.q_raw[l].shape))
            if qs is not None:
                g.q_raw_scale[l].copy_(qs.reshape(g.q_raw_scale[l].shape))
        torch.cuda.synchronize()

    def check(self, got, rows, q, w, what):
        ref = indexer.score(rows, q, w)
        M = indexer.error_scale(rows, q, w)
        return assert_scores_close(got, ref, M, TOL, what)


CASES = {
    "bf16-n3000": (lambda: shrunk(workload(1), capacity=3000), "bf16"),
    "e4m3-n5000x2": (lambda: shrunk(workload(3), capacity=5000, batch=2), "e4m3"),
    "seg-e4m3-n4096x2": (lambda: shrunk(workload(3), capacity=4096, batch=2), "seg"),
    "ragged-bf16-n2500x3": (lambda: shrunk(workload(2), capacity=2500, batch=3), "bf16"),
}


@pytest.mark.parametrize("name", list(CASES))
def test_latent_scan_on_oracle_operands(ctx, name):
    mk, kind = CASES[name]
    s = Stored(ctx, mk(), kind)
    wl, inp = s.wl, s.inp
    worst = 0.0
    for l in (0, wl.group - 1):
        dump = torch.full((wl.batch, 1, wl.capacity), float("nan"), device=DEV)
        s.g.score_topk(l, dump=dump)
        torch.cuda.synchronize()
        assert li.li_device_status(ctx, s.g.ws) == "LI_OK"
        d = dump.cpu().numpy()
        for b in range(wl.batch):
            n = int(inp.lengths[b])
            worst = max(worst, s.check(d[b, 0, :n], s.rows[b, :n], s.q[l][b, 0], inp.w[l][b, 0],
                                       f"{name} layer {l} seq {b}"))
            assert np.all(np.isnan(d[b, 0, n:]))
    print(f"{name}: max |gpu - oracle| / M = {worst:.2e}")


@pytest.mark.parametrize("name", ["bf16-n3000", "e4m3-n5000x2", "seg-e4m3-n4096x2"])
def test_follower_gather_on_oracle_operands(ctx, name):
    """The row gather: an oracle-made candidate list (seeded, ascending, with
    the first and the last valid position) selects the rows to rescore."""
    mk, kind = CASES[name]
    s = Stored(ctx, mk(), kind)
    wl, inp = s.wl, s.inp
    rng = np.random.default_rng(11)
    cand = np.full((wl.batch, 1, wl.B), -1, np.int32)
    cand_n = np.zeros((wl.batch, 1), np.int32)
    for b in range(wl.batch):
        n = int(inp.lengths[b])
        m = min(wl.B, n) - (b % 2) * 7          # one list shorter than the budget
        pick = np.union1d([0, n - 1], rng.choice(n, size=m, replace=False))[:m]
        cand[b, 0, :m] = np.sort(pick)
        cand_n[b, 0] = m
    s.g.cand.copy_(torch.from_numpy(cand).to(DEV))
    s.g.cand_n.copy_(torch.from_numpy(cand_n).to(DEV))
    worst = 0.0
    for l in range(1, wl.group):
        fdump = torch.full((wl.batch, 1, wl.B), float("nan"), device=DEV)
        s.g.hs_follower(l, dump=fdump)
        torch.cuda.synchronize()
        assert li.li_device_status(ctx, s.g.ws) == "LI_OK"
        fd = fdump.cpu().numpy()
        for b in range(wl.batch):
            m = int(cand_n[b, 0])
            toks = cand[b, 0, :m]
            worst = max(worst, s.check(fd[b, 0, :m], s.rows[b, toks], s.q[l][b, 0], inp.w[l][b, 0],
                                       f"{name} follower {l} seq {b}"))
    print(f"{name} follower: max |gpu - oracle| / M = {worst:.2e}")


@pytest.mark.parametrize("kind", ["bf16", "e4m3"])
def test_dsa_key_scan_on_oracle_operands(ctx, kind):
    wl = shrunk(workload(1 if kind == "bf16" else 3), capacity=3000, batch=2)
    s = Stored(ctx, wl, kind, dsa_layer=1)
    inp = s.inp
    dump = torch.full((wl.batch, 1, wl.capacity), float("nan"), device=DEV)
    s.g.dsa_score_topk(1, dump=dump)
    torch.cuda.synchronize()
    assert li.li_device_status(ctx, s.g.ws) == "LI_OK"
    d = dump.cpu().numpy()
    worst = 0.0
    for b in range(wl.batch):
        n = int(inp.lengths[b])
        worst = max(worst, s.check(d[b, 0, :n], s.keys[b, :n], s.q_raw[b, 0], inp.w[1][b, 0], f"dsa {kind} seq {b}"))
    print(f"dsa {kind}: max |gpu - oracle| / M = {worst:.2e}")


def test_prefill_chunk_on_oracle_operands(ctx):
    """Several query rows per MMA (8 queries x 32 heads) and the epilogue
    that reads 64 tensor-memory columns per wait, with the causal mask."""
    wl = replace(shrunk(workload(4), capacity=1500, queries=96), k=200)
    s = Stored(ctx, wl, "bf16")
    inp = s.inp
    dump = torch.full((1, wl.queries, wl.capacity), float("nan"), device=DEV)
    s.g.score_topk(2, dump=dump)
    torch.cuda.synchronize()
    assert li.li_device_status(ctx, s.g.ws) == "LI_OK"
    d = dump.cpu().numpy()
    worst = 0.0
    for t in range(wl.queries):
        n = indexer.valid_length(inp.lengths[0], inp.q_pos[0, t])
        worst = max(worst, s.check(d[0, t, :n], s.rows[0, :n], s.q[2][0, t], inp.w[2][0, t], f"prefill query {t}"))
        assert np.all(np.isnan(d[0, t, n:]))
    print(f"prefill: max |gpu - oracle| / M = {worst:.2e}")


def test_a_dropped_head_would_fail(ctx):
    """The tolerance is tight enough to see one head's contribution: the
    oracle score without its largest-weight head misses the GPU's score by
    far more than 2e-5 M on most positions."""
    wl = shrunk(workload(1), capacity=3000)
    s = Stored(ctx, wl, "bf16")
    dump = torch.full((1, 1, wl.capacity), float("nan"), device=DEV)
    s.g.score_topk(0, dump=dump)
    torch.cuda.synchronize()
    d = dump.cpu().numpy()[0, 0]
    q, w = s.q[0][0, 0].copy(), s.inp.w[0][0, 0].astype(np.float64)
    h = int(np.argmax(np.abs(w)))
    w_drop = w.copy()
    w_drop[h] = 0
    rows = s.rows[0]
    ref_drop = indexer.score(rows, q, w_drop)
    M = indexer.error_scale(rows, q, w)
    err = np.abs(d - ref_drop) / M
    assert np.mean(err > TOL) > 0.3
