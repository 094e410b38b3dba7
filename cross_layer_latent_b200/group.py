"""One layer group's indexer state on the GPU, wired through the C ABI.

LatentIndex (paperlayer summary of arXiv 2610.04635) keeps one shared latent
cache per group of G layers, built by the anchor (first) layer (Sec. 3.1);
each layer absorbs its decoder into its query and selects its own top-k
(Sec. 3.1, Sec. B.2); with hierarchical selection the anchor proposes B
candidates and the followers rescore only those (Sec. 3.2, Sec. C.4).  The
DSA-style comparison path keeps one key cache per layer (Sec. 1, Sec. B.3).

This module only allocates device buffers with torch and calls the library's
entry points in order; every arithmetic step runs in libli's kernels.
"""
from typing import List, Optional

import torch

from ._binding import (LI_BF16, LI_E4M3, LI_F32, Cache, Context, LatentTransform, Query, li_absorb_query,
                       li_absorb_query_group, li_append_latent, li_append_latent_ex, li_dsa_score_topk,
                       li_hs_anchor_candidates, li_hs_follower_refine, li_score_topk, workspace)

TORCH_DTYPE = {LI_F32: torch.float32, LI_BF16: torch.bfloat16, LI_E4M3: torch.uint8}


def _cache(batch, capacity, dim, dtype, device, scale_split: int = 0) -> Cache:
    scale = None
    if dtype == LI_E4M3:
        shape = (batch, capacity, 2) if scale_split else (batch, capacity)
        scale = torch.ones(*shape, dtype=torch.float32, device=device)
    return Cache(data=torch.zeros(batch, capacity, dim, dtype=TORCH_DTYPE[dtype], device=device),
                 lengths=torch.zeros(batch, dtype=torch.int32, device=device), scale=scale, dtype=dtype,
                 scale_split=scale_split)


class GroupIndexer:
    """Buffers and calls for one group: latent cache, per-layer absorbed
    queries and selections, HS candidates, optional DSA key caches."""

    def __init__(self, ctx: Context, *, batch: int, capacity: int, d_c: int, H: int, d_k: int, G: int = 4,
                 dtype: int = LI_BF16, k: int = 2048, B: Optional[int] = None, T: int = 1, dsa: bool = False,
                 device: Optional[str] = None, transform: Optional[LatentTransform] = None,
                 scale_split: int = 0):
        """transform: the two-branch latent's row transforms applied by every
        append to the shared latent (rotary branch rotated at the row's
        position, LayerNorm on the NoPE branch); scale_split > 0 stores the
        latent as segmented fp8 (E4M3 only)."""
        self.ctx = ctx
        self.transform = transform
        self.device = device or f"cuda:{ctx.device}"
        self.batch, self.capacity, self.d_c, self.H, self.d_k = batch, capacity, d_c, H, d_k
        self.G, self.dtype, self.k, self.B, self.T = G, dtype, k, B, T
        dev, tdt = self.device, TORCH_DTYPE[dtype]
        self.latent = _cache(batch, capacity, d_c, dtype, dev, scale_split)
        self.keys: List[Cache] = [_cache(batch, capacity, d_k, dtype, dev) for _ in range(G)] if dsa else []
        # per-layer queries, layer-major: layer l's are the contiguous slice [l]
        e4 = dtype == LI_E4M3
        self.q_abs_all = torch.zeros(G, batch, T, H, d_c, dtype=tdt, device=dev)
        self.q_abs_scale_all = torch.ones(G, batch, T, H, device=dev) if e4 else None
        self.w_all = torch.zeros(G, batch, T, H, device=dev)
        self.q_abs = list(self.q_abs_all.unbind(0))
        self.q_abs_scale = list(self.q_abs_scale_all.unbind(0)) if e4 else [None] * G
        self.w = list(self.w_all.unbind(0))
        self.q_raw = [torch.zeros(batch, T, H, d_k, dtype=tdt, device=dev) for _ in range(G)] if dsa else []
        self.q_raw_scale = [torch.ones(batch, T, H, device=dev) if e4 else None for _ in range(G)] if dsa else []
        self.beta: List[Optional[torch.Tensor]] = [None] * G
        self.q_pos: Optional[torch.Tensor] = None
        self.idx = [torch.full((batch, T, k), -1, dtype=torch.int32, device=dev) for _ in range(G)]
        self.score = [torch.zeros(batch, T, k, device=dev) for _ in range(G)]
        if B is not None:
            self.cand = torch.full((batch, T, B), -1, dtype=torch.int32, device=dev)
            self.cand_n = torch.zeros(batch, T, dtype=torch.int32, device=dev)
        self.ws = workspace(ctx, batch, T, capacity, H, k, B or 0, device=dev)

    # ------------------------------------------------------------ loading a prefix
    def load(self, lengths, W_K, q, w, latent=None, hidden=None, W_down=None, q_pos=None, dsa_keys=True):
        """Fill the caches with a prefix and set every layer's queries.

        lengths [batch] valid rows; latent [batch, >= max(lengths), d_c] fp32
        (or hidden [batch, ..., d_model] with W_down [d_c, d_model], built into
        the latent by the library); W_K per layer [d_k, d_c]; q per layer
        [batch, T, H, d_k]; w per layer [batch, T, H]; q_pos [batch, T] for
        prefill queries.  Arrays may be NumPy or torch; the DSA key caches (if
        any) receive key = W_K c, built by the library from the fp32 latent."""
        dev = self.device
        as_t = lambda x: torch.as_tensor(x).to(dev)  # noqa: E731
        lengths = as_t(lengths).to(torch.int32)
        maxlen = int(lengths.max().item())
        if hidden is not None:
            self.append(as_t(hidden)[:, :maxlen].contiguous(), as_t(W_down))
            c_src = self.latent.data[:, :maxlen].float().contiguous() if self.keys else None
        else:
            c_src = as_t(latent)[:, :maxlen].float().contiguous()
            self.append(c_src)
        self.set_lengths(lengths)
        for l, kc in enumerate(self.keys if dsa_keys else []):
            kc.lengths.zero_()
            li_append_latent(self.ctx, kc, c_src, as_t(W_K[l]).float().contiguous(), maxlen, self.ws)
            kc.lengths.copy_(lengths)
        if q_pos is not None:
            self.q_pos = as_t(q_pos).to(torch.int32).contiguous()
        for l in range(self.G):
            self.set_queries(l, as_t(q[l]).float().contiguous(), as_t(W_K[l]).float().contiguous(),
                             as_t(w[l]).float().contiguous())

    # ------------------------------------------------------------ construction (a1)
    def append(self, h: torch.Tensor, W_down: Optional[torch.Tensor] = None, stream=None):
        """Append T new tokens per sequence to the shared latent cache:
        h [batch, T, d_model] with W_down [d_c, d_model], or the fp32 latent
        [batch, T, d_c] itself when W_down is None."""
        li_append_latent_ex(self.ctx, self.latent, h, W_down, h.shape[1], self.transform, self.ws, stream)

    def append_keys(self, layer: int, h: torch.Tensor, W_k: Optional[torch.Tensor] = None, stream=None):
        """Append to layer `layer`'s DSA key cache (key = W_k h)."""
        li_append_latent(self.ctx, self.keys[layer], h, W_k, h.shape[1], self.ws, stream)

    def set_lengths(self, lengths: torch.Tensor):
        self.latent.lengths.copy_(lengths)
        for kc in self.keys:
            kc.lengths.copy_(lengths)

    # ------------------------------------------------------------ absorption (a2)
    def set_queries(self, layer: int, q: torch.Tensor, W_K: Optional[torch.Tensor], w: torch.Tensor,
                    b_K: Optional[torch.Tensor] = None, stream=None):
        """q [batch, T, H, d_k] (f32 or bf16), W_K [d_k, d_c] (same dtype),
        w [batch, T, H] f32.  Absorbs the decoder (and, for the DSA path,
        converts the raw query to the cache dtype)."""
        self.w[layer].copy_(w)
        beta = None
        if b_K is not None:
            beta = torch.zeros(self.batch, self.T, self.H, device=self.device)
        li_absorb_query(self.ctx, q, W_K, self.d_c, self.dtype, self.q_abs[layer], self.q_abs_scale[layer],
                        b_K=b_K, beta=beta, stream=stream)
        self.beta[layer] = beta
        if self.q_raw:
            li_absorb_query(self.ctx, q, None, self.d_k, self.dtype, self.q_raw[layer], self.q_raw_scale[layer],
                            stream=stream)

    def query(self, layer: int) -> Query:
        return Query(q=self.q_abs[layer], w=self.w[layer], q_scale=self.q_abs_scale[layer],
                     beta=self.beta[layer], q_pos=self.q_pos, dtype=self.dtype)

    def raw_query(self, layer: int) -> Query:
        return Query(q=self.q_raw[layer], w=self.w[layer], q_scale=self.q_raw_scale[layer], q_pos=self.q_pos,
                     dtype=self.dtype)

    # ------------------------------------------------------------ scoring and selection (a3-a7)
    def score_topk(self, layer: int, dump: Optional[torch.Tensor] = None, stream=None):
        li_score_topk(self.ctx, self.latent, self.query(layer), self.k, self.idx[layer], self.score[layer], dump,
                      self.ws, stream)
        return self.idx[layer]

    def set_group_queries(self, q: torch.Tensor, W_K: List[torch.Tensor], w: torch.Tensor, stream=None):
        """Training-aware instantiation (Sec. D.2): every layer's query and
        head weights come from the anchor's hidden state, so the group's
        queries arrive together.  q [batch, G, H, d_k] (f32 or bf16) is
        absorbed with the G decoders W_K[l] [d_k, d_c] (q's dtype) in one
        launch, stacked as q_group [batch, G, H, d_c]; w [batch, G, H] f32 is
        kept as the group's head weights (not copied)."""
        if self.T != 1:
            raise ValueError("the fused group scan stacks decode queries (T = 1)")
        if not hasattr(self, "q_group"):
            dev, G, b = self.device, self.G, self.batch
            self.q_group = torch.empty(b, G, self.H, self.d_c, dtype=TORCH_DTYPE[self.dtype], device=dev)
            self.q_group_scale = torch.empty(b, G, self.H, device=dev) if self.dtype == LI_E4M3 else None
            self.idx_group = torch.full((b, G, self.k), -1, dtype=torch.int32, device=dev)
            self.score_group = torch.zeros(b, G, self.k, device=dev)
            self.ws_group = workspace(self.ctx, b, G, self.capacity, self.H, self.k, 0, device=dev)
        li_absorb_query_group(self.ctx, q, W_K, self.d_c, self.dtype, self.q_group, self.q_group_scale, stream)
        self.w_group = w

    def fused_group_score_topk(self, dump: Optional[torch.Tensor] = None, stream=None):
        """Full LatentIndex for all G layers of a decode token with one pass
        over the shared latent: the queries set by set_group_queries are the
        G query rows of each sequence, and the scan takes up to 256 // H of
        them per MMA (G * H columns at G = 4, H = 64: one read of the latent
        for the whole group).  Selections land in idx_group [batch, G, k];
        dump, if given, is [batch, G, capacity]."""
        if not hasattr(self, "w_group"):
            raise RuntimeError("set_group_queries must come first")
        q = Query(q=self.q_group, w=self.w_group, q_scale=self.q_group_scale, beta=None, q_pos=None, dtype=self.dtype)
        li_score_topk(self.ctx, self.latent, q, self.k, self.idx_group, self.score_group, dump, self.ws_group, stream)
        return self.idx_group

    def hs_anchor(self, layer: int = 0, dump: Optional[torch.Tensor] = None, stream=None):
        li_hs_anchor_candidates(self.ctx, self.latent, self.query(layer), self.B, self.k, self.cand, self.cand_n,
                                self.idx[layer], self.score[layer], dump, self.ws, stream)
        return self.idx[layer]

    def hs_follower(self, layer: int, dump: Optional[torch.Tensor] = None, stream=None):
        li_hs_follower_refine(self.ctx, self.latent, self.query(layer), self.cand, self.cand_n, self.B, self.k,
                              self.idx[layer], self.score[layer], dump, self.ws, stream)
        return self.idx[layer]

    def dsa_score_topk(self, layer: int, dump: Optional[torch.Tensor] = None, stream=None):
        li_dsa_score_topk(self.ctx, self.keys[layer], self.raw_query(layer), self.k, self.idx[layer],
                          self.score[layer], dump, self.ws, stream)
        return self.idx[layer]

    def hs_step(self, stream=None):
        """One HS decode step of the group: anchor proposes, followers refine."""
        self.hs_anchor(0, stream=stream)
        for l in range(1, self.G):
            self.hs_follower(l, stream=stream)

    def full_step(self, stream=None):
        """Full-prefix LatentIndex: every layer scans the shared latent."""
        for l in range(self.G):
            self.score_topk(l, stream=stream)

    def dsa_step(self, stream=None):
        """DSA-style comparison: every layer scans its own key cache."""
        for l in range(self.G):
            self.dsa_score_topk(l, stream=stream)
