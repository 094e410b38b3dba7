"""ctypes binding of libli (include/li.h): argument marshalling only.

Every function here has the name of the C entry point it calls and forwards
device pointers taken from torch tensors; all arithmetic runs in the
library's CUDA kernels.  Importing fails loudly when libli.so is missing:
there is no fallback path.
"""
import ctypes
import os
from dataclasses import dataclass
from typing import List, Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libli.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m cross_layer_latent_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

# li_status / li_dtype values (include/li.h)
LI_OK = 0
STATUS_NAMES = {0: "LI_OK", 1: "LI_ERR_ARG", 2: "LI_ERR_SHAPE", 3: "LI_ERR_DTYPE", 4: "LI_ERR_ALIGN",
                5: "LI_ERR_WORKSPACE", 6: "LI_ERR_CAPACITY", 7: "LI_ERR_CUDA",
                8: "LI_ERR_DEVICE_TIMEOUT", 9: "LI_ERR_UNSUPPORTED", 10: "LI_ERR_INDEX"}
STATUS = {v: k for k, v in STATUS_NAMES.items()}
LI_F32, LI_BF16, LI_E4M3 = 0, 1, 2
_DTYPE_CODE = {torch.float32: LI_F32, torch.bfloat16: LI_BF16, torch.float8_e4m3fn: LI_E4M3,
               torch.uint8: LI_E4M3}


class LiError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status
        self.name = STATUS_NAMES.get(status, str(status))


class c_li_cache(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("lengths", ctypes.c_void_p),
                ("batch", ctypes.c_int32), ("capacity", ctypes.c_int32), ("dim", ctypes.c_int32),
                ("dtype", ctypes.c_int), ("scale_split", ctypes.c_int32)]


class c_li_latent_transform(ctypes.Structure):
    _fields_ = [("rope_offset", ctypes.c_int32), ("rope_dim", ctypes.c_int32), ("rope_sources", ctypes.c_int32),
                ("inv_freq", ctypes.c_void_p), ("norm_offset", ctypes.c_int32), ("norm_dim", ctypes.c_int32),
                ("norm_gamma", ctypes.c_void_p), ("norm_beta", ctypes.c_void_p), ("norm_eps", ctypes.c_float)]


class c_li_query(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("dtype", ctypes.c_int), ("q_scale", ctypes.c_void_p),
                ("beta", ctypes.c_void_p), ("w", ctypes.c_void_p), ("T", ctypes.c_int32),
                ("H", ctypes.c_int32), ("q_pos", ctypes.c_void_p)]


class c_li_profile_record(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_char * 48), ("ms", ctypes.c_float), ("grid", ctypes.c_int32),
                ("block", ctypes.c_int32), ("smem", ctypes.c_int32)]


_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_sigs = {
    "li_create": (_I, [ctypes.POINTER(_P), _I]),
    "li_destroy": (_I, [_P]),
    "li_last_error": (ctypes.c_char_p, [_P]),
    "li_status_string": (ctypes.c_char_p, [_I]),
    "li_workspace_bytes": (_SZ, [_P, _I, _I, _I, _I, _I, _I]),
    "li_device_status": (_I, [_P, _P, _P, ctypes.POINTER(_I)]),
    "li_set_wait_limit": (_I, [_P, ctypes.c_uint64]),
    "li_append_latent": (_I, [_P, ctypes.POINTER(c_li_cache), _P, _I, _I, _P, _I, _P, _SZ, _P]),
    "li_append_latent_ex": (_I, [_P, ctypes.POINTER(c_li_cache), _P, _I, _I, _P, _I,
                                 ctypes.POINTER(c_li_latent_transform), _P, _SZ, _P]),
    "li_absorb_query_group": (_I, [_P, _P, _I, _I, _I, _I, _I, ctypes.POINTER(_P), _I, _I, _P, _P, _P]),
    "li_absorb_query": (_I, [_P, _P, _I, _I, _I, _I, _P, _I64, _P, _I64, _I, _I, _P, _P, _P, _P]),
    "li_score_topk": (_I, [_P, ctypes.POINTER(c_li_cache), ctypes.POINTER(c_li_query), _I, _P, _P, _P, _P,
                           _SZ, _P]),
    "li_score_topk_static": (_I, [_P, ctypes.POINTER(c_li_cache), ctypes.POINTER(c_li_query), _I, _P, _P, _P,
                                  _P]),
    "li_hs_anchor_candidates": (_I, [_P, ctypes.POINTER(c_li_cache), ctypes.POINTER(c_li_query), _I, _I, _P,
                                     _P, _P, _P, _P, _P, _SZ, _P]),
    "li_hs_follower_refine": (_I, [_P, ctypes.POINTER(c_li_cache), ctypes.POINTER(c_li_query), _P, _P, _I, _I,
                                   _P, _P, _P, _P, _SZ, _P]),
    "li_dsa_score_topk": (_I, [_P, ctypes.POINTER(c_li_cache), ctypes.POINTER(c_li_query), _I, _P, _P, _P, _P,
                               _SZ, _P]),
    "li_topk": (_I, [_P, _P, _I, _I, _I64, _P, _I, _P, _P, _P, _SZ, _P]),
    "li_recall_workspace_bytes": (_SZ, [_P, _I, _I, _I, _I]),
    "li_attention_recall": (_I, [_P, _P, _I, _I, _I, _P, _P, _I, _I, _P, _P, _P, _SZ, _P]),
    "li_set_trace": (_I, [_P, _P, _SZ]),
    "li_profile_enable": (_I, [_P, _I]),
    "li_profile_read": (_I, [_P, ctypes.POINTER(c_li_profile_record), _I, ctypes.POINTER(_I)]),
    "li_profile_reset": (_I, [_P]),
}
for _name, (_res, _args) in _sigs.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTED = tuple(_sigs)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _dtype(t: torch.Tensor) -> int:
    return _DTYPE_CODE[t.dtype]


class Context:
    """Owns one li_ctx (host state only)."""

    def __init__(self, device: int = 0):
        h = ctypes.c_void_p()
        st = _lib.li_create(ctypes.byref(h), int(device))
        if st != LI_OK:
            raise LiError(st, f"li_create(device={device}) failed")
        self.handle = h
        self.device = device

    def check(self, status: int):
        if status != LI_OK:
            msg = _lib.li_last_error(self.handle)
            raise LiError(status, msg.decode() if msg else "")

    def close(self):
        if self.handle:
            _lib.li_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


@dataclass
class Cache:
    """A latent or key cache: data [batch, capacity, dim] (float32, bfloat16 or
    uint8 e4m3 codes), scale [batch, capacity] float32 (e4m3 only; with
    segmented fp8, scale_split > 0, [batch, capacity, 2]), lengths [batch]
    int32."""
    data: torch.Tensor
    lengths: torch.Tensor
    scale: Optional[torch.Tensor] = None
    dtype: Optional[int] = None
    scale_split: int = 0

    def c(self) -> c_li_cache:
        b, cap, dim = self.data.shape
        dt = self.dtype if self.dtype is not None else _dtype(self.data)
        return c_li_cache(_ptr(self.data), _ptr(self.scale), _ptr(self.lengths), b, cap, dim, dt,
                          int(self.scale_split))


@dataclass
class LatentTransform:
    """The two-branch latent's row transforms (li_latent_transform): rotary
    range [rope_offset, rope_offset + rope_dim) with inv_freq [rope_dim /
    (2 rope_sources)] float32, LayerNorm range [norm_offset, norm_offset +
    norm_dim) with optional gamma / beta [norm_dim] float32."""
    rope_offset: int = 0
    rope_dim: int = 0
    rope_sources: int = 1
    inv_freq: Optional[torch.Tensor] = None
    norm_offset: int = 0
    norm_dim: int = 0
    gamma: Optional[torch.Tensor] = None
    beta: Optional[torch.Tensor] = None
    eps: float = 1e-6

    def c(self) -> c_li_latent_transform:
        return c_li_latent_transform(self.rope_offset, self.rope_dim, self.rope_sources, _ptr(self.inv_freq),
                                     self.norm_offset, self.norm_dim, _ptr(self.gamma), _ptr(self.beta),
                                     float(self.eps))


@dataclass
class Query:
    """Queries of one layer: q [batch, T, H, dim], w [batch, T, H] float32,
    optional q_scale / beta [batch, T, H] float32 and q_pos [batch, T] int32."""
    q: torch.Tensor
    w: torch.Tensor
    q_scale: Optional[torch.Tensor] = None
    beta: Optional[torch.Tensor] = None
    q_pos: Optional[torch.Tensor] = None
    dtype: Optional[int] = None

    def c(self) -> c_li_query:
        b, T, H, dim = self.q.shape
        dt = self.dtype if self.dtype is not None else _dtype(self.q)
        return c_li_query(_ptr(self.q), dt, _ptr(self.q_scale), _ptr(self.beta), _ptr(self.w), T, H,
                          _ptr(self.q_pos))


def li_create(device: int = 0) -> Context:
    return Context(device)


def li_destroy(ctx: Context):
    ctx.close()


def li_status_string(status: int) -> str:
    return _lib.li_status_string(int(status)).decode()


def li_workspace_bytes(ctx: Optional[Context], batch: int, T: int, capacity: int, H: int, k: int, B: int) -> int:
    return int(_lib.li_workspace_bytes(ctx.handle if ctx else None, batch, T, capacity, H, k, B))


def workspace(ctx: Context, batch: int, T: int, capacity: int, H: int, k: int, B: int = 0,
              device=None) -> torch.Tensor:
    """A zero-filled workspace of li_workspace_bytes(...) bytes (256-byte aligned)."""
    n = li_workspace_bytes(ctx, batch, T, capacity, H, k, B)
    ws = torch.zeros(n, dtype=torch.uint8, device=device or f"cuda:{ctx.device}")
    assert ws.data_ptr() % 256 == 0
    return ws


def li_device_status(ctx: Context, ws: torch.Tensor, stream=None) -> str:
    out = ctypes.c_int(0)
    ctx.check(_lib.li_device_status(ctx.handle, _ptr(ws), _stream(stream), ctypes.byref(out)))
    return STATUS_NAMES.get(out.value, str(out.value))


def li_set_wait_limit(ctx: Context, ns: int):
    ctx.check(_lib.li_set_wait_limit(ctx.handle, int(ns)))


def li_append_latent(ctx: Context, cache: Cache, h: torch.Tensor, W_down: Optional[torch.Tensor], T: int,
                     ws: torch.Tensor, stream=None):
    d_model = h.shape[-1]
    cc = cache.c()
    ctx.check(_lib.li_append_latent(ctx.handle, ctypes.byref(cc), _ptr(h), _dtype(h), d_model, _ptr(W_down),
                                    int(T), _ptr(ws), ws.numel(), _stream(stream)))


def li_append_latent_ex(ctx: Context, cache: Cache, h: torch.Tensor, W_down: Optional[torch.Tensor], T: int,
                        tf: Optional[LatentTransform], ws: torch.Tensor, stream=None):
    d_model = h.shape[-1]
    cc = cache.c()
    ct = tf.c() if tf is not None else None
    ctx.check(_lib.li_append_latent_ex(ctx.handle, ctypes.byref(cc), _ptr(h), _dtype(h), d_model, _ptr(W_down),
                                       int(T), ctypes.byref(ct) if ct is not None else None, _ptr(ws), ws.numel(),
                                       _stream(stream)))


def li_absorb_query(ctx: Context, q: torch.Tensor, W_K: Optional[torch.Tensor], d_c: int, out_dtype: int,
                    q_abs: torch.Tensor, q_abs_scale: Optional[torch.Tensor] = None,
                    b_K: Optional[torch.Tensor] = None, beta: Optional[torch.Tensor] = None,
                    W_K_head_stride: int = 0, b_K_head_stride: int = 0, stream=None):
    """q [..., H, d_k] -> q_abs [..., H, d_c] (n_tok = product of the leading dims)."""
    H, d_k = q.shape[-2], q.shape[-1]
    n_tok = q.numel() // (H * d_k)
    ctx.check(_lib.li_absorb_query(ctx.handle, _ptr(q), _dtype(q), n_tok, H, d_k, _ptr(W_K), int(W_K_head_stride),
                                   _ptr(b_K), int(b_K_head_stride), int(d_c), int(out_dtype), _ptr(q_abs),
                                   _ptr(q_abs_scale), _ptr(beta), _stream(stream)))


def li_score_topk(ctx: Context, cache: Cache, query: Query, k: int, out_idx: torch.Tensor,
                  out_score: Optional[torch.Tensor], scores_dump: Optional[torch.Tensor], ws: torch.Tensor,
                  stream=None):
    cc, qq = cache.c(), query.c()
    ctx.check(_lib.li_score_topk(ctx.handle, ctypes.byref(cc), ctypes.byref(qq), int(k), _ptr(out_idx),
                                 _ptr(out_score), _ptr(scores_dump), _ptr(ws), ws.numel(), _stream(stream)))


def li_score_topk_static(ctx: Context, cache: Cache, query: Query, k: int, out_idx: torch.Tensor,
                         out_score: Optional[torch.Tensor] = None, device_status: Optional[torch.Tensor] = None,
                         stream=None):
    """li_score_topk with the library's fixed internal scratch instead of a workspace."""
    cc, qq = cache.c(), query.c()
    ctx.check(_lib.li_score_topk_static(ctx.handle, ctypes.byref(cc), ctypes.byref(qq), int(k), _ptr(out_idx),
                                        _ptr(out_score), _ptr(device_status), _stream(stream)))


def li_dsa_score_topk(ctx: Context, key_cache: Cache, query: Query, k: int, out_idx: torch.Tensor,
                      out_score: Optional[torch.Tensor], scores_dump: Optional[torch.Tensor], ws: torch.Tensor,
                      stream=None):
    cc, qq = key_cache.c(), query.c()
    ctx.check(_lib.li_dsa_score_topk(ctx.handle, ctypes.byref(cc), ctypes.byref(qq), int(k), _ptr(out_idx),
                                     _ptr(out_score), _ptr(scores_dump), _ptr(ws), ws.numel(), _stream(stream)))


def li_hs_anchor_candidates(ctx: Context, cache: Cache, query: Query, B: int, k: int, cand: torch.Tensor,
                            cand_n: torch.Tensor, anchor_idx: torch.Tensor, anchor_score: Optional[torch.Tensor],
                            scores_dump: Optional[torch.Tensor], ws: torch.Tensor, stream=None):
    cc, qq = cache.c(), query.c()
    ctx.check(_lib.li_hs_anchor_candidates(ctx.handle, ctypes.byref(cc), ctypes.byref(qq), int(B), int(k),
                                           _ptr(cand), _ptr(cand_n), _ptr(anchor_idx), _ptr(anchor_score),
                                           _ptr(scores_dump), _ptr(ws), ws.numel(), _stream(stream)))


def li_hs_follower_refine(ctx: Context, cache: Cache, query: Query, cand: torch.Tensor, cand_n: torch.Tensor,
                          B: int, k: int, out_idx: torch.Tensor, out_score: Optional[torch.Tensor],
                          scores_dump: Optional[torch.Tensor], ws: torch.Tensor, stream=None):
    cc, qq = cache.c(), query.c()
    ctx.check(_lib.li_hs_follower_refine(ctx.handle, ctypes.byref(cc), ctypes.byref(qq), _ptr(cand),
                                         _ptr(cand_n), int(B), int(k), _ptr(out_idx), _ptr(out_score),
                                         _ptr(scores_dump), _ptr(ws), ws.numel(), _stream(stream)))


def li_absorb_query_group(ctx: Context, q: torch.Tensor, W_K: List[torch.Tensor], d_c: int, out_dtype: int,
                          q_abs: torch.Tensor, q_abs_scale: Optional[torch.Tensor] = None, stream=None):
    """q [batch, G, H, d_k] (f32 or bf16), W_K: G decoders [d_k, d_c] of q's
    dtype -> q_abs [batch, G, H, d_c] (and q_abs_scale [batch, G, H] for e4m3)."""
    batch, G, H, d_k = q.shape
    ptrs = (_P * G)(*[W.data_ptr() for W in W_K])
    ctx.check(_lib.li_absorb_query_group(ctx.handle, _ptr(q), _dtype(q), batch, G, H, d_k, ptrs, int(d_c),
                                         int(out_dtype), _ptr(q_abs), _ptr(q_abs_scale), _stream(stream)))


def li_topk(ctx: Context, scores: torch.Tensor, k: int, out_idx: torch.Tensor, out_score: Optional[torch.Tensor],
            ws: torch.Tensor, lengths: Optional[torch.Tensor] = None, n: Optional[int] = None, stream=None):
    """scores [rows, stride] float32; row r selects among its first n (or lengths[r]) entries."""
    rows, stride = scores.shape
    n = stride if n is None else n
    ctx.check(_lib.li_topk(ctx.handle, _ptr(scores), rows, int(n), int(scores.stride(0)), _ptr(lengths), int(k),
                           _ptr(out_idx), _ptr(out_score), _ptr(ws), ws.numel(), _stream(stream)))


def li_attention_recall(ctx: Context, probs: torch.Tensor, sel: torch.Tensor, K: int,
                        lengths: Optional[torch.Tensor] = None, mean: bool = True, ws: Optional[torch.Tensor] = None,
                        stream=None):
    """probs [rows, H, N] float32, sel [rows, k] int32 (-1 padded).  Returns
    (recall [rows, H], mean_recall [rows] or None) as device tensors."""
    rows, H, N = probs.shape
    k = sel.shape[-1]
    need = int(_lib.li_recall_workspace_bytes(ctx.handle, rows, H, N, int(K)))
    if ws is None or ws.numel() < need:
        ws = torch.zeros(need, dtype=torch.uint8, device=probs.device)
    rec = torch.empty(rows, H, device=probs.device)
    mrec = torch.empty(rows, device=probs.device) if mean else None
    ctx.check(_lib.li_attention_recall(ctx.handle, _ptr(probs), rows, H, N, _ptr(lengths), _ptr(sel), int(k), int(K),
                                       _ptr(rec), _ptr(mrec), _ptr(ws), ws.numel(), _stream(stream)))
    return rec, mrec


def li_set_trace(ctx: Context, buf: Optional[torch.Tensor]):
    """Diagnostic per-tile trace of the scoring kernels into buf (uint8/int64
    device tensor of >= 32768 bytes, viewed as [8, 64, 8] int64), or None."""
    ctx.check(_lib.li_set_trace(ctx.handle, _ptr(buf), 0 if buf is None else buf.numel() * buf.element_size()))


def li_profile_enable(ctx: Context, enable: bool = True):
    ctx.check(_lib.li_profile_enable(ctx.handle, 1 if enable else 0))


def li_profile_read(ctx: Context):
    count = ctypes.c_int(0)
    ctx.check(_lib.li_profile_read(ctx.handle, None, 0, ctypes.byref(count)))
    n = count.value
    recs = (c_li_profile_record * max(n, 1))()
    ctx.check(_lib.li_profile_read(ctx.handle, recs, n, ctypes.byref(count)))
    return [dict(kernel=recs[i].kernel.decode(), ms=recs[i].ms, grid=recs[i].grid, block=recs[i].block,
                 smem=recs[i].smem) for i in range(n)]


def li_profile_reset(ctx: Context):
    ctx.check(_lib.li_profile_reset(ctx.handle))
