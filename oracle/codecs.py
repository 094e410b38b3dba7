"""Cache element codecs, written from the format definitions.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py): never called by the library.

* bf16: the upper 16 bits of an IEEE-754 binary32; encoding picks the nearer
  of the two bf16 values that bracket x, ties to the one with an even last
  mantissa bit (round-to-nearest-even).
* e4m3 (OCP 8-bit floating point, "E4M3"): 1 sign bit, 4 exponent bits with
  bias 7, 3 mantissa bits; exponent 0 is subnormal (m * 2^-9); S.1111.111 is
  NaN; there are no infinities; the largest finite magnitude is 1.75 * 2^8 =
  448.  Encoding is round-to-nearest-even with saturation to +-448.
* Per-token e4m3 scaling (the fp8 latent cache of the LatentIndex summary,
  Sec. B.2 "segmented FP8 execution", one scale per token in this build):
  scale = fp32(amax) / 448 in binary32 division (1 when amax = 0); each code is
  e4m3(c_i / scale) with binary32 division.
"""
import numpy as np

# ----------------------------------------------------------------------------- bf16

def bf16_decode(bits: np.ndarray) -> np.ndarray:
    """uint16 bf16 codes -> float32 values (exact: the code is the high half)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_encode(x: np.ndarray) -> np.ndarray:
    """float32 -> uint16 bf16 codes, round to nearest, ties to even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    sign = u & np.uint32(0x80000000)
    mag = u & np.uint32(0x7FFFFFFF)
    lo = mag & np.uint32(0xFFFF0000)                 # bracket below (toward zero)
    hi = lo + np.uint32(0x10000)                     # bracket above (may reach +inf)
    v = mag.view(np.float32).astype(np.float64)
    v_lo = lo.view(np.float32).astype(np.float64)
    with np.errstate(invalid="ignore", over="ignore"):
        v_hi = hi.view(np.float32).astype(np.float64)
        # IEEE rounding treats the step past the largest finite value as 2^128:
        # inputs at or beyond that midpoint round to infinity.
        v_hi = np.where(hi == np.uint32(0x7F800000), 2.0 ** 128, v_hi)
        d_lo = v - v_lo
        d_hi = v_hi - v
    lo_even = ((lo >> np.uint32(16)) & np.uint32(1)) == 0
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ~lo_even)
    out = np.where(take_hi, hi, lo)
    is_nan = mag > np.uint32(0x7F800000)
    is_inf = mag == np.uint32(0x7F800000)
    out = np.where(is_inf, np.uint32(0x7F800000), out)
    out = np.where(is_nan, np.uint32(0x7FC00000), out)
    return ((out | sign) >> np.uint32(16)).astype(np.uint16)


# ----------------------------------------------------------------------------- e4m3

E4M3_MAX = 448.0


def _e4m3_value(code: int) -> float:
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * m * 2.0 ** -9
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


E4M3_TABLE = np.array([_e4m3_value(c) for c in range(256)], dtype=np.float64)
# Non-negative finite codes 0x00..0x7E in increasing value order.
_POS_CODES = np.arange(0x7F, dtype=np.int64)
_POS_VALUES = E4M3_TABLE[:0x7F]


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)].astype(np.float32)


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """float32 -> uint8 e4m3 codes: nearest finite value, ties to the even code,
    saturating at +-448; NaN -> S.1111.111."""
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x.astype(np.float64))
    neg = np.signbit(x)
    nan = np.isnan(x)
    a = np.where(nan, 0.0, a)
    j = np.searchsorted(_POS_VALUES, a, side="left")          # first value >= a
    j_hi = np.clip(j, 0, 0x7E)
    j_lo = np.clip(j - 1, 0, 0x7E)
    d_hi = np.abs(_POS_VALUES[j_hi] - a)
    d_lo = np.abs(a - _POS_VALUES[j_lo])
    tie = d_hi == d_lo
    pick_hi = (d_hi < d_lo) | (tie & ((_POS_CODES[j_hi] & 1) == 0))
    code = np.where(pick_hi, _POS_CODES[j_hi], _POS_CODES[j_lo])
    code = np.where(a > E4M3_MAX, 0x7E, code)
    code = np.where(nan, 0x7F, code)
    code = code | np.where(neg, 0x80, 0)
    return code.astype(np.uint8)


def e4m3_encode_bruteforce(x: np.ndarray) -> np.ndarray:
    """Same mapping by exhaustive search over all finite codes (small inputs)."""
    out = []
    for v in np.asarray(x, dtype=np.float32).ravel().tolist():
        if v != v:
            out.append(0x7F | (0x80 if np.signbit(np.float32(v)) else 0))
            continue
        a = abs(v)
        best, bestd = None, None
        for c in range(0x7F):
            d = abs(E4M3_TABLE[c] - a)
            if bestd is None or d < bestd or (d == bestd and (c & 1) == 0 and (best & 1) == 1):
                best, bestd = c, d
        out.append(best | (0x80 if np.signbit(np.float32(v)) else 0))
    return np.array(out, dtype=np.uint8).reshape(np.shape(x))


def e4m3_quantize_rows(c: np.ndarray):
    """Per-row (per-token) e4m3 quantisation of float32 rows [..., d].

    Returns (codes uint8 [..., d], scale float32 [...])."""
    c = np.asarray(c, dtype=np.float32)
    amax = np.max(np.abs(c), axis=-1)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    q = (c / scale[..., None]).astype(np.float32)
    return e4m3_encode(q), scale


def e4m3_dequantize_rows(codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    return e4m3_decode(codes).astype(np.float64) * np.asarray(scale, np.float64)[..., None]


def e4m3_quantize_rows_segmented(c: np.ndarray, split: int):
    """Segmented fp8 (LatentIndex summary, Sec. B.2 and Sec. C.1): each row
    [..., d] is quantised as two independent segments, elements [0, split)
    and [split, d), each with its own per-row scale (the two branches of
    the latent keep their own range).  Returns (codes uint8 [..., d],
    scale float32 [..., 2])."""
    c = np.asarray(c, dtype=np.float32)
    c0, s0 = e4m3_quantize_rows(c[..., :split])
    c1, s1 = e4m3_quantize_rows(c[..., split:])
    return np.concatenate([c0, c1], axis=-1), np.stack([s0, s1], axis=-1)


def e4m3_dequantize_rows_segmented(codes: np.ndarray, scale: np.ndarray, split: int) -> np.ndarray:
    scale = np.asarray(scale, np.float64)
    return np.concatenate([e4m3_dequantize_rows(codes[..., :split], scale[..., 0]),
                           e4m3_dequantize_rows(codes[..., split:], scale[..., 1])], axis=-1)
