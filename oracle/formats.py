"""Storage formats of the KV cache and the indexer, decoded and encoded exactly.

The pages store an entry's rotary dimensions in BF16 and the rest in FP8
("DeepSeek-V4 Explained: ...", section "The attention stack, and why it is two
mechanisms"); "DeepSeek-V4: Making a Million Tokens Affordable", section "Two
ways to shrink attention, interleaved", gives the same split as about halving
the cache.  The pages name the formats only; the codecs below are written from
the formats' own definitions:

* FP8 e4m3 ("e4m3fn" of the OCP 8-bit floating-point spec): 1 sign bit,
  4 exponent bits with bias 7, 3 mantissa bits; exponent field 0 is
  subnormal (m * 2^-9); exponent 15 with mantissa 7 is NaN; no infinities;
  largest finite 448.
* bfloat16: the upper 16 bits of an IEEE binary32.

Reading (the pages give no scale rule): the FP8 part of a row carries one
float32 scale sigma = the smallest power of two with amax / sigma <= 448
(sigma = 1 for an all-zero row), and code = RNE-satfinite(x / sigma); a
power-of-two scale makes x / sigma exact, so the encoding is unambiguous.

Row layout (``kv_format``): ``f32`` D float32; ``bf16`` D bfloat16;
``mixed`` D+80 bytes = e4m3 codes of dims [0, D-64) | bfloat16 of the 64
rotary dims | float32 scale | zero pad.
"""

import numpy as np

F8_MAX = 448.0


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
# non-negative finite values in code order 0x00..0x7E (strictly increasing)
_E4M3_POS = E4M3_TABLE[:0x7F].copy()


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Round to nearest e4m3 value, ties to the even code, saturating at +-448."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), F8_MAX)
    hi = np.searchsorted(_E4M3_POS, a, side="left")          # first value >= a
    hi = np.minimum(hi, 0x7E)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _E4M3_POS[lo]
    d_hi = _E4M3_POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    exact = _E4M3_POS[hi] == a
    code = np.where(exact, hi, code).astype(np.uint8)
    sign = np.signbit(x)
    return np.where(sign, code | 0x80, code).astype(np.uint8)


def bf16_decode(bits: np.ndarray) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def bf16_encode(x: np.ndarray) -> np.ndarray:
    """Round a real value to the nearest bfloat16 (8 significant bits), ties to even.

    Valid for the normal range, which is all the operator produces; zero maps to
    (signed) zero.
    """
    x = np.asarray(x, dtype=np.float64)
    f, e = np.frexp(x)                      # x = f * 2^e, 0.5 <= |f| < 1
    q = np.rint(np.ldexp(f, 8))             # 8 significant bits, half-to-even
    y = np.ldexp(q, e - 8).astype(np.float32)
    return (y.view(np.uint32) >> 16).astype(np.uint16)


def pow2_scale(amax: np.ndarray) -> np.ndarray:
    """Smallest power of two sigma with amax / sigma <= 448; 1 where amax == 0.

    448 = 0.875 * 2^9.  With amax = f * 2^e (0.5 <= f < 1), amax <= 448 * 2^k
    holds first at k = e - 9 when f <= 0.875, else at k = e - 8.
    """
    amax = np.asarray(amax, dtype=np.float64)
    f, e = np.frexp(amax)
    k = np.where(f <= 0.875, e - 9, e - 8)
    return np.where(amax == 0, 1.0, np.ldexp(1.0, k))


def row_bytes(fmt: str, D: int) -> int:
    return {"f32": 4 * D, "bf16": 2 * D, "mixed": D + 80}[fmt]


def decode_rows(rows: np.ndarray, fmt: str, D: int, d_rope: int = 64) -> np.ndarray:
    """Stored rows uint8 [..., row_bytes] -> exact values float64 [..., D]."""
    rows = np.ascontiguousarray(rows, dtype=np.uint8)
    lead = rows.shape[:-1]
    if fmt == "f32":
        return rows.view(np.float32).reshape(lead + (D,)).astype(np.float64)
    if fmt == "bf16":
        return bf16_decode(rows.view(np.uint16).reshape(lead + (D,)))
    if fmt == "mixed":
        dn = D - d_rope
        nope = e4m3_decode(rows[..., :dn])
        rope = bf16_decode(np.ascontiguousarray(rows[..., dn:dn + 2 * d_rope]).view(np.uint16))
        scale = np.ascontiguousarray(rows[..., D + 64:D + 68]).view(np.float32).reshape(lead).astype(np.float64)
        return np.concatenate([nope * scale[..., None], rope], axis=-1)
    raise ValueError(fmt)


def encode_rows(x: np.ndarray, fmt: str, d_rope: int = 64) -> np.ndarray:
    """Values float64 [..., D] -> stored rows uint8 [..., row_bytes]."""
    x = np.asarray(x, dtype=np.float64)
    lead, D = x.shape[:-1], x.shape[-1]
    if fmt == "f32":
        return x.astype(np.float32).view(np.uint8).reshape(lead + (4 * D,))
    if fmt == "bf16":
        return bf16_encode(x).view(np.uint8).reshape(lead + (2 * D,))
    if fmt == "mixed":
        dn = D - d_rope
        out = np.zeros(lead + (D + 80,), dtype=np.uint8)
        nope = x[..., :dn]
        sigma = pow2_scale(np.max(np.abs(nope), axis=-1))
        out[..., :dn] = e4m3_encode(nope / sigma[..., None])
        out[..., dn:dn + 2 * d_rope] = bf16_encode(x[..., dn:]).view(np.uint8).reshape(lead + (2 * d_rope,))
        out[..., D + 64:D + 68] = sigma.astype(np.float32).reshape(lead + (1,)).view(np.uint8)
        return out
    raise ValueError(fmt)


def decode_act(a: np.ndarray, fmt: str) -> np.ndarray:
    """Activation tensors (queries, raw rows, gates): float32 or bf16 bits -> float64."""
    if fmt == "f32":
        return np.asarray(a, dtype=np.float32).astype(np.float64)
    if fmt == "bf16":
        return bf16_decode(a)
    raise ValueError(fmt)


def decode_idx(codes: np.ndarray, fmt: str) -> np.ndarray:
    """Index keys / queries: float32 values or e4m3 codes -> float64 (before the scale)."""
    if fmt == "f32":
        return np.asarray(codes, dtype=np.float32).astype(np.float64)
    if fmt == "e4m3":
        return e4m3_decode(codes)
    raise ValueError(fmt)
