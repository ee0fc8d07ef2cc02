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


# --------------------------------------------------------------------------- FP4 (e2m1) index keys
#
# "DeepSeek-V4: Making a Million Tokens Affordable", "Two ways to shrink attention, interleaved":
# the indexer's attention runs in FP4.  The format is read as OCP e2m1 (1 sign bit, 2 exponent bits
# with bias 1, 1 mantissa bit; exponent field 0 is subnormal m * 0.5; no infinities or NaN; largest
# finite 6) with block scaling.  Reading of the scales (the pages give none): a key of d dims has one
# power-of-two scale sigma (the smallest with max|k| / sigma <= 6) and, per block of 32 dims, an
# offset delta_b in 0..7 that scales the block further down by 2^-delta_b (the largest delta_b with
# max_block|k| * 2^delta_b / sigma <= 6, capped at 7): value = code * sigma * 2^-delta_b.  Codes are
# round-to-nearest-even with saturation at 6, two per byte (the even dim in the low nibble).  The scale
# word of a key packs the exponent of sigma (+127) in bits 0..7 and delta_b in bits 8 + 4b .. 11 + 4b.

E2M1_MAX = 6.0
FP4_BLOCK = 32


def _e2m1_value(code: int) -> float:
    s = -1.0 if code & 0x8 else 1.0
    e = (code >> 1) & 0x3
    m = code & 0x1
    if e == 0:
        return s * m * 0.5
    return s * (1.0 + m / 2.0) * 2.0 ** (e - 1)


E2M1_TABLE = np.array([_e2m1_value(c) for c in range(16)], dtype=np.float64)
_E2M1_POS = E2M1_TABLE[:8].copy()          # 0, 0.5, 1, 1.5, 2, 3, 4, 6 (strictly increasing)


def e2m1_encode(x: np.ndarray) -> np.ndarray:
    """Round to the nearest e2m1 value, ties to the even code, saturating at +-6 (uint8 codes 0..15)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E2M1_MAX)
    hi = np.minimum(np.searchsorted(_E2M1_POS, a, side="left"), 7)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _E2M1_POS[lo]
    d_hi = _E2M1_POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(_E2M1_POS[hi] == a, hi, code).astype(np.uint8)
    return np.where(np.signbit(x) & (code != 0), code | 0x8, code).astype(np.uint8)


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    return E2M1_TABLE[np.asarray(codes, dtype=np.uint8) & 0xF]


def fp4_pack(codes: np.ndarray) -> np.ndarray:
    """[..., d] codes (d even) -> [..., d/2] bytes, the even dim in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def fp4_unpack(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def pow2_scale_fp4(amax: np.ndarray) -> np.ndarray:
    """Smallest power of two sigma with amax / sigma <= 6; 1 where amax == 0.  6 = 0.75 * 2^3: with
    amax = f * 2^e (0.5 <= f < 1) the bound holds first at k = e - 3 when f <= 0.75, else e - 2."""
    amax = np.asarray(amax, dtype=np.float64)
    f, e = np.frexp(amax)
    k = np.where(f <= 0.75, e - 3, e - 2)
    return np.where(amax == 0, 1.0, np.ldexp(1.0, k))


def encode_fp4_keys(x: np.ndarray):
    """Keys float64 [..., d] (d a multiple of 32) -> (packed codes uint8 [..., d/2], scale words uint32 [...])."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    nb = d // FP4_BLOCK
    blocks = x.reshape(x.shape[:-1] + (nb, FP4_BLOCK))
    bmax = np.max(np.abs(blocks), axis=-1)                              # [..., nb]
    sigma = pow2_scale_fp4(np.max(bmax, axis=-1))                       # [...]
    # delta_b: largest integer with bmax * 2^delta / sigma <= 6, in 0..7
    ratio = bmax / sigma[..., None]                                     # <= 6
    delta = np.zeros_like(bmax, dtype=np.int64)
    for dd in range(1, 8):
        delta = np.where(ratio * 2.0 ** dd <= E2M1_MAX, dd, delta)
    bscale = sigma[..., None] * np.exp2(-delta.astype(np.float64))      # [..., nb]
    codes = e2m1_encode(blocks / bscale[..., None]).reshape(x.shape)
    e = np.round(np.log2(sigma)).astype(np.int64) + 127
    word = e.astype(np.uint64)
    for b in range(nb):
        word = word | (delta[..., b].astype(np.uint64) << np.uint64(8 + 4 * b))
    return fp4_pack(codes), word.astype(np.uint32)


def decode_fp4_keys(packed: np.ndarray, words: np.ndarray) -> np.ndarray:
    """(packed codes [..., d/2], scale words [...]) -> exact values float64 [..., d]."""
    codes = fp4_unpack(packed)
    d = codes.shape[-1]
    nb = d // FP4_BLOCK
    w = np.asarray(words, dtype=np.uint32).astype(np.int64)
    sigma = np.exp2((w & 0xFF) - 127.0)
    vals = e2m1_decode(codes).reshape(codes.shape[:-1] + (nb, FP4_BLOCK))
    delta = np.stack([(w >> (8 + 4 * b)) & 0xF for b in range(nb)], axis=-1).astype(np.float64)
    return (vals * (sigma[..., None] * np.exp2(-delta))[..., None]).reshape(codes.shape)


def encode_scaled_e4m3(x: np.ndarray):
    """Values float64 [..., d] -> (e4m3 codes uint8 [..., d], float32 scale [...]) with one power-of-two
    scale per leading index (the row-scale rule of the mixed rows: max|x| / scale <= 448)."""
    x = np.asarray(x, dtype=np.float64)
    sigma = pow2_scale(np.max(np.abs(x), axis=-1))
    return e4m3_encode(x / sigma[..., None]), sigma.astype(np.float32)


def encode_idx(x: np.ndarray, fmt: str, role: str = "key"):
    """Index keys / queries in storage form: (codes, scales).  e4m3: scaled codes as encode_scaled_e4m3;
    f32: the float32 values with scale 1; e2m1: keys as encode_fp4_keys (packed codes, scale words),
    queries (role "query") as e4m3."""
    x = np.asarray(x, dtype=np.float64)
    if fmt == "e2m1":
        return encode_fp4_keys(x) if role == "key" else encode_scaled_e4m3(x)
    if fmt == "e4m3":
        return encode_scaled_e4m3(x)
    if fmt == "f32":
        return x.astype(np.float32), np.ones(x.shape[:-1], np.float32)
    raise ValueError(fmt)


def decode_idx_keys(codes: np.ndarray, scales: np.ndarray, fmt: str) -> np.ndarray:
    """Stored index keys -> exact values, scales applied (e2m1: block scales included)."""
    if fmt == "e2m1":
        return decode_fp4_keys(codes, scales)
    return decode_idx(codes, fmt) * np.asarray(scales, np.float64)[..., None]


def decode_idx(codes: np.ndarray, fmt: str) -> np.ndarray:
    """Index keys / queries: float32 values or e4m3 codes -> float64 (before the scale)."""
    if fmt == "f32":
        return np.asarray(codes, dtype=np.float32).astype(np.float64)
    if fmt == "e4m3":
        return e4m3_decode(codes)
    raise ValueError(fmt)
