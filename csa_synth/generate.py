"""Seeded synthetic tensors in the operator's storage formats.

Values are Gaussian as the workloads state: raw rows, gate logits, biases,
queries, sink logits and indexer head weights N(0,1); index keys N(0, 1/d_I);
cached rows (compressed entries and window rows, which in a model come out of
an RMSNorm) N(0,1).  Tensors stored as BF16 or FP8-e4m3 are produced by
torch's own dtype casts of those draws; FP8 tensors get a random power-of-two
scale per row from {2^-4, 2^-5, 2^-6} so the codes stay inside e4m3's range.

Byte layout of one stored KV row (``kv_format``):

* ``f32``   -- D little-endian float32.
* ``bf16``  -- D bfloat16.
* ``mixed`` -- D+80 bytes: e4m3 codes of dims [0, D-64) at byte 0, bfloat16
  of the rotary dims [D-64, D) at byte D-64, the float32 row scale at byte
  D+64, zero padding to D+80 (a multiple of 16 bytes).

Nothing here pools, normalises, rotates, scores, selects or attends.
"""

import zlib

import numpy as np
import torch

from .configs import Layer, Workload, raw_ring_rows, row_bytes

_FP8_SCALE_EXPONENTS = np.array([4, 5, 6], dtype=np.int64)


def stream(seed: int, tag: str, layer: int = 0) -> np.random.Generator:
    """An independent Philox stream for one tensor of one workload."""
    key = (int(seed) << 40) ^ (zlib.crc32(tag.encode()) << 8) ^ int(layer)
    return np.random.Generator(np.random.Philox(key=key))


def _normal(rng, shape, std=1.0):
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _e4m3_codes(x: np.ndarray) -> np.ndarray:
    x = np.clip(x, -448.0, 448.0).astype(np.float32)
    t = torch.from_numpy(np.ascontiguousarray(x)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def _fp8_with_row_scale(rng_val, rng_exp, shape, std=1.0):
    """Codes [..., d] and per-row scales [...] with value = code * scale ~ N(0, std^2)."""
    z = _normal(rng_val, shape)
    e = rng_exp.choice(_FP8_SCALE_EXPONENTS, size=shape[:-1])
    codes = _e4m3_codes(z * np.exp2(e)[..., None].astype(np.float32))
    scale = (np.exp2(-e.astype(np.float64)) * std).astype(np.float32)
    return codes, scale


def act_array(rng, shape, fmt, std=1.0):
    """Activation-typed tensor (queries, raw rows, gate logits): float32 or bf16 bits."""
    x = _normal(rng, shape, std)
    if fmt == "f32":
        return x
    if fmt == "bf16":
        return _bf16_bits(x)
    raise ValueError(fmt)


def kv_rows(seed: int, tag: str, layer_idx: int, lead_shape, layer: Layer) -> np.ndarray:
    """Random stored KV rows, uint8 [*lead_shape, row_bytes]."""
    D = layer.D
    rb = row_bytes(layer)
    rng = stream(seed, tag, layer_idx)
    if layer.kv_format == "f32":
        return _normal(rng, tuple(lead_shape) + (D,)).view(np.uint8)
    if layer.kv_format == "bf16":
        return _bf16_bits(_normal(rng, tuple(lead_shape) + (D,))).view(np.uint8)
    if layer.kv_format == "mixed":
        dn = D - layer.d_rope
        codes, scale = _fp8_with_row_scale(rng, stream(seed, tag + ".exp", layer_idx),
                                           tuple(lead_shape) + (dn,))
        rope = _bf16_bits(_normal(stream(seed, tag + ".rope", layer_idx),
                                  tuple(lead_shape) + (layer.d_rope,)))
        out = np.zeros(tuple(lead_shape) + (rb,), dtype=np.uint8)
        out[..., :dn] = codes
        out[..., dn:dn + 2 * layer.d_rope] = rope.view(np.uint8).reshape(tuple(lead_shape) + (2 * layer.d_rope,))
        out[..., D + 64:D + 68] = scale.reshape(tuple(lead_shape) + (1,)).view(np.uint8).reshape(tuple(lead_shape) + (4,))
        return out
    raise ValueError(layer.kv_format)


# magnitudes of the 8 non-negative e2m1 codes are 0, .5, 1, 1.5, 2, 3, 4, 6: a draw is binned at the
# midpoints between them (random bytes in the FP4 key layout; nothing here scores or selects)
_E2M1_MIDPOINTS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])


def _fp4_keys(seed, layer_idx, lead_shape, d):
    """Random FP4 index keys in storage form: packed e2m1 codes [..., d/2] (even dim in the low
    nibble) of draws N(0, 2^2), and scale words [...] holding a per-key exponent from {-6, -5, -4}
    (+127, bits 0..7) and per-32-dim block offsets from {0, 1, 2} (bits 8+4b..11+4b)."""
    z = _normal(stream(seed, "idx_k", layer_idx), tuple(lead_shape) + (d,), 2.0)
    mag = np.digitize(np.abs(z), _E2M1_MIDPOINTS).astype(np.uint8)
    codes = np.where((z < 0) & (mag > 0), mag | 0x8, mag).astype(np.uint8)
    packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
    e = stream(seed, "idx_k.exp", layer_idx).choice(np.array([-6, -5, -4]), size=tuple(lead_shape))
    off = stream(seed, "idx_k.blk", layer_idx).integers(0, 3, size=tuple(lead_shape) + (d // 32,))
    word = (e + 127).astype(np.uint64)
    for b in range(d // 32):
        word = word | (off[..., b].astype(np.uint64) << np.uint64(8 + 4 * b))
    return packed, word.astype(np.uint32)


def index_keys(seed, layer_idx, lead_shape, layer: Layer):
    """Index keys N(0, 1/d_I): (keys, scales).  f32: keys float32, scales all 1.  e2m1: packed FP4
    codes and scale words (_fp4_keys)."""
    std = 1.0 / np.sqrt(layer.d_I)
    shape = tuple(lead_shape) + (layer.d_I,)
    if layer.idx_format == "e2m1":
        return _fp4_keys(seed, layer_idx, lead_shape, layer.d_I)
    if layer.idx_format == "f32":
        return _normal(stream(seed, "idx_k", layer_idx), shape, std), np.ones(lead_shape, np.float32)
    return _fp8_with_row_scale(stream(seed, "idx_k", layer_idx), stream(seed, "idx_k.exp", layer_idx),
                               shape, std)


def index_queries(seed, layer_idx, lead_shape, layer: Layer):
    """Index queries N(0,1) per head: (queries, scales) with scales [*lead_shape, H_I] (e4m3 codes
    for both the e4m3 and the e2m1 key formats)."""
    shape = tuple(lead_shape) + (layer.H_I, layer.d_I)
    if layer.idx_format == "f32":
        return _normal(stream(seed, "idx_q", layer_idx), shape), np.ones(shape[:-1], np.float32)
    return _fp8_with_row_scale(stream(seed, "idx_q", layer_idx), stream(seed, "idx_q.exp", layer_idx), shape)


def _common(wl: Workload, li: int, layer: Layer, lead):
    seed = wl.seed
    d = {
        "sinks": _normal(stream(seed, "sinks", li), (layer.H,)),
        "pos_bias": _normal(stream(seed, "pos_bias", li), ((1 + layer.ov) * layer.m, layer.D)),
        "gamma_kv": np.ones(layer.D, np.float32),
        "gamma_q": np.ones(layer.D, np.float32),
        "q": act_array(stream(seed, "q", li), tuple(lead) + (layer.H, layer.D), layer.act_format),
    }
    if layer.kind == "csa":
        iq, iqs = index_queries(seed, li, lead, layer)
        d["idx_q"], d["idx_q_scale"] = iq, iqs
        d["head_w"] = _normal(stream(seed, "head_w", li), tuple(lead) + (layer.H_I,))
    return d


def index_stream_inputs(wl: Workload, li: int, lead_shape, layer: Layer):
    """Inputs of the index side produced in a step: index-key stream rings and new rows, its slot
    biases, the query latent c [*lead, r] N(0,1) and the up-projection W [H_I*d_I, r] N(0, 1/r)."""
    B = lead_shape[0]
    rr = raw_ring_rows(layer)
    r = layer.idx_rank
    return {
        "idx_raw_ring": act_array(stream(wl.seed, "idx_raw_ring", li), (B, rr, layer.d_I), layer.act_format),
        "idx_gate_ring": act_array(stream(wl.seed, "idx_gate_ring", li), (B, rr, layer.d_I), layer.act_format),
        "idx_x_new": act_array(stream(wl.seed, "idx_x_new", li), tuple(lead_shape) + (layer.d_I,), layer.act_format),
        "idx_g_new": act_array(stream(wl.seed, "idx_g_new", li), tuple(lead_shape) + (layer.d_I,), layer.act_format),
        "idx_pos_bias": _normal(stream(wl.seed, "idx_pos_bias", li), ((1 + layer.ov) * layer.m, layer.d_I)),
        "c_q": act_array(stream(wl.seed, "c_q", li), tuple(lead_shape) + (r,), layer.act_format),
        "W_iq": act_array(stream(wl.seed, "W_iq", li), (layer.H_I * layer.d_I, r), layer.act_format,
                          std=1.0 / np.sqrt(r)),
    }


def decode_inputs(wl: Workload, li: int = 0, n=None, entry_cap=None, indexed=False):
    """State and step inputs of one decode step of layer ``li`` (with ``indexed``, also the inputs of
    the index side produced in the step: index_stream_inputs).

    The step is for token t = pos0 + n - 1 of every sequence.  Caches hold
    random stored rows: entries [B, entry_cap, row], window ring
    [B, window, row] (row of raw position r at slot r mod window), raw and
    gate rings [B, (1+ov)m, D] (slot r mod (1+ov)m) holding the rows before t.
    The new token's raw row and gate row are step inputs.
    """
    layer = wl.layers[li]
    n = wl.n if n is None else n
    B = wl.B
    N = n // layer.m
    cap = max(N, 1) if entry_cap is None else entry_cap
    rr = raw_ring_rows(layer)
    d = _common(wl, li, layer, (B,))
    d.update({
        "n": n,
        "t": np.full(B, wl.pos0 + n - 1, dtype=np.int64),
        "entries": kv_rows(wl.seed, "entries", li, (B, cap), layer),
        "window": kv_rows(wl.seed, "window", li, (B, layer.window), layer),
        "raw_ring": act_array(stream(wl.seed, "raw_ring", li), (B, rr, layer.D), layer.act_format),
        "gate_ring": act_array(stream(wl.seed, "gate_ring", li), (B, rr, layer.D), layer.act_format),
        "x_new": act_array(stream(wl.seed, "x_new", li), (B, layer.D), layer.act_format),
        "g_new": act_array(stream(wl.seed, "g_new", li), (B, layer.D), layer.act_format),
    })
    if layer.kind == "csa":
        d["idx_k"], d["idx_k_scale"] = index_keys(wl.seed, li, (B, cap), layer)
        if indexed:
            d.update(index_stream_inputs(wl, li, (B,), layer))
    return d


def compress_inputs(wl: Workload, li: int = 0, n_rows=None, first_row=0):
    """Uncompressed rows [B, n_rows, D] for raw positions first_row.. and their gate logits."""
    layer = wl.layers[li]
    n_rows = wl.n if n_rows is None else n_rows
    return {
        "raw": act_array(stream(wl.seed, "raw", li), (wl.B, n_rows, layer.D), layer.act_format),
        "gate": act_array(stream(wl.seed, "gate", li), (wl.B, n_rows, layer.D), layer.act_format),
        "first_row": first_row,
        "pos_bias": _normal(stream(wl.seed, "pos_bias", li), ((1 + layer.ov) * layer.m, layer.D)),
        "gamma_kv": np.ones(layer.D, np.float32),
    }


def prefill_inputs(wl: Workload, li: int = 0, Tq=None, prefix=None):
    """Inputs of one chunked-prefill call: Tq new tokens after a prefix of ``prefix`` tokens.

    Queries are at positions prefix .. prefix+Tq-1 (pos0 = 0).  The entry cache
    holds random rows for the prefix's complete entries and room for the
    chunk's; index keys are given for every entry (the chunk's too).  The raw
    rows cover positions [prefix - ov*m, prefix + Tq) so the chunk's first
    entry has its look-back rows.  The window buffer is a ring of
    Tq + window rows holding random rows for the prefix's last window-1
    positions; the chunk's rows are appended by the operator.
    """
    layer = wl.layers[li]
    Tq = wl.Tq if Tq is None else Tq
    prefix = (wl.n - wl.Tq) if prefix is None else prefix
    n = prefix + Tq
    B = wl.B
    N_total = n // layer.m
    look = layer.ov * layer.m
    first_row = max(0, (prefix // layer.m - layer.ov) * layer.m)
    d = _common(wl, li, layer, (B, Tq))
    d.update({
        "prefix": prefix,
        "n": n,
        "Tq": Tq,
        "t": (prefix + np.arange(Tq, dtype=np.int64))[None, :].repeat(B, 0),
        "entries": kv_rows(wl.seed, "entries", li, (B, N_total), layer),
        "window": kv_rows(wl.seed, "window", li, (B, Tq + layer.window), layer),
        "raw": act_array(stream(wl.seed, "raw", li), (B, n - first_row, layer.D), layer.act_format),
        "gate": act_array(stream(wl.seed, "gate", li), (B, n - first_row, layer.D), layer.act_format),
        "raw_first_row": first_row,
    })
    if layer.kind == "csa":
        d["idx_k"], d["idx_k_scale"] = index_keys(wl.seed, li, (B, N_total), layer)
    return d
