"""Pins of the oracle's storage codecs against the format definitions and library casts."""

import numpy as np
import pytest
import torch

from oracle import formats as F


def test_e4m3_table_matches_format_definition():
    # e4m3fn: bias 7, 3 mantissa bits, subnormal quantum 2^-9, max 448, 0x7F NaN.
    assert F.E4M3_TABLE[0x00] == 0.0
    assert F.E4M3_TABLE[0x01] == 2.0 ** -9
    assert F.E4M3_TABLE[0x07] == 7 * 2.0 ** -9
    assert F.E4M3_TABLE[0x08] == 2.0 ** -6
    assert F.E4M3_TABLE[0x38] == 1.0
    assert F.E4M3_TABLE[0x3C] == 1.5
    assert F.E4M3_TABLE[0x7E] == 448.0
    assert np.isnan(F.E4M3_TABLE[0x7F]) and np.isnan(F.E4M3_TABLE[0xFF])
    assert F.E4M3_TABLE[0xB8] == -1.0
    pos = F.E4M3_TABLE[:0x7F]
    assert np.all(np.diff(pos) > 0)


def test_e4m3_decode_matches_torch_for_every_code():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = F.e4m3_decode(np.arange(256, dtype=np.uint8))
    both_nan = np.isnan(ref) & np.isnan(ours)
    assert np.all(both_nan | (ref == ours))


def test_e4m3_encode_roundtrips_every_finite_code():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    back = F.e4m3_encode(F.e4m3_decode(codes))
    assert np.array_equal(back, codes)


def test_e4m3_encode_matches_torch_rne_sweep():
    rng = np.random.default_rng(7)
    vals = F.E4M3_TABLE[:0x7F]
    mids = (vals[1:] + vals[:-1]) / 2                          # exact ties
    x = np.concatenate([rng.uniform(-448, 448, 20000), rng.normal(0, 1, 20000), rng.normal(0, 0.01, 5000),
                        mids, -mids, vals, -vals]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = F.e4m3_encode(x.astype(np.float64))
    assert np.array_equal(ours, ref)


def test_e4m3_encode_saturates():
    assert F.e4m3_encode(np.array([1000.0]))[0] == 0x7E
    assert F.e4m3_encode(np.array([-1e9]))[0] == 0xFE
    assert F.e4m3_encode(np.array([470.0]))[0] == 0x7E


def test_bf16_encode_matches_torch():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.normal(0, 1, 50000), rng.normal(0, 1e4, 5000), rng.normal(0, 1e-4, 5000)]).astype(np.float32)
    # exact halfway cases between neighbouring bf16 values
    b = (x.view(np.uint32) & 0xFFFF0000) | 0x00008000
    x = np.concatenate([x, b.view(np.float32), np.array([0.0, -0.0], np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ours = F.bf16_encode(x.astype(np.float64))
    assert np.array_equal(ours, ref)
    assert np.array_equal(F.bf16_decode(ref), torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).double().numpy())


def test_pow2_scale_is_smallest_fitting_power_of_two():
    rng = np.random.default_rng(5)
    amax = np.concatenate([rng.lognormal(0, 4, 2000), [448.0, 448.0 * 2 ** -7, 448.0 * 1.0000001, 1.0, 224.0, 3.5]])
    sig = F.pow2_scale(amax)
    for a, s in zip(amax, sig):
        k = -200
        while a / 2.0 ** k > 448.0:        # brute force search
            k += 1
        while a / 2.0 ** (k - 1) <= 448.0:
            k -= 1
        assert s == 2.0 ** k, (a, s, k)
    assert F.pow2_scale(np.array([0.0]))[0] == 1.0


@pytest.mark.parametrize("fmt", ["f32", "bf16", "mixed"])
def test_row_codec_roundtrip(fmt):
    rng = np.random.default_rng(11)
    D = 512
    x = rng.normal(0, 1, (64, D))
    rows = F.encode_rows(x, fmt)
    assert rows.shape == (64, F.row_bytes(fmt, D))
    y = F.decode_rows(rows, fmt, D)
    tol = {"f32": 1e-7, "bf16": 2 ** -8, "mixed": 2 ** -3}[fmt]
    assert np.all(np.abs(y - x) <= tol * np.abs(x) + 1e-3 * (fmt == "mixed"))
    if fmt != "mixed":   # (mixed: a row max that rounds down to 224*sigma halves sigma on re-encode)
        assert np.array_equal(F.encode_rows(y, fmt), rows)
    else:
        assert np.allclose(F.decode_rows(F.encode_rows(y, fmt), fmt, D), y, rtol=0, atol=1e-12)


def test_mixed_row_layout():
    D = 512
    x = np.zeros(D)
    x[0], x[447], x[448], x[511] = 448.0, -1.0, 2.5, -3.0
    row = F.encode_rows(x[None], "mixed")[0]
    assert row.shape == (592,)
    assert row[0] == 0x7E and row[447] == 0xB8          # sigma = 1
    assert np.frombuffer(row[448:450].tobytes(), np.uint16)[0] == 0x4020   # 2.5 in bf16
    assert np.frombuffer(row[574:576].tobytes(), np.uint16)[0] == 0xC040   # -3.0 in bf16
    assert np.frombuffer(row[576:580].tobytes(), np.float32)[0] == 1.0
    assert not row[580:].any()


# ----------------------------------------------------------------------------- FP4 (e2m1) index keys

def test_e2m1_table_matches_format_definition():
    # 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit; exponent 0 is subnormal m * 0.5
    expect = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert np.array_equal(F.E2M1_TABLE[:8], expect)
    assert np.array_equal(F.E2M1_TABLE[8:], [-v for v in expect])


def test_e2m1_encode_roundtrips_and_rounds_to_nearest_even():
    for c in range(16):
        v = F.E2M1_TABLE[c]
        got = F.e2m1_encode(np.array([v]))[0]
        assert F.E2M1_TABLE[got] == v                       # -0 may come back as +0
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for x, y in ties.items():
        assert F.e2m1_decode(F.e2m1_encode(np.array([x, -x]))).tolist() == [y, -y]
    assert F.e2m1_decode(F.e2m1_encode(np.array([7.0, 1e9, -6.5]))).tolist() == [6.0, 6.0, -6.0]
    rng = np.random.default_rng(0)
    x = rng.uniform(-6, 6, 20000)
    d = np.abs(F.e2m1_decode(F.e2m1_encode(x))[:, None] - x[:, None])
    best = np.min(np.abs(F.E2M1_TABLE[None, :] - x[:, None]), axis=1)
    assert np.allclose(d[:, 0], best)                       # always a nearest value


def test_fp4_pack_order_and_roundtrip():
    c = np.arange(16, dtype=np.uint8)
    p = F.fp4_pack(c)
    assert p[0] == (0 | (1 << 4)) and p[7] == (14 | (15 << 4))
    assert np.array_equal(F.fp4_unpack(p), c)


def test_fp4_block_scales_follow_their_rule():
    rng = np.random.default_rng(1)
    x = rng.normal(size=(200, 128)) * np.exp2(rng.integers(-10, 10, size=(200, 1)))
    x[:, 32:64] *= np.exp2(-rng.integers(0, 12, size=(200, 1)))      # blocks of very different size
    packed, words = F.encode_fp4_keys(x)
    w = words.astype(np.int64)
    sigma = np.exp2((w & 0xFF) - 127.0)
    amax = np.abs(x).max(1)
    assert np.all(amax / sigma <= 6) and np.all(amax / sigma > 3)     # the smallest power of two
    for b in range(4):
        delta = (w >> (8 + 4 * b)) & 0xF
        bmax = np.abs(x[:, 32 * b:32 * b + 32]).max(1)
        assert np.all((delta >= 0) & (delta <= 7))
        fits = bmax * np.exp2(delta) / sigma <= 6
        assert np.all(fits)
        more = bmax * np.exp2(delta + 1) / sigma <= 6
        assert np.all(~more | (delta == 7))                         # the largest offset that fits
    v = F.decode_fp4_keys(packed, words)
    # within half a code step of each block's scale (the e2m1 spacing at the value's size)
    bs = np.repeat(np.stack([sigma * np.exp2(-((w >> (8 + 4 * b)) & 0xF)) for b in range(4)], 1), 32, axis=1)
    a = np.abs(x / bs)
    step = np.where(a < 2, 0.5, np.where(a < 4, 1.0, 2.0))
    assert np.all(np.abs(v - x) <= 0.5 * step * bs + 1e-300)


def test_fp4_scores_equal_fp8_scores_on_exactly_representable_keys():
    # keys built from e2m1 values times powers of two are exact in both formats: same scores
    rng = np.random.default_rng(2)
    from oracle import csa as O
    from csa_synth.configs import CSA_PRO, scaled_layer
    codes = rng.integers(0, 16, size=(50, 128)).astype(np.uint8)
    k = F.e2m1_decode(codes) * np.exp2(rng.integers(-6, -2, size=(50, 1)))
    q = rng.normal(size=(32, 128))
    qc, qs = F.encode_scaled_e4m3(q)
    w = rng.normal(size=32)
    k8, s8 = F.encode_scaled_e4m3(k)
    k4, w4 = F.encode_fp4_keys(k)
    L8 = O.LayerSpec.of(scaled_layer(CSA_PRO))
    L4 = O.LayerSpec.of(scaled_layer(CSA_PRO, idx_format="e2m1"))
    a8 = O.index_operands(L8, qc, k8, s8)
    a4 = O.index_operands(L4, qc, k4, w4)
    assert np.allclose(a8[1] * a8[2][:, None], a4[1] * a4[2][:, None], rtol=0, atol=0)
    s_8 = O.index_scores(a8[0], qs, w, a8[1], a8[2])
    s_4 = O.index_scores(a4[0], qs, w, a4[1], a4[2])
    assert np.allclose(s_8, s_4, rtol=1e-14, atol=0)
