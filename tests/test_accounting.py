"""Pins of the KV / FLOP accounting tool against what the pages print and against closed forms.

Exact: the entry counts of "Decoding DeepSeek-V4" ("Compressing the past": 250,000 entries grouped
by 4 and 7,813 grouped by 128 at a million tokens), the 8x of a 512 latent against a 4096-wide K/V
("DeepSeek-V4, explained."), the 0.013% window share and m'/m = 32 ("Two ways to shrink attention,
interleaved"), and each layer's bytes and FLOPs against its formula written out by hand.
Banded: the reproduction of Figure 1's values at one million tokens (V4-Pro 27% of V3.2's FLOPs and
10% of its cache, V4-Flash 10% and 7%) rests on readings the pages do not fix (the V3.2 cache and
indexer, the layer alternation, the FP8-equivalent weights), so it is held to +-40% of each figure,
to the ordering of the models and to the shape of the curves over context length.
"""

import pytest

from long_context_sparse_csa_b200 import accounting as A


def test_entry_counts_at_a_million_tokens():
    assert A.entries_seen(10 ** 6, 4) == 250_000
    assert A.entries_seen(10 ** 6, 128, partial=True) == 7_813
    assert A.entries_seen(10 ** 6, 128) == 7_812          # complete groups only (what a query sees)
    assert A.entries_seen(1 << 20, 4) == 262_144 and A.entries_seen(1 << 20, 128) == 8_192


def test_latent_window_and_ratio_facts():
    assert 4096 / 512 == 8
    assert round(100 * 128 / 10 ** 6, 3) == 0.013
    csa, hca = A._v4_kinds(128)
    assert hca.m // csa.m == 32


def test_layer_bytes_and_flops_closed_forms():
    csa, hca = A._v4_kinds(128)
    n = 131_072
    assert A.layer_kv_bytes(csa, n) == (n // 4) * (580 + 132) + 128 * 580
    assert A.layer_kv_bytes(hca, n) == (n // 128) * 580 + 128 * 580
    f = A.layer_flops(csa, n)
    assert f["indexer"] == 2 * 32 * 128 * (n // 4)
    assert f["attention"] == 2 * 128 * (512 + 512) * (1024 + 128)
    assert f["fp8_equiv"] == 0.5 * f["indexer"] + 2 * f["attention"]
    g = A.layer_flops(hca, n)
    assert g["indexer"] == 0 and g["attention"] == 2 * 128 * 1024 * (n // 128 + 128)
    # short contexts: the selection and the window saturate at what exists
    assert A.layer_flops(csa, 40)["attention"] == 2 * 128 * 1024 * (10 + 40)


def test_alternation_counts():
    pro, flash = A.v4_pro(), A.v4_flash()
    assert len(pro.layers) == 61 and len(flash.layers) == 43
    assert sum(k.name == "csa" for k in pro.layers) == 31 and sum(k.name == "hca" for k in pro.layers) == 30


def _at(rows, n, model):
    return [r for r in rows if r["context"] == n and r["model"] == model][0]


@pytest.mark.parametrize("model,flops,kv", [("V4-Pro", 0.27, 0.10), ("V4-Flash", 0.10, 0.07)])
def test_figure_1_values_at_a_million_tokens(model, flops, kv):
    r = _at(A.figure1(), 10 ** 6, model)
    assert flops / 1.4 <= r["flops_vs_v3_2"] <= flops * 1.4
    assert kv / 1.4 <= r["kv_vs_v3_2"] <= kv * 1.4


def test_figure_1_shape():
    rows = A.figure1()
    ctx = sorted({r["context"] for r in rows})
    for model in ("V4-Pro", "V4-Flash"):
        f = [_at(rows, n, model)["flops_vs_v3_2"] for n in ctx if n != 10 ** 6]
        assert all(a > b for a, b in zip(f, f[1:])), "the FLOP gap widens with context"
    for n in ctx:
        assert _at(rows, n, "V4-Flash")["flops_vs_v3_2"] < _at(rows, n, "V4-Pro")["flops_vs_v3_2"]
        assert _at(rows, n, "V4-Flash")["kv_vs_v3_2"] < _at(rows, n, "V4-Pro")["kv_vs_v3_2"]


def test_against_gqa8_roughly_two_percent_and_halved_by_mixed_rows():
    g = A.gqa8_comparison(10 ** 6)
    assert 0.01 <= g["mixed_vs_gqa8"] <= 0.03
    assert 0.4 <= g["mixed_vs_bf16"] <= 0.7
    assert abs(A.mixed_vs_bf16_row_ratio() - 580 / 1024) < 1e-12
