"""Pins of the oracle's index-key production and low-rank index query (readings R14, R15).

Index keys pool the index-key stream with the compressor's per-channel softmax and no norm or
rotation; the index query is the up-projection of the query's low-rank latent, q_h = W_h c.  The
pins: special cases that reduce to closed forms (equal gates give the window mean, a single row is
itself, a +60 bias selects its slot, an identity projection of rank d_I returns the latent),
linearity, the storage rule of the scales, and the decode step's in-step production agreeing with
the batch definitions.  Page: "DeepSeek-V4 Explained: ...", "The attention stack, and why it is two
mechanisms" (a low-rank lightning indexer over the compressed entries).
"""

import numpy as np
import pytest

from csa_synth import decode_inputs, get_workload
from csa_synth.configs import Workload, scaled_layer, CSA_PRO
from oracle import csa as O
from oracle import formats as F


def test_index_key_with_equal_gates_is_the_window_mean_unnormalised():
    rng = np.random.default_rng(0)
    x = rng.normal(size=(12, 128)) * 3.0
    keys = O.compress_index_keys(x, np.zeros_like(x), np.zeros((8, 128)), 4, 1, [0, 1, 2])
    assert np.allclose(keys[0], x[0:4].mean(0), atol=1e-14)          # entry 0: its own 4 rows
    assert np.allclose(keys[2], x[4:12].mean(0), atol=1e-14)         # overlap: 2m rows
    assert not np.isclose(np.sqrt(np.mean(keys[2] ** 2)), 1.0)       # no RMSNorm


def test_index_key_single_row_is_itself_and_bias_selects():
    rng = np.random.default_rng(1)
    x, gte = rng.normal(size=(2, 9, 64))
    keys = O.compress_index_keys(x, gte, np.zeros((1, 64)), 1, 0, range(9))
    assert np.allclose(keys, x, atol=1e-14)
    bias = np.zeros((8, 64))
    bias[5] = 60.0                                                    # slot 5 of entry 1 = raw row 5
    k1 = O.compress_index_keys(x, np.zeros_like(x), bias, 4, 1, [1])[0]
    assert np.allclose(k1, x[5], atol=1e-12)


def test_index_storage_rule():
    rng = np.random.default_rng(2)
    v = rng.normal(size=(50, 128)) * np.exp2(rng.integers(-8, 8, size=(50, 1)))
    codes, sig = F.encode_idx(v, "e4m3")
    amax = np.abs(v).max(1)
    assert np.all(np.log2(sig) == np.round(np.log2(sig)))           # powers of two
    assert np.all(amax / sig <= 448) and np.all(amax / sig > 224)     # the smallest such power
    back = F.e4m3_decode(codes) * sig[:, None]
    # round to nearest: within half a quantum of e4m3 (3 mantissa bits) around each value
    q = np.exp2(np.floor(np.log2(np.maximum(np.abs(v / sig[:, None]), 2.0 ** -6))) - 3) * sig[:, None]
    assert np.all(np.abs(back - v) <= 0.5 * q + 1e-30)
    f, one = F.encode_idx(v, "f32")
    assert np.array_equal(f, v.astype(np.float32)) and np.all(one == 1)


def test_identity_projection_of_rank_d_I_returns_the_latent():
    rng = np.random.default_rng(3)
    H_I, d_I = 4, 16
    c = rng.normal(size=d_I)
    W = np.concatenate([np.eye(d_I)] * H_I)                          # [H_I * d_I, r = d_I]
    q = O.index_query(c, W, H_I, d_I)
    assert q.shape == (H_I, d_I) and np.allclose(q, c[None], atol=0)


def test_index_query_is_linear_in_the_latent():
    rng = np.random.default_rng(4)
    H_I, d_I, r = 3, 8, 20
    W = rng.normal(size=(H_I * d_I, r))
    c1, c2 = rng.normal(size=(2, r))
    assert np.allclose(O.index_query(c1 + 2 * c2, W, H_I, d_I),
                       O.index_query(c1, W, H_I, d_I) + 2 * O.index_query(c2, W, H_I, d_I), atol=1e-12)
    # head h uses rows [h d_I, (h+1) d_I) of W
    assert np.allclose(O.index_query(c1, W, H_I, d_I)[1], W[d_I:2 * d_I] @ c1, atol=1e-12)


@pytest.mark.parametrize("n", [4 * 300, 4 * 300 + 2])
def test_decode_step_produces_key_and_query_as_defined(n):
    """In-step production (the token completes a group when n is a multiple of m) against the
    batch definitions over the same rows, and the step's output against decode_step fed with them."""
    layer = scaled_layer(CSA_PRO, H=4, top_k=16, H_I=4)
    wl = Workload(name="t", mode="decode", B=2, n=n, layers=(layer,), seed=5)
    d = decode_inputs(wl, 0, indexed=True)
    L = O.LayerSpec.of(layer)
    for b in range(2):
        res = O.decode_step_indexed(L, d, b)
        t = int(d["t"][b])
        rr = 8
        ring_x = F.decode_act(d["idx_raw_ring"][b], "bf16").copy()
        ring_g = F.decode_act(d["idx_gate_ring"][b], "bf16").copy()
        ring_x[t % rr] = F.decode_act(d["idx_x_new"][b], "bf16")
        ring_g[t % rr] = F.decode_act(d["idx_g_new"][b], "bf16")
        if (t + 1) % 4 == 0:
            i, codes, scale = res["index_key"]
            assert i == (t + 1) // 4 - 1
            rows = np.arange(t - 7, t + 1)
            key = O.pool_entry(ring_x[rows % rr], ring_g[rows % rr], d["idx_pos_bias"], rows - (i - 1) * 4)
            c2, s2 = F.encode_idx(key[None], "e4m3")
            assert np.array_equal(codes, c2[0]) and scale == s2[0]
        else:
            assert "index_key" not in res
        q = O.index_query(F.decode_act(d["c_q"][b], "bf16"), F.decode_act(d["W_iq"], "bf16"), 4, 128)
        qc, qs = F.encode_idx(q, "e4m3")
        assert np.array_equal(res["idx_q"][0], qc) and np.array_equal(res["idx_q"][1], qs)
        # decode_step fed with the produced key and query gives the same output
        d2 = dict(d)
        d2["idx_q"], d2["idx_q_scale"] = d["idx_q"].copy(), d["idx_q_scale"].copy()
        d2["idx_q"][b], d2["idx_q_scale"][b] = qc, qs
        if "index_key" in res:
            d2["idx_k"], d2["idx_k_scale"] = d["idx_k"].copy(), d["idx_k_scale"].copy()
            d2["idx_k"][b, res["index_key"][0]] = res["index_key"][1]
            d2["idx_k_scale"][b, res["index_key"][0]] = res["index_key"][2]
        ref = O.decode_step(L, d2, b)
        assert np.array_equal(ref["topk"], res["topk"]) and np.allclose(ref["o"], res["o"], atol=0)
