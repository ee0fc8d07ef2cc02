"""Pins of the oracle's method against what the pages and mathematics fix.

Each test checks the oracle against something other than itself: a closed
form, an invariant, a library routine (torch's scaled_dot_product_attention,
numpy's sort), brute force on tiny inputs, the pages' worked counts, or a
case worked by hand.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import csa as O
from oracle import formats as F
from csa_synth import get_workload
from csa_synth.configs import Layer

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- rotary / norm

def test_rope_first_pair_is_rotation_by_position_radians():
    # theta_0 = base^0 = 1: the first rotary pair turns by exactly t radians.
    x = np.zeros(8)
    x[4], x[5] = 1.0, 0.0
    y = O.rope(x, 3.0, 4, 10000.0)
    assert np.allclose(y[4:6], [math.cos(3.0), math.sin(3.0)], atol=1e-15)
    assert np.allclose(y[:4], 0)


def test_rope_second_pair_frequency():
    # theta_1 = base^(-2/d_rope)
    x = np.zeros(4)
    x[2] = 1.0
    y = O.rope(x, 7.0, 4, 10000.0)
    a = 7.0 * 10000.0 ** (-0.5)
    assert np.allclose(y[2:4], [math.cos(a), math.sin(a)], atol=1e-15)


def test_rope_is_an_isometry_with_inverse_and_relative_dots():
    rng = np.random.default_rng(0)
    x, y = rng.normal(size=(2, 512))
    for t in [0, 5, 4096, 10 ** 6, 2 ** 20 - 1]:
        xr = O.rope(x, t, 64, 10000.0)
        assert np.isclose(np.linalg.norm(xr), np.linalg.norm(x), rtol=1e-13)
        assert np.allclose(O.rope(xr, -t, 64, 10000.0), x, atol=1e-12)
        assert np.array_equal(xr[:448], x[:448])
    # <R_a x, R_b y> = <x, R_(b-a) y>
    a, b = 1000003, 999
    lhs = O.rope(x, a, 64, 10000.0) @ O.rope(y, b, 64, 10000.0)
    rhs = x @ O.rope(y, b - a, 64, 10000.0)
    assert np.isclose(lhs, rhs, rtol=1e-10)


def test_rms_norm_unit_rms_and_constant_vector():
    rng = np.random.default_rng(1)
    x = rng.normal(0, 3, (10, 512))
    y = O.rms_norm(x, np.ones(512), 0.0)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-14)
    c = 0.25
    y = O.rms_norm(np.full(4, c), np.ones(4), 1e-6)
    assert np.allclose(y, c / math.sqrt(c * c + 1e-6), rtol=1e-15)
    g = np.array([1.0, 2.0, 0.5, -1.0])
    assert np.allclose(O.rms_norm(np.full(4, c), g, 1e-6), g * c / math.sqrt(c * c + 1e-6))


# ----------------------------------------------------------------------------- compression

def test_pool_single_row_is_identity():
    # m = 1, no overlap: each entry pools exactly its own row
    rng = np.random.default_rng(2)
    raw, gate = rng.normal(size=(2, 10, 16))
    bias = rng.normal(size=(1, 16))
    for i in range(10):
        rows, slots = O.entry_rows(i, 1, 0)
        assert list(rows) == [i]
        assert np.allclose(O.pool_entry(raw[rows], gate[rows], bias, slots), raw[i])


def test_pool_equal_logits_is_window_mean():
    rng = np.random.default_rng(3)
    raw = rng.normal(size=(40, 32))
    gate = np.zeros((40, 32))
    bias = np.zeros((8, 32))
    for i in range(10):
        rows, slots = O.entry_rows(i, 4, 1)
        exp_rows = list(range(max(0, (i - 1) * 4), (i + 1) * 4))
        assert list(rows) == exp_rows
        assert np.allclose(O.pool_entry(raw[rows], gate[rows], bias, slots), raw[exp_rows].mean(0), atol=1e-15)


@pytest.mark.parametrize("m,ov", [(4, 1), (4, 0), (128, 0), (2, 1)])
def test_pool_large_bias_selects_the_slot(m, ov):
    # A bias of +60 on window slot j makes the softmax pick raw row (i-ov)*m + j.
    rng = np.random.default_rng(4)
    n = 6 * m
    raw = rng.normal(size=(n, 8))
    gate = rng.normal(size=(n, 8))
    for i in [2, 5]:
        for j in sorted({0, m - 1, (1 + ov) * m - 1, m}):
            if j >= (1 + ov) * m:
                continue
            bias = np.zeros(((1 + ov) * m, 8))
            bias[j] = 60.0
            rows, slots = O.entry_rows(i, m, ov)
            e = O.pool_entry(raw[rows], gate[rows], bias, slots)
            assert np.allclose(e, raw[(i - ov) * m + j], rtol=0, atol=1e-15)


def test_pool_is_convex_per_channel():
    rng = np.random.default_rng(5)
    raw, gate = rng.normal(size=(2, 64, 24))
    gate *= 5
    bias = rng.normal(size=(8, 24)) * 5
    for i in range(16):
        rows, slots = O.entry_rows(i, 4, 1)
        e = O.pool_entry(raw[rows], gate[rows], bias, slots)
        assert np.all(e <= raw[rows].max(0) + 1e-14) and np.all(e >= raw[rows].min(0) - 1e-14)


def test_first_entry_uses_only_its_own_rows():
    rows, slots = O.entry_rows(0, 4, 1)
    assert list(rows) == [0, 1, 2, 3] and list(slots) == [4, 5, 6, 7]


def test_entry_counts_fall_by_m():
    with open(os.path.join(GOLDEN, "page_counts.json")) as f:
        g = json.load(f)
    e = g["entries_at_1m"]
    # grouped by 4: a decimal million splits into whole groups
    assert int(O.n_visible(e["tokens"] - 1, 0, 4)) == e["group_4"]
    # grouped by 128: the page counts the trailing partial group (ceil); only complete entries are visible
    assert int(O.n_visible(e["tokens"] - 1, 0, 128)) == e["group_128"] - 1
    assert -(-e["tokens"] // 128) == e["group_128"]
    c = g["counting_example"]
    assert int(O.n_visible(c["tokens"] - 1, 0, c["group"])) == c["entries"]
    assert c["tokens"] // c["entries"] == c["cheaper"]
    t = g["cache_table"]
    merged = int(O.n_visible(t["rows"] - 1, 0, t["rows_merged_by"]))
    assert merged * t["cols"] == t["after_row_merge"]
    assert merged * t["cols_cut_to"] == t["after_both"] and t["total"] // t["after_both"] == t["reduction"]
    s = g["selection_example"]
    scores = np.random.default_rng(0).normal(size=s["entries"])
    assert int(O.n_visible(s["passages"] - 1, 0, s["passages"] // s["entries"])) == s["entries"]
    assert (O.top_k(scores, s["read"]) >= 0).sum() == s["read"]
    hp = g["hyper_parameters"]
    assert hp["hca_m"] == hp["hca_over_csa"] * hp["csa_m"]
    # workload counts: N = floor(n / m)
    for name, N in [("csa_decode_tiny_2k", 512), ("hca_decode_128k", 1024), ("csa_decode_128k", 32768)]:
        wl = get_workload(name)
        assert int(O.n_visible(wl.n - 1, 0, wl.layers[0].m)) == N
    wl = get_workload("csa_hca_decode_1m")
    assert [int(O.n_visible(wl.n - 1, 0, L.m)) for L in wl.layers] == [262144, 8192]
    wl = get_workload("csa_prefill_8k")
    assert int(O.n_visible(wl.n - 1, 0, 4)) == 18432 and 65536 // 4 == 16384
    w = g["window_share"]
    assert round(100 * w["window"] / w["tokens"], 3) == w["percent"]


def test_visibility_and_window_edges():
    assert int(O.n_visible(2, 0, 4)) == 0 and int(O.n_visible(3, 0, 4)) == 1
    assert int(O.n_visible(10, 8, 4)) == 0 and int(O.n_visible(11, 8, 4)) == 1
    assert list(O.window_row_ids(0, 0, 128)) == [0]
    assert list(O.window_row_ids(200, 0, 128)) == list(range(73, 201))
    assert len(O.window_row_ids(10 ** 6, 0, 128)) == 128


# ----------------------------------------------------------------------------- index + top-k

def test_single_head_index_ranking_equals_sorted_dot_products():
    rng = np.random.default_rng(6)
    ik = rng.normal(size=(300, 16))
    iq = rng.normal(size=(1, 16))
    s = O.index_scores(iq, np.ones(1), np.ones(1), ik, np.ones(300))
    d = ik @ iq[0]
    assert np.allclose(s, np.maximum(d, 0))
    k = 20
    top = O.top_k(s, k)
    assert set(top) == set(np.argsort(-d)[:k])


def test_index_scores_scale_and_relu():
    rng = np.random.default_rng(7)
    ik = rng.normal(size=(50, 8))
    iq = rng.normal(size=(4, 8))
    w = np.abs(rng.normal(size=4))
    s1 = O.index_scores(iq, np.ones(4), w, ik, np.ones(50))
    s2 = O.index_scores(iq, np.ones(4), w, ik, np.full(50, 4.0))
    assert np.allclose(s2, 4 * s1)
    s3 = O.index_scores(iq, np.full(4, 0.5), w, ik, np.ones(50))
    assert np.allclose(s3, 0.5 * s1)
    # negated keys: every head whose dot was positive becomes ReLU-zero and vice versa
    s4 = O.index_scores(iq, np.ones(4), w, -ik, np.ones(50))
    dots = ik @ iq.T
    assert np.allclose(s1 + s4, np.abs(dots) @ w)
    assert np.all(s1 >= 0)


def test_top_k_brute_force_with_ties():
    rng = np.random.default_rng(8)
    for trial in range(200):
        N = int(rng.integers(1, 12))
        k = int(rng.integers(1, 14))
        s = rng.integers(0, 4, N).astype(float)          # many ties
        got = O.top_k(s, k)
        sel = [int(i) for i in got if i >= 0]
        assert len(sel) == min(N, k) and sel == sorted(sel)
        assert list(got[len(sel):]) == [-1] * (k - len(sel))
        rest = [i for i in range(N) if i not in sel]
        for a in sel:
            for b in rest:
                assert s[a] > s[b] or (s[a] == s[b] and a < b)
        assert np.array_equal(got, O.top_k_fast(s, k))


def test_top_k_fast_matches_reference_on_large_inputs():
    rng = np.random.default_rng(9)
    s = np.round(rng.normal(size=5000), 2)
    assert np.array_equal(O.top_k(s, 300), O.top_k_fast(s, 300))


# ----------------------------------------------------------------------------- attention

def _sdpa_with_sink(qt, rows, sinks, scale):
    """Library attention: the sink is one extra key whose logit is s_h and whose value is zero."""
    H, D = qt.shape
    R = rows.shape[0]
    q = torch.from_numpy(qt).view(1, H, 1, D)
    k = torch.from_numpy(rows).view(1, 1, R, D).expand(1, H, R, D)
    v = k
    bias = torch.zeros(1, H, 1, R + 1, dtype=torch.float64)
    kk = torch.cat([k, torch.zeros(1, H, 1, D, dtype=torch.float64)], dim=2)
    vv = torch.cat([v, torch.zeros(1, H, 1, D, dtype=torch.float64)], dim=2)
    # make the extra key's logit exactly s_h: zero key + additive bias s_h
    bias[0, :, 0, R] = torch.from_numpy(np.asarray(sinks, np.float64))
    o = torch.nn.functional.scaled_dot_product_attention(q, kk, vv, attn_mask=bias, scale=scale)
    return o.view(H, D).numpy()


def test_attend_matches_library_attention_with_sink_as_extra_key():
    rng = np.random.default_rng(10)
    H, D, R = 8, 128, 77
    q = rng.normal(size=(H, D))
    rows = rng.normal(size=(R, D))
    sinks = rng.normal(size=H)
    gq = rng.uniform(0.5, 1.5, D)
    t = 12345
    o = O.attend(q, t, rows, sinks, gq, 64, 10000.0)
    qt = O.prep_query(q, gq, t, 64, 10000.0)
    ref = O.rope(_sdpa_with_sink(qt, rows, sinks, 1 / math.sqrt(D)), -t, 64, 10000.0)
    assert np.allclose(o, ref, atol=1e-12)


def test_sink_to_minus_infinity_is_plain_softmax():
    rng = np.random.default_rng(11)
    H, D, R = 4, 64, 30
    q, rows = rng.normal(size=(H, D)), rng.normal(size=(R, D))
    o = O.attend(q, 0, rows, np.full(H, -1e4), np.ones(D), 64, 10000.0)
    qt = O.prep_query(q, np.ones(D), 0, 64, 10000.0)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(qt).view(1, H, 1, D), torch.from_numpy(rows).view(1, 1, R, D).expand(1, H, R, D),
        torch.from_numpy(rows).view(1, 1, R, D).expand(1, H, R, D), scale=1 / 8.0).view(H, D).numpy()
    assert np.allclose(o, ref, atol=1e-13)


def test_sink_lets_weights_sum_below_one_with_closed_form():
    rng = np.random.default_rng(12)
    H, D, R = 3, 16, 9
    q = rng.normal(size=(H, D))
    rows = rng.normal(size=(R, D))
    sinks = np.array([0.0, 2.0, -3.0])
    p = O.attention_probs(q, 0, rows, sinks, np.ones(D), 4, 10000.0)
    assert np.all(p.sum(1) < 1)
    # equal logits c: every p_j = 1 / (R + e^(s - c)); a zero query makes c = 0
    p0 = O.attention_probs(np.zeros((H, D)), 0, rows, sinks, np.ones(D), 4, 10000.0)
    assert np.allclose(p0, (1 / (R + np.exp(sinks)))[:, None])
    # single key: o = (1 - p_sink) * k at t = 0 (the output rotation is the identity)
    k = rng.normal(size=(1, D))
    o = O.attend(q, 0, k, sinks, np.ones(D), 4, 10000.0)
    qt = O.prep_query(q, np.ones(D), 0, 4, 10000.0)
    l = qt @ k[0] / 4.0
    p1 = 1 / (1 + np.exp(sinks - l))
    assert np.allclose(o, p1[:, None] * k, atol=1e-14)


def _tiny_layer(**kw):
    base = dict(kind="csa", m=4, ov=1, top_k=8, H=4, D=128, H_I=2, d_I=32,
                kv_format="f32", idx_format="f32", act_format="f32")
    base.update(kw)
    return Layer(**base)


def _state_from_raw(layer, n, seed, pos0):
    """Caches built from raw rows through the oracle's own compress / window steps (f32 rows)."""
    rng = np.random.default_rng(seed)
    D, m, ov = layer.D, layer.m, layer.ov
    raw = rng.normal(size=(n, D))
    gate = rng.normal(size=(n, D))
    bias = rng.normal(size=((1 + ov) * m, D))
    L = O.LayerSpec.of(layer, pos0)
    t = pos0 + n - 1
    N = n // m
    ent = O.compress(raw, gate, bias, np.ones(D), m, ov, 64, 10000.0, pos0, range(N))
    rr = (1 + ov) * m
    raw_ring = np.zeros((rr, D))
    gate_ring = np.zeros((rr, D))
    for r in range(max(0, n - rr), n):
        raw_ring[r % rr], gate_ring[r % rr] = raw[r], gate[r]
    window = np.zeros((layer.window, D))
    for r in range(max(0, n - layer.window), n):
        window[r % layer.window] = O.rope(raw[r], pos0 + r, 64, 10000.0)
    st = {
        "t": np.array([t]), "x_new": raw[n - 1:n].astype(np.float32), "g_new": gate[n - 1:n].astype(np.float32),
        "entries": F.encode_rows(ent, "f32")[None], "window": F.encode_rows(window, "f32")[None],
        "raw_ring": raw_ring[None].astype(np.float32), "gate_ring": gate_ring[None].astype(np.float32),
        "pos_bias": bias, "gamma_kv": np.ones(D), "gamma_q": np.ones(D),
        "q": rng.normal(size=(1, layer.H, D)).astype(np.float32), "sinks": rng.normal(size=layer.H),
        "idx_q": rng.normal(size=(1, layer.H_I, layer.d_I)).astype(np.float32),
        "idx_q_scale": np.ones((1, layer.H_I), np.float32),
        "head_w": rng.normal(size=(1, layer.H_I)),
        "idx_k": rng.normal(size=(1, max(N, 1), layer.d_I)).astype(np.float32),
        "idx_k_scale": np.ones((1, max(N, 1)), np.float32),
    }
    return L, st, raw


@pytest.mark.parametrize("delta", [1, 4096, 10 ** 6])
def test_output_carries_only_relative_positions(delta):
    layer = _tiny_layer()
    L0, st0, _ = _state_from_raw(layer, 203, 13, 0)
    L1, st1, _ = _state_from_raw(layer, 203, 13, delta)
    o0 = O.decode_step(L0, st0, 0)["o"]
    o1 = O.decode_step(L1, st1, 0)["o"]
    assert np.allclose(o0, o1, atol=1e-9)


def test_shift_invariance_fails_without_inverse_rope():
    # sanity of the pin: without the output's inverse rotation the result moves with the shift
    rng = np.random.default_rng(14)
    q, base_rows = rng.normal(size=(2, 16)), rng.normal(size=(5, 16))
    pos = np.arange(5) * 3

    def out(delta):
        rows = np.stack([O.rope(base_rows[j], pos[j] + delta, 8, 1e4) for j in range(5)])
        t = 20 + delta
        return O.attend(q, t, rows, np.zeros(2), np.ones(16), 8, 1e4), t

    (o0, t0), (o1, t1) = out(0), out(7)
    assert np.allclose(o0, o1, atol=1e-12)
    assert not np.allclose(O.rope(o0, t0, 8, 1e4), O.rope(o1, t1, 8, 1e4), atol=1e-3)


def test_full_top_k_and_window_is_dense_attention():
    # "if k covers every block, S_t is the whole past and the layer is dense attention again"
    n = 37
    layer = _tiny_layer(top_k=64, window=64)
    L, st, raw = _state_from_raw(layer, n, 15, 0)
    res = O.decode_step(L, st, 0)
    N = n // 4
    assert list(res["topk"][:N]) == list(range(N)) and np.all(res["topk"][N:] == -1)
    ent = F.decode_rows(st["entries"][0][:N], "f32", 128)
    if (n) % 4 == 0:
        ent[-1] = F.decode_rows(res["entry"][1], "f32", 128)
    allraw = np.stack([O.rope(raw[r], r, 64, 10000.0) for r in range(n)])
    rows = np.concatenate([ent, allraw])
    qt = O.prep_query(st["q"][0].astype(np.float64), np.ones(128), n - 1, 64, 10000.0)
    ref = O.rope(_sdpa_with_sink(qt, rows, st["sinks"], 1 / math.sqrt(128)), -(n - 1), 64, 10000.0)
    assert np.allclose(res["o"], ref, atol=1e-6)       # window rows were stored as f32


def test_attended_row_count_freezes_at_k_plus_w():
    layer = _tiny_layer(top_k=8, window=16)
    for n in [5, 20, 33, 64, 120, 200]:
        L, st, _ = _state_from_raw(layer, n, 16, 0)
        res = O.decode_step(L, st, 0)
        assert res["n_rows"] == min(n // 4, 8) + min(n, 16)


def test_decode_compress_matches_batch_compress():
    # the step's on-the-fly compression of the completed group equals compressing it from all rows
    layer = _tiny_layer()
    n = 48
    L, st, raw = _state_from_raw(layer, n, 17, 0)
    res = O.decode_step(L, st, 0)
    i, row = res["entry"]
    assert i == n // 4 - 1
    assert np.allclose(F.decode_rows(row, "f32", 128), F.decode_rows(st["entries"][0][i], "f32", 128), atol=1e-6)


# ----------------------------------------------------------------------------- hand-worked case

def test_hand_worked_tiny_case():
    """D=4, d_r=2, m=2 (overlap), n=6, k=1, w=2, one query head, one indexer head.

    Raw rows x0..x5, all gate logits and biases 0 (so each entry is its window's mean):
      x0=[2,0,0,0] x1=[0,2,0,0] x2=[2,2,0,0] x3=[-2,2,0,0] x4=[0,0,1,0] x5=[0,0,0,1]
    Entries (t = 5 sees entries 0,1,2):
      e0 = mean(x0,x1) = [1,1,0,0];  e1 = mean(x0..x3) = [.5,1.5,0,0];  e2 = mean(x2..x5) = [0,1,.25,.25]
    Index keys k0=[1,0], k1=[0,1], k2=[1,1], query [1,.5], w=1 -> scores 1, .5, 1.5 -> top-1 = {2}.
    e2 after RMSNorm: ms = (1 + .0625 + .0625)/4 = .28125 -> scale 1/sqrt(.281251);
      rotary pair (dims 2,3) = (.25,.25)*scale turned by angle 4 (position i*m = 4, theta_0 = 1).
    Window rows (raw 4, 5) turned at their positions: x4 -> [0,0,cos4,sin4], x5 -> [0,0,-sin5,cos5].
    Query q=[0,2,0,0]: RMSNorm -> [0, 2/sqrt(1+1e-6), 0, 0]; its rotary pair is zero.
    Logits (scale 1/sqrt(4)): l(e2) = q1*e2_1/2, l(w4) = l(w5) = 0; sink s = 0.
    p = e^l / (e^0 + sum e^l); o = sum p_j row_j, then dims 2,3 turned by -5.
    """
    c4, s4, c5, s5 = math.cos(4), math.sin(4), math.cos(5), math.sin(5)
    sc = 1 / math.sqrt(0.28125 + 1e-6)
    e2 = [0.0, sc, 0.25 * sc * (c4 - s4), 0.25 * sc * (s4 + c4)]
    w4 = [0.0, 0.0, c4, s4]
    w5 = [0.0, 0.0, -s5, c5]
    q1 = 2 / math.sqrt(1 + 1e-6)
    l_e2 = q1 * e2[1] / 2
    Z = 1 + math.exp(l_e2) + 2
    p = [math.exp(l_e2) / Z, 1 / Z, 1 / Z]
    o = [p[0] * e2[d] + p[1] * w4[d] + p[2] * w5[d] for d in range(4)]
    c, s = math.cos(-5), math.sin(-5)
    expect = [o[0], o[1], o[2] * c - o[3] * s, o[2] * s + o[3] * c]
    assert abs(p[0] - 0.6872) < 1e-3           # checked by calculator: e^1.8856 / (3 + e^1.8856)

    layer = Layer(kind="csa", m=2, ov=1, top_k=1, H=1, D=4, d_rope=2, window=2, H_I=1, d_I=2,
                  kv_format="f32", idx_format="f32", act_format="f32")
    L = O.LayerSpec.of(layer)
    x = np.array([[2, 0, 0, 0], [0, 2, 0, 0], [2, 2, 0, 0], [-2, 2, 0, 0], [0, 0, 1, 0], [0, 0, 0, 1]], float)
    zeros = np.zeros((6, 4))
    bias = np.zeros((4, 4))
    ent = O.compress(x, zeros, bias, np.ones(4), 2, 1, 2, 10000.0, 0, range(3))
    assert np.allclose(ent[2], e2, atol=1e-15)
    assert np.allclose(ent[0], np.array([1, 1, 0, 0]) / math.sqrt(0.5 + 1e-6), atol=1e-15)
    window = np.zeros((2, 4))
    window[4 % 2] = O.rope(x[4], 4, 2, 10000.0)
    st = {
        "t": np.array([5]), "x_new": x[5:6].astype(np.float32), "g_new": np.zeros((1, 4), np.float32),
        "entries": F.encode_rows(ent, "f32")[None], "window": F.encode_rows(window, "f32")[None],
        "raw_ring": x[2:6][[2, 3, 0, 1]][None].astype(np.float32),    # slot r mod 4 holds raw row r
        "gate_ring": np.zeros((1, 4, 4), np.float32), "pos_bias": bias, "gamma_kv": np.ones(4),
        "gamma_q": np.ones(4), "q": np.array([[[0, 2, 0, 0]]], np.float32), "sinks": np.zeros(1),
        "idx_q": np.array([[[1, 0.5]]], np.float32), "idx_q_scale": np.ones((1, 1), np.float32),
        "head_w": np.ones((1, 1)), "idx_k": np.array([[[1, 0], [0, 1], [1, 1]]], np.float32),
        "idx_k_scale": np.ones((1, 3), np.float32),
    }
    res = O.decode_step(L, st, 0)
    assert np.allclose(res["scores"], [1, 0.5, 1.5])
    assert list(res["topk"]) == [2]
    assert res["n_rows"] == 3
    assert np.allclose(res["o"][0], expect, atol=1e-6)
