"""Pins of the oracle's chunked-prefill functions (prefill_caches, prefill_query).

A chunk of Tq tokens appended at once must give exactly what Tq successive
decode steps give when they are fed the same raw rows one token at a time:
the same compressed entries (the range [prefix/m, n/m) and nothing else),
the same window rows in their ring slots, and the same output per query,
each query seeing only the entries complete at its own position.  decode_step
is pinned on its own (hand-worked case, dense brute force, shift invariance),
so this ties the chunk path to it.  A second test runs the hand-worked
D = 4 case of test_oracle_method as a 2-token chunk and checks both outputs
against values worked out by hand.

Pages: an entry pools m tokens with a 2m-row overlap, the sequence still
shrinks m-fold, and a 128-token window stays uncompressed ("DeepSeek-V4:
Making a Million Tokens Affordable", "Two ways to shrink attention,
interleaved").
"""

import math

import numpy as np
import pytest

from csa_synth import get_workload, prefill_inputs
from csa_synth.configs import Layer, Workload
from oracle import csa as O
from oracle import formats as F


def _decode_state(L, pf, b, j, entries, win_ring):
    """Decode-step inputs for query j of the chunk, built from running caches (window ring of
    capacity w, raw/gate rings of (1+ov)m rows holding the rows before the token), all in the
    chunk's own storage formats."""
    first = pf["raw_first_row"]
    r = int(pf["t"][b, j]) - L.pos0
    rr = (1 + L.ov) * L.m
    raw, gate = pf["raw"][b], pf["gate"][b]
    ring_x = np.zeros((rr,) + raw.shape[1:], raw.dtype)
    ring_g = np.zeros((rr,) + gate.shape[1:], gate.dtype)
    for q in range(max(first, r - rr + 1), r):
        ring_x[q % rr] = raw[q - first]
        ring_g[q % rr] = gate[q - first]
    st = {
        "t": np.array([pf["t"][b, j]]),
        "x_new": pf["raw"][b][r - first][None], "g_new": pf["gate"][b][r - first][None],
        "entries": entries[None], "window": win_ring[None],
        "raw_ring": ring_x[None], "gate_ring": ring_g[None],
        "pos_bias": pf["pos_bias"], "gamma_kv": pf["gamma_kv"], "gamma_q": pf["gamma_q"],
        "q": pf["q"][b, j][None], "sinks": pf["sinks"],
    }
    if L.kind == "csa":
        st.update({"idx_q": pf["idx_q"][b, j][None], "idx_q_scale": pf["idx_q_scale"][b, j][None],
                   "head_w": pf["head_w"][b, j][None], "idx_k": pf["idx_k"][b][None],
                   "idx_k_scale": pf["idx_k_scale"][b][None]})
    return st


CASES = [
    # (layer, prefix, Tq): ragged prefix and chunk lengths, both kinds, all row formats
    (Layer(kind="csa", m=4, ov=1, top_k=8, H=4, D=128, H_I=2, d_I=32, window=16,
           kv_format="f32", idx_format="f32", act_format="f32"), 4 * 9 + 2, 23),
    (Layer(kind="csa", m=4, ov=1, top_k=6, H=2, D=512, H_I=2, d_I=128, window=8,
           kv_format="mixed", idx_format="e4m3", act_format="bf16"), 4 * 5 + 3, 14),
    (Layer(kind="hca", m=8, ov=0, top_k=0, H=2, D=128, window=8,
           kv_format="bf16", idx_format="e4m3", act_format="bf16"), 8 * 3 + 5, 21),
    (Layer(kind="csa", m=4, ov=1, top_k=8, H=2, D=128, H_I=2, d_I=32, window=16,
           kv_format="f32", idx_format="f32", act_format="f32"), 0, 11),     # from an empty cache
]


@pytest.mark.parametrize("layer,prefix,Tq", CASES)
def test_chunk_equals_successive_decode_steps(layer, prefix, Tq):
    wl = Workload(name="t", mode="prefill", B=1, n=prefix + Tq, layers=(layer,), seed=31, Tq=Tq)
    pf = prefill_inputs(wl, Tq=Tq, prefix=prefix)
    L = O.LayerSpec.of(layer)
    ents, win, e0, ne = O.prefill_caches(L, pf, 0)
    # the entry range: exactly the entries the chunk completes
    assert (e0, ne) == (prefix // layer.m, (prefix + Tq) // layer.m - prefix // layer.m)
    assert np.array_equal(ents[:e0], pf["entries"][0][:e0])
    assert np.array_equal(ents[e0 + ne:], pf["entries"][0][e0 + ne:])
    chunk = [O.prefill_query(L, pf, ents, win, 0, j) for j in range(Tq)]

    cap = win.shape[0]
    w = layer.window
    entries = pf["entries"][0].copy()
    win_ring = np.zeros((w, win.shape[1]), np.uint8)
    for r in range(max(0, prefix - w + 1), prefix):
        win_ring[r % w] = pf["window"][0][r % cap]
    for j in range(Tq):
        st = _decode_state(L, pf, 0, j, entries, win_ring)
        res = O.decode_step(L, st, 0)
        r = prefix + j
        win_ring[r % w] = res["window_row"]
        if "entry" in res:
            i, row = res["entry"]
            assert e0 <= i < e0 + ne
            entries[i] = row
        # per-query visibility: the decode step at position t sees n_visible(t) entries
        if layer.kind == "csa":
            assert np.array_equal(res["topk"], chunk[j]["topk"]), f"query {j}: selection differs"
            assert len(res["scores"]) == (r + 1) // layer.m
        assert np.allclose(res["o"], chunk[j]["o"], rtol=0, atol=1e-12), f"query {j}: output differs"
        # the chunk's window ring holds this token's row at slot r mod cap
        assert np.array_equal(win[r % cap], res["window_row"])
    assert np.array_equal(entries, ents)


def test_hand_worked_case_as_a_two_token_chunk():
    """The D=4, m=2 (overlap), k=1, w=2 case of test_oracle_method, appended as rows 4 and 5.

    Rows 0..3 are the prefix (entries 0 and 1 complete, row 3's window row cached).  The chunk
    compresses entry 2 from rows 2..5 (completed by row 5) and appends window rows 4 and 5.
    Query 0 (t = 4) sees entries 0 and 1: scores 1 and 0.5 -> top-1 = {0}; window rows 3 and 4.
      e0 = [1,1,0,0] / sqrt(0.5 + 1e-6) (its rotary pair is zero, so the rotation leaves it);
      w3 = x3 = [-2,2,0,0] (zero rotary pair); w4 = [0,0,cos4,sin4].
      q~ = [0, q1, 0, 0] with q1 = 2/sqrt(1+1e-6); logits (scale 1/2): q1*e0_1/2, q1*2/2, 0.
    Query 1 (t = 5) is the decode case worked in test_oracle_method.
    """
    layer = Layer(kind="csa", m=2, ov=1, top_k=1, H=1, D=4, d_rope=2, window=2, H_I=1, d_I=2,
                  kv_format="f32", idx_format="f32", act_format="f32")
    L = O.LayerSpec.of(layer)
    x = np.array([[2, 0, 0, 0], [0, 2, 0, 0], [2, 2, 0, 0], [-2, 2, 0, 0], [0, 0, 1, 0], [0, 0, 0, 1]], float)
    zeros = np.zeros((6, 4))
    bias = np.zeros((4, 4))
    e01 = O.compress(x, zeros, bias, np.ones(4), 2, 1, 2, 10000.0, 0, range(2))
    entries = np.zeros((3, 16), np.uint8)
    entries[:2] = F.encode_rows(e01, "f32")
    window = np.zeros((4, 16), np.uint8)                  # ring of Tq + w = 4 rows
    window[3 % 4] = F.encode_rows(O.rope(x[3], 3, 2, 10000.0), "f32")
    q = np.array([0, 2, 0, 0], np.float32)
    pf = {
        "prefix": 4, "n": 6, "Tq": 2, "t": np.array([[4, 5]]), "entries": entries[None], "window": window[None],
        "raw": x[2:6][None].astype(np.float32), "gate": np.zeros((1, 4, 4), np.float32), "raw_first_row": 2,
        "pos_bias": bias, "gamma_kv": np.ones(4), "gamma_q": np.ones(4),
        "q": np.stack([q, q])[None, :, None, :], "sinks": np.zeros(1),
        "idx_q": np.array([[[[1, 0.5]], [[1, 0.5]]]], np.float32), "idx_q_scale": np.ones((1, 2, 1), np.float32),
        "head_w": np.ones((1, 2, 1)), "idx_k": np.array([[[1, 0], [0, 1], [1, 1]]], np.float32),
        "idx_k_scale": np.ones((1, 3), np.float32),
    }
    ents, win, e0, ne = O.prefill_caches(L, pf, 0)
    assert (e0, ne) == (2, 1)
    c4, s4, c5, s5 = math.cos(4), math.sin(4), math.cos(5), math.sin(5)
    sc = 1 / math.sqrt(0.28125 + 1e-6)
    e2 = [0.0, sc, 0.25 * sc * (c4 - s4), 0.25 * sc * (s4 + c4)]
    assert np.allclose(F.decode_rows(ents[2], "f32", 4), e2, atol=1e-6)
    assert np.allclose(F.decode_rows(win[4 % 4], "f32", 4), [0, 0, c4, s4], atol=1e-7)
    assert np.allclose(F.decode_rows(win[5 % 4], "f32", 4), [0, 0, -s5, c5], atol=1e-7)
    assert np.allclose(F.decode_rows(win[3], "f32", 4), [-2, 2, 0, 0])   # the prefix's row is kept

    q1 = 2 / math.sqrt(1 + 1e-6)
    # query 0
    r0 = O.prefill_query(L, pf, ents, win, 0, 0)
    assert np.allclose(r0["scores"], [1.0, 0.5]) and list(r0["topk"]) == [0]
    e0v = [1 / math.sqrt(0.5 + 1e-6), 1 / math.sqrt(0.5 + 1e-6), 0.0, 0.0]
    rows = [e0v, [-2.0, 2.0, 0.0, 0.0], [0.0, 0.0, c4, s4]]
    logits = [q1 * e0v[1] / 2, q1 * 2 / 2, 0.0]
    Z = 1 + sum(math.exp(v) for v in logits)
    o = [sum(math.exp(logits[k]) / Z * rows[k][d] for k in range(3)) for d in range(4)]
    c, s = math.cos(-4), math.sin(-4)
    expect0 = [o[0], o[1], o[2] * c - o[3] * s, o[2] * s + o[3] * c]
    assert np.allclose(r0["o"][0], expect0, atol=1e-6)
    # query 1: the decode case worked by hand
    r1 = O.prefill_query(L, pf, ents, win, 0, 1)
    assert np.allclose(r1["scores"], [1.0, 0.5, 1.5]) and list(r1["topk"]) == [2]
    w4, w5 = [0.0, 0.0, c4, s4], [0.0, 0.0, -s5, c5]
    l_e2 = q1 * e2[1] / 2
    Z = 1 + math.exp(l_e2) + 2
    p = [math.exp(l_e2) / Z, 1 / Z, 1 / Z]
    o = [p[0] * e2[d] + p[1] * w4[d] + p[2] * w5[d] for d in range(4)]
    c, s = math.cos(-5), math.sin(-5)
    expect1 = [o[0], o[1], o[2] * c - o[3] * s, o[2] * s + o[3] * c]
    assert np.allclose(r1["o"][0], expect1, atol=1e-6)


def test_prefill_workload_entry_range_and_ring_size():
    # the chunked-prefill workload: 8,192 queries after 65,536 tokens complete entries 16,384..18,431
    wl = get_workload("csa_prefill_8k")
    layer = wl.layer()
    prefix, n = wl.n - wl.Tq, wl.n
    assert (prefix // layer.m, n // layer.m) == (16384, 18432)
    # the window ring of the chunk holds Tq + w rows, enough for every query's w rows
    assert wl.Tq + layer.window - 1 <= wl.Tq + layer.window
