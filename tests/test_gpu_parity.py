"""GPU parity: the CUDA path through the C ABI against the float64 oracle.

Every input is seeded and synthetic (csa_synth); every expected value comes
from oracle/.  Sizes span several tiles with ragged tails; the full-size
workloads are checked on their own launch configuration.
"""

import json
import os

import numpy as np
import pytest
import torch

from csa_synth import compress_inputs, decode_inputs, get_workload, prefill_inputs
from csa_synth.configs import CSA_PRO, HCA_128K, HCA_PRO, Layer, Workload, raw_ring_rows, scaled_layer
from long_context_sparse_csa_b200 import binding as C
from long_context_sparse_csa_b200.state import LayerState
from oracle import csa as O
from oracle import formats as F

import _gpu_util
from _gpu_util import assert_out_close, assert_rows_match, check_topk, dev, host, out_values

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    C.lib()
    yield
    torch.cuda.synchronize()
    # measured error statistics of the parity cases, written when CSA_PARITY_STATS names a file
    out = os.environ.get("CSA_PARITY_STATS")
    if out:
        with open(out, "w") as f:
            json.dump(_gpu_util.STATS, f, indent=1)


def _layer(**kw):
    base = dict(kind="csa", m=4, ov=1, top_k=64, H=8, D=128, H_I=4, d_I=64,
                kv_format="f32", idx_format="f32", act_format="f32")
    base.update(kw)
    return Layer(**base)


def _no_device_error(ws):
    assert C.csa_device_error(ws) == 0


# ----------------------------------------------------------------------------- compression + window append

@pytest.mark.parametrize("kv,act,D,m,ov", [("f32", "f32", 128, 4, 1), ("bf16", "bf16", 512, 4, 1),
                                           ("mixed", "bf16", 512, 4, 1), ("mixed", "bf16", 512, 128, 0),
                                           ("bf16", "bf16", 512, 128, 0)])
def test_compress_parity(kv, act, D, m, ov):
    layer = _layer(kv_format=kv, act_format=act, D=D, m=m, ov=ov, H=64 if D == 512 else 8)
    n = 1000 if m == 4 else 1400                         # ragged: n is not a multiple of m
    wl = Workload(name="t", mode="decode", B=2, n=n, layers=(layer,), seed=21)
    ci = compress_inputs(wl, n_rows=n)
    rng = np.random.default_rng(5)
    gamma = rng.uniform(0.5, 1.5, D).astype(np.float32)
    N = n // m
    rb = F.row_bytes(kv, D)
    entries = torch.zeros((2, N + 3, rb), dtype=torch.uint8, device="cuda")
    window = torch.zeros((2, 128, rb), dtype=torch.uint8, device="cuda")
    st = LayerState(layer, 2, entries=entries, window=window, raw=dev(ci["raw"]), gate=dev(ci["gate"]),
                    pos_bias=dev(ci["pos_bias"]), gamma_kv=dev(gamma))
    q_pos = torch.arange(n, device="cuda", dtype=torch.int64).repeat(2, 1).contiguous()
    C.csa_compress(st.L, st.cache(), st.params(), q_pos, n)
    torch.cuda.synchronize()
    got = host(entries)
    for b in range(2):
        ref = O.compress(F.decode_act(ci["raw"][b], act), F.decode_act(ci["gate"][b], act), ci["pos_bias"], gamma,
                         m, ov, 64, 10000.0, 0, range(N))
        assert_rows_match(got[b, :N], ref, kv, D)
        assert not got[b, N:].any(), "entries past the last complete group must not be written"


@pytest.mark.parametrize("kv,act,D", [("f32", "f32", 128), ("bf16", "bf16", 512), ("mixed", "bf16", 512)])
def test_append_window_parity(kv, act, D):
    layer = _layer(kv_format=kv, act_format=act, D=D, H=64 if D == 512 else 8)
    B, n, Tq, pos0 = 2, 700, 300, 12345
    wl = Workload(name="t", mode="decode", B=B, n=n, layers=(layer,), seed=22)
    ci = compress_inputs(wl, n_rows=n)
    rb = F.row_bytes(kv, D)
    cap = Tq + 128
    window = torch.zeros((B, cap, rb), dtype=torch.uint8, device="cuda")
    entries = torch.zeros((B, 1, rb), dtype=torch.uint8, device="cuda")
    raw = dev(ci["raw"])
    gate = dev(ci["gate"])
    st = LayerState(layer, B, pos0, entries=entries, window=window, raw=raw, gate=gate)
    first = n - Tq
    q_pos = (pos0 + torch.arange(first, n, device="cuda", dtype=torch.int64)).repeat(B, 1).contiguous()
    C.csa_append(st.L, st.cache(), None, None, q_pos, Tq)
    torch.cuda.synchronize()
    got = host(window)
    for b in range(B):
        x = F.decode_act(ci["raw"][b], act)
        for r in range(first, n, 37):
            ref = O.rope(x[r], pos0 + r, 64, 10000.0)
            assert_rows_match(got[b, r % cap][None], ref[None], kv, D, max_code_mismatch=1.0)


# ----------------------------------------------------------------------------- indexer + top-k

def _index_case(wl, li=0, n=None):
    d = decode_inputs(wl, li, n=n)
    layer = wl.layers[li]
    st = LayerState.from_arrays(layer, wl.B, d)
    return d, layer, st


@pytest.mark.parametrize("name,n", [("csa_decode_tiny_2k", None), ("csa_decode_128k", 20000 * 4 + 3),
                                    ("csa_decode_128k", None)])
def test_index_topk_parity(name, n):
    wl = get_workload(name)
    d, layer, st = _index_case(wl, n=n)
    B = wl.B
    cap = d["entries"].shape[1]
    topk = torch.full((B, layer.top_k), -7, dtype=torch.int32, device="cuda")
    scores = torch.zeros((B, cap), dtype=torch.float32, device="cuda")
    ws = st.workspace("index_topk", 1, cap)
    q_pos = dev(d["t"])
    C.csa_index_topk(st.L, st.cache(), dev(d["idx_q"]), dev(d["idx_q_scale"]), dev(d["head_w"]), q_pos, 1, cap,
                     topk, scores, ws)
    torch.cuda.synchronize()
    _no_device_error(ws)
    got_s, got_k = host(scores), host(topk)
    for b in range(B):
        nv = int(O.n_visible(d["t"][b], 0, layer.m))
        iq = F.decode_idx(d["idx_q"][b], layer.idx_format)
        ik = F.decode_idx(d["idx_k"][b][:nv], layer.idx_format)
        ref = O.index_scores(iq, d["idx_q_scale"][b], d["head_w"][b], ik, d["idx_k_scale"][b][:nv])
        scale = np.abs(ref).max() + 1e-30
        assert np.max(np.abs(got_s[b, :nv] - ref)) <= 1e-5 * scale + 1e-7
        check_topk(got_k[b], ref, layer.top_k)


@pytest.mark.parametrize("n", [9000, 160000])
def test_topk_ties_go_to_smaller_index(n):
    # identical index keys: every visible entry scores the same -> the k smallest indices
    # (n = 160000: 40,000 entries, the multi-CTA path with every candidate tied at the k-th key)
    wl = get_workload("csa_decode_128k", B=2, n=n)
    d, layer, st = _index_case(wl)
    d["idx_k"][:] = d["idx_k"][:, :1]
    d["idx_k_scale"][:] = d["idx_k_scale"][:, :1]
    st = LayerState.from_arrays(layer, wl.B, d)
    cap = d["entries"].shape[1]
    topk = torch.zeros((2, layer.top_k), dtype=torch.int32, device="cuda")
    ws = st.workspace("index_topk", 1, cap)
    C.csa_index_topk(st.L, st.cache(), dev(d["idx_q"]), dev(d["idx_q_scale"]), dev(d["head_w"]), dev(d["t"]), 1,
                     cap, topk, None, ws)
    got = host(topk)
    assert np.array_equal(got, np.tile(np.arange(layer.top_k), (2, 1)))


def test_topk_long_row_with_duplicated_keys():
    # blocks of 7 identical keys: many exact ties around the k-th score in a multi-CTA row
    wl = get_workload("csa_decode_128k", B=2, n=4 * 70001)
    d, layer, st = _index_case(wl)
    d["idx_k"][:] = np.repeat(d["idx_k"][:, ::7], 7, axis=1)[:, :d["idx_k"].shape[1]]
    d["idx_k_scale"][:] = np.repeat(d["idx_k_scale"][:, ::7], 7, axis=1)[:, :d["idx_k"].shape[1]]
    st = LayerState.from_arrays(layer, wl.B, d)
    cap = d["entries"].shape[1]
    topk = torch.zeros((2, layer.top_k), dtype=torch.int32, device="cuda")
    ws = st.workspace("index_topk", 1, cap)
    C.csa_index_topk(st.L, st.cache(), dev(d["idx_q"]), dev(d["idx_q_scale"]), dev(d["head_w"]), dev(d["t"]), 1,
                     cap, topk, None, ws)
    got = host(topk)
    for b in range(2):
        iq = F.decode_idx(d["idx_q"][b], layer.idx_format)
        ref = O.index_scores(iq, d["idx_q_scale"][b], d["head_w"][b], F.decode_idx(d["idx_k"][b], "e4m3"),
                             d["idx_k_scale"][b])
        check_topk(got[b], ref, layer.top_k)


def test_topk_fewer_visible_than_k_pads():
    wl = get_workload("csa_decode_128k", B=3, n=2000)
    d, layer, st = _index_case(wl)
    d["t"] = np.array([3, 500, 1999], dtype=np.int64)        # 1, 125, 500 visible entries (< k = 1024)
    cap = d["entries"].shape[1]
    topk = torch.zeros((3, layer.top_k), dtype=torch.int32, device="cuda")
    ws = st.workspace("index_topk", 1, cap)
    C.csa_index_topk(st.L, st.cache(), dev(d["idx_q"]), dev(d["idx_q_scale"]), dev(d["head_w"]), dev(d["t"]), 1,
                     cap, topk, None, ws)
    got = host(topk)
    for b, nv in enumerate([1, 125, 500]):
        assert np.array_equal(got[b, :nv], np.arange(nv)) and np.all(got[b, nv:] == -1)


# ----------------------------------------------------------------------------- fused decode steps

def _oracle_step(layer, d, b, pos0=0):
    L = O.LayerSpec.of(layer, pos0)
    return O.decode_step(L, d, b)


def _run_decode(wl, li=0, n=None, d=None, sharp=1.0):
    layer = wl.layers[li]
    if d is None:
        d = decode_inputs(wl, li, n=n)
    st = LayerState.from_arrays(layer, wl.B, d)
    if sharp != 1.0:
        st.L.softmax_scale = sharp / np.sqrt(layer.D)
    B, H, D = wl.B, layer.H, layer.D
    cap = d["entries"].shape[1]
    out_dtype = torch.float32 if layer.act_format == "f32" else torch.int16
    out = torch.zeros((B, H, D), dtype=out_dtype, device="cuda")
    ws = st.workspace("decode_step", 1, cap)
    q_pos = dev(d["t"])
    topk = None
    if layer.kind == "csa":
        topk = torch.zeros((B, layer.top_k), dtype=torch.int32, device="cuda")
        C.csa_decode_step(st.L, st.cache(), st.params(), dev(d["q"]), dev(d["idx_q"]), dev(d["idx_q_scale"]),
                          dev(d["head_w"]), dev(d["x_new"]), dev(d["g_new"]), q_pos, out, topk, ws)
    else:
        C.hca_decode_step(st.L, st.cache(), st.params(), dev(d["q"]), dev(d["x_new"]), dev(d["g_new"]), q_pos,
                          out, ws)
    torch.cuda.synchronize()
    _no_device_error(ws)
    return d, st, out, topk


def _check_decode(wl, li=0, n=None, bs=None, sharp=1.0, rel_l2=1e-2, max_abs=2e-2, mean_abs=2e-3):
    layer = wl.layers[li]
    d, st, out, topk = _run_decode(wl, li, n, sharp=sharp)
    got = out_values(out, layer.act_format)
    ents, wins = host(st.entries), host(st.window)
    for b in (range(wl.B) if bs is None else bs):
        L = O.LayerSpec.of(layer)
        if sharp != 1.0:
            L.scale = sharp / np.sqrt(layer.D)
        ref = O.decode_step(L, d, b)
        t = int(d["t"][b])
        # the appended window row and the compressed entry
        x_new = F.decode_act(d["x_new"][b], layer.act_format)
        assert_rows_match(wins[b, t % layer.window][None], O.rope(x_new, t, 64, layer.rope_base)[None],
                          layer.kv_format, layer.D, max_code_mismatch=1.0)
        if "entry" in ref:
            i = ref["entry"][0]
            rr = raw_ring_rows(layer)
            raw = F.decode_act(d["raw_ring"][b], layer.act_format).copy()
            gate = F.decode_act(d["gate_ring"][b], layer.act_format).copy()
            raw[t % rr], gate[t % rr] = x_new, F.decode_act(d["g_new"][b], layer.act_format)
            rows, slots = O.entry_rows(i, layer.m, layer.ov)
            e = O.pool_entry(raw[rows % rr], gate[rows % rr], d["pos_bias"], slots)
            e = O.rope(O.rms_norm(e, d["gamma_kv"], layer.eps), i * layer.m, 64, layer.rope_base)
            assert_rows_match(ents[b, i][None], e[None], layer.kv_format, layer.D, max_code_mismatch=1.0)
        if layer.kind == "csa":
            tk = host(topk)[b]
            swapped = check_topk(tk, ref["scores"], layer.top_k)
            if swapped:
                # a tie-band swap: attend over the GPU's (valid) selection
                d2 = dict(d)
                ref = _oracle_with_selection(L, d, b, tk)
        assert_out_close(got[b], ref["o"], max_abs=max_abs, mean_abs=mean_abs, rel_l2=rel_l2,
                         tag=f"{wl.name}/L{li}/n={n}/b={b}/sharp={sharp}")


def _oracle_with_selection(L, d, b, sel):
    t = int(d["t"][b])
    res = O.decode_step(L, d, b)
    ents = d["entries"][b].copy()
    if "entry" in res:
        ents[res["entry"][0]] = res["entry"][1]
    window = d["window"][b].copy()
    window[(t - L.pos0) % L.window] = res["window_row"]
    ids = np.asarray(sel)[np.asarray(sel) >= 0]
    rows = np.concatenate([F.decode_rows(ents[ids], L.kv_format, L.D),
                           F.decode_rows(window[O.window_row_ids(t, L.pos0, L.window) % L.window], L.kv_format, L.D)])
    q = F.decode_act(d["q"][b], L.act_format)
    return {"o": O.attend(q, t, rows, d["sinks"], d["gamma_q"], 64, L.rope_base, L.scale, L.eps)}


def test_decode_tiny_csa_fp32():
    wl = get_workload("csa_decode_tiny_2k")
    d, st, out, topk = _run_decode(wl)
    ref = _oracle_step(wl.layers[0], d, 0)
    got = out_values(out, "f32")
    assert_out_close(got[0], ref["o"], max_abs=1e-4, mean_abs=1e-5, rel_l2=1e-4)
    check_topk(host(topk)[0], ref["scores"], 64)


def test_decode_tiny_end_to_end_from_raw_rows():
    """Config built from raw rows through the operator itself: compress all entries, append the window,
    then one fused decode step; checked against the oracle doing the same from the same raw rows."""
    wl = get_workload("csa_decode_tiny_2k")
    layer = wl.layers[0]
    n, D = wl.n, layer.D
    ci = compress_inputs(wl, n_rows=n)
    d = decode_inputs(wl)
    N = n // layer.m
    rb = F.row_bytes("f32", D)
    entries = torch.zeros((1, N, rb), dtype=torch.uint8, device="cuda")
    window = torch.zeros((1, 128, rb), dtype=torch.uint8, device="cuda")
    raw_all, gate_all = dev(ci["raw"]), dev(ci["gate"])
    st = LayerState(layer, 1, entries=entries, window=window, raw=raw_all, gate=gate_all,
                    idx_keys=dev(d["idx_k"]), idx_key_scale=dev(d["idx_k_scale"]), pos_bias=dev(ci["pos_bias"]),
                    gamma_kv=dev(d["gamma_kv"]), gamma_q=dev(d["gamma_q"]), sinks=dev(d["sinks"]))
    q_all = torch.arange(n, device="cuda", dtype=torch.int64)[None].contiguous()
    C.csa_compress(st.L, st.cache(), st.params(), q_all[:, : n - 1].contiguous(), n - 1)
    C.csa_append(st.L, st.cache(), None, None, q_all[:, n - 128: n - 1].contiguous(), 127)
    # decode step for the last token with rings holding rows n-8 .. n-2
    rr = raw_ring_rows(layer)
    raw_ring = torch.zeros((1, rr, D), dtype=torch.float32, device="cuda")
    gate_ring = torch.zeros_like(raw_ring)
    for r in range(n - rr, n - 1):
        raw_ring[0, r % rr] = raw_all[0, r]
        gate_ring[0, r % rr] = gate_all[0, r]
    st.raw, st.gate = raw_ring, gate_ring
    out = torch.zeros((1, layer.H, D), dtype=torch.float32, device="cuda")
    topk = torch.zeros((1, layer.top_k), dtype=torch.int32, device="cuda")
    ws = st.workspace("decode_step", 1, N)
    C.csa_decode_step(st.L, st.cache(), st.params(), dev(d["q"]), dev(d["idx_q"]), dev(d["idx_q_scale"]),
                      dev(d["head_w"]), raw_all[:, n - 1].contiguous(), gate_all[:, n - 1].contiguous(),
                      dev(d["t"]), out, topk, ws)
    torch.cuda.synchronize()
    # oracle from the same raw rows
    raw = ci["raw"][0].astype(np.float64)
    gate = ci["gate"][0].astype(np.float64)
    ents = O.compress(raw, gate, ci["pos_bias"], d["gamma_kv"], 4, 1, 64, 10000.0, 0, range(N))
    win = np.stack([O.rope(raw[r], r, 64, 10000.0) for r in range(n - 128, n)])
    assert_rows_match(host(entries)[0], ents, "f32", D)
    assert_rows_match(host(window)[0][np.arange(n - 128, n) % 128], win, "f32", D)
    iq = d["idx_q"][0].astype(np.float64)
    s = O.index_scores(iq, d["idx_q_scale"][0], d["head_w"][0], d["idx_k"][0].astype(np.float64), d["idx_k_scale"][0])
    sel = host(topk)[0]
    check_topk(sel, s, 64)
    rows = np.concatenate([ents[sel], win])
    ref = O.attend(d["q"][0].astype(np.float64), n - 1, rows, d["sinks"], d["gamma_q"], 64, 10000.0)
    assert_out_close(out_values(out, "f32")[0], ref, max_abs=1e-4, mean_abs=1e-5, rel_l2=1e-4)


def test_decode_hca_128k():
    _check_decode(get_workload("hca_decode_128k"))


def test_decode_csa_128k():
    _check_decode(get_workload("csa_decode_128k"))


def test_decode_csa_128k_sharp_logits():
    # Logits 8x sharper than 1/sqrt(D).  The kernel rounds q~ to bf16 (relative 2^-9 per element), so a
    # logit moves by up to ~8 * 2^-9 * sum|q_d k_d| / sqrt(D) ~ 0.04 and the output, dominated by a few
    # keys of size ~3, by up to ~0.1: the bound here is 4x the standard one.
    _check_decode(get_workload("csa_decode_128k", B=2), sharp=8.0, rel_l2=4e-2, max_abs=8e-2, mean_abs=8e-3)


@pytest.mark.parametrize("li", [0, 1])
def test_decode_1m_interleaved(li):
    _check_decode(get_workload("csa_hca_decode_1m"), li=li)


@pytest.mark.parametrize("n", [1, 3, 4, 130, 4099])
def test_decode_short_contexts(n):
    # empty, sub-group, first group, ragged window, fewer entries than k
    wl = get_workload("csa_decode_128k", B=2)
    _check_decode(wl, n=n)
    wl = get_workload("csa_hca_decode_1m")
    _check_decode(wl, li=1, n=n)


def test_decode_hca_bf16_rows_128_heads():
    # dense attention on bf16 rows with 128 heads: the tcgen05 kernel's bf16 row path
    wl = get_workload("hca_decode_128k", B=2, layers=(scaled_layer(HCA_128K, H=128),))
    _check_decode(wl)


def test_decode_csa_bf16_rows():
    # top-k attention on bf16 rows: the mma.sync kernel's bf16 tile path
    wl = get_workload("csa_decode_128k", B=2, layers=(scaled_layer(CSA_PRO, kv_format="bf16"),))
    _check_decode(wl)


def test_decode_per_sequence_positions():
    wl = get_workload("csa_decode_128k", B=3, n=6000)
    layer = wl.layers[0]
    d = decode_inputs(wl)
    d["t"] = np.array([5999, 4003, 777], dtype=np.int64)
    d_st, st, out, topk = _run_decode(wl, d=d)
    got = out_values(out, layer.act_format)
    for b in range(3):
        ref = _oracle_step(layer, d, b)
        sw = check_topk(host(topk)[b], ref["scores"], layer.top_k)
        if sw:
            ref = _oracle_with_selection(O.LayerSpec.of(layer), d, b, host(topk)[b])
        assert_out_close(got[b], ref["o"])


def test_decode_hca_per_sequence_positions():
    # HCA steps of one call where one sequence's token completes a group (its new entry joins in the
    # combine) and the others' do not; every token's own window row joins there too
    wl = get_workload("hca_decode_128k", B=3)
    layer = wl.layers[0]
    d = decode_inputs(wl)
    d["t"] = np.array([131071, 130999, 1500], dtype=np.int64)
    _, st, out, _ = _run_decode(wl, d=d)
    got = out_values(out, layer.act_format)
    for b in range(3):
        ref = _oracle_step(layer, d, b)
        assert_out_close(got[b], ref["o"], tag=f"hca positions b{b}")


# ----------------------------------------------------------------------------- chunked prefill

def _prefill_case(wl, Tq=None, prefix=None):
    layer = wl.layers[0]
    pf = prefill_inputs(wl, Tq=Tq, prefix=prefix)
    st = LayerState.from_arrays(layer, wl.B, pf, raw_key="raw", gate_key="gate", raw_base=pf["raw_first_row"])
    n_max = pf["n"] // layer.m
    out = torch.zeros((wl.B, pf["Tq"], layer.H, layer.D), dtype=torch.int16, device="cuda")
    topk = torch.zeros((wl.B, pf["Tq"], layer.top_k), dtype=torch.int32, device="cuda")
    ws = st.workspace("prefill", pf["Tq"], n_max)
    opt = lambda k: dev(pf[k]) if pf.get(k) is not None else None  # noqa: E731  (HCA layers have no indexer)
    C.csa_prefill(st.L, st.cache(), st.params(), dev(pf["q"]), opt("idx_q"), opt("idx_q_scale"),
                  opt("head_w"), dev(pf["t"]), pf["Tq"], n_max, out, topk if layer.kind == "csa" else None, ws)
    torch.cuda.synchronize()
    _no_device_error(ws)
    return pf, st, out, topk


def _check_prefill(wl, Tq, prefix, queries):
    layer = wl.layers[0]
    pf, st, out, topk = _prefill_case(wl, Tq, prefix)
    L = O.LayerSpec.of(layer)
    ents, win, e0, ne = O.prefill_caches(L, pf, 0)
    # caches written by the operator
    raw = F.decode_act(pf["raw"][0], layer.act_format)
    gate = F.decode_act(pf["gate"][0], layer.act_format)
    vals = O.compress(raw, gate, pf["pos_bias"], pf["gamma_kv"], layer.m, layer.ov, 64, layer.rope_base, 0,
                      range(e0, e0 + ne), raw_first_row=pf["raw_first_row"])
    assert_rows_match(host(st.entries)[0, e0:e0 + ne], vals, layer.kv_format, layer.D)
    got = out_values(out, layer.act_format)[0]
    tk = host(topk)[0]
    for j in queries:
        ref = O.prefill_query(L, pf, ents, win, 0, j)
        if layer.kind == "csa" and check_topk(tk[j], ref["scores"], layer.top_k):
            t = int(pf["t"][0, j])
            ids = tk[j][tk[j] >= 0]
            rows = np.concatenate([F.decode_rows(ents[ids], layer.kv_format, layer.D),
                                   F.decode_rows(win[O.window_row_ids(t, 0, layer.window) % win.shape[0]],
                                                 layer.kv_format, layer.D)])
            ref = {"o": O.attend(F.decode_act(pf["q"][0, j], layer.act_format), t, rows, pf["sinks"],
                                 pf["gamma_q"], 64, layer.rope_base)}
        assert_out_close(got[j], ref["o"])


def test_prefill_small_ragged():
    wl = get_workload("csa_prefill_8k")
    _check_prefill(wl, Tq=301, prefix=4096 + 2, queries=range(0, 301, 7))


def test_prefill_from_empty_cache():
    wl = get_workload("csa_prefill_8k")
    _check_prefill(wl, Tq=200, prefix=0, queries=[0, 1, 2, 3, 4, 5, 50, 127, 128, 129, 199])


def test_prefill_hca_dense():
    # HCA chunked prefill: every query of the chunk attends densely (200 query rows: the mma.sync
    # kernel; calls of at most 8 rows take the tcgen05 kernel, which the decode tests cover)
    wl = get_workload("csa_prefill_8k", layers=(HCA_PRO,))
    _check_prefill(wl, Tq=200, prefix=4096 + 2, queries=[0, 1, 62, 63, 64, 127, 128, 199])


def test_prefill_hca_dense_64_heads():
    # HCA chunked prefill with 64 heads of bf16 rows: the persistent tcgen05 prefill kernel over dense
    # slot lists (about 33 entries and up to 128 window rows: a full tile and a ragged one)
    layer = scaled_layer(HCA_PRO, H=64, kv_format="bf16")
    wl = get_workload("csa_prefill_8k", layers=(layer,))
    _check_prefill(wl, Tq=200, prefix=4096 + 2, queries=[0, 1, 62, 63, 64, 127, 128, 199])


def test_prefill_window_rows_dominate():
    # window rows four times larger than usual (raw rows and stored window rows scaled by 4, exactly):
    # the window's tile, the query's last, raises every head's running maximum by more than the
    # kernel's margin, so the accumulated output and sums are rescaled mid-query
    wl = get_workload("csa_prefill_8k")
    layer = wl.layers[0]
    Tq, prefix = 96, 4096 + 2
    pf = prefill_inputs(wl, Tq=Tq, prefix=prefix)
    pf["raw"] = F.bf16_encode(F.decode_act(pf["raw"], "bf16") * 4.0)
    pf["window"] = _scaled_rows(pf["window"], layer.kv_format, layer.D, 4.0)
    st = LayerState.from_arrays(layer, wl.B, pf, raw_key="raw", gate_key="gate", raw_base=pf["raw_first_row"])
    n_max = pf["n"] // layer.m
    out = torch.zeros((wl.B, Tq, layer.H, layer.D), dtype=torch.int16, device="cuda")
    topk = torch.zeros((wl.B, Tq, layer.top_k), dtype=torch.int32, device="cuda")
    ws = st.workspace("prefill", Tq, n_max)
    C.csa_prefill(st.L, st.cache(), st.params(), dev(pf["q"]), dev(pf["idx_q"]), dev(pf["idx_q_scale"]),
                  dev(pf["head_w"]), dev(pf["t"]), Tq, n_max, out, topk, ws)
    torch.cuda.synchronize()
    _no_device_error(ws)
    L = O.LayerSpec.of(layer)
    ents, win, _, _ = O.prefill_caches(L, pf, 0)
    got = out_values(out, layer.act_format)[0]
    tk = host(topk)[0]
    # values and logits of the window keys are 4x the usual: the bf16 roundings of q~ and P move a
    # logit of size |l| by about |l| 2^-8, so the absolute bars scale by 4 x 4 and the relative L2 bar
    # by 4 (a missed or wrong rescale would put the error at the size of the output itself)
    for j in range(0, Tq, 5):
        ref = O.prefill_query(L, pf, ents, win, 0, j)
        assert check_topk(tk[j], ref["scores"], layer.top_k) == 0
        assert_out_close(got[j], ref["o"], max_abs=0.32, mean_abs=0.032, rel_l2=4e-2, tag=f"window x4 q{j}")
    worst = max((x for x in _gpu_util.STATS if x["tag"].startswith("window x4")), key=lambda x: x["rel_l2"])
    print("window x4 worst:", worst)


def test_prefill_full_size_sampled():
    wl = get_workload("csa_prefill_8k")
    Tq = wl.Tq
    queries = list(range(0, Tq, 512)) + [Tq - 1]
    _check_prefill(wl, Tq=Tq, prefix=None, queries=queries)


# ----------------------------------------------------------------------------- the attention calls on their own

def _scaled_rows(rows, fmt, D, factor):
    """Stored rows whose values are exactly `factor` (a power of two) times the given ones."""
    return F.encode_rows(F.decode_rows(rows, fmt, D) * factor, fmt)


def _direct_attend(name, li, Tq=1, B=None, window_factor=1.0, logit_sharp=1.0):
    """csa_sparse_attend (oracle top-k fed in) or hca_attend called directly on the stored caches.

    Queries j < Tq of sequence b sit at positions t - Tq + 1 + j.  The window buffer holds
    Tq + w - 1 rows, so every query finds its w rows.  With window_factor != 1 the window rows are
    scaled by that power of two and the logit scale divided by it: logits keep their size while the
    raw partial scores grow by the factor."""
    over = {} if B is None else {"B": B}
    wl = get_workload(name, **over)
    layer = wl.layers[li]
    d = decode_inputs(wl, li)
    B, H, D, w = wl.B, layer.H, layer.D, layer.window
    cap_w = w + Tq - 1 if Tq > 1 else w
    if cap_w != w:
        from csa_synth.generate import kv_rows
        d["window"] = kv_rows(wl.seed, "window_chunk", li, (B, cap_w), layer)
    if window_factor != 1.0:
        d["window"] = _scaled_rows(d["window"], layer.kv_format, D, window_factor)
    t_last = int(d["t"][0])
    t = np.array([[t_last - Tq + 1 + j for j in range(Tq)] for _ in range(B)], dtype=np.int64)
    from csa_synth.generate import act_array, stream
    q = d["q"] if Tq == 1 else act_array(stream(wl.seed, "q_chunk", li), (B, Tq, H, D), layer.act_format)
    st = LayerState.from_arrays(layer, B, d)
    scale = logit_sharp / (window_factor * np.sqrt(D))
    if scale != 1.0 / np.sqrt(D):
        st.L.softmax_scale = scale
    L = O.LayerSpec.of(layer)
    L.scale = scale
    out_dtype = torch.float32 if layer.act_format == "f32" else torch.int16
    out = torch.zeros((B, Tq, H, D), dtype=out_dtype, device="cuda")
    q_pos = dev(t.reshape(-1))
    refs, sels = [], []
    for b in range(B):
        for j in range(Tq):
            tj = int(t[b, j])
            nv = int(O.n_visible(tj, 0, layer.m))
            if layer.kind == "csa":
                iq = F.decode_idx(d["idx_q"][b], layer.idx_format)
                s = O.index_scores(iq, d["idx_q_scale"][b], d["head_w"][b],
                                   F.decode_idx(d["idx_k"][b][:nv], layer.idx_format), d["idx_k_scale"][b][:nv])
                sel = O.top_k_fast(s, layer.top_k)
                ids = sel[sel >= 0]
            else:
                sel, ids = None, np.arange(nv)
            sels.append(sel)
            rows = np.concatenate([F.decode_rows(d["entries"][b][ids], layer.kv_format, D),
                                   F.decode_rows(d["window"][b][O.window_row_ids(tj, 0, w) % cap_w],
                                                 layer.kv_format, D)])
            qv = F.decode_act(q.reshape(B, Tq, H, D)[b, j], layer.act_format)
            refs.append(O.attend(qv, tj, rows, d["sinks"], d["gamma_q"], 64, layer.rope_base, scale, layer.eps))
    cap = d["entries"].shape[1]
    if layer.kind == "csa":
        topk = dev(np.stack(sels).astype(np.int32))
        ws = st.workspace("sparse_attend", Tq, cap)
        C.csa_sparse_attend(st.L, st.cache(), st.params(), dev(q), q_pos, Tq, topk, out, ws)
    else:
        ws = st.workspace("hca_attend", Tq, cap)
        C.hca_attend(st.L, st.cache(), st.params(), dev(q), q_pos, Tq, cap, out, ws)
    torch.cuda.synchronize()
    _no_device_error(ws)
    got = out_values(out, layer.act_format).reshape(B * Tq, H, D)
    return got, np.stack(refs)


@pytest.mark.parametrize("name,li,Tq,B", [("csa_decode_tiny_2k", 0, 1, None), ("csa_decode_128k", 0, 1, None),
                                          ("csa_hca_decode_1m", 0, 1, None), ("csa_decode_128k", 0, 3, 2),
                                          ("csa_decode_128k", 0, 16, 1)])
def test_sparse_attend_direct(name, li, Tq, B):
    # oracle top-k fed in; Tq = 3 x B = 2 is 6 query rows (the tcgen05 kernel), Tq = 16 the mma.sync one
    got, ref = _direct_attend(name, li, Tq, B)
    tight = name == "csa_decode_tiny_2k"
    for r in range(len(ref)):
        if tight:
            assert_out_close(got[r], ref[r], max_abs=1e-4, mean_abs=1e-5, rel_l2=1e-4)
        else:
            assert_out_close(got[r], ref[r], tag=f"sparse_attend/{name}/Tq={Tq}/row{r}")


@pytest.mark.parametrize("name,li,Tq,B", [("hca_decode_128k", 0, 1, None), ("csa_hca_decode_1m", 1, 1, None),
                                          ("csa_hca_decode_1m", 1, 4, 2)])
def test_hca_attend_direct(name, li, Tq, B):
    got, ref = _direct_attend(name, li, Tq, B)
    for r in range(len(ref)):
        assert_out_close(got[r], ref[r], tag=f"hca_attend/{name}/Tq={Tq}/row{r}")


def _assert_relative(got, ref, rel_l2, rel_max):
    d = np.abs(got - ref)
    assert np.all(np.isfinite(got)), "non-finite outputs"
    scale = np.abs(ref).max()
    assert d.max() <= rel_max * scale, f"max-abs {d.max()} vs {rel_max} x {scale}"
    rl2 = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rl2 <= rel_l2, f"relative L2 {rl2}"


@pytest.mark.parametrize("name,li", [("csa_decode_128k", 0), ("csa_hca_decode_1m", 1), ("hca_decode_128k", 0)])
@pytest.mark.parametrize("sharp", [1.0, 8.0])
def test_large_window_rows(name, li, sharp):
    """Window rows 1024x larger than the entries (raw activations are not normalised) with the logit
    scale divided by 1024: the logits keep their size, but the raw partial scores reach ~7e4, beyond
    fp16's range, so any half-precision exchange of unscaled partial scores would overflow.  With
    the x8 sharper logits the bars are 4x wider (the bf16 rounding of q~ moves such logits more)."""
    got, ref = _direct_attend(name, li, 1, 2 if name != "hca_decode_128k" else None, window_factor=1024.0,
                              logit_sharp=sharp)
    k = 1.0 if sharp == 1.0 else 4.0
    for r in range(len(ref)):
        _assert_relative(got[r], ref[r], rel_l2=1e-2 * k, rel_max=2e-2 * k)
