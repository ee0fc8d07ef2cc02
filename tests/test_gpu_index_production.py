"""GPU parity of the index side produced on the device: index keys compressed from the index-key
stream (csa_index_keys), low-rank index queries (csa_index_query), and the decode step that makes
both before scoring (csa_decode_step_indexed), against the oracle's definitions (R14, R15).

Keys and queries are quantised codes decided by floating point: the GPU forms them in float32, the
oracle in float64, so a value that sits on a rounding midpoint may land one code apart.  They are
compared within one e4m3 quantum of the oracle's exact value; the step's selection and output are
then checked against the oracle fed with the codes the GPU wrote (the decision taken in the
kernel's precision), after those codes were validated.
"""

import numpy as np
import pytest
import torch

from csa_synth import compress_inputs, decode_inputs, get_workload
from csa_synth.configs import CSA_PRO, Workload, raw_ring_rows, scaled_layer
from csa_synth.generate import act_array, index_stream_inputs, stream
from long_context_sparse_csa_b200 import binding as C
from long_context_sparse_csa_b200.state import LayerState, to_device
from oracle import csa as O
from oracle import formats as F

from _gpu_util import assert_out_close, check_topk, dev, host, out_values

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    C.lib()
    yield
    torch.cuda.synchronize()


def _assert_codes_close(codes, scales, ref_vals, max_mismatch=2e-3):
    """GPU e4m3 codes x scales vs exact values: within one quantum of the coarser scale."""
    g = F.e4m3_decode(codes) * scales[..., None].astype(np.float64)
    x = np.asarray(ref_vals, np.float64)
    _, sig_o = F.encode_idx(x, "e4m3")
    sig = np.maximum(scales.astype(np.float64), sig_o.astype(np.float64))[..., None]
    ay = np.abs(x / sig)
    quantum = np.exp2(np.maximum(np.floor(np.log2(np.maximum(ay, 2.0 ** -6))), -6) - 3) * sig
    err = np.abs(g - x)
    bad = err > quantum + 1e-6 * np.abs(x)
    assert not bad.any(), f"{bad.sum()} values beyond one quantum (worst {err[bad].max()})"
    assert np.mean(scales == sig_o) > 0.99
    ref_codes, _ = F.encode_idx(x, "e4m3")
    assert np.mean(ref_codes != codes) <= max_mismatch


@pytest.mark.parametrize("fmt,n", [("e4m3", 1003), ("f32", 517)])
def test_index_keys_from_a_chunk(fmt, n):
    layer = scaled_layer(CSA_PRO, idx_format=fmt, H=8)
    wl = Workload(name="t", mode="prefill", B=2, n=n, layers=(layer,), seed=41)
    st_in = index_stream_inputs(wl, 0, (2, n), layer)
    raw = act_array(stream(41, "idx_raw_chunk"), (2, n, 128), "bf16")
    gate = act_array(stream(41, "idx_gate_chunk"), (2, n, 128), "bf16")
    N = n // 4
    keys = torch.zeros((2, N + 2, 128), dtype=torch.uint8 if fmt == "e4m3" else torch.float32, device="cuda")
    ks = torch.zeros((2, N + 2), dtype=torch.float32, device="cuda")
    entries = torch.zeros((2, N + 2, 592), dtype=torch.uint8, device="cuda")
    window = torch.zeros((2, 128, 592), dtype=torch.uint8, device="cuda")
    raw_d, gate_d = dev(raw), dev(gate)
    st = LayerState(layer, 2, entries=entries, window=window, raw=raw_d, gate=gate_d, idx_keys=keys, idx_key_scale=ks)
    bias = to_device(np.asarray(st_in["idx_pos_bias"], np.float32))
    S = C.make_index_stream(raw_d, gate_d, bias)
    q_pos = torch.arange(n, device="cuda", dtype=torch.int64).repeat(2, 1).contiguous()
    C.csa_index_keys(st.L, st.cache(), S, None, None, q_pos, n)
    torch.cuda.synchronize()
    got, gs = host(keys), host(ks)
    for b in range(2):
        ref = O.compress_index_keys(F.decode_act(raw[b], "bf16"), F.decode_act(gate[b], "bf16"),
                                    st_in["idx_pos_bias"], 4, 1, range(N))
        if fmt == "e4m3":
            _assert_codes_close(got[b, :N], gs[b, :N], ref)
        else:
            assert np.allclose(got[b, :N], ref, rtol=1e-5, atol=1e-6) and np.all(gs[b, :N] == 1)
        assert not got[b, N:].any(), "entries past the last complete group are not written"


@pytest.mark.parametrize("rows,rank,H_I", [(37, 512, 32), (1, 1536, 16), (8, 128, 64), (3, 48, 8)])
def test_index_query_projection(rows, rank, H_I):
    layer = scaled_layer(CSA_PRO, H_I=H_I, idx_rank=rank)
    L = C.layer_from_spec(layer, 1)
    c = act_array(stream(42, "c"), (rows, rank), "bf16")
    W = act_array(stream(42, "W"), (H_I * 128, rank), "bf16", std=1.0 / np.sqrt(rank))
    q = torch.zeros((rows, H_I, 128), dtype=torch.uint8, device="cuda")
    qs = torch.zeros((rows, H_I), dtype=torch.float32, device="cuda")
    C.csa_index_query(L, dev(c), dev(W), rank, rows, q, qs)
    torch.cuda.synchronize()
    Wv = F.decode_act(W, "bf16")
    ref = np.stack([O.index_query(F.decode_act(c[r], "bf16"), Wv, H_I, 128) for r in range(rows)])
    _assert_codes_close(host(q), host(qs), ref)


def _indexed_case(name, B=None, n=None):
    over = {}
    if B is not None:
        over["B"] = B
    if n is not None:
        over["n"] = n
    wl = get_workload(name, **over)
    layer = wl.layers[0]
    d = decode_inputs(wl, 0, indexed=True)
    st = LayerState.from_arrays(layer, wl.B, d)
    # the struct holds raw device pointers: keep the tensors alive on the state object
    st.idx_rings = (to_device(d["idx_raw_ring"]), to_device(d["idx_gate_ring"]),
                    to_device(np.asarray(d["idx_pos_bias"], np.float32)))
    S = C.make_index_stream(*st.idx_rings)
    return wl, layer, d, st, S


@pytest.mark.parametrize("name,B,n", [("csa_decode_128k", 2, None), ("csa_decode_128k", 3, 4 * 5000 + 2),
                                      ("csa_hca_decode_1m", None, None)])
def test_decode_step_indexed(name, B, n):
    wl, layer, d, st, S = _indexed_case(name, B, n)
    Bq = wl.B
    cap = d["entries"].shape[1]
    ws = st.workspace("decode_step_indexed", 1, cap)
    out = torch.zeros((Bq, layer.H, layer.D), dtype=torch.int16, device="cuda")
    topk = torch.zeros((Bq, layer.top_k), dtype=torch.int32, device="cuda")
    keep = {k: dev(d[k]) for k in ("q", "c_q", "W_iq", "head_w", "x_new", "g_new", "idx_x_new", "idx_g_new", "t")}
    C.csa_decode_step_indexed(st.L, st.cache(), st.params(), S, keep["q"], keep["c_q"], keep["W_iq"], layer.idx_rank,
                              keep["head_w"], keep["x_new"], keep["g_new"], keep["idx_x_new"], keep["idx_g_new"],
                              keep["t"], out, topk, ws)
    torch.cuda.synchronize()
    assert C.csa_device_error(ws) == 0
    oq, nq = C.csa_debug_workspace_segment(st.L, "decode_step_indexed", 1, cap, "index_query")
    os_, ns = C.csa_debug_workspace_segment(st.L, "decode_step_indexed", 1, cap, "index_query_scale")
    gq = host(ws[oq:oq + nq]).reshape(Bq, layer.H_I, layer.d_I)
    gqs = host(ws[os_:os_ + ns]).view(np.float32).reshape(Bq, layer.H_I)
    keys, kscale = host(st.idx_keys), host(st.idx_key_scale)
    got = out_values(out, layer.act_format)
    L = O.LayerSpec.of(layer)
    for b in range(Bq):
        res = O.decode_step_indexed(L, d, b)
        qv = O.index_query(F.decode_act(d["c_q"][b], "bf16"), F.decode_act(d["W_iq"], "bf16"), layer.H_I, layer.d_I)
        _assert_codes_close(gq[b], gqs[b], qv)
        d2 = dict(d)
        d2["idx_q"], d2["idx_q_scale"] = d["idx_q"].copy(), d["idx_q_scale"].copy()
        d2["idx_q"][b], d2["idx_q_scale"][b] = gq[b], gqs[b]
        if "index_key" in res:
            i = res["index_key"][0]
            t = int(d["t"][b])
            rr = raw_ring_rows(layer)
            rx = F.decode_act(d["idx_raw_ring"][b], "bf16").copy()
            rg = F.decode_act(d["idx_gate_ring"][b], "bf16").copy()
            rx[t % rr] = F.decode_act(d["idx_x_new"][b], "bf16")
            rg[t % rr] = F.decode_act(d["idx_g_new"][b], "bf16")
            rows = np.arange(t - rr + 1, t + 1)
            kv = O.pool_entry(rx[rows % rr], rg[rows % rr], d["idx_pos_bias"], rows - (i - layer.ov) * layer.m)
            _assert_codes_close(keys[b, i][None], kscale[b, i][None], kv[None], max_mismatch=1.0)
            d2["idx_k"], d2["idx_k_scale"] = d["idx_k"].copy(), d["idx_k_scale"].copy()
            d2["idx_k"][b, i], d2["idx_k_scale"][b, i] = keys[b, i], kscale[b, i]
        ref = O.decode_step(L, d2, b)
        check_topk(host(topk)[b], ref["scores"], layer.top_k)
        assert_out_close(got[b], ref["o"], tag=f"indexed/{name}/b{b}")
