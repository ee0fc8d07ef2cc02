"""GPU parity of the FP4 indexer: e2m1 index keys with block scales (idx_format "e2m1"), e4m3 index
queries, against the oracle's FP4 codec and scores.

The FP4 codes and their block offsets are exact e4m3 values on the device, so the scores agree with
the float64 oracle to float32 accumulation: the same element-wise bar as the FP8 indexer, and the
top-k sets bit-exact outside the 1e-4 tie band.  Key production in FP4 is compared within half a
code step of each key's block scale (a float32 value on a rounding midpoint may land one code apart).
"""

import numpy as np
import pytest
import torch

from csa_synth import decode_inputs, get_workload, prefill_inputs
from csa_synth.configs import CSA_PRO, CSA_PREFILL, Workload, scaled_layer
from csa_synth.generate import act_array, index_stream_inputs, stream
from long_context_sparse_csa_b200 import binding as C
from long_context_sparse_csa_b200.state import LayerState, to_device
from oracle import csa as O
from oracle import formats as F

from _gpu_util import assert_out_close, check_topk, dev, host, out_values

pytestmark = pytest.mark.gpu

FP4_PRO = scaled_layer(CSA_PRO, idx_format="e2m1")


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    C.lib()
    yield
    torch.cuda.synchronize()


def _scores_ref(layer, d, b):
    nv = int(O.n_visible(d["t"][b], 0, layer.m))
    L = O.LayerSpec.of(layer)
    iq, ik, iks = O.index_operands(L, d["idx_q"][b], d["idx_k"][b][:nv], d["idx_k_scale"][b][:nv])
    return O.index_scores(iq, d["idx_q_scale"][b], d["head_w"][b], ik, iks)


# entry counts that are multiples of 4 take the tensor-core kernel (block-scaled MMA); 20,001 entries
# take the warp-level kernel
@pytest.mark.parametrize("B,n", [(2, 4 * 20000 + 3), (3, 4 * 3000 + 1), (1, 1 << 20), (2, 4 * 20001 + 1)])
def test_fp4_index_topk(B, n):
    wl = Workload(name="t", mode="decode", B=B, n=n, layers=(FP4_PRO,), seed=51)
    d = decode_inputs(wl)
    st = LayerState.from_arrays(FP4_PRO, B, d)
    cap = d["entries"].shape[1]
    topk = torch.full((B, FP4_PRO.top_k), -7, dtype=torch.int32, device="cuda")
    scores = torch.zeros((B, cap), dtype=torch.float32, device="cuda")
    ws = st.workspace("index_topk", 1, cap)
    C.csa_index_topk(st.L, st.cache(), dev(d["idx_q"]), dev(d["idx_q_scale"]), dev(d["head_w"]), dev(d["t"]), 1, cap,
                     topk, scores, ws)
    torch.cuda.synchronize()
    assert C.csa_device_error(ws) == 0
    got_s, got_k = host(scores), host(topk)
    for b in range(B):
        ref = _scores_ref(FP4_PRO, d, b)
        nv = len(ref)
        assert np.max(np.abs(got_s[b, :nv] - ref)) <= 1e-5 * np.abs(ref).max() + 1e-7
        check_topk(got_k[b], ref, FP4_PRO.top_k)


def test_fp4_decode_step():
    wl = Workload(name="t", mode="decode", B=2, n=131072, layers=(FP4_PRO,), seed=52)
    d = decode_inputs(wl)
    st = LayerState.from_arrays(FP4_PRO, 2, d)
    cap = d["entries"].shape[1]
    out = torch.zeros((2, FP4_PRO.H, FP4_PRO.D), dtype=torch.int16, device="cuda")
    topk = torch.zeros((2, FP4_PRO.top_k), dtype=torch.int32, device="cuda")
    ws = st.workspace("decode_step", 1, cap)
    C.csa_decode_step(st.L, st.cache(), st.params(), dev(d["q"]), dev(d["idx_q"]), dev(d["idx_q_scale"]),
                      dev(d["head_w"]), dev(d["x_new"]), dev(d["g_new"]), dev(d["t"]), out, topk, ws)
    torch.cuda.synchronize()
    assert C.csa_device_error(ws) == 0
    got = out_values(out, "bf16")
    for b in range(2):
        ref = O.decode_step(O.LayerSpec.of(FP4_PRO), d, b)
        assert check_topk(host(topk)[b], ref["scores"], FP4_PRO.top_k) == 0
        assert_out_close(got[b], ref["o"], tag=f"fp4 decode b{b}")


def test_fp4_index_keys_from_a_chunk():
    n = 1003
    wl = Workload(name="t", mode="prefill", B=2, n=n, layers=(FP4_PRO,), seed=53)
    st_in = index_stream_inputs(wl, 0, (2, n), FP4_PRO)
    raw = act_array(stream(53, "idx_raw_chunk"), (2, n, 128), "bf16")
    gate = act_array(stream(53, "idx_gate_chunk"), (2, n, 128), "bf16")
    N = n // 4
    keys = torch.zeros((2, N + 2, 64), dtype=torch.uint8, device="cuda")
    words = torch.zeros((2, N + 2), dtype=torch.int32, device="cuda")
    entries = torch.zeros((2, N + 2, 592), dtype=torch.uint8, device="cuda")
    window = torch.zeros((2, 128, 592), dtype=torch.uint8, device="cuda")
    raw_d, gate_d = dev(raw), dev(gate)
    bias = to_device(np.asarray(st_in["idx_pos_bias"], np.float32))
    st = LayerState(FP4_PRO, 2, entries=entries, window=window, raw=raw_d, gate=gate_d, idx_keys=keys,
                    idx_key_scale=words)
    S = C.make_index_stream(raw_d, gate_d, bias)
    q_pos = torch.arange(n, device="cuda", dtype=torch.int64).repeat(2, 1).contiguous()
    C.csa_index_keys(st.L, st.cache(), S, None, None, q_pos, n)
    torch.cuda.synchronize()
    gk, gw = host(keys), host(words).view(np.uint32)
    for b in range(2):
        ref = O.compress_index_keys(F.decode_act(raw[b], "bf16"), F.decode_act(gate[b], "bf16"),
                                    st_in["idx_pos_bias"], 4, 1, range(N))
        rk, rw = F.encode_fp4_keys(ref)
        assert np.mean(gw[b, :N] == rw) > 0.99, "scale words (sigma and block offsets) agree"
        v = F.decode_fp4_keys(gk[b, :N], gw[b, :N])
        wv = gw[b, :N].astype(np.int64)
        bs = np.repeat(np.stack([np.exp2((wv & 0xFF) - 127.0 - ((wv >> (8 + 4 * k)) & 0xF)) for k in range(4)], 1),
                       32, axis=1)
        a = np.abs(ref / bs)
        step = np.where(a < 2, 0.5, np.where(a < 4, 1.0, 2.0))
        assert np.all(np.abs(v - ref) <= 0.5 * step * bs * (1 + 1e-5) + 1e-12)
        assert np.mean(gk[b, :N] != rk) <= 2e-3
        assert not gk[b, N:].any()


def test_fp4_indexed_decode_step():
    # index keys produced in FP4 and the index query in e4m3, then scored and selected
    wl = get_workload("csa_decode_128k", B=2, layers=(FP4_PRO,))
    d = decode_inputs(wl, 0, indexed=True)
    st = LayerState.from_arrays(FP4_PRO, 2, d)
    rings = (to_device(d["idx_raw_ring"]), to_device(d["idx_gate_ring"]),
             to_device(np.asarray(d["idx_pos_bias"], np.float32)))
    S = C.make_index_stream(*rings)
    cap = d["entries"].shape[1]
    ws = st.workspace("decode_step_indexed", 1, cap)
    out = torch.zeros((2, FP4_PRO.H, FP4_PRO.D), dtype=torch.int16, device="cuda")
    topk = torch.zeros((2, FP4_PRO.top_k), dtype=torch.int32, device="cuda")
    k = {x: dev(d[x]) for x in ("q", "c_q", "W_iq", "head_w", "x_new", "g_new", "idx_x_new", "idx_g_new", "t")}
    C.csa_decode_step_indexed(st.L, st.cache(), st.params(), S, k["q"], k["c_q"], k["W_iq"], FP4_PRO.idx_rank,
                              k["head_w"], k["x_new"], k["g_new"], k["idx_x_new"], k["idx_g_new"], k["t"], out, topk,
                              ws)
    torch.cuda.synchronize()
    assert C.csa_device_error(ws) == 0
    oq, nq = C.csa_debug_workspace_segment(st.L, "decode_step_indexed", 1, cap, "index_query")
    os_, ns = C.csa_debug_workspace_segment(st.L, "decode_step_indexed", 1, cap, "index_query_scale")
    gq = host(ws[oq:oq + nq]).reshape(2, FP4_PRO.H_I, FP4_PRO.d_I)
    gqs = host(ws[os_:os_ + ns]).view(np.float32).reshape(2, FP4_PRO.H_I)
    keys, words = host(st.idx_keys), host(st.idx_key_scale).view(np.uint32)
    got = out_values(out, "bf16")
    L = O.LayerSpec.of(FP4_PRO)
    for b in range(2):
        res = O.decode_step_indexed(L, d, b)
        i = res["index_key"][0]
        # the produced key's values (GPU codes) against the oracle's: within half a code step
        ok_words = words[b, i] == res["index_key"][2]
        assert ok_words or abs(int(words[b, i] & 0xFF) - int(res["index_key"][2] & 0xFF)) <= 1
        d2 = dict(d)
        d2["idx_q"], d2["idx_q_scale"] = d["idx_q"].copy(), d["idx_q_scale"].copy()
        d2["idx_q"][b], d2["idx_q_scale"][b] = gq[b], gqs[b]
        d2["idx_k"], d2["idx_k_scale"] = d["idx_k"].copy(), d["idx_k_scale"].copy()
        d2["idx_k"][b, i], d2["idx_k_scale"][b, i] = keys[b, i], words[b, i]
        ref = O.decode_step(L, d2, b)
        check_topk(host(topk)[b], ref["scores"], FP4_PRO.top_k)
        assert_out_close(got[b], ref["o"], tag=f"fp4 indexed b{b}")


@pytest.mark.parametrize("prefix", [4096 + 2, 4096 + 6])
def test_fp4_prefill_small(prefix):
    # chunked prefill with FP4 keys, then top-k and attention: 1,048 entries (a multiple of 4) take the
    # tensor-core indexer, 1,049 the CUDA-core one
    layer = scaled_layer(CSA_PREFILL, idx_format="e2m1")
    wl = get_workload("csa_prefill_8k", layers=(layer,))
    pf = prefill_inputs(wl, Tq=97, prefix=prefix)
    st = LayerState.from_arrays(layer, 1, pf, raw_key="raw", gate_key="gate", raw_base=pf["raw_first_row"])
    n_max = pf["n"] // layer.m
    assert st.idx_keys.shape[1] % 4 == (0 if prefix == 4098 else 1)
    out = torch.zeros((1, 97, layer.H, layer.D), dtype=torch.int16, device="cuda")
    topk = torch.zeros((1, 97, layer.top_k), dtype=torch.int32, device="cuda")
    ws = st.workspace("prefill", 97, n_max)
    C.csa_prefill(st.L, st.cache(), st.params(), dev(pf["q"]), dev(pf["idx_q"]), dev(pf["idx_q_scale"]),
                  dev(pf["head_w"]), dev(pf["t"]), 97, n_max, out, topk, ws)
    torch.cuda.synchronize()
    assert C.csa_device_error(ws) == 0
    L = O.LayerSpec.of(layer)
    ents, win, _, _ = O.prefill_caches(L, pf, 0)
    got = out_values(out, "bf16")[0]
    tk = host(topk)[0]
    for j in range(0, 97, 12):
        ref = O.prefill_query(L, pf, ents, win, 0, j)
        assert check_topk(tk[j], ref["scores"], layer.top_k) == 0
        assert_out_close(got[j], ref["o"], tag=f"fp4 prefill q{j}")
