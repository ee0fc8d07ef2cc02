"""Failure detection on the GPU, in the forms that fault nothing.

* A bounded wait that runs out: the wait-probe kernel waits, with the library's
  own bounded-wait helper and a 100 us limit, on an mbarrier phase that nothing
  completes; it must set the timeout bit of the error word, csa_device_error
  must report CSA_ERR_DEVICE_TIMEOUT, and the next ordinary call must run clean.
* An inconsistent top-k histogram, injected from the host into the
  caller-owned workspace: the multi-CTA top-k must notice that its histogram
  and the scores disagree, set bit 2, pad the row with -1, leave the
  workspace's histograms zeroed, and the next call on the same workspace must
  give the exact selection again.
"""

import numpy as np
import pytest
import torch

from csa_synth import decode_inputs, get_workload
from long_context_sparse_csa_b200 import binding as C
from long_context_sparse_csa_b200.state import LayerState
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


def _decode_tiny_step(ws=None):
    wl = get_workload("csa_decode_tiny_2k")
    layer = wl.layers[0]
    d = decode_inputs(wl)
    st = LayerState.from_arrays(layer, wl.B, d)
    cap = d["entries"].shape[1]
    if ws is None:
        ws = st.workspace("decode_step", 1, cap)
    out = torch.zeros((1, layer.H, layer.D), dtype=torch.float32, device="cuda")
    topk = torch.zeros((1, layer.top_k), dtype=torch.int32, device="cuda")
    C.csa_decode_step(st.L, st.cache(), st.params(), dev(d["q"]), dev(d["idx_q"]), dev(d["idx_q_scale"]),
                      dev(d["head_w"]), dev(d["x_new"]), dev(d["g_new"]), dev(d["t"]), out, topk, ws)
    torch.cuda.synchronize()
    ref = O.decode_step(O.LayerSpec.of(layer), d, 0)
    assert_out_close(out_values(out, "f32")[0], ref["o"], max_abs=1e-4, mean_abs=1e-5, rel_l2=1e-4)
    return ws


def test_bounded_wait_gives_up_and_reports():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    assert C.csa_device_error(ws) == 0
    C.csa_debug_wait_probe(ws, 100_000)              # 100 us, on a phase nothing completes
    torch.cuda.synchronize()
    st = C.lib().csa_device_error(C.ptr(ws), ws.numel(), C._stream(), None)
    assert st == 5, "CSA_ERR_DEVICE_TIMEOUT expected"
    assert C.csa_device_error(ws) == 0, "the word is cleared by the read"
    # the context is intact: an ordinary decode step runs and matches the oracle, with a clean word
    ws2 = _decode_tiny_step()
    assert C.csa_device_error(ws2) == 0


def test_bounded_wait_probe_rejects_bad_limits():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    for bad in (0, 2_000_000_000):
        with pytest.raises(C.CsaError):
            C.csa_debug_wait_probe(ws, bad)


def test_inconsistent_histogram_is_detected_and_cleaned():
    # 20,000 entries per row: the multi-CTA top-k, fed by the indexer's histogram
    wl = get_workload("csa_decode_128k", B=2, n=4 * 20000)
    layer = wl.layers[0]
    d = decode_inputs(wl)
    st = LayerState.from_arrays(layer, wl.B, d)
    cap = d["entries"].shape[1]
    ws = st.workspace("index_topk", 1, cap)
    off, nbytes = C.csa_debug_workspace_segment(st.L, "index_topk", 1, cap, "topk_histogram")
    assert nbytes == 2 * (4096 + 4 + 4096) * 4
    hist = ws[off:off + nbytes].view(torch.int32)
    hist[4095] += 1_000_000                           # row 0: a million phantom scores in the top bin
    topk = torch.zeros((2, layer.top_k), dtype=torch.int32, device="cuda")
    args = (dev(d["idx_q"]), dev(d["idx_q_scale"]), dev(d["head_w"]), dev(d["t"]))
    C.csa_index_topk(st.L, st.cache(), *args, 1, cap, topk, None, ws)
    torch.cuda.synchronize()
    got = host(topk)
    assert C.csa_device_error(ws) == 2
    assert np.all(got[0] == -1), "the inconsistent row is padded with -1"
    refs = []
    for b in range(2):
        iq = F.decode_idx(d["idx_q"][b], layer.idx_format)
        refs.append(O.index_scores(iq, d["idx_q_scale"][b], d["head_w"][b], F.decode_idx(d["idx_k"][b], "e4m3"),
                                   d["idx_k_scale"][b]))
    check_topk(got[1], refs[1], layer.top_k)          # the other row is unaffected
    assert not hist.any(), "the top-k leaves its histograms and counters zeroed"
    # the same workspace, no injection: exact selections and a clean word
    C.csa_index_topk(st.L, st.cache(), *args, 1, cap, topk, None, ws)
    torch.cuda.synchronize()
    assert C.csa_device_error(ws) == 0
    got = host(topk)
    for b in range(2):
        check_topk(got[b], refs[b], layer.top_k)
