"""csa_decode_step_scratch: the decode step on the library's static device scratch.

The entry point takes no workspace and allocates nothing; its workspace is a fixed
CSA_SCRATCH_BYTES array in static device memory.  The CPU test checks the host-side
size limit (an oversize call is rejected before any device work); the GPU test runs
two calls in a row on the same scratch and checks each against the float64 oracle, and plants a
device error with dirty top-k histograms in the scratch to check that the next call cleans them.
This file is collected last, after every other user of the library in the run.
"""

import ctypes

import numpy as np
import pytest

from csa_synth import decode_inputs, get_workload
from long_context_sparse_csa_b200 import binding as C

SCRATCH_BYTES = 16 << 20
ERR_WORKSPACE = 3


def _layer(kind="csa", B=1):
    wl = get_workload("csa_hca_decode_1m")
    spec = [s for s in wl.layers if s.kind == kind][0]
    return C.layer_from_spec(spec, B)


def test_scratch_limit_covers_1m_context_batch_1():
    L = _layer()
    need = C.lib().csa_workspace_size(ctypes.byref(L), 3, 1, 1 << 18)
    assert 0 < need <= SCRATCH_BYTES


def test_oversize_call_rejected_on_host():
    # 2^22 entries need > 16 MiB of scores alone: rejected before any CUDA call (none exists here)
    L = _layer()
    need = C.lib().csa_workspace_size(ctypes.byref(L), 3, 1, 1 << 22)
    assert need > SCRATCH_BYTES
    cache = C.CsaCache(entry_cap=1 << 22, window_cap=128)
    params = C.CsaParams()
    st = C.lib().csa_decode_step_scratch(ctypes.byref(L), ctypes.byref(cache), ctypes.byref(params), None, None,
                                         None, None, None, None, None, None, None, None, None)
    assert st == ERR_WORKSPACE
    assert b"static scratch" in C.lib().csa_last_error()


def test_null_layer_rejected():
    st = C.lib().csa_decode_step_scratch(None, None, None, None, None, None, None, None, None, None, None, None,
                                         None, None)
    assert st != 0


@pytest.mark.gpu
def test_two_calls_in_a_row_match_oracle():
    import torch

    from _gpu_util import assert_out_close, check_topk, dev, host, out_values
    from long_context_sparse_csa_b200.state import LayerState
    from oracle import csa as O

    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    wl = get_workload("csa_decode_128k", B=4)     # 11.7 MB of workspace: inside the 16 MiB scratch
    layer = wl.layers[0]
    d = decode_inputs(wl, 0)
    st = LayerState.from_arrays(layer, wl.B, d)
    out_dtype = torch.float32 if layer.act_format == "f32" else torch.int16
    args = [dev(d[k]) for k in ("q", "idx_q", "idx_q_scale", "head_w", "x_new", "g_new", "t")]
    refs = [O.decode_step(O.LayerSpec.of(layer), d, b) for b in range(wl.B)]
    outs = [torch.zeros((wl.B, layer.H, layer.D), dtype=out_dtype, device="cuda") for _ in range(2)]
    topks = [torch.zeros((wl.B, layer.top_k), dtype=torch.int32, device="cuda") for _ in range(2)]
    free = []
    for call, (out, topk) in enumerate(zip(outs, topks)):
        torch.cuda.synchronize()
        before = torch.cuda.mem_get_info()[0]
        code = C.csa_decode_step_scratch(st.L, st.cache(), st.params(), *args, out, topk, read_device_error=True)
        assert code == 0, f"call {call}: device error word {code}"
        torch.cuda.synchronize()
        free.append((before, torch.cuda.mem_get_info()[0]))
        got = out_values(out, layer.act_format)
        idx = host(topk)
        for b in range(wl.B):
            assert_out_close(got[b], refs[b]["o"], tag=f"scratch call {call} b{b}")
            check_topk(idx[b], refs[b]["scores"], layer.top_k)
    # once the module is loaded (first call), a call allocates nothing: free device memory is
    # unchanged across the second call
    assert free[1][0] == free[1][1]


@pytest.mark.gpu
def test_dirty_scratch_is_cleaned_after_a_device_error():
    # a device error left by an earlier call (error word set, a million phantom counts in row 0's
    # top-k histogram): a call with device_error NULL must still select and attend exactly (its guard
    # kernel zero-fills the histograms because the word is set), and keep the word for the next
    # reporting call, which then returns it and zero-fills the scratch
    import torch

    from _gpu_util import assert_out_close, check_topk, dev, host, out_values
    from long_context_sparse_csa_b200.state import LayerState
    from oracle import csa as O

    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    wl = get_workload("csa_decode_128k", B=2)
    layer = wl.layers[0]
    d = decode_inputs(wl, 0)
    st = LayerState.from_arrays(layer, wl.B, d)
    cap = d["entries"].shape[1]
    args = [dev(d[k]) for k in ("q", "idx_q", "idx_q_scale", "head_w", "x_new", "g_new", "t")]
    out_dtype = torch.float32 if layer.act_format == "f32" else torch.int16
    refs = [O.decode_step(O.LayerSpec.of(layer), d, b) for b in range(wl.B)]
    err_off, _ = C.csa_debug_workspace_segment(st.L, "decode_step", 1, cap, "error_word")
    h_off, h_bytes = C.csa_debug_workspace_segment(st.L, "decode_step", 1, cap, "topk_histogram")
    assert h_bytes > 0, "the workload takes the multi-CTA top-k"
    hist = torch.zeros(h_bytes // 4, dtype=torch.int32, device="cuda")
    hist[4095] = 1_000_000
    C.csa_debug_scratch_copy(h_off, hist, to_scratch=True)
    C.csa_debug_scratch_copy(err_off, torch.tensor([2], dtype=torch.int32, device="cuda"), to_scratch=True)

    out = torch.zeros((wl.B, layer.H, layer.D), dtype=out_dtype, device="cuda")
    topk = torch.zeros((wl.B, layer.top_k), dtype=torch.int32, device="cuda")
    C.csa_decode_step_scratch(st.L, st.cache(), st.params(), *args, out, topk, read_device_error=False)
    torch.cuda.synchronize()
    got, idx = out_values(out, layer.act_format), host(topk)
    for b in range(wl.B):
        check_topk(idx[b], refs[b]["scores"], layer.top_k)
        assert_out_close(got[b], refs[b]["o"], tag=f"after a dirty scratch b{b}")
    back = torch.ones(h_bytes // 4, dtype=torch.int32, device="cuda")
    C.csa_debug_scratch_copy(h_off, back, to_scratch=False)
    assert not back.any(), "the histograms are zero after the call"
    # the planted word is kept for the next reporting call, which returns it and restores the scratch
    code = C.csa_decode_step_scratch(st.L, st.cache(), st.params(), *args, out, topk, read_device_error=True)
    assert code == 2
    code = C.csa_decode_step_scratch(st.L, st.cache(), st.params(), *args, out, topk, read_device_error=True)
    assert code == 0
    for b in range(wl.B):
        check_topk(host(topk)[b], refs[b]["scores"], layer.top_k)


def test_scratch_copy_rejects_ranges_outside_the_array():
    buf = (ctypes.c_char * 16)()
    st = C.lib().csa_debug_scratch_copy(SCRATCH_BYTES - 8, ctypes.cast(buf, ctypes.c_void_p), 16, 1, None)
    assert st != 0
    assert b"outside the static scratch" in C.lib().csa_last_error()
