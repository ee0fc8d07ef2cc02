"""csa_decode_step_scratch: the decode step on the library's static device scratch.

The entry point takes no workspace and allocates nothing; its workspace is a fixed
CSA_SCRATCH_BYTES array in static device memory.  The CPU test checks the host-side
size limit (an oversize call is rejected before any device work); the GPU test runs
two calls in a row on the same scratch and checks each against the float64 oracle.
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
