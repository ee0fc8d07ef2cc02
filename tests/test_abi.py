"""The C-ABI library loads, exports every entry point include/csa.h declares, and
rejects bad arguments on the host before any launch (no GPU needed)."""

import ctypes
import os
import re

import pytest
import torch

from long_context_sparse_csa_b200 import binding as C

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "csa.h")).read()
    return sorted(set(re.findall(r"CSA_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = _declared()
    for want in ["csa_compress", "csa_index_topk", "csa_sparse_attend", "hca_attend", "csa_decode_step",
                 "hca_decode_step", "csa_prefill", "csa_append", "csa_workspace_size", "csa_last_error"]:
        assert want in names


def test_library_exports_every_declared_symbol():
    h = C.lib()
    for name in _declared():
        assert hasattr(h, name), name
    assert set(_declared()) == set(C.EXPORTED)


def test_version_and_row_bytes():
    assert "sm_100a" in C.csa_version()
    for fmt, rb in [("f32", 2048), ("bf16", 1024), ("mixed", 592)]:
        L = C.make_layer("csa", 1, 128, 512, 4, 1, 1024, 128, 32, 128, kv_format=fmt)
        assert C.csa_row_bytes(L) == rb


def test_layer_struct_matches_c_layout():
    assert ctypes.sizeof(C.CsaLayer) == 80
    assert C.CsaLayer.rope_base.offset == 56 and C.CsaLayer.pos0.offset == 72
    assert ctypes.sizeof(C.CsaCache) == 80
    assert ctypes.sizeof(C.CsaParams) == 32


def _bad_layer(**kw):
    base = dict(kind="csa", B=1, H=128, D=512, m=4, overlap=1, top_k=1024, window=128, H_I=32, d_I=128,
                kv_format="mixed")
    base.update(kw)
    return C.make_layer(**base)


@pytest.mark.parametrize("kw,status", [(dict(D=100), 2), (dict(d_rope=32), 2), (dict(m=0), 1), (dict(overlap=2), 1),
                                       (dict(top_k=0), 1), (dict(B=0), 1), (dict(window=0), 1),
                                       (dict(d_I=100), 2)])
def test_invalid_layers_rejected_on_host(kw, status):
    L = _bad_layer(**kw)
    cache = C.CsaCache()
    params = C.CsaParams()
    q_pos = torch.zeros(1, dtype=torch.int64)
    with pytest.raises(C.CsaError) as e:
        C._check(C.lib().csa_compress(ctypes.byref(L), ctypes.byref(cache), ctypes.byref(params),
                                      ctypes.c_void_p(q_pos.data_ptr()), 1, None))
    assert e.value.status == status
    assert C.csa_workspace_size(L, "decode_step", 1, 1024) == 0


def test_null_pointers_and_workspace_rejected():
    L = _bad_layer()
    h = C.lib()
    cache = C.CsaCache()
    params = C.CsaParams()
    st = h.csa_decode_step(ctypes.byref(L), ctypes.byref(cache), ctypes.byref(params), *([None] * 9), None, 0, None)
    assert st == 1 and b"NULL" in h.csa_last_error()
    # a layer with every pointer set but no workspace
    buf = torch.zeros(1 << 24, dtype=torch.uint8)
    p = (buf.data_ptr() + 255) // 256 * 256
    ws = p + 4096
    cache = C.CsaCache(p, 1024, p, p, p, 128, p, p, 8, 0)
    params = C.CsaParams(p, p, p, p)
    st = h.csa_decode_step(ctypes.byref(L), ctypes.byref(cache), ctypes.byref(params), *([ctypes.c_void_p(p)] * 9),
                           None, 0, None)
    assert st == 3, h.csa_last_error()
    need = C.csa_workspace_size(L, "decode_step", 1, 1024)
    assert need > 1024 * 4
    st = h.csa_decode_step(ctypes.byref(L), ctypes.byref(cache), ctypes.byref(params), *([ctypes.c_void_p(p)] * 9),
                           ctypes.c_void_p(ws), need - 1, None)
    assert st == 3
    # misaligned pointer
    cache2 = C.CsaCache(p + 4, 1024, p, p, p, 128, p, p, 8, 0)
    st = h.csa_decode_step(ctypes.byref(L), ctypes.byref(cache2), ctypes.byref(params), *([ctypes.c_void_p(p)] * 9),
                           ctypes.c_void_p(ws), need, None)
    assert st == 1 and b"aligned" in h.csa_last_error()


def test_unsupported_attention_shape_is_reported():
    # 48 heads of D=512: neither the tensor-core kernel (H % 32) nor the generic one (H <= 32)
    L = _bad_layer(kind="hca", H=48, top_k=0, H_I=0, d_I=0, m=128, overlap=0)
    h = C.lib()
    buf = torch.zeros(1 << 20, dtype=torch.uint8)
    base = (buf.data_ptr() + 255) // 256 * 256
    p = ctypes.c_void_p(base)
    cache = C.CsaCache(base, 16, None, None, base, 128, None, None, 0, 0)
    params = C.CsaParams(None, None, None, base)
    need = C.csa_workspace_size(L, "hca_attend", 1, 16)
    st = h.hca_attend(ctypes.byref(L), ctypes.byref(cache), ctypes.byref(params), p, p, 1, 16, p, p, need, None)
    assert st == 2, h.csa_last_error()


def test_workspace_of_many_query_rows_has_no_per_tile_partials():
    # 128 heads of 512 dims: decode-like calls (a few query rows) take the tcgen05 kernel, whose
    # per-query slot tiles each leave a partial (about 132 KB) plus a bf16 q~ row block; a chunk of
    # 8,192 queries takes the mma.sync kernel instead, so its workspace stays far from the
    # 8,192 x 18 x 132 KB = 19 GB the tile partials would need
    from csa_synth.configs import CSA_PRO
    dec = C.layer_from_spec(CSA_PRO, 1)
    need_dec = C.csa_workspace_size(dec, "decode_step", 1, 1 << 18)
    one = C.layer_from_spec(CSA_PRO, 1)
    need_pf = C.csa_workspace_size(one, "prefill", 8192, 18432)
    scores = 8192 * 18432 * 4
    assert need_dec > 18 * 128 * 512 * 2                # the decode step's 18 bf16 partials are there
    assert need_pf < scores + (1 << 30)                 # scores + top-k + modest scratch, no 19 GB
