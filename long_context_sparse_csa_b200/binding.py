"""ctypes binding of libcsa.so: the C ABI declared in include/csa.h, one Python
function per entry point with the same name.

Only argument marshalling happens here (torch tensors -> device pointers,
layer / cache / parameter structs, the current CUDA stream); every step of
the operator runs in the library's kernels.  A missing or unloadable library
raises immediately -- there is no fallback path.
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa.so")

FMT = {"f32": 0, "bf16": 1, "mixed": 2, "e4m3": 3, "e2m1": 4}
SEGMENT = {"error_word": 0, "scores": 1, "topk_histogram": 2, "topk": 3, "partials": 4, "index_query": 5,
           "index_query_scale": 6}
KIND = {"csa": 0, "hca": 1}
OP = {"index_topk": 0, "sparse_attend": 1, "hca_attend": 2, "decode_step": 3, "prefill": 4, "decode_step_indexed": 5}
STATUS = {0: "CSA_OK", 1: "CSA_ERR_INVALID_ARG", 2: "CSA_ERR_UNSUPPORTED", 3: "CSA_ERR_WORKSPACE",
          4: "CSA_ERR_CUDA", 5: "CSA_ERR_DEVICE_TIMEOUT"}


class CsaError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


class CsaLayer(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("B", ctypes.c_int32), ("H", ctypes.c_int32), ("D", ctypes.c_int32),
                ("d_rope", ctypes.c_int32), ("m", ctypes.c_int32), ("overlap", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("window", ctypes.c_int32), ("H_I", ctypes.c_int32),
                ("d_I", ctypes.c_int32), ("kv_format", ctypes.c_int32), ("idx_format", ctypes.c_int32),
                ("act_format", ctypes.c_int32), ("rope_base", ctypes.c_double), ("eps", ctypes.c_float),
                ("softmax_scale", ctypes.c_float), ("pos0", ctypes.c_int64)]


class CsaCache(ctypes.Structure):
    _fields_ = [("entries", ctypes.c_void_p), ("entry_cap", ctypes.c_int64), ("idx_keys", ctypes.c_void_p),
                ("idx_key_scale", ctypes.c_void_p), ("window", ctypes.c_void_p), ("window_cap", ctypes.c_int64),
                ("raw", ctypes.c_void_p), ("gate", ctypes.c_void_p), ("raw_cap", ctypes.c_int64),
                ("raw_base", ctypes.c_int64)]


class CsaParams(ctypes.Structure):
    _fields_ = [("pos_bias", ctypes.c_void_p), ("gamma_kv", ctypes.c_void_p), ("gamma_q", ctypes.c_void_p),
                ("sinks", ctypes.c_void_p)]


class CsaIndexStream(ctypes.Structure):
    _fields_ = [("raw", ctypes.c_void_p), ("gate", ctypes.c_void_p), ("pos_bias", ctypes.c_void_p)]


_P = ctypes.c_void_p
_STREAM_S = ctypes.POINTER(CsaIndexStream)
_LAYER = ctypes.POINTER(CsaLayer)
_CACHE = ctypes.POINTER(CsaCache)
_PARAMS = ctypes.POINTER(CsaParams)
_I32, _I64, _SZ = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t

_SIGS = {
    "csa_row_bytes": (_SZ, [_LAYER]),
    "csa_workspace_size": (_SZ, [_LAYER, _I32, _I32, _I64]),
    "csa_last_error": (ctypes.c_char_p, []),
    "csa_version": (ctypes.c_char_p, []),
    "csa_profile_events": (None, [_P, _P]),
    "csa_launch_count": (ctypes.c_uint64, []),
    "csa_profile_timeline": (None, [_P, _I32]),
    "csa_profile_timeline_count": (_I32, []),
    "csa_device_error": (ctypes.c_int, [_P, _SZ, _P, ctypes.POINTER(_I32)]),
    "csa_append": (ctypes.c_int, [_LAYER, _CACHE, _P, _P, _P, _I32, _P]),
    "csa_compress": (ctypes.c_int, [_LAYER, _CACHE, _PARAMS, _P, _I32, _P]),
    "csa_index_topk": (ctypes.c_int, [_LAYER, _CACHE, _P, _P, _P, _P, _I32, _I64, _P, _P, _P, _SZ, _P]),
    "csa_sparse_attend": (ctypes.c_int, [_LAYER, _CACHE, _PARAMS, _P, _P, _I32, _P, _P, _P, _SZ, _P]),
    "hca_attend": (ctypes.c_int, [_LAYER, _CACHE, _PARAMS, _P, _P, _I32, _I64, _P, _P, _SZ, _P]),
    "csa_decode_step": (ctypes.c_int, [_LAYER, _CACHE, _PARAMS, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "hca_decode_step": (ctypes.c_int, [_LAYER, _CACHE, _PARAMS, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "csa_decode_step_scratch": (ctypes.c_int, [_LAYER, _CACHE, _PARAMS, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                               ctypes.POINTER(_I32), _P]),
    "csa_prefill": (ctypes.c_int, [_LAYER, _CACHE, _PARAMS, _P, _P, _P, _P, _P, _I32, _I64, _P, _P, _P, _SZ, _P]),
    "csa_debug_workspace_segment": (ctypes.c_int, [_LAYER, _I32, _I32, _I64, _I32, ctypes.POINTER(_SZ),
                                                   ctypes.POINTER(_SZ)]),
    "csa_debug_wait_probe": (ctypes.c_int, [_P, _SZ, ctypes.c_uint64, _P]),
    "csa_debug_scratch_copy": (ctypes.c_int, [_SZ, _P, _SZ, _I32, _P]),
    "csa_index_keys": (ctypes.c_int, [_LAYER, _CACHE, _STREAM_S, _P, _P, _P, _I32, _P]),
    "csa_index_query": (ctypes.c_int, [_LAYER, _P, _P, _I32, _I32, _P, _P, _P]),
    "csa_decode_step_indexed": (ctypes.c_int, [_LAYER, _CACHE, _PARAMS, _STREAM_S, _P, _P, _P, _I32, _P, _P, _P, _P,
                                               _P, _P, _P, _P, _P, _SZ, _P]),
    "csa_shard_candidates": (ctypes.c_int, [_LAYER, _P, _I64, _P, _I64, _P, _P, _P]),
    "csa_shard_select": (ctypes.c_int, [_LAYER, _I32, _P, _P, _P, _P]),
    "csa_sparse_attend_partial": (ctypes.c_int, [_LAYER, _CACHE, _PARAMS, _P, _P, _P, _I64, _I32, _P, _P, _SZ, _P]),
    "csa_attend_merge": (ctypes.c_int, [_LAYER, _PARAMS, _P, _I32, _P, _P, _P]),
}

EXPORTED = tuple(_SIGS)

_lib = None


def lib():
    """The loaded library; raises if it was not built (no fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m long_context_sparse_csa_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(h, name)
            f.restype = res
            f.argtypes = args
        _lib = h
    return _lib


def _check(status):
    if status != 0:
        raise CsaError(status, lib().csa_last_error().decode())


def ptr(t):
    """Device (or host) address of a tensor, or None."""
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def make_layer(kind, B, H, D, m, overlap, top_k=0, window=128, H_I=0, d_I=0, kv_format="bf16",
               idx_format="e4m3", act_format="bf16", rope_base=10000.0, eps=1e-6, softmax_scale=0.0,
               pos0=0, d_rope=64) -> CsaLayer:
    return CsaLayer(KIND[kind], B, H, D, d_rope, m, overlap, top_k, window, H_I, d_I, FMT[kv_format],
                    FMT[idx_format], FMT[act_format], float(rope_base), float(eps), float(softmax_scale), int(pos0))


def layer_from_spec(layer, B, pos0=0) -> CsaLayer:
    """CsaLayer from a csa_synth.configs.Layer."""
    return make_layer(layer.kind, B, layer.H, layer.D, layer.m, layer.ov, layer.top_k, layer.window, layer.H_I,
                      layer.d_I, layer.kv_format, layer.idx_format, layer.act_format, layer.rope_base, layer.eps,
                      0.0, pos0, layer.d_rope)


def make_cache(entries, window, raw=None, gate=None, idx_keys=None, idx_key_scale=None, raw_base=0) -> CsaCache:
    """Cache struct over tensors shaped [B, cap, ...] (entries, window, raw, gate, idx keys)."""
    return CsaCache(entries.data_ptr(), entries.shape[1], idx_keys.data_ptr() if idx_keys is not None else None,
                    idx_key_scale.data_ptr() if idx_key_scale is not None else None, window.data_ptr(),
                    window.shape[1], raw.data_ptr() if raw is not None else None,
                    gate.data_ptr() if gate is not None else None, raw.shape[1] if raw is not None else 0, raw_base)


def make_index_stream(raw, gate, pos_bias) -> CsaIndexStream:
    """Index-key stream struct over rings [B, raw_cap, d_I] and the slot biases [(1+ov)m, d_I]."""
    return CsaIndexStream(raw.data_ptr(), gate.data_ptr(), pos_bias.data_ptr())


def make_params(pos_bias=None, gamma_kv=None, gamma_q=None, sinks=None) -> CsaParams:
    g = lambda t: t.data_ptr() if t is not None else None  # noqa: E731
    return CsaParams(g(pos_bias), g(gamma_kv), g(gamma_q), g(sinks))


# ----------------------------------------------------------------------------- entry points
def csa_row_bytes(L: CsaLayer) -> int:
    return lib().csa_row_bytes(ctypes.byref(L))


def csa_workspace_size(L: CsaLayer, op: str, Tq: int, entry_cap: int) -> int:
    return lib().csa_workspace_size(ctypes.byref(L), OP[op], Tq, entry_cap)


def csa_version() -> str:
    return lib().csa_version().decode()


def csa_profile_events(ev_start, ev_stop):
    """Record these torch.cuda.Events around each later indexer-score launch (None, None: off)."""
    h = lib()
    if ev_start is None or ev_stop is None:
        h.csa_profile_events(None, None)
    else:
        h.csa_profile_events(ctypes.c_void_p(ev_start.cuda_event), ctypes.c_void_p(ev_stop.cuda_event))


_timeline_keep = None


def csa_profile_timeline(events):
    """Arm a timeline of torch.cuda.Events (recorded before each later launch); None disarms."""
    global _timeline_keep
    h = lib()
    if not events:
        h.csa_profile_timeline(None, 0)
        _timeline_keep = None
        return
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    _timeline_keep = arr
    h.csa_profile_timeline(ctypes.cast(arr, ctypes.c_void_p), len(events))


def csa_profile_timeline_count() -> int:
    return lib().csa_profile_timeline_count()


def csa_launch_count() -> int:
    return lib().csa_launch_count()


def csa_device_error(workspace, stream=None) -> int:
    """OR of the workspace's error word (None: skipped) and the library's own word; both cleared."""
    code = _I32(0)
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().csa_device_error(ptr(workspace), nbytes, _stream(stream), ctypes.byref(code))
    if st not in (0, 5):
        _check(st)
    return code.value


def csa_debug_workspace_segment(L, op, Tq, entry_cap, segment):
    """(byte offset, bytes) of a workspace segment (test aid)."""
    off, nb = _SZ(0), _SZ(0)
    _check(lib().csa_debug_workspace_segment(ctypes.byref(L), OP[op], Tq, entry_cap, SEGMENT[segment],
                                             ctypes.byref(off), ctypes.byref(nb)))
    return off.value, nb.value


def csa_debug_wait_probe(workspace, limit_ns, stream=None):
    """Launch the bounded-wait probe: its wait runs out after limit_ns and sets the error word (test aid)."""
    _check(lib().csa_debug_wait_probe(ptr(workspace), workspace.numel() * workspace.element_size(), int(limit_ns),
                                      _stream(stream)))


def csa_debug_scratch_copy(offset, buf, to_scratch, stream=None):
    """Copy between a tensor and the static scratch at byte `offset` (test aid; synchronises)."""
    _check(lib().csa_debug_scratch_copy(int(offset), ptr(buf), buf.numel() * buf.element_size(),
                                        1 if to_scratch else 0, _stream(stream)))


def csa_append(L, cache, x_new, g_new, q_pos, Tq, stream=None):
    _check(lib().csa_append(ctypes.byref(L), ctypes.byref(cache), ptr(x_new), ptr(g_new), ptr(q_pos), Tq,
                            _stream(stream)))


def csa_compress(L, cache, params, q_pos, Tq, stream=None):
    _check(lib().csa_compress(ctypes.byref(L), ctypes.byref(cache), ctypes.byref(params), ptr(q_pos), Tq,
                              _stream(stream)))


def csa_index_topk(L, cache, idx_q, idx_q_scale, head_w, q_pos, Tq, n_max, topk_idx, scores, workspace,
                   stream=None):
    _check(lib().csa_index_topk(ctypes.byref(L), ctypes.byref(cache), ptr(idx_q), ptr(idx_q_scale), ptr(head_w),
                                ptr(q_pos), Tq, n_max, ptr(topk_idx), ptr(scores), ptr(workspace),
                                workspace.numel() * workspace.element_size(), _stream(stream)))


def csa_sparse_attend(L, cache, params, q, q_pos, Tq, topk_idx, out, workspace, stream=None):
    _check(lib().csa_sparse_attend(ctypes.byref(L), ctypes.byref(cache), ctypes.byref(params), ptr(q), ptr(q_pos),
                                   Tq, ptr(topk_idx), ptr(out), ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream)))


def hca_attend(L, cache, params, q, q_pos, Tq, n_max, out, workspace, stream=None):
    _check(lib().hca_attend(ctypes.byref(L), ctypes.byref(cache), ctypes.byref(params), ptr(q), ptr(q_pos), Tq,
                            n_max, ptr(out), ptr(workspace), workspace.numel() * workspace.element_size(),
                            _stream(stream)))


def csa_decode_step(L, cache, params, q, idx_q, idx_q_scale, head_w, x_new, g_new, q_pos, out, topk_idx,
                    workspace, stream=None):
    _check(lib().csa_decode_step(ctypes.byref(L), ctypes.byref(cache), ctypes.byref(params), ptr(q), ptr(idx_q),
                                 ptr(idx_q_scale), ptr(head_w), ptr(x_new), ptr(g_new), ptr(q_pos), ptr(out),
                                 ptr(topk_idx), ptr(workspace), workspace.numel() * workspace.element_size(),
                                 _stream(stream)))


def csa_decode_step_scratch(L, cache, params, q, idx_q, idx_q_scale, head_w, x_new, g_new, q_pos, out, topk_idx,
                            read_device_error=False, stream=None):
    """csa_decode_step on the library's static device scratch (no workspace argument).  With
    read_device_error the call synchronises and returns the device error word (else None)."""
    code = _I32(0)
    st = lib().csa_decode_step_scratch(ctypes.byref(L), ctypes.byref(cache), ctypes.byref(params), ptr(q),
                                       ptr(idx_q), ptr(idx_q_scale), ptr(head_w), ptr(x_new), ptr(g_new),
                                       ptr(q_pos), ptr(out), ptr(topk_idx),
                                       ctypes.byref(code) if read_device_error else None, _stream(stream))
    if read_device_error and st == 5:      # CSA_ERR_DEVICE_TIMEOUT: the device error word is the result
        return code.value
    _check(st)
    return code.value if read_device_error else None


def hca_decode_step(L, cache, params, q, x_new, g_new, q_pos, out, workspace, stream=None):
    _check(lib().hca_decode_step(ctypes.byref(L), ctypes.byref(cache), ctypes.byref(params), ptr(q), ptr(x_new),
                                 ptr(g_new), ptr(q_pos), ptr(out), ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream)))


def csa_prefill(L, cache, params, q, idx_q, idx_q_scale, head_w, q_pos, Tq, n_max, out, topk_idx, workspace,
                stream=None):
    _check(lib().csa_prefill(ctypes.byref(L), ctypes.byref(cache), ctypes.byref(params), ptr(q), ptr(idx_q),
                             ptr(idx_q_scale), ptr(head_w), ptr(q_pos), Tq, n_max, ptr(out), ptr(topk_idx),
                             ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def csa_index_keys(L, cache, index_stream, x_new, g_new, q_pos, Tq, stream=None):
    _check(lib().csa_index_keys(ctypes.byref(L), ctypes.byref(cache), ctypes.byref(index_stream), ptr(x_new),
                                ptr(g_new), ptr(q_pos), Tq, _stream(stream)))


def csa_index_query(L, c, W, rank, rows, idx_q, idx_q_scale, stream=None):
    _check(lib().csa_index_query(ctypes.byref(L), ptr(c), ptr(W), rank, rows, ptr(idx_q), ptr(idx_q_scale),
                                 _stream(stream)))


def csa_decode_step_indexed(L, cache, params, index_stream, q, c, W, rank, head_w, x_new, g_new, idx_x_new,
                            idx_g_new, q_pos, out, topk_idx, workspace, stream=None):
    _check(lib().csa_decode_step_indexed(ctypes.byref(L), ctypes.byref(cache), ctypes.byref(params),
                                         ctypes.byref(index_stream), ptr(q), ptr(c), ptr(W), rank, ptr(head_w),
                                         ptr(x_new), ptr(g_new), ptr(idx_x_new), ptr(idx_g_new), ptr(q_pos), ptr(out),
                                         ptr(topk_idx), ptr(workspace), workspace.numel() * workspace.element_size(),
                                         _stream(stream)))


def csa_shard_candidates(L, scores, n_local, topk_local, entry_offset, cand_score, cand_idx, stream=None):
    _check(lib().csa_shard_candidates(ctypes.byref(L), ptr(scores), n_local, ptr(topk_local), entry_offset,
                                      ptr(cand_score), ptr(cand_idx), _stream(stream)))


def csa_shard_select(L, shards, cand_score, cand_idx, topk_idx, stream=None):
    _check(lib().csa_shard_select(ctypes.byref(L), shards, ptr(cand_score), ptr(cand_idx), ptr(topk_idx),
                                  _stream(stream)))


def csa_sparse_attend_partial(L, cache, params, q, q_pos, topk_idx, entry_offset, with_window, partial, workspace,
                              stream=None):
    _check(lib().csa_sparse_attend_partial(ctypes.byref(L), ctypes.byref(cache), ctypes.byref(params), ptr(q),
                                           ptr(q_pos), ptr(topk_idx), entry_offset, 1 if with_window else 0,
                                           ptr(partial), ptr(workspace), workspace.numel() * workspace.element_size(),
                                           _stream(stream)))


def csa_attend_merge(L, params, q_pos, parts, partials, out, stream=None):
    _check(lib().csa_attend_merge(ctypes.byref(L), ctypes.byref(params), ptr(q_pos), parts, ptr(partials), ptr(out),
                                  _stream(stream)))
