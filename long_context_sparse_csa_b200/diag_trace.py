"""Per-CTA phase timelines of the decode kernels (diagnostics; needs a GPU and the trace library).

    python -m long_context_sparse_csa_b200.build --trace
    python -m long_context_sparse_csa_b200.diag_trace attend|index|compress [--workload NAME]

The trace library is the product's kernels built with CSA_TRACE: selected threads record
%globaltimer (ns) or clock64 at fixed points into small device arrays, which this module reads
back after each call.  Every timing below is a median over the traced CTAs, in µs from the first
traced CTA's start; the L2 is cleaned by a 256 MB read before each call unless stated.  The
numbers come from a build that is not the product's (the records cost a few instructions), so they
explain where time goes; they are not the benchmark.
"""

import argparse
import ctypes
import os

import numpy as np
import torch

from . import binding as C
from .build import TRACE_LIB
from .state import LayerState, to_device


def _lib():
    if not os.path.exists(TRACE_LIB):
        raise SystemExit(f"{TRACE_LIB} is missing: python -m long_context_sparse_csa_b200.build --trace")
    C.LIB_PATH = TRACE_LIB
    return C.lib()


def _rel(buf, n_ctas):
    """int64 µs relative to the earliest start (slot 0), NaN where a slot was not written."""
    b = buf[:n_ctas].astype(np.int64)
    t0 = int(b[:, 0][b[:, 0] > 0].min())
    out = (b - t0) / 1000.0
    out[buf[:n_ctas] == 0] = np.nan
    return out


def _flush():
    big = torch.ones(256 << 20, dtype=torch.uint8, device="cuda")
    return lambda: (big.sum(), torch.cuda.synchronize())


def trace_attend(wl):
    """tcgen05 attention of each layer: set-up, row copies and conversion, partial S, the pair's
    score exchange, softmax, P.V and the partials' epilogue."""
    from csa_synth import decode_inputs
    h = _lib()
    h.csa_trace_read_a.argtypes = [ctypes.c_void_p]
    flush = _flush()
    phases = [(0, "start"), (1, "set-up done"), (7, "raw half rows landed"), (2, "half rows converted"),
              (3, "partial S done"), (4, "pair barrier, first phase awaited"), (8, "peer's partial scores in"),
              (9, "softmax done (P in shared memory)"), (5, "P.V issued"), (10, "O ready"),
              (11, "partials written"), (6, "end")]
    for li, layer in enumerate(wl.layers):
        d = decode_inputs(wl, li)
        st = LayerState.from_arrays(layer, wl.B, d)
        cap = d["entries"].shape[1]
        io = {k: to_device(d[k]) for k in ("q", "t")}
        out = torch.zeros((wl.B, layer.H, layer.D), dtype=torch.int16, device="cuda")
        ws = st.workspace("decode_step", 1, cap)        # covers either attention call
        topk = None
        if layer.kind == "csa":
            rng = np.random.default_rng(0)
            sel = np.sort(rng.choice(cap, layer.top_k, replace=False)).astype(np.int32)
            topk = torch.from_numpy(np.tile(sel, (wl.B, 1))).cuda()
        for _ in range(3):
            flush()
            if layer.kind == "csa":
                C.csa_sparse_attend(st.L, st.cache(), st.params(), io["q"], io["t"], 1, topk, out, ws)
            else:
                C.hca_attend(st.L, st.cache(), st.params(), io["q"], io["t"], 1, cap, out, ws)
            torch.cuda.synchronize()
        buf = np.zeros((320, 16), dtype=np.uint64)
        h.csa_trace_read_a(buf.ctypes.data)
        n = int((buf[:, 0] > 0).sum())
        T = _rel(buf, n)
        cyc = buf[:n, 12:16].astype(np.int64)
        print(f"{layer.kind} attention, {n} CTAs traced (query row 0)")
        for s, name in phases:
            print(f"  {name:40s} median {np.nanmedian(T[:, s]):6.2f}  max {np.nanmax(T[:, s]):6.2f}")
        print("  softmax cycles (median): max pass %d, exp pass %d, P stores %d" %
              tuple(np.median(np.diff(cyc, axis=1), axis=0)))


def trace_index(wl):
    """CSA indexer (per-tile copy, MMA and epilogue times) and the split top-k's phases."""
    from csa_synth import decode_inputs
    h = _lib()
    h.csa_trace_read.argtypes = [ctypes.c_void_p, ctypes.c_int]
    h.csa_trace_read_t.argtypes = [ctypes.c_void_p]
    li = [i for i, l in enumerate(wl.layers) if l.kind == "csa"][0]
    layer = wl.layers[li]
    d = decode_inputs(wl, li)
    st = LayerState.from_arrays(layer, wl.B, d)
    cap = d["entries"].shape[1]
    topk = torch.zeros((wl.B, layer.top_k), dtype=torch.int32, device="cuda")
    ws = st.workspace("index_topk", 1, cap)
    args = [to_device(d[k]) for k in ("idx_q", "idx_q_scale", "head_w", "t")]
    flush = _flush()
    for _ in range(3):
        flush()
        C.csa_index_topk(st.L, st.cache(), *args[:3], args[3], 1, cap, topk, None, ws)
        torch.cuda.synchronize()
    buf = np.zeros((320, 80), dtype=np.uint64)
    h.csa_trace_read(buf.ctypes.data, buf.size)
    n = int((buf[:, 0] > 0).sum())
    T = _rel(buf, n)
    print(f"indexer, {n} CTAs: set-up done {np.nanmedian(T[:, 1]):.2f}")
    print("  tile   issued   landed   accumulator ready   epilogue done")
    for k in range(16):
        if np.all(np.isnan(T[:, 18 + k])):
            break
        print("  %4d  %7.2f  %7.2f  %18.2f  %14.2f" % (k, np.nanmedian(T[:, 2 + k]), np.nanmedian(T[:, 18 + k]),
                                                     np.nanmedian(T[:, 34 + k]), np.nanmedian(T[:, 50 + k])))
    print(f"  epilogue warps reach the final barrier: median {np.nanmedian(T[:, 70]):.2f}, max {np.nanmax(T[:, 70]):.2f}")
    tb = np.zeros((80, 24), dtype=np.uint64)
    h.csa_trace_read_t(tb.ctypes.data)
    g = int((tb[:, 0] > 0).sum())
    TT = _rel(tb, g)
    print(f"split top-k, {g} CTAs (all CTAs: median and max; the last CTA's phases: max)")
    for s, name in [(0, "start"), (1, "first-level bin found"), (2, "slice filtered"), (3, "ticket taken"),
                    (8, "last CTA begins"), (9, "second-level bin found"), (10, "slice offsets"),
                    (4, "list loads issued, histograms cleared"), (11, "list in registers"),
                    (12, "third-level histogram"), (5, "threshold key found"), (7, "end")]:
        print(f"  {name:40s} median {np.nanmedian(TT[:, s]):7.2f}  max {np.nanmax(TT[:, s]):7.2f}")


def trace_compress(wl):
    """Append+compress of each layer: phases of CTA 0 and its cycle split (pooling, wait at the
    row-group merge, merge, RMSNorm with the cluster reduction)."""
    from csa_synth import decode_inputs
    h = _lib()
    h.csa_trace_read_c.argtypes = [ctypes.c_void_p]
    flush = _flush()
    buf = np.zeros((4, 16), dtype=np.uint64)
    for li, layer in enumerate(wl.layers):
        d = decode_inputs(wl, li)
        st = LayerState.from_arrays(layer, wl.B, d)
        t = to_device(d["t"])
        for label, clean in (("back to back", False), ("after a 256 MB read", True)):
            for _ in range(3):
                if clean:
                    flush()
                C.csa_compress(st.L, st.cache(), st.params(), t, 1)
                torch.cuda.synchronize()
            h.csa_trace_read_c(buf.ctypes.data)
            row = buf[0 if layer.m == 4 else 1].astype(np.int64)
            us = [round((row[i] - row[0]) / 1000, 2) for i in range(9)]
            cyc = [int(row[11] - row[10]), int(row[14] - row[11]), int(row[12] - row[14]), int(row[13] - row[12])]
            print(f"{layer.kind} compress, {label}: CTA 0 phases (µs) {us}; cycles pool {cyc[0]}, "
                  f"merge wait {cyc[1]}, merge {cyc[2]}, norm {cyc[3]}")


def main():
    p = argparse.ArgumentParser()
    p.add_argument("what", choices=["attend", "index", "compress"])
    p.add_argument("--workload", default="csa_hca_decode_1m")
    a = p.parse_args()
    from csa_synth import get_workload
    wl = get_workload(a.workload)
    {"attend": trace_attend, "index": trace_index, "compress": trace_compress}[a.what](wl)


if __name__ == "__main__":
    main()
