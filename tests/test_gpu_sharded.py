"""Context-sharded CSA decode on one GPU: G ranks emulated in sequence, their all-gathers replaced by
stacking the ranks' tensors in rank order (the same bytes a collective would deliver), checked
against the oracle over the unsharded caches: the global top-k bit-exact outside the tie band and
identical on every rank, the merged output within the operator's bars."""

import numpy as np
import pytest
import torch

from csa_synth import decode_inputs, get_workload
from long_context_sparse_csa_b200 import binding as C
from long_context_sparse_csa_b200.sharded import GpuBackend, Shard, shard_bounds
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


@pytest.mark.parametrize("name,G,B,n", [("csa_decode_128k", 2, 2, None), ("csa_decode_128k", 3, 1, 4 * 9001 + 3),
                                        ("csa_hca_decode_1m", 4, None, None), ("csa_decode_128k", 5, 2, 4 * 900)])
def test_sharded_decode_matches_unsharded(name, G, B, n):
    over = {}
    if B is not None:
        over["B"] = B
    if n is not None:
        over["n"] = n
    wl = get_workload(name, **over)
    layer = wl.layers[0]
    d = decode_inputs(wl, 0)
    Bq = wl.B
    N = d["entries"].shape[1]
    backends = []
    for r, (off, cnt) in enumerate(shard_bounds(N, G)):
        sub = dict(d)
        sub["entries"] = np.ascontiguousarray(d["entries"][:, off:off + cnt])
        sub["idx_k"] = np.ascontiguousarray(d["idx_k"][:, off:off + cnt])
        sub["idx_k_scale"] = np.ascontiguousarray(d["idx_k_scale"][:, off:off + cnt])
        backends.append(GpuBackend(LayerState.from_arrays(layer, Bq, sub), Shard(r, G, off, cnt)))
    q, iq, iqs, hw, qp = (dev(d[k]) for k in ("q", "idx_q", "idx_q_scale", "head_w", "t"))
    cands = [be.local_candidates(iq, iqs, hw, qp) for be in backends]
    all_s = torch.stack([c[0].clone() for c in cands])
    all_i = torch.stack([c[1].clone() for c in cands])
    topks = [be.select(all_s, all_i).clone() for be in backends]
    parts = torch.stack([be.partial_attend(q, qp, topks[r]).clone() for r, be in enumerate(backends)])
    out = torch.zeros((Bq, layer.H, layer.D), dtype=torch.int16, device="cuda")
    backends[0].merge(qp, parts, out)
    torch.cuda.synchronize()
    for be in backends:
        assert be.device_errors() == 0
    for r in range(1, G):
        assert torch.equal(topks[r], topks[0]), "every rank picks the same global top-k"
    got = out_values(out, layer.act_format)
    tk = host(topks[0])
    L = O.LayerSpec.of(layer)
    for b in range(Bq):
        t = int(d["t"][b])
        nv = int(O.n_visible(t, 0, layer.m))
        iqv, ik, iks = O.index_operands(L, d["idx_q"][b], d["idx_k"][b][:nv], d["idx_k_scale"][b][:nv])
        s = O.index_scores(iqv, d["idx_q_scale"][b], d["head_w"][b], ik, iks)
        check_topk(tk[b], s, layer.top_k)
        ids = tk[b][tk[b] >= 0]
        rows = np.concatenate([F.decode_rows(d["entries"][b][ids], layer.kv_format, layer.D),
                               F.decode_rows(d["window"][b][O.window_row_ids(t, 0, layer.window) % layer.window],
                                             layer.kv_format, layer.D)])
        ref = O.attend(F.decode_act(d["q"][b], layer.act_format), t, rows, d["sinks"], d["gamma_q"], 64,
                       layer.rope_base, None, layer.eps)
        assert_out_close(got[b], ref, tag=f"sharded/{name}/G={G}/b{b}")
