"""The sharded decode step's host side (long_context_sparse_csa_b200.sharded.decode_step) over real
collectives: two gloo ranks on the CPU, each holding half of a sequence's entries, exchange their
candidates and partials with torch.distributed.all_gather.  The per-rank compute is a CPU stand-in
written from the oracle's definitions (scores, top-k, the partial (O/l, m, l) of a key set, the merge
with the sink and the inverse rotation), so the test checks the step's dataflow and exchanges: the
result must equal the oracle's attention over the unsharded caches, identically on both ranks."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from csa_synth import decode_inputs
from csa_synth.configs import CSA_PRO, Workload, scaled_layer
from long_context_sparse_csa_b200.sharded import Shard, decode_step, dist_all_gather, shard_bounds
from oracle import csa as O
from oracle import formats as F

LAYER = scaled_layer(CSA_PRO, H=4, top_k=32, window=16)
LOG2E = 1.4426950408889634


def _inputs():
    wl = Workload(name="t", mode="decode", B=2, n=4 * 700 + 1, layers=(LAYER,), seed=61)
    return decode_inputs(wl, 0)


class CpuBackend:
    """Oracle-based stand-in for the per-rank kernels (test only)."""

    def __init__(self, d, shard):
        self.d, self.shard = d, shard
        self.L = O.LayerSpec.of(LAYER)

    def local_candidates(self, idx_q, idx_q_scale, head_w, q_pos):
        k = LAYER.top_k
        B = len(self.d["t"])
        cs = torch.full((B, k), -float("inf"), dtype=torch.float64)
        ci = torch.full((B, k), -1, dtype=torch.int64)
        off, cnt = self.shard.offset, self.shard.count
        for b in range(B):
            nv = int(O.n_visible(self.d["t"][b], 0, LAYER.m))
            hi = min(off + cnt, nv)
            if hi <= off:
                continue
            iq, ik, iks = O.index_operands(self.L, self.d["idx_q"][b], self.d["idx_k"][b][off:hi],
                                           self.d["idx_k_scale"][b][off:hi])
            s = O.index_scores(iq, self.d["idx_q_scale"][b], self.d["head_w"][b], ik, iks)
            sel = O.top_k_fast(s, k)
            m = sel >= 0
            cs[b, :m.sum()] = torch.from_numpy(s[sel[m]])
            ci[b, :m.sum()] = torch.from_numpy(sel[m] + off)
        return cs, ci

    def select(self, all_s, all_i):
        W, B, k = all_s.shape
        out = torch.full((B, k), -1, dtype=torch.int64)
        for b in range(B):
            s = all_s[:, b].reshape(-1).numpy()
            i = all_i[:, b].reshape(-1).numpy()
            keep = i >= 0
            order = sorted(zip(-s[keep], i[keep]))[:k]
            pick = np.sort(np.array([x[1] for x in order], dtype=np.int64))
            out[b, :len(pick)] = torch.from_numpy(pick)
        return out

    def partial_attend(self, q, q_pos, topk):
        B = len(self.d["t"])
        H, D = LAYER.H, LAYER.D
        part = torch.zeros((B, H, D + 2), dtype=torch.float64)
        off, cnt = self.shard.offset, self.shard.count
        for b in range(B):
            t = int(self.d["t"][b])
            ids = topk[b].numpy()
            own = ids[(ids >= off) & (ids < off + cnt)]
            rows = [F.decode_rows(self.d["entries"][b][own], LAYER.kv_format, D)]
            if self.shard.rank == 0:
                w = O.window_row_ids(t, 0, LAYER.window) % LAYER.window
                rows.append(F.decode_rows(self.d["window"][b][w], LAYER.kv_format, D))
            rows = np.concatenate(rows)
            qt = O.prep_query(F.decode_act(self.d["q"][b], "bf16"), self.d["gamma_q"], t, 64, LAYER.rope_base)
            if len(rows) == 0:
                part[b, :, D] = -float("inf")
                continue
            z = (qt @ rows.T) / np.sqrt(D) * LOG2E
            m = z.max(axis=1)
            e = np.exp2(z - m[:, None])
            l = e.sum(axis=1)
            part[b, :, :D] = torch.from_numpy((e @ rows) / l[:, None])
            part[b, :, D] = torch.from_numpy(m)
            part[b, :, D + 1] = torch.from_numpy(l)
        return part

    def merge(self, q_pos, all_p, out):
        W, B, H, D2 = all_p.shape
        D = D2 - 2
        p = all_p.numpy()
        for b in range(B):
            sk = np.asarray(self.d["sinks"], np.float64) * LOG2E
            M = np.maximum(sk, p[:, b, :, D].max(axis=0))
            w = p[:, b, :, D + 1] * np.exp2(p[:, b, :, D] - M[None])        # [W, H]
            w = np.where(np.isfinite(p[:, b, :, D]), w, 0.0)
            z = np.exp2(sk - M) + w.sum(axis=0)
            o = (w[:, :, None] * p[:, b, :, :D]).sum(axis=0) / z[:, None]
            out[b] = torch.from_numpy(O.rope(o, -float(self.d["t"][b]), 64, LAYER.rope_base))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        d = _inputs()
        off, cnt = shard_bounds(d["entries"].shape[1], world)[rank]
        be = CpuBackend(d, Shard(rank, world, off, cnt))
        out = torch.zeros((2, LAYER.H, LAYER.D), dtype=torch.float64)
        topk = decode_step(be, None, None, None, None, None, out, dist_all_gather())
        np.save(os.path.join(out_dir, f"out{rank}.npy"), out.numpy())
        np.save(os.path.join(out_dir, f"topk{rank}.npy"), topk.numpy())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_give_the_unsharded_result(tmp_path):
    port = _free_port()
    mp.start_processes(_rank, args=(2, port, str(tmp_path)), nprocs=2, start_method="spawn", join=True)
    d = _inputs()
    o0, o1 = np.load(tmp_path / "out0.npy"), np.load(tmp_path / "out1.npy")
    t0, t1 = np.load(tmp_path / "topk0.npy"), np.load(tmp_path / "topk1.npy")
    assert np.array_equal(t0, t1) and np.array_equal(o0, o1)
    L = O.LayerSpec.of(LAYER)
    for b in range(2):
        t = int(d["t"][b])
        nv = int(O.n_visible(t, 0, LAYER.m))
        iq, ik, iks = O.index_operands(L, d["idx_q"][b], d["idx_k"][b][:nv], d["idx_k_scale"][b][:nv])
        s = O.index_scores(iq, d["idx_q_scale"][b], d["head_w"][b], ik, iks)
        sel = O.top_k_fast(s, LAYER.top_k)
        assert np.array_equal(t0[b], sel)
        ids = sel[sel >= 0]
        rows = np.concatenate([F.decode_rows(d["entries"][b][ids], LAYER.kv_format, LAYER.D),
                               F.decode_rows(d["window"][b][O.window_row_ids(t, 0, LAYER.window) % LAYER.window],
                                             LAYER.kv_format, LAYER.D)])
        want = O.attend(F.decode_act(d["q"][b], "bf16"), t, rows, d["sinks"], d["gamma_q"], 64, LAYER.rope_base)
        assert np.allclose(o0[b], want, atol=1e-10), np.abs(o0[b] - want).max()


def test_shard_bounds_cover_every_entry_once():
    for n, w in [(10, 3), (262144, 8), (7, 7), (5, 8)]:
        b = shard_bounds(n, w)
        assert len(b) == w and b[0][0] == 0
        assert sum(c for _, c in b) == n
        assert all(b[i][0] + b[i][1] == b[i + 1][0] for i in range(w - 1))
