"""Context-sharded CSA decode of one long sequence over ranks (one process per GPU): the host side.

Each rank holds a contiguous shard of the sequence's compressed entries and index keys (entries
[offset, offset + count) at slots 0.. of its caches) and every rank holds the query.  One decode step:

  1. the rank scores its shard and selects its local top-k (csa_index_topk with the layer's pos0
     moved to pos0 + offset * m, so a shard entry is visible exactly when its global position is);
  2. csa_shard_candidates turns those into (score, global index) candidates;
  3. all ranks all-gather the candidates ([world, B, k]);
  4. csa_shard_select picks the global top-k from them, the same on every rank;
  5. each rank attends the selected entries it holds, rank 0 also the window rows
     (csa_sparse_attend_partial), into a partial (O/l, m, l) per query and head;
  6. all ranks all-gather the partials ([world, B, H, D + 2]);
  7. csa_attend_merge merges them with the sink and the inverse rotation into the output.

Steps 3 and 6 are the only exchanges: 8 bytes per candidate (B * k * world) and (D + 2) * 4 bytes per
query head and rank.  The result is that of csa_sparse_attend over the unsharded caches with the
unsharded top-k: an entry in the global top-k is in its own shard's top-k, and attention over
disjoint key sets merges exactly by log-sum-exp weights with the sink counted once.

This module only marshals: every step runs in the library's kernels, and the collectives are the
caller's (torch.distributed over NCCL on GPUs; any all-gather with the same contract elsewhere).
"""

import torch

from . import binding as C


def shard_bounds(n_entries: int, world: int):
    """Contiguous split of n_entries over world ranks: [(offset, count)] (the first ranks get one
    more entry when the split is uneven)."""
    base, extra = divmod(n_entries, world)
    out, off = [], 0
    for r in range(world):
        cnt = base + (1 if r < extra else 0)
        out.append((off, cnt))
        off += cnt
    return out


class Shard:
    """One rank's part of the sequence: its rank, the world size and its entry range."""

    def __init__(self, rank: int, world: int, offset: int, count: int):
        self.rank, self.world, self.offset, self.count = rank, world, offset, count


class GpuBackend:
    """The library's calls for the steps of one rank, with the device buffers they need.

    state: the rank's LayerState (caches holding its shard; the window ring on every rank, attended by
    rank 0 only); B queries of one token each."""

    def __init__(self, state, shard: Shard):
        self.st, self.shard = state, shard
        spec = state.spec
        B, k, dev = state.B, spec.top_k, state.entries.device
        self.L = state.L
        # the indexer's layer: shard entry i is visible iff pos0 + (offset + i + 1) m - 1 <= t
        self.L_idx = C.CsaLayer.from_buffer_copy(state.L)
        self.L_idx.pos0 = state.L.pos0 + shard.offset * spec.m
        self.topk_local = torch.empty((B, k), dtype=torch.int32, device=dev)
        self.scores = torch.empty((B, max(shard.count, 1)), dtype=torch.float32, device=dev)
        self.cand_s = torch.empty((B, k), dtype=torch.float32, device=dev)
        self.cand_i = torch.empty((B, k), dtype=torch.int32, device=dev)
        self.topk = torch.empty((B, k), dtype=torch.int32, device=dev)
        self.partial = torch.empty((B, spec.H, spec.D + 2), dtype=torch.float32, device=dev)
        self.ws_idx = state.workspace("index_topk", 1, max(shard.count, 1))
        self.ws_att = state.workspace("sparse_attend", 1, state.entries.shape[1])

    def local_candidates(self, idx_q, idx_q_scale, head_w, q_pos):
        C.csa_index_topk(self.L_idx, self.st.cache(), idx_q, idx_q_scale, head_w, q_pos, 1, self.shard.count,
                         self.topk_local, self.scores, self.ws_idx)
        C.csa_shard_candidates(self.L, self.scores, self.shard.count, self.topk_local, self.shard.offset,
                               self.cand_s, self.cand_i)
        return self.cand_s, self.cand_i

    def select(self, all_s, all_i):
        C.csa_shard_select(self.L, all_s.shape[0], all_s.contiguous(), all_i.contiguous(), self.topk)
        return self.topk

    def partial_attend(self, q, q_pos, topk):
        C.csa_sparse_attend_partial(self.L, self.st.cache(), self.st.params(), q, q_pos, topk, self.shard.offset,
                                    self.shard.rank == 0, self.partial, self.ws_att)
        return self.partial

    def merge(self, q_pos, all_p, out):
        C.csa_attend_merge(self.L, self.st.params(), q_pos, all_p.shape[0], all_p.contiguous(), out)

    def device_errors(self):
        return C.csa_device_error(self.ws_idx) | C.csa_device_error(self.ws_att)


def decode_step(backend, q, idx_q, idx_q_scale, head_w, q_pos, out, all_gather):
    """One sharded decode step on this rank; all_gather(t) returns the ranks' tensors stacked on a new
    leading axis, in rank order.  Returns the global top-k (identical on every rank)."""
    cand_s, cand_i = backend.local_candidates(idx_q, idx_q_scale, head_w, q_pos)
    all_s, all_i = all_gather(cand_s), all_gather(cand_i)
    topk = backend.select(all_s, all_i)
    part = backend.partial_attend(q, q_pos, topk)
    backend.merge(q_pos, all_gather(part), out)
    return topk


def dist_all_gather(group=None):
    """all_gather over torch.distributed (NCCL for device tensors, gloo for host tensors)."""
    import torch.distributed as dist

    def gather(t):
        parts = [torch.empty_like(t) for _ in range(dist.get_world_size(group))]
        dist.all_gather(parts, t.contiguous(), group=group)
        return torch.stack(parts)

    return gather
