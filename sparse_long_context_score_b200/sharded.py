"""Context-sharded decode: one IndexShare group over a context spread across GPUs.

"Le contexte d'un million de tokens", Service efficace pour un million de contextes: a
long context is served by spreading it over several GPUs (the pages give no algorithm).
Every rank holds the contiguous range ``[offset, offset + Ns)`` of every sequence's cached
tokens (index keys and compressed rows).  One decode step of a group:

1. the rank scores its shard and keeps its own top-k (``dsa_index_score``, ``dsa_topk``),
   turned into (score, global position) candidates (``dsa_shard_candidates``);
2. the candidates of all ranks are all-gathered (shard-major) and every rank keeps the k
   best (``dsa_merge_candidates``): the row's index list, identical to the unsharded
   top-k, since a token in the row's top-k is in its own shard's top-k;
3. per layer, each rank attends over the selected rows it holds and also returns the
   log-sum-exp of their logits (``dsa_sparse_attn_shard``); the partials are all-gathered
   and combined (``dsa_merge_partials``).

Every step of the computation is a libdsa kernel; torch only allocates device memory and
runs the all-gathers (NCCL between GPUs).  The exchange logic takes its kernels from an
``ops`` object and its collectives from a ``comm`` object, so that the same code is
exercised with other implementations of either in tests.
"""
from __future__ import annotations

from types import SimpleNamespace


def shard_bounds(n_total: int, world: int):
    """Contiguous, balanced shards of the positions [0, n_total): a list of (offset, size)."""
    return [(r * n_total // world, (r + 1) * n_total // world - r * n_total // world) for r in range(world)]


def cuda_ops(device=None):
    """The library's kernels (CUDA tensors in, CUDA tensors out)."""
    from . import (dsa_index_score, dsa_merge_candidates, dsa_merge_partials, dsa_shard_candidates,
                   dsa_sparse_attn_shard, dsa_topk)
    return SimpleNamespace(
        index_score=lambda iq, w, ik, q_pos0: dsa_index_score(iq, w, ik, q_pos0),
        topk=lambda scores, q_pos0, k: dsa_topk(scores, q_pos0, k),
        candidates=lambda scores, idx, offset: dsa_shard_candidates(scores, idx, offset),
        merge_candidates=lambda cand_score, cand_pos, k: dsa_merge_candidates(cand_score, cand_pos, k),
        attn_shard=lambda q, kv, idx, offset, scale: dsa_sparse_attn_shard(q, kv, idx, offset, scale),
        merge_partials=lambda outs, lses: dsa_merge_partials(outs, lses),
    )


class TorchComm:
    """All-gather over a torch.distributed process group (NCCL for CUDA tensors, gloo on
    the CPU): ``all_gather(t)`` returns the ranks' tensors stacked along a new first axis,
    rank order."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def all_gather(self, t):
        import torch
        t = t.contiguous()
        out = torch.empty((self.world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
        if t.is_cuda:
            self.dist.all_gather_into_tensor(out, t, group=self.group)
        else:
            self.dist.all_gather(list(out.unbind(0)), t, group=self.group)
        return out


def local_candidates(ops, iq, w, ik_shard, q_pos: int, offset: int, k: int):
    """Step 1 on this rank's shard: (cand_score [B,T,k], cand_pos [B,T,k] global).
    ``q_pos`` is the global position of query 0 (query t sees positions <= q_pos + t)."""
    q_pos0 = q_pos - offset
    scores = ops.index_score(iq, w, ik_shard, q_pos0)
    idx = ops.topk(scores, q_pos0, k)
    return ops.candidates(scores, idx, offset)


def sharded_group_forward(comm, ops, iq, w, ik_shard, qs, kv_shards, q_pos: int, offset: int, k: int,
                          scale: float):
    """One IndexShare group on this rank's context shard; every rank calls it with its own
    shard (``offset`` = the global position of its first cached token) and the same
    queries.  Returns (idx [B,T,k] global positions, [out_l [B,T,H,512] for each layer]),
    the same on every rank and equal to the unsharded group's."""
    cand_score, cand_pos = local_candidates(ops, iq, w, ik_shard, q_pos, offset, k)
    idx = ops.merge_candidates(comm.all_gather(cand_score), comm.all_gather(cand_pos), k)
    outs = []
    for q, kv in zip(qs, kv_shards):
        out, lse = ops.attn_shard(q, kv, idx, offset, scale)
        outs.append(ops.merge_partials(comm.all_gather(out), comm.all_gather(lse)))
    return idx, outs
