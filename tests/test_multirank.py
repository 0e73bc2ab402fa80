"""The multi-GPU path's host logic, on CPU with two gloo ranks.

bench.py --gpus N runs one process per GPU; every rank decodes its own batch (the path
shards by sequence, so there is no data-path collective), the slowest rank sets the step
time, and the job's throughput counts the units of all ranks.  These pieces are checked
here with world_size 2 over gloo; the CUDA work itself is covered by the GPU tests."""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import synth
        from synth import configs as C
        w = C.WORKLOADS["decode128k"]
        # per-rank inputs differ (weak scaling: each rank its own batch)
        key = bench.rank_key(w.key(synth.KIND_IK), rank)
        sample = synth.int17_bf16(key, (4, 128))
        gathered = [None] * world
        dist.all_gather_object(gathered, sample.tobytes())
        # the slowest rank sets the step time
        mine = [1.0 + rank, 10.0 - rank, 3.0]
        mx = bench.max_over_ranks(mine, world)
        thr = bench.job_throughput(w.B * w.T, world, mx[0])
        out[rank] = (gathered, mx, thr)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    g0, mx0, thr0 = out[0]
    g1, mx1, thr1 = out[1]
    assert g0 == g1 and g0[0] != g0[1]          # both ranks saw both samples; they differ
    assert mx0 == mx1 == [2.0, 10.0, 3.0]        # element-wise max over the two ranks
    assert thr0 == thr1 == pytest.approx(8 * 1 * 2 / 2.0e-3)


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks([1.5, 2.5], 1) == [1.5, 2.5]
    assert bench.job_throughput(8, 1, 0.1) == pytest.approx(80000.0)


def _oracle_shard_ops(orc):
    """The context-shard steps computed by the CPU oracle, with torch CPU tensors where the
    exchange needs them (test-only stand-ins for the library's kernels)."""
    import torch
    from types import SimpleNamespace

    def tn(t):
        return t.numpy() if isinstance(t, torch.Tensor) else t

    def candidates(scores, idx, offset):
        s, i = tn(scores), tn(idx)
        v = i >= 0
        cs = np.where(v, np.take_along_axis(s, np.maximum(i, 0), axis=2), -np.inf).astype(np.float32)
        cp = np.where(v, i + offset, -1).astype(np.int32)
        return torch.from_numpy(cs), torch.from_numpy(cp)

    def merge_candidates(cs, cp, k):
        cs, cp = tn(cs), tn(cp)                       # [W, B, T, kc], shard-major
        W, B, T, kc = cs.shape
        cs = np.moveaxis(cs, 0, 2).reshape(B, T, W * kc)
        cp = np.moveaxis(cp, 0, 2).reshape(B, T, W * kc)
        return orc.merge_candidates(cs, cp, k)

    def attn_shard(q, kv, idx, offset, scale):
        out, lse = orc.sparse_attn_partial(q, kv, tn(idx), offset, scale)
        return torch.from_numpy(out), torch.from_numpy(lse)

    return SimpleNamespace(
        index_score=lambda iq, w, ik, q_pos0: orc.index_score(iq, w, ik, q_pos0).astype(np.float32),
        topk=lambda scores, q_pos0, k: orc.topk(scores, q_pos0, k),
        candidates=candidates, merge_candidates=merge_candidates, attn_shard=attn_shard,
        merge_partials=lambda outs, lses: orc.merge_partials(tn(outs), tn(lses)))


def _shard_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from sparse_long_context_score_b200 import sharded
        from synth import configs as C
        orc = oracle.default()
        w = C.scaled(C.WORKLOADS["decode1m"], B=2, N=700, q_pos0=699, k=64, H=16, L=2, groups=1)
        iq, wt, ik, qs, kvs = C.host_group_inputs(w)
        offset, size = sharded.shard_bounds(w.N, world)[rank]
        comm = sharded.TorchComm()
        idx, outs = sharded.sharded_group_forward(
            comm, _oracle_shard_ops(orc), iq, wt, ik[:, offset:offset + size].copy(), qs,
            [kv[:, offset:offset + size].copy() for kv in kvs], w.q_pos0, offset, w.k, C.SCALE)
        out[rank] = (np.asarray(idx).tobytes(), [np.asarray(o).tobytes() for o in outs])
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_context_sharded_group_on_two_gloo_ranks(orc):
    """The context-sharded group (exchange logic of sparse_long_context_score_b200.sharded,
    steps by the oracle) over two ranks: the same index list and outputs on both ranks,
    equal to the unsharded group's."""
    from synth import configs as C
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_shard_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    w = C.scaled(C.WORKLOADS["decode1m"], B=2, N=700, q_pos0=699, k=64, H=16, L=2, groups=1)
    iq, wt, ik, qs, kvs = C.host_group_inputs(w)
    ridx, routs = orc.group_forward(iq, wt, ik, qs, kvs, w.q_pos0, w.k, C.SCALE)
    for rank in range(world):
        idx_b, outs_b = out[rank]
        idx = np.frombuffer(idx_b, dtype=np.int32).reshape(ridx.shape)
        assert np.array_equal(idx, ridx)
        for l in range(w.L):
            got = np.frombuffer(outs_b[l], dtype=np.float64).reshape(routs[l].shape)
            assert np.allclose(got, routs[l], rtol=0, atol=1e-9)
