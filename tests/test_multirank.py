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
