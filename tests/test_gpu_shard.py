"""Parity of the context-sharded decode kernels against the CPU oracle, and the sharded
group on one GPU (W shards run one after the other in one process, the all-gathers
replaced by stacking the shards' tensors) against the unsharded oracle group."""
import numpy as np
import pytest

import synth
from gpu_util import assert_close, dev, dev_bf16, host
from synth import configs as C

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import sparse_long_context_score_b200 as m
    from sparse_long_context_score_b200 import build
    build.build()
    m.lib()
    return m


def _attn_case(seed, B, T, N, H, k):
    key = lambda kind: synth.stream_key(seed, synth.tensor_id(kind))
    q = synth.normal_bf16(key(synth.KIND_Q), (B, T, H, 576))
    kv = synth.normal_bf16(key(synth.KIND_KV), (B, N, 576))
    r = np.random.default_rng(seed)
    idx = np.stack([np.stack([np.sort(r.choice(N, size=k, replace=False)) for _ in range(T)]) for _ in range(B)])
    return q, kv, idx.astype(np.int32)


@pytest.mark.parametrize("B,N,H,k,lo,hi", [(2, 3000, 64, 2048, 1000, 2200), (3, 1200, 16, 300, 0, 600),
                                          (1, 5000, 64, 2048, 4000, 5000), (2, 900, 32, 64, 850, 900)])
def test_attn_shard_matches_oracle(dsa, orc, B, N, H, k, lo, hi):
    """Attention over the selected rows of the shard [lo, hi): output and log-sum-exp."""
    q, kv, idx = _attn_case(600 + N + lo, B, 1, N, H, k)
    idx[0, 0, :5] = -1                                  # padding is skipped too
    shard = np.ascontiguousarray(kv[:, lo:hi])
    out, lse = dsa.dsa_sparse_attn_shard(dev_bf16(q), dev_bf16(shard), dev(idx), lo, C.SCALE)
    rout, rlse = orc.sparse_attn_partial(q, shard, idx, lo, C.SCALE)
    assert_close(host(out), rout, "shard attention")
    got = host(lse).astype(np.float64)
    fin = np.isfinite(rlse)
    assert np.array_equal(np.isfinite(got), fin)
    assert np.all(np.abs(got[fin] - rlse[fin]) <= 1e-4 * np.maximum(1.0, np.abs(rlse[fin])))


def test_shard_candidates(dsa):
    r = np.random.default_rng(3)
    B, T, N, k, offset = 2, 1, 500, 64, 12345
    scores = r.standard_normal((B, T, N)).astype(np.float32)
    idx = np.sort(r.choice(N, size=(B, T, k)), axis=2).astype(np.int32)
    idx[1, 0, -7:] = -1
    cs, cp = dsa.dsa_shard_candidates(dev(scores), dev(idx), offset)
    v = idx >= 0
    want_s = np.where(v, np.take_along_axis(scores, np.maximum(idx, 0), axis=2), -np.inf).astype(np.float32)
    assert np.array_equal(host(cs), want_s)
    assert np.array_equal(host(cp), np.where(v, idx + offset, -1))


@pytest.mark.parametrize("W,kc,k", [(3, 64, 100), (8, 2048, 2048), (2, 40, 128), (5, 300, 7)])
def test_merge_candidates_matches_oracle(dsa, orc, W, kc, k):
    """Candidates of W shards (ascending positions per shard, shards in order, heavy ties,
    padding) merged into the k best, against the oracle."""
    r = np.random.default_rng(W * 1000 + kc)
    B, T = 3, 1
    span = 4 * kc
    cs = (r.integers(-30, 31, size=(W, B, T, kc)) / 8).astype(np.float32)
    cp = np.empty((W, B, T, kc), np.int32)
    for w in range(W):
        for b in range(B):
            cp[w, b, 0] = np.sort(r.choice(span, size=kc, replace=False)) + w * span
    cp[1 % W, 0, 0, kc // 2:] = -1                     # a shard with fewer candidates
    cs[0, 2, 0, :3] = np.nan
    got = host(dsa.dsa_merge_candidates(dev(cs), dev(cp), k))
    want = orc.merge_candidates(np.moveaxis(cs, 0, 2).reshape(B, T, W * kc),
                                np.moveaxis(cp, 0, 2).reshape(B, T, W * kc), k)
    assert np.array_equal(got, want)


def test_merge_partials_matches_oracle(dsa, orc):
    r = np.random.default_rng(9)
    W, B, T, H = 4, 2, 1, 64
    outs = r.standard_normal((W, B, T, H, 512)).astype(np.float32)
    lses = (r.standard_normal((W, B, T, H)) * 5).astype(np.float32)
    lses[2, 0, 0, :10] = -np.inf                       # a shard without rows for some heads
    lses[:, 1, 0, 3] = -np.inf                         # a head no shard selects
    got = host(dsa.dsa_merge_partials(dev(outs), dev(lses)))
    want = orc.merge_partials(outs.astype(np.float64), lses.astype(np.float64))
    assert_close(got, want, "merged partials")
    assert np.all(got[1, 0, 3] == 0)


@pytest.mark.parametrize("W", [2, 3])
def test_sharded_group_matches_unsharded_oracle(dsa, orc, W):
    """The sharded group's kernels, W shards in one process: the index list equals the
    unsharded oracle's bit for bit, the outputs within the tolerance."""
    import torch
    from sparse_long_context_score_b200 import sharded
    w = C.scaled(C.WORKLOADS["decode1m"], B=2, N=9000, q_pos0=8999, groups=1)
    iq, wt, ik, qs, kvs = C.host_group_inputs(w)
    ridx, routs = orc.group_forward(iq, wt, ik, qs, kvs, w.q_pos0, w.k, C.SCALE)
    ops = sharded.cuda_ops()
    bounds = sharded.shard_bounds(w.N, W)
    cands = [sharded.local_candidates(ops, dev_bf16(iq), dev(wt), dev_bf16(np.ascontiguousarray(ik[:, o:o + n])),
                                      w.q_pos0, o, w.k) for o, n in bounds]
    idx = ops.merge_candidates(torch.stack([c[0] for c in cands]), torch.stack([c[1] for c in cands]), w.k)
    assert np.array_equal(host(idx), ridx)
    for l in range(w.L):
        parts = [ops.attn_shard(dev_bf16(qs[l]), dev_bf16(np.ascontiguousarray(kvs[l][:, o:o + n])), idx, o, C.SCALE)
                 for o, n in bounds]
        out = ops.merge_partials(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))
        assert_close(host(out), routs[l], f"sharded layer {l}")
    torch.cuda.synchronize()
    assert dsa.dsa_check_device_status() == 0
