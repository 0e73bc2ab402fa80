"""Parity of the indexer over an FP8 (E4M3) index-key cache against the CPU oracle.

On the workload's integer inputs (the same integers as the bf16 indexer, as E4M3 bytes)
every product and partial sum is an integer below 2^14, exact in any f32 accumulation
order, so the scores must match the oracle bit for bit and the decode step's index lists
must equal the oracle's.  On arbitrary finite E4M3 bytes the products are still exact but
the f32 sums round; there the bound is relative to the score of |q| and |k|."""
import numpy as np
import pytest

import synth
from gpu_util import assert_close, dev, host
from synth import configs as C

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import sparse_long_context_score_b200 as m
    from sparse_long_context_score_b200 import build
    build.build()
    m.lib()
    return m


def _inputs(seed, B, T, N):
    key = lambda kind: synth.stream_key(seed, synth.tensor_id(kind))
    q = synth.int17_e4m3(key(synth.KIND_IQ), (B, T, 32, 128))
    w = synth.pow2_f32(key(synth.KIND_W), (B, T, 32))
    k = synth.int17_e4m3(key(synth.KIND_IK), (B, N, 128))
    return q, w, k


def _visible(B, T, N, q_pos0):
    t = np.arange(T)[:, None]
    s = np.arange(N)[None, :]
    return np.broadcast_to(s <= q_pos0 + t, (B, T, N))


@pytest.mark.parametrize("B,T,N,q_pos0", [
    (1, 1, 4096, 4095),      # tiny decode
    (3, 1, 5000, 4999),      # several sequences, ragged last key tile
    (2, 1, 300, 150),        # part of the cache not yet visible
    (1, 20, 3000, 2980),     # prefill: three 8-query groups, the last one ragged
    (2, 9, 129, 120),        # one key past a tile, causal cut inside it
    (1, 1, 1, 0),            # a single cached token
])
def test_index_score_e4m3_exact(dsa, orc, B, T, N, q_pos0):
    q, w, k = _inputs(5100 + N + T, B, T, N)
    got = host(dsa.dsa_index_score_e4m3(dev(q), dev(w), dev(k), q_pos0))
    ref = orc.index_score_e4m3(q, w, k, q_pos0)
    vis = _visible(B, T, N, q_pos0)
    assert np.array_equal(got[vis].astype(np.float64), ref[vis])


def test_index_score_e4m3_matches_bf16_on_integers(dsa):
    """The same integers as bf16 and as E4M3 give the same f32 scores."""
    B, T, N = 2, 1, 7000
    key = lambda kind: synth.stream_key(77, synth.tensor_id(kind))
    q8 = synth.int17_e4m3(key(synth.KIND_IQ), (B, T, 32, 128))
    k8 = synth.int17_e4m3(key(synth.KIND_IK), (B, N, 128))
    qb = synth.int17_bf16(key(synth.KIND_IQ), (B, T, 32, 128))
    kb = synth.int17_bf16(key(synth.KIND_IK), (B, N, 128))
    w = synth.pow2_f32(key(synth.KIND_W), (B, T, 32))
    from gpu_util import dev_bf16
    a = host(dsa.dsa_index_score_e4m3(dev(q8), dev(w), dev(k8), N - 1))
    b = host(dsa.dsa_index_score(dev_bf16(qb), dev(w), dev_bf16(kb), N - 1))
    assert np.array_equal(a, b)


def test_index_score_e4m3_arbitrary_bytes(dsa, orc):
    """Every finite E4M3 byte (subnormals included) in q and k."""
    rng = np.random.default_rng(5)
    B, T, N = 2, 3, 1500
    finite = np.array([b for b in range(256) if (b & 0x7F) != 0x7F], np.uint8)
    q = rng.choice(finite, size=(B, T, 32, 128)).astype(np.uint8)
    k = rng.choice(finite, size=(B, N, 128)).astype(np.uint8)
    w = synth.pow2_f32(synth.stream_key(78, synth.tensor_id(synth.KIND_W)), (B, T, 32))
    q_pos0 = N - T
    got = host(dsa.dsa_index_score_e4m3(dev(q), dev(w), dev(k), q_pos0))
    ref = orc.index_score_e4m3(q, w, k, q_pos0)
    mag = orc.index_score_e4m3(q & 0x7F, w, k & 0x7F, q_pos0)   # sum_h w_h sum_d |q_d k_d|
    vis = _visible(B, T, N, q_pos0)
    # each score is a sum of at most 32 x 128 exact products: f32 summation in any order
    # errs by less than 4096 * 2^-24 of the sum of their magnitudes
    err = np.abs(got[vis].astype(np.float64) - ref[vis])
    assert np.all(err <= 4096 * 2.0 ** -24 * mag[vis] + 1e-30)


@pytest.mark.parametrize("B,G", [(3, 2), (2, 1)])
def test_decode_step_e4m3_matches_oracle(dsa, orc, B, G):
    """dsa_decode_step with an E4M3 index-key cache: the oracle's index list (E4M3 scores,
    then the select) bit for bit, attention within the tolerance."""
    import torch
    from gpu_util import dev_bf16
    w = C.scaled(C.WORKLOADS["decode1m"], B=B, N=9000, q_pos0=8999, groups=G)
    groups, ref = [], []
    for g in range(G):
        _, wt, _, qs, kvs = C.host_group_inputs(w, g)
        iq = synth.int17_e4m3(w.key(synth.KIND_IQ, g, 0, 0), (w.B, 1, 32, 128))
        ik = synth.int17_e4m3(w.key(synth.KIND_IK, g), (w.B, w.N, 128))
        ridx = orc.topk(orc.index_score_e4m3(iq, wt, ik, w.q_pos0), w.q_pos0, w.k)
        routs = [orc.sparse_attn(qs[l], kvs[l], ridx, C.SCALE) for l in range(w.L)]
        ref.append((ridx, routs))
        groups.append(dict(iq=dev(iq), w=dev(wt), ik=dev(ik), qs=[dev_bf16(x) for x in qs],
                           kvs=[dev_bf16(x) for x in kvs],
                           idx=torch.empty(B, 1, w.k, dtype=torch.int32, device="cuda"),
                           outs=[torch.empty(B, 1, w.H, 512, dtype=torch.float32, device="cuda") for _ in range(w.L)]))
    dsa.dsa_decode_step(groups, w.k, C.SCALE)
    torch.cuda.synchronize()
    assert dsa.dsa_check_device_status() == 0
    for g in range(G):
        ridx, routs = ref[g]
        assert np.array_equal(host(groups[g]["idx"]), ridx), f"group {g}"
        for l in range(w.L):
            assert_close(host(groups[g]["outs"][l]), routs[l], f"group {g} layer {l}")
