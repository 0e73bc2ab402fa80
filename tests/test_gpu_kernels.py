"""Parity of each C-ABI step against the CPU oracle on the same seeded inputs.

Indexer scores and top-k indices must match bit-exactly on the workloads' integer-valued
inputs; attention outputs within max|d| <= 2e-3 * max|ref| + 1e-3."""
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


def _indexer_inputs(seed, B, T, N, kind="int"):
    key = lambda kd: synth.stream_key(seed, synth.tensor_id(kd))
    if kind == "int":
        q = synth.int17_bf16(key(synth.KIND_IQ), (B, T, 32, 128))
        k = synth.int17_bf16(key(synth.KIND_IK), (B, N, 128))
        w = synth.pow2_f32(key(synth.KIND_W), (B, T, 32))
    else:
        q = synth.normal_bf16(key(synth.KIND_IQ), (B, T, 32, 128))
        k = synth.normal_bf16(key(synth.KIND_IK), (B, N, 128))
        w = synth.unit_f32(key(synth.KIND_W), (B, T, 32)) + np.float32(0.5)
    return q, w, k


@pytest.mark.parametrize("B,T,N,q_pos0", [(1, 1, 4096, 4095), (3, 1, 4099, 4098), (2, 1, 1, 0), (1, 1, 17, 16),
                                         (2, 1, 300, 100), (1, 37, 530, 493), (2, 5, 1000, 10)])
def test_index_score_exact(dsa, orc, B, T, N, q_pos0):
    q, w, k = _indexer_inputs(100 + N + T, B, T, N)
    got = host(dsa.dsa_index_score(dev_bf16(q), dev(w), dev_bf16(k), q_pos0))
    ref = orc.index_score(q, w, k, q_pos0)
    for t in range(T):
        vis = min(N, q_pos0 + t + 1)
        assert np.array_equal(got[:, t, :vis].astype(np.float64), ref[:, t, :vis]), (t, vis)


def test_index_score_general_values(dsa, orc):
    q, w, k = _indexer_inputs(7, 2, 3, 2000, kind="normal")
    got = host(dsa.dsa_index_score(dev_bf16(q), dev(w), dev_bf16(k), 1999))
    ref = orc.index_score(q, w, k, 1999)
    assert np.allclose(got, ref, rtol=1e-5, atol=1e-4)


def _score_rows(seed, B, T, N, levels):
    key = synth.stream_key(seed, synth.tensor_id(synth.KIND_SCORES))
    u = synth.unit_f32(key, (B, T, N)).astype(np.float64) + 0.5
    return (np.floor(u * levels) / 64.0).astype(np.float32)


@pytest.mark.parametrize("B,T,N,q_pos0,k,levels", [
    (1, 1, 4096, 4095, 256, 1 << 20), (2, 1, 4096, 4095, 256, 50), (3, 1, 10000, 9999, 2048, 1 << 16),
    (2, 1, 70000, 69999, 2048, 3000), (1, 1, 200, 199, 2048, 10), (1, 1, 1, 0, 1, 5), (2, 1, 8193, 8192, 7, 100),
    (1, 1, 33000, 32999, 1, 1 << 22), (1, 9, 3000, 2990, 2048, 1000), (1, 4, 20000, 2040, 2048, 1 << 20),
    (1, 1, 50000, 49999, 2048, 1),
    # one cluster of 8 CTAs with 32 keys per thread; equal keys down to the index digits
    (1, 1, 200000, 199999, 2048, 1 << 18), (2, 1, 150000, 149999, 2048, 3),
    # decode128k rows: one cluster of 8 CTAs per row (merge path; heavy ties: digit path)
    (8, 1, 131072, 131071, 2048, 1 << 20), (8, 1, 131072, 131071, 2048, 5),
    # shapes for the scan kernels: more rows than one wave of clusters, rows too long
    (1, 160, 3000, 2900, 256, 1000), (1, 1, 300000, 299999, 2048, 1 << 20), (1, 1, 300000, 299999, 2048, 7),
])
def test_topk_exact(dsa, orc, B, T, N, q_pos0, k, levels):
    sc = _score_rows(N + k + levels, B, T, N, levels)
    got = host(dsa.dsa_topk(dev(sc), q_pos0, k))
    ref = orc.topk(sc, q_pos0, k)
    assert np.array_equal(got, ref)


def test_topk_special_values(dsa, orc):
    N, k = 9000, 300
    sc = _score_rows(5, 1, 3, N, 1000)
    sc[0, 0, ::7] = -0.0
    sc[0, 0, 1::7] = 0.0
    sc[0, 1, ::5] = np.nan
    sc[0, 1, 3::11] = np.inf
    sc[0, 2, :] = -sc[0, 2, :]
    sc[0, 2, 17] = -np.inf
    got = host(dsa.dsa_topk(dev(sc), N - 1, k))
    assert np.array_equal(got, orc.topk(sc, N - 1, k))
    allzero = np.zeros((1, 1, N), np.float32)
    allzero[0, 0, ::2] = -0.0
    assert np.array_equal(host(dsa.dsa_topk(dev(allzero), N - 1, k)), orc.topk(allzero, N - 1, k))


def test_topk_candidate_overflow_path(dsa, orc):
    # the scan kernels (20 rows of 300000: too long for a cluster, too many chunks for one
    # cooperative launch), with more than 8192 elements in the threshold bin: resolved
    # from the row itself
    B, N, k = 20, 300000, 2048
    sc = np.full((B, 1, N), 1.5, np.float32)
    for b in range(1, B):
        sc[b, 0, 100 * b::2 + b % 3] = 1.75 + 0.25 * (b % 2)
    got = host(dsa.dsa_topk(dev(sc), N - 1, k))
    assert np.array_equal(got, orc.topk(sc, N - 1, k))


def _attn_case(seed, B, T, N, H, k, invalid_frac=0.0):
    key = lambda kd: synth.stream_key(seed, synth.tensor_id(kd))
    q = synth.normal_bf16(key(synth.KIND_Q), (B, T, H, 576))
    kv = synth.normal_bf16(key(synth.KIND_KV), (B, N, 576))
    r = np.random.default_rng(seed)
    idx = np.stack([np.stack([np.sort(r.choice(N, size=k, replace=False)) for _ in range(T)]) for _ in range(B)])
    idx = idx.astype(np.int32)
    if invalid_frac:
        idx[r.random(idx.shape) < invalid_frac] = -1
    return q, kv, idx


@pytest.mark.parametrize("B,T,N,H,k,inv", [(1, 1, 4096, 16, 256, 0.0), (2, 1, 5000, 64, 2048, 0.0),
                                          (1, 3, 3000, 64, 33, 0.1), (3, 1, 700, 32, 1, 0.0),
                                          (1, 2, 900, 48, 100, 0.5), (2, 2, 2500, 64, 2048, 0.02)])
def test_sparse_attn(dsa, orc, B, T, N, H, k, inv):
    q, kv, idx = _attn_case(B * 1000 + k + H, B, T, N, H, k, inv)
    got = host(dsa.dsa_sparse_attn(dev_bf16(q), dev_bf16(kv), dev(idx), C.SCALE))
    ref = orc.sparse_attn(q, kv, idx, C.SCALE)
    assert_close(got, ref, "sparse attention")


@pytest.mark.parametrize("rows", [21, 24, 29, 37])
def test_sparse_attn_uneven_splits(dsa, orc, rows):
    """Row counts whose key splits (148 SMs: 7, 6, 5 or 4 CTAs per row) cut the [H][512]
    output into slices of unequal length, so the split reduction's received slices do not
    tile the block exactly."""
    N, H, k = 3000, 64, 2048
    q, kv, idx = _attn_case(9000 + rows, rows, 1, N, H, k, 0.01)
    got = host(dsa.dsa_sparse_attn(dev_bf16(q), dev_bf16(kv), dev(idx), C.SCALE))
    ref = orc.sparse_attn(q, kv, idx, C.SCALE)
    assert_close(got, ref, f"sparse attention, {rows} rows")


def test_sparse_attn_empty_rows_are_zero(dsa):
    q, kv, idx = _attn_case(3, 1, 2, 100, 16, 40)
    idx[0, 1, :] = -1
    got = host(dsa.dsa_sparse_attn(dev_bf16(q), dev_bf16(kv), dev(idx), C.SCALE))
    assert np.all(got[0, 1] == 0)
