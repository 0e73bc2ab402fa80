"""Pins for the CPU oracle: checks against facts fixed by the pages and by mathematics.

Each pin takes an ``oracle.Oracle`` and raises AssertionError when the oracle disagrees
with something other than itself: the hand-worked golden example, a closed form, a
special case that reduces to a library routine (numpy matmul / lexsort, torch's
scaled-dot-product attention), or an invariant.  They are chosen so that a plausible
mistake anywhere in the oracle (a dropped term, a wrong sign or index, a transposed
operand, an off-by-one in the mask) fails at least one of them; the planted-mistake test
checks exactly that.
"""
from __future__ import annotations

import math
import os

import numpy as np

import synth
from synth import configs as C

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def bf(x) -> np.ndarray:
    """float values that are exact in bf16 -> bf16 bit patterns."""
    x = np.asarray(x, dtype=np.float32)
    bits = synth.f32_to_bf16_bits(x)
    assert np.array_equal(synth.bf16_bits_to_f32(bits), x), "value not exact in bf16"
    return bits


def f(bits) -> np.ndarray:
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def load_golden(name: str) -> dict:
    out = {}
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, *vals = line.split()
            out[key] = vals
    return out


def _rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


# ----------------------------------------------------------------------------- indexer

def pin_indexer_golden(o):
    g = load_golden("indexer_worked_example.txt")
    nh, hd = int(g["heads"][0]), int(g["head_dim"][0])
    q = bf(np.array(g["q"], dtype=np.float32).reshape(1, 1, nh, hd))
    w = np.array(g["w"], dtype=np.float32).reshape(1, 1, nh)
    keys = [g[f"k{i}"] for i in range(4)]
    k = bf(np.array(keys, dtype=np.float32).reshape(1, 4, hd))
    q_pos0 = int(g["q_pos0"][0])
    s = o.index_score(q, w, k, q_pos0)
    want = np.array([float(x) for x in g["score"]])
    assert np.array_equal(s[0, 0], want), (s[0, 0], want)
    sf = s.astype(np.float32)
    assert o.topk(sf, q_pos0, 2)[0, 0].tolist() == [int(x) for x in g["top2"]]
    assert o.topk(sf, q_pos0, 5)[0, 0].tolist() == [int(x) for x in g["top5"]]


def pin_indexer_nonnegative_is_matmul(o):
    """With q >= 0 and k >= 0 no dot product is negative, ReLU is the identity, and
    I(t,s) = (sum_h w[t,h] q[t,h]) . k[s]: one matrix product."""
    r = _rng(1)
    B, T, nh, hd, N = 2, 3, 5, 16, 40
    qv = r.integers(0, 9, size=(B, T, nh, hd)).astype(np.float32)
    kv = r.integers(0, 9, size=(B, N, hd)).astype(np.float32)
    w = np.ldexp(1.0, -r.integers(1, 7, size=(B, T, nh))).astype(np.float32)
    s = o.index_score(bf(qv), w, bf(kv), q_pos0=N - 1)
    qsum = np.einsum("bth,bthd->btd", w.astype(np.float64), qv.astype(np.float64))
    want = np.matmul(qsum, np.swapaxes(kv.astype(np.float64), 1, 2))
    assert np.array_equal(s, want)


def pin_indexer_relu_zero(o):
    """q >= 0 and k <= 0: every dot product is <= 0, so every visible score is 0."""
    r = _rng(2)
    qv = r.integers(0, 9, size=(1, 2, 4, 8)).astype(np.float32)
    kv = -r.integers(0, 9, size=(1, 30, 8)).astype(np.float32)
    w = np.full((1, 2, 4), 0.5, dtype=np.float32)
    s = o.index_score(bf(qv), w, bf(kv), q_pos0=29)
    assert np.array_equal(s[0, 0], np.zeros(30))


def pin_indexer_one_hot(o):
    """q[t,h] = a_h e_{i_h}, k[s] = b_s e_{j_s}: I(t,s) = sum_h w_h max(0, a_h b_s)[i_h = j_s]."""
    r = _rng(3)
    nh, hd, N = 6, 8, 25
    a = r.integers(-8, 9, size=nh)
    ih = r.integers(0, hd, size=nh)
    bs = r.integers(-8, 9, size=N)
    js = r.integers(0, hd, size=N)
    qv = np.zeros((1, 1, nh, hd), np.float32)
    qv[0, 0, np.arange(nh), ih] = a
    kv = np.zeros((1, N, hd), np.float32)
    kv[0, np.arange(N), js] = bs
    w = np.ldexp(1.0, -r.integers(1, 7, size=(1, 1, nh))).astype(np.float32)
    s = o.index_score(bf(qv), w, bf(kv), q_pos0=N - 1)
    for sidx in range(N):
        want = sum(float(w[0, 0, h]) * max(0, int(a[h]) * int(bs[sidx])) * (ih[h] == js[sidx])
                   for h in range(nh))
        assert s[0, 0, sidx] == want, (sidx, s[0, 0, sidx], want)


def pin_indexer_causal(o):
    """Query t sees exactly the positions s <= q_pos0 + t (and s < N)."""
    r = _rng(4)
    B, T, nh, hd, N, q_pos0 = 1, 5, 2, 8, 12, 6
    qv = r.integers(-8, 9, size=(B, T, nh, hd)).astype(np.float32)
    kv = r.integers(-8, 9, size=(B, N, hd)).astype(np.float32)
    w = np.full((B, T, nh), 0.25, np.float32)
    s = o.index_score(bf(qv), w, bf(kv), q_pos0)
    for t in range(T):
        vis = min(N, q_pos0 + t + 1)
        assert np.all(np.isfinite(s[0, t, :vis])) and np.all(s[0, t, vis:] == -np.inf), t
    full = o.index_score(bf(qv), w, bf(kv), q_pos0=N - 1)
    for t in range(T):
        vis = min(N, q_pos0 + t + 1)
        assert np.array_equal(s[0, t, :vis], full[0, t, :vis])


def pin_indexer_head_and_weight_structure(o):
    """Permuting heads (with their weights) changes nothing; doubling w doubles I;
    swapping batch items swaps the score rows."""
    r = _rng(5)
    B, T, nh, hd, N = 2, 2, 6, 16, 50
    qv = r.integers(-8, 9, size=(B, T, nh, hd)).astype(np.float32)
    kv = r.integers(-8, 9, size=(B, N, hd)).astype(np.float32)
    w = np.ldexp(1.0, -r.integers(1, 7, size=(B, T, nh))).astype(np.float32)
    base = o.index_score(bf(qv), w, bf(kv), N - 1)
    perm = r.permutation(nh)
    assert np.array_equal(o.index_score(bf(qv[:, :, perm]), w[:, :, perm], bf(kv), N - 1), base)
    assert np.array_equal(o.index_score(bf(qv), 2 * w, bf(kv), N - 1), 2 * base)
    sw = o.index_score(bf(qv[::-1].copy()), w[::-1].copy(), bf(kv[::-1].copy()), N - 1)
    assert np.array_equal(sw, base[::-1])


def pin_indexer_exact_on_workload_inputs(o):
    """On the workloads' inputs (integers in [-8,8], w in {2^-1..2^-6}) every score is a
    multiple of 2^-6 below 2^17, so it is exact in float32 (24-bit significand)."""
    w = C.scaled(C.WORKLOADS["tiny"], N=300, q_pos0=299)
    iq, wt, ik, _, _ = C.host_group_inputs(w, with_attention=False)
    s = o.index_score(iq, wt, ik, w.q_pos0)
    m = s * 64.0
    assert np.array_equal(m, np.round(m)) and np.all(s >= 0) and np.all(s < 2 ** 17)
    assert np.array_equal(s.astype(np.float32).astype(np.float64), s)


# ----------------------------------------------------------------------------- top-k

def _lexsort_topk(row: np.ndarray, vis: int, k: int) -> list:
    """Library reference: numpy lexsort by (score descending, index ascending)."""
    sc = row[:vis].astype(np.float64)
    key = np.where(np.isnan(sc), -np.inf, sc)
    nanrank = np.isnan(sc).astype(np.int64)          # numbers before NaN
    order = np.lexsort((np.arange(vis), -key, nanrank))
    take = sorted(order[:k].tolist())
    return take + [-1] * (k - len(take))


def pin_topk_matches_lexsort(o):
    r = _rng(6)
    for N, k, spread in [(1, 1, 5), (7, 3, 3), (100, 10, 1000), (257, 64, 4), (1000, 999, 50),
                         (1000, 1000, 50), (1000, 1500, 50), (4096, 256, 7)]:
        sc = (r.integers(0, spread, size=(2, 3, N)) * 0.015625).astype(np.float32)
        idx = o.topk(sc, N - 1, k)
        for b in range(2):
            for t in range(3):
                assert idx[b, t].tolist() == _lexsort_topk(sc[b, t], N, k), (N, k, b, t)


def pin_topk_ties(o):
    N, k = 500, 37
    sc = np.full((1, 1, N), 3.5, np.float32)
    assert o.topk(sc, N - 1, k)[0, 0].tolist() == list(range(k))
    # two-valued row: every 1.0 is taken before any 0.0; among equals the lower index
    r = _rng(7)
    row = (r.random(N) < 0.05).astype(np.float32)
    ones = np.flatnonzero(row == 1.0).tolist()
    zeros = np.flatnonzero(row == 0.0).tolist()
    want = ones[:k] if len(ones) >= k else ones + zeros[: k - len(ones)]
    assert o.topk(row[None, None], N - 1, k)[0, 0].tolist() == sorted(want)
    # -0 and +0 are equal scores: the lower index wins
    row = np.array([-0.0, 0.0, -0.0, 0.0, -1.0], np.float32)
    assert o.topk(row[None, None], 4, 2)[0, 0].tolist() == [0, 1]
    # a NaN ranks below every number
    row = np.array([np.nan, -5.0, np.nan, 2.0], np.float32)
    assert o.topk(row[None, None], 3, 3)[0, 0].tolist() == [0, 1, 3]


def pin_topk_causal_and_padding(o):
    r = _rng(8)
    T, N, q_pos0, k = 6, 40, 20, 24
    sc = r.random((1, T, N)).astype(np.float32)
    idx = o.topk(sc, q_pos0, k)
    for t in range(T):
        vis = min(N, q_pos0 + t + 1)
        row = idx[0, t]
        valid = row[row >= 0]
        assert len(valid) == min(k, vis) and np.all(row[len(valid):] == -1)
        assert np.all(valid <= q_pos0 + t) and np.all(np.diff(valid) > 0)
        if vis <= k:
            assert valid.tolist() == list(range(vis))
        assert row.tolist() == _lexsort_topk(sc[0, t], vis, k)


def pin_topk_selection_invariant(o):
    """Every selected score >= every unselected visible score; equal scores split by index."""
    r = _rng(9)
    N, k = 3000, 200
    sc = (r.integers(0, 300, size=(4, 1, N)) * 0.5).astype(np.float32)
    idx = o.topk(sc, N - 1, k)
    for b in range(4):
        sel = idx[b, 0]
        mask = np.zeros(N, bool)
        mask[sel] = True
        lo = sc[b, 0][mask].min()
        assert sc[b, 0][~mask].max() <= lo
        tied_out = np.flatnonzero((~mask) & (sc[b, 0] == lo))
        tied_in = np.flatnonzero(mask & (sc[b, 0] == lo))
        if len(tied_out):
            assert tied_in.max() < tied_out.min()


# ----------------------------------------------------------------------------- attention

def _attn_inputs(seed, B=1, T=2, H=3, N=60, k=20, dqk=576):
    r = _rng(seed)
    q = bf((r.integers(-64, 65, size=(B, T, H, dqk)) / 64.0).astype(np.float32))
    kv = bf((r.integers(-64, 65, size=(B, N, dqk)) / 64.0).astype(np.float32))
    idx = np.stack([np.stack([np.sort(r.choice(N, size=k, replace=False)) for _ in range(T)])
                    for _ in range(B)]).astype(np.int32)
    return q, kv, idx


def pin_attn_single_row(o):
    """One valid index: the softmax weight is 1 and the output is that row's value part."""
    q, kv, _ = _attn_inputs(10)
    idx = np.full((1, 2, 5), -1, np.int32)
    idx[0, 0, 3] = 17
    idx[0, 1, 0] = 42
    out = o.sparse_attn(q, kv, idx, C.SCALE)
    for t, row in ((0, 17), (1, 42)):
        for h in range(3):
            assert np.array_equal(out[0, t, h], f(kv[0, row, :512]))


def pin_attn_uniform_logits(o):
    """q = 0: all logits equal, the output is the plain mean of the selected value rows."""
    q, kv, idx = _attn_inputs(11)
    q[:] = 0
    out = o.sparse_attn(q, kv, idx, C.SCALE)
    for t in range(2):
        want = f(kv[0, idx[0, t], :512]).mean(axis=0)
        for h in range(3):
            assert np.allclose(out[0, t, h], want, rtol=0, atol=1e-13)


def pin_attn_matches_torch_sdpa(o):
    """The selected-row attention equals torch's scaled_dot_product_attention (float64)
    over the gathered rows, with the value = the first 512 columns."""
    import torch
    q, kv, idx = _attn_inputs(12, B=2, T=2, H=4, N=80, k=33)
    out = o.sparse_attn(q, kv, idx, C.SCALE)
    for b in range(2):
        for t in range(2):
            rows = torch.from_numpy(f(kv[b, idx[b, t]]))            # [k, 576]
            qq = torch.from_numpy(f(q[b, t]))                        # [H, 576]
            ref = torch.nn.functional.scaled_dot_product_attention(
                qq[None], rows[None], rows[None, :, :512], scale=C.SCALE)[0]
            assert np.allclose(out[b, t], ref.numpy(), rtol=1e-12, atol=1e-13)


def pin_attn_dense_masked(o):
    """Sparse attention == dense softmax over all N positions with -inf outside the set."""
    q, kv, idx = _attn_inputs(13, B=2, T=3, H=2, N=90, k=31)
    idx[1, 2, 5:9] = -1
    a = o.sparse_attn(q, kv, idx, C.SCALE)
    d = o.sparse_attn(q, kv, idx, C.SCALE, dense_masked=True)
    assert np.allclose(a, d, rtol=1e-12, atol=1e-13)


def pin_attn_order_and_padding_invariance(o):
    q, kv, idx = _attn_inputs(14)
    base = o.sparse_attn(q, kv, idx, C.SCALE)
    r = _rng(15)
    shuffled = idx.copy()
    for t in range(2):
        shuffled[0, t] = r.permutation(shuffled[0, t])
    assert np.allclose(o.sparse_attn(q, kv, shuffled, C.SCALE), base, rtol=1e-12, atol=1e-13)
    padded = np.concatenate([idx, np.full((1, 2, 7), -1, np.int32)], axis=2)
    assert np.allclose(o.sparse_attn(q, kv, padded, C.SCALE), base, rtol=1e-12, atol=1e-13)
    # the output is a convex combination of the selected value rows
    for t in range(2):
        vals = f(kv[0, idx[0, t], :512])
        assert np.all(base[0, t] <= vals.max(0) + 1e-12) and np.all(base[0, t] >= vals.min(0) - 1e-12)


def pin_attn_empty_selection_is_zero(o):
    q, kv, _ = _attn_inputs(16)
    idx = np.full((1, 2, 4), -1, np.int32)
    assert np.array_equal(o.sparse_attn(q, kv, idx, C.SCALE), np.zeros((1, 2, 3, 512)))


# ----------------------------------------------------------------------------- group

def pin_group_shares_one_index_list(o):
    """Indexer + top-k once, then every layer attends over the same, unchanged list."""
    w = C.scaled(C.WORKLOADS["tiny"], N=200, q_pos0=199, k=32, H=2, L=4)
    iq, wt, ik, qs, kvs = C.host_group_inputs(w)
    idx, outs = o.group_forward(iq, wt, ik, qs, kvs, w.q_pos0, w.k, C.SCALE)
    sc = o.index_score(iq, wt, ik, w.q_pos0).astype(np.float32)
    assert np.array_equal(idx, o.topk(sc, w.q_pos0, w.k))
    for l in range(4):
        assert np.array_equal(outs[l], o.sparse_attn(qs[l], kvs[l], idx, C.SCALE))
    # reuse: with compute_indices off the caller's list is used unchanged
    mine = np.sort(_rng(17).choice(w.N, size=(1, 1, w.k), replace=False), axis=-1).astype(np.int32)
    idx2, outs2 = o.group_forward(iq, wt, ik, qs, kvs, w.q_pos0, w.k, C.SCALE,
                                  compute_indices=False, idx_shared=mine.copy())
    assert np.array_equal(idx2, mine)
    assert np.array_equal(outs2[2], o.sparse_attn(qs[2], kvs[2], mine, C.SCALE))


def pin_mtp_draft_rows_never_attended(o):
    """MTP reuse: the step-1 query sits at the last target position, so the draft rows
    appended after it are never selected, and steps 2.. reuse that list: changing the
    draft rows changes no output."""
    w = C.scaled(C.WORKLOADS["mtp"], B=2, N=150 + 3, q_pos0=149, k=40, H=2, L=1, steps=3)
    iq, wt, ik, _, kvs = C.host_group_inputs(w)
    kv = kvs[0].copy()
    idx = None
    outs_a, outs_b = [], []
    kv_b = kv.copy()
    kv_b[:, 150:, :] = bf(np.full((2, 3, 576), 8.0, np.float32))  # loud draft rows
    ik_b = ik.copy()
    ik_b[:, 150:, :] = bf(np.full((2, 3, 128), 8.0, np.float32))
    for step in range(w.steps):
        q = synth.normal_bf16(w.key(synth.KIND_Q, 0, 0, step), (w.B, 1, w.H, 576))
        ia, oa = o.group_forward(iq, wt, ik, [q], [kv], w.q_pos0, w.k, C.SCALE,
                                 compute_indices=(step == 0), idx_shared=idx)
        ib, ob = o.group_forward(iq, wt, ik_b, [q], [kv_b], w.q_pos0, w.k, C.SCALE,
                                 compute_indices=(step == 0), idx_shared=None if step == 0 else idx)
        if step == 0:
            idx = ia.copy()
        assert np.array_equal(ia, idx) and np.array_equal(ib, idx)
        assert np.all(idx < 150)
        assert np.array_equal(oa[0], ob[0])


# ------------------------------------------------------------------ MTP verify step
# "GLM-5.2 MTP IndexShare inference", Rejection Sampling: the acceptance rate is the sum
# over the vocabulary of the smaller of the two probabilities.  The accept / resample rule
# read from it is the standard speculative-sampling rule; its defining property is that
# the token it emits is distributed as the target distribution p.

def _dist(seed, V, rows, temp=1.0):
    """rows float32 probability vectors of length V (softmax of Gaussian logits, f32)."""
    r = _rng(seed)
    z = (r.standard_normal((rows, V)) * temp).astype(np.float32)
    e = np.exp(z - z.max(axis=1, keepdims=True), dtype=np.float32)
    return (e / e.sum(axis=1, keepdims=True, dtype=np.float32)).astype(np.float32)


def pin_verify_identical_distributions(o):
    """p == q: the acceptance rate is 1 and every draft token is kept."""
    p = _dist(5, 300, 6).reshape(2, 3, 300)
    draft = np.array([[3, 77, 299], [0, 150, 12]], np.int32)
    u = np.full((2, 3), 0.999, np.float32)
    a, acc, tok, alen = o.verify(p, p, draft, u, np.full((2, 3), 0.5, np.float32))
    assert np.allclose(a, 1.0, atol=1e-6)
    assert np.all(acc == 1) and np.array_equal(tok, draft) and np.all(alen == 3)


def pin_verify_disjoint_supports(o):
    """Disjoint supports: the acceptance rate is 0, every draft token is rejected and the
    replacement comes from the target's support."""
    V = 10
    p = np.zeros((1, 2, V), np.float32)
    q = np.zeros((1, 2, V), np.float32)
    p[..., :5] = 0.2
    q[..., 5:] = 0.2
    a, acc, tok, alen = o.verify(p, q, np.array([[7, 9]], np.int32), np.array([[0.0, 0.5]], np.float32),
                                 np.array([[0.1, 0.95]], np.float32))
    assert np.allclose(a, 0.0) and np.all(acc == 0) and alen[0] == 0
    assert tok[0, 0] == 0 and tok[0, 1] == 4  # inverse CDF of the uniform residual over 0..4


def pin_verify_alpha_is_one_minus_tv(o):
    """sum_v min(p_v, q_v) = (sum p + sum q)/2 - (1/2) sum |p - q| for any vectors, which is
    1 - TV(p, q) for normalised ones."""
    p = _dist(6, 4096, 8).reshape(2, 4, 4096)
    q = _dist(7, 4096, 8, temp=1.5).reshape(2, 4, 4096)
    a, _, _, _ = o.verify(p, q, np.zeros((2, 4), np.int32), np.zeros((2, 4), np.float32),
                          np.zeros((2, 4), np.float32))
    pd, qd = p.astype(np.float64), q.astype(np.float64)
    assert np.allclose(a, 0.5 * (pd.sum(axis=2) + qd.sum(axis=2)) - 0.5 * np.abs(pd - qd).sum(axis=2), atol=1e-12)
    assert np.allclose(a, 1.0 - 0.5 * np.abs(pd - qd).sum(axis=2), atol=2e-5)
    assert np.all((a > 0.0) & (a < 1.0))


def _grid(m):
    return ((np.arange(m) + 0.5) / m).astype(np.float32)


def pin_verify_accept_probability(o):
    """Over a fine grid of u, the draft token x is accepted with frequency min(1, p_x/q_x)."""
    p = np.array([0.4, 0.1, 0.3, 0.15, 0.05], np.float32)
    q = np.array([0.2, 0.3, 0.3, 0.05, 0.15], np.float32)
    M = 1000
    u = _grid(M)
    for x in range(5):
        P = np.broadcast_to(p, (1, M, 5)).copy()
        Q = np.broadcast_to(q, (1, M, 5)).copy()
        _, acc, _, _ = o.verify(P, Q, np.full((1, M), x, np.int32), u.reshape(1, M), np.zeros((1, M), np.float32))
        assert abs(acc.mean() - min(1.0, float(p[x]) / float(q[x]))) <= 2.0 / M, x


def pin_verify_output_is_distributed_as_target(o):
    """Speculative sampling's defining property: with x ~ q, u and u2 uniform, the emitted
    token is distributed as p.  Enumerated on a tiny vocabulary: x weighted by q_x, u and
    u2 on fine grids."""
    p = np.array([0.05, 0.35, 0.2, 0.25, 0.15], np.float32)
    q = np.array([0.3, 0.1, 0.2, 0.05, 0.35], np.float32)
    M = 200
    uu, vv = np.meshgrid(_grid(M), _grid(M), indexing="ij")
    n = M * M
    out = np.zeros(5)
    for x in range(5):
        P = np.broadcast_to(p, (1, n, 5)).copy()
        Q = np.broadcast_to(q, (1, n, 5)).copy()
        _, acc, tok, _ = o.verify(P, Q, np.full((1, n), x, np.int32), uu.reshape(1, n), vv.reshape(1, n))
        out += float(q[x]) * np.bincount(tok.ravel(), minlength=5) / n
        # a resampled token always has p > q
        rej = tok[acc == 0]
        assert np.all(p[rej] > q[rej])
    assert np.allclose(out, p, atol=0.01), out


def pin_verify_accepted_length_is_leading_run(o):
    """The sequence is cut at its first rejection: accepted_len counts the leading
    accepted positions only."""
    V = 4
    p = np.tile(np.array([0.7, 0.1, 0.1, 0.1], np.float32), (3, 5, 1))
    q = np.tile(np.array([0.1, 0.7, 0.1, 0.1], np.float32), (3, 5, 1))
    # token 0 (p > q) is always accepted; token 1 with u near 1 is rejected
    draft = np.array([[0, 0, 1, 0, 0], [1, 0, 0, 0, 0], [0, 0, 0, 0, 0]], np.int32)
    u = np.full((3, 5), 0.99, np.float32)
    _, acc, tok, alen = o.verify(p, q, draft, u, np.full((3, 5), 0.3, np.float32))
    assert alen.tolist() == [2, 0, 5]
    assert acc.sum() == 13 and tok[0, 2] == 0 and tok[1, 0] == 0
    del V


# ------------------------------------------------------------------ FP8 index keys
# "Le contexte d'un million de tokens", Entraînement par renforcement: an FP8 KV cache.
# Read as E4M3; its values are fixed by the format's definition.

def pin_e4m3_decode_reference_values(o):
    """E4M3 reference values: 1.0, 2.0, 3.0, the largest finite 448, the smallest normal
    2^-6, the smallest subnormal 2^-9, signed zero, NaN only at S.1111.111, and the
    positive codes ordered as their values."""
    ref = {0x00: 0.0, 0x38: 1.0, 0x40: 2.0, 0x44: 3.0, 0x7E: 448.0, 0x08: 2.0 ** -6, 0x01: 2.0 ** -9,
           0x07: 7 * 2.0 ** -9, 0x3F: 1.875, 0xB8: -1.0, 0xFE: -448.0}
    for b, v in ref.items():
        assert o.e4m3_to_double(b) == v, hex(b)
    assert math.copysign(1.0, o.e4m3_to_double(0x80)) == -1.0 and o.e4m3_to_double(0x80) == 0.0
    assert math.isnan(o.e4m3_to_double(0x7F)) and math.isnan(o.e4m3_to_double(0xFF))
    pos = [o.e4m3_to_double(b) for b in range(0x7F)]
    assert all(a < b for a, b in zip(pos, pos[1:]))


def pin_index_score_e4m3_equals_bf16_on_integers(o):
    """The workload's integer-valued keys and queries encoded as E4M3 and as bf16 give
    the same scores (the values are exact in both formats)."""
    key = lambda kind: synth.stream_key(91, synth.tensor_id(kind))
    q8 = synth.int17_e4m3(key(synth.KIND_IQ), (2, 3, 32, 128))
    k8 = synth.int17_e4m3(key(synth.KIND_IK), (2, 300, 128))
    qb = synth.int17_bf16(key(synth.KIND_IQ), (2, 3, 32, 128))
    kb = synth.int17_bf16(key(synth.KIND_IK), (2, 300, 128))
    w = synth.pow2_f32(key(synth.KIND_W), (2, 3, 32))
    a = o.index_score_e4m3(q8, w, k8, 200)
    b = o.index_score(qb, w, kb, 200)
    assert np.array_equal(a, b)
    assert np.isinf(a[:, 0, 201:]).all() and np.isfinite(a[:, 2, :203]).all()


def pin_index_score_e4m3_one_hot(o):
    """q[t,h] = e_h and k[s] = e_h for all heads: I = sum_h w[t,h] (E4M3 1.0 = 0x38)."""
    q = np.zeros((1, 1, 4, 8), np.uint8)
    for h in range(4):
        q[0, 0, h, h] = 0x38
    k = np.zeros((1, 2, 8), np.uint8)
    k[0, 0, :4] = 0x38   # dot 1 with every head
    k[0, 1, :4] = 0xB8   # dot -1: ReLU gives 0
    w = np.array([[[0.5, 0.25, 0.125, 0.0625]]], np.float32)
    s = o.index_score_e4m3(q, w, k, 1)
    assert s[0, 0, 0] == 0.9375 and s[0, 0, 1] == 0.0


# ---------------------------------------------------------------- context-sharded decode

def pin_partial_single_row_lse_is_logit(o):
    """One selected row in the shard: its value part is the output and the log-sum-exp is
    its logit scale * q . kv (computed here with numpy, in float64)."""
    q, kv, _ = _attn_inputs(30, N=60)
    offset = 1000                      # the shard holds global positions 1000..1059
    idx = np.full((1, 2, 4), -1, np.int32)
    idx[0, 0, 1] = offset + 17
    idx[0, 1, 3] = offset + 59
    idx[0, 1, 0] = 5                   # outside the shard: skipped
    out, lse = o.sparse_attn_partial(q, kv, idx, offset, C.SCALE)
    for t, row in ((0, 17), (1, 59)):
        for h in range(3):
            assert np.array_equal(out[0, t, h], f(kv[0, row, :512]))
            want = C.SCALE * float(np.dot(f(q[0, t, h]), f(kv[0, row])))
            assert abs(lse[0, t, h] - want) <= 1e-12 * max(1.0, abs(want))


def pin_partial_uniform_logits_lse_is_log_count(o):
    """q = 0: every logit is 0, so the log-sum-exp is ln(number of rows in the shard)."""
    q, kv, idx = _attn_inputs(31, N=60, k=20)
    q[:] = 0
    offset = 300
    gidx = idx + offset
    gidx[0, 1, :7] = -1                # 13 rows left in query 1
    _, lse = o.sparse_attn_partial(q, kv, gidx, offset, C.SCALE)
    assert np.allclose(lse[0, 0], math.log(20), rtol=0, atol=1e-13)
    assert np.allclose(lse[0, 1], math.log(13), rtol=0, atol=1e-13)


def pin_partial_whole_cache_equals_sparse_attn(o):
    """A shard holding the whole cache (offset 0) is the unsharded attention."""
    q, kv, idx = _attn_inputs(32, B=2, T=2, H=2, N=50, k=12)
    out, _ = o.sparse_attn_partial(q, kv, idx, 0, C.SCALE)
    assert np.array_equal(out, o.sparse_attn(q, kv, idx, C.SCALE))


def pin_merged_partials_equal_unsharded_attention(o):
    """Three contiguous shards of the cache: their partials combined by log-sum-exp equal
    the attention over the whole selection (float64, to rounding)."""
    q, kv, idx = _attn_inputs(33, B=2, T=2, H=3, N=90, k=30)
    full = o.sparse_attn(q, kv, idx, C.SCALE)
    outs, lses = [], []
    for lo, hi in ((0, 25), (25, 61), (61, 90)):
        out, lse = o.sparse_attn_partial(q, kv[:, lo:hi].copy(), idx, lo, C.SCALE)
        outs.append(out)
        lses.append(lse)
    merged = o.merge_partials(np.stack(outs), np.stack(lses))
    assert np.allclose(merged, full, rtol=0, atol=1e-12)


def pin_merge_partials_one_shard_empty(o):
    """A shard without selected rows (lse = -inf) contributes nothing; all empty gives 0."""
    outs = np.zeros((2, 1, 4), np.float64)
    outs[0, 0] = [1.0, -2.0, 3.0, 0.5]
    lses = np.array([[0.7], [-np.inf]])
    assert np.array_equal(o.merge_partials(outs, lses)[0], outs[0, 0])
    assert np.array_equal(o.merge_partials(outs, np.full((2, 1), -np.inf))[0], np.zeros(4))


def pin_merge_partials_weights(o):
    """Two shards with log-sum-exps ln 1 and ln 3: weights 1/4 and 3/4 (closed form)."""
    outs = np.zeros((2, 1, 2), np.float64)
    outs[0, 0] = [4.0, 0.0]
    outs[1, 0] = [0.0, 8.0]
    got = o.merge_partials(outs, np.array([[0.0], [math.log(3.0)]]))[0]
    assert np.allclose(got, [1.0, 6.0], rtol=0, atol=1e-14)


def _shard_candidates(o, row_scores, bounds, k):
    """Per shard: the oracle's top-k of the shard's scores (positions local), mapped to
    global positions, with their scores; -1 / -inf padding."""
    T = row_scores.shape[0]
    score, pos = [], []
    for lo, hi in bounds:
        loc = o.topk(row_scores[None, :, lo:hi].copy(), hi - lo - 1, k)[0]
        g = np.where(loc >= 0, loc + lo, -1).astype(np.int32)
        sc = np.where(loc >= 0, np.take_along_axis(row_scores[:, lo:hi], np.maximum(loc, 0), axis=1),
                      -np.inf).astype(np.float32)
        score.append(sc)
        pos.append(g)
    return np.concatenate(score, axis=1), np.concatenate(pos, axis=1)


def pin_sharded_topk_equals_full_topk(o):
    """Top-k per contiguous shard, then the k best candidates, equals the top-k of the
    whole row (numpy lexsort of the full row) -- with many ties across shard borders."""
    r = _rng(34)
    T, N, k = 3, 997, 40
    scores = r.integers(-20, 21, size=(T, N)).astype(np.float32) / 4   # heavy ties
    bounds = ((0, 250), (250, 251), (251, 700), (700, N))
    cs, cp = _shard_candidates(o, scores, bounds, k)
    got = o.merge_candidates(cs, cp, k)
    for t in range(T):
        assert got[t].tolist() == _lexsort_topk(scores[t], N, k)


def pin_merge_candidates_ties_and_padding(o):
    """Equal scores go to the lower position whatever the candidate order; fewer than k
    candidates are all kept, ascending, then -1."""
    score = np.array([[5.0, 7.0, 5.0, 5.0, 1.0, 0.0]], np.float32)
    pos = np.array([[90, 40, 10, 60, -1, 3]], np.int32)
    assert o.merge_candidates(score, pos, 3)[0].tolist() == [10, 40, 60]
    assert o.merge_candidates(score, pos, 8)[0].tolist() == [3, 10, 40, 60, 90, -1, -1, -1]


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
