"""Parity of the MTP verify step (dsa_verify) against the CPU oracle.

Accept flags, emitted tokens and accepted lengths must match bit for bit (both sides take
the decisions exactly: one float32 product for the accept test, integer weights for the
resample); the acceptance rate sum_v min(p_v, q_v) within float32 summation error."""
import numpy as np
import pytest

import synth
from gpu_util import dev, host

pytestmark = pytest.mark.gpu

VOCAB = 151552  # a GLM-sized vocabulary; the pages do not fix it


@pytest.fixture(scope="module")
def dsa():
    import sparse_long_context_score_b200 as m
    from sparse_long_context_score_b200 import build
    build.build()
    m.lib()
    return m


def _softmax_f32(z):
    z = z.astype(np.float32)
    e = np.exp(z - z.max(axis=-1, keepdims=True), dtype=np.float32)
    return (e / e.sum(axis=-1, keepdims=True, dtype=np.float32)).astype(np.float32)


def _case(seed, B, S, V, temp_q=1.3):
    key = lambda kind, layer=0: synth.stream_key(seed, synth.tensor_id(kind, 0, layer))
    zp = synth.bf16_bits_to_f32(synth.normal_bf16(key(synth.KIND_Q, 0), (B, S, V))) * 2.0
    zq = synth.bf16_bits_to_f32(synth.normal_bf16(key(synth.KIND_Q, 1), (B, S, V))) * 2.0 * temp_q + zp * 0.5
    p, q = _softmax_f32(zp), _softmax_f32(zq)
    u = (synth.unit_f32(key(synth.KIND_SCORES, 0), (B, S)) + np.float32(0.5)).astype(np.float32)
    u2 = (synth.unit_f32(key(synth.KIND_SCORES, 1), (B, S)) + np.float32(0.5)).astype(np.float32)
    # draft tokens drawn from q (inverse CDF of a third uniform)
    u3 = synth.unit_f32(key(synth.KIND_SCORES, 2), (B, S)).astype(np.float64) + 0.5
    cdf = np.cumsum(q.astype(np.float64), axis=-1)
    draft = np.minimum((cdf < u3[..., None] * cdf[..., -1:]).sum(axis=-1), V - 1).astype(np.int32)
    return p, q, draft, u, u2


def _compare(dsa, orc, p, q, draft, u, u2):
    a, acc, tok, alen = dsa.dsa_verify(dev(p), dev(q), dev(draft), dev(u), dev(u2))
    ra, racc, rtok, ralen = orc.verify(p, q, draft, u, u2)
    assert np.array_equal(host(acc), racc)
    assert np.array_equal(host(tok), rtok)
    assert np.array_equal(host(alen), ralen)
    assert np.allclose(host(a).astype(np.float64), ra, atol=1e-5, rtol=0)
    return racc, ralen


def test_verify_mtp_shape(dsa, orc):
    """16 sequences x 7 draft positions over a 151552-entry vocabulary."""
    racc, ralen = _compare(dsa, orc, *_case(71, 16, 7, VOCAB))
    assert 0 < racc.mean() < 1  # both decisions occur


def test_verify_scalar_path_and_small_vocab(dsa, orc):
    _compare(dsa, orc, *_case(72, 3, 5, 1001))          # V not a multiple of 4
    _compare(dsa, orc, *_case(73, 2, 4, 37, temp_q=3.0))


def test_verify_enumerated_tiny_vocab(dsa, orc):
    """Every (draft, u, u2) on grids over a 5-token vocabulary: the same decisions as the
    oracle everywhere, including on the boundaries of the inverse CDF."""
    p = np.array([0.05, 0.35, 0.2, 0.25, 0.15], np.float32)
    q = np.array([0.3, 0.1, 0.2, 0.05, 0.35], np.float32)
    M = 64
    g = ((np.arange(M) + 0.5) / M).astype(np.float32)
    uu, vv = np.meshgrid(g, g, indexing="ij")
    n = M * M
    for x in range(5):
        P = np.ascontiguousarray(np.broadcast_to(p, (1, n, 5)))
        Q = np.ascontiguousarray(np.broadcast_to(q, (1, n, 5)))
        _compare(dsa, orc, P, Q, np.full((1, n), x, np.int32), uu.reshape(1, n).copy(), vv.reshape(1, n).copy())


def test_verify_special_distributions(dsa, orc):
    V = 4096
    p, q, draft, u, u2 = _case(74, 2, 3, V)
    _compare(dsa, orc, p, p.copy(), draft, u, u2)          # identical: all accepted
    dis_p = np.zeros_like(p)
    dis_q = np.zeros_like(q)
    dis_p[..., : V // 2] = 2.0 / V
    dis_q[..., V // 2:] = 2.0 / V
    _compare(dsa, orc, dis_p, dis_q, np.full_like(draft, V - 1), u, u2)  # disjoint: all rejected


def test_verify_rejects_out_of_range_draft(dsa):
    p, q, draft, u, u2 = _case(75, 1, 2, 512)
    draft = np.array([[512, -3]], np.int32)
    _, acc, tok, alen = dsa.dsa_verify(dev(p), dev(q), dev(draft), dev(u), dev(u2))
    assert host(acc).tolist() == [[0, 0]] and host(tok).tolist() == [[-1, -1]] and host(alen).tolist() == [0]


def test_verify_vocab_beyond_one_step_per_chunk(dsa, orc):
    """Vocabularies whose warp segments hold more steps than the kernel keeps chunk sums
    for: a chunk spans two steps (scalar loads at 800001 entries, 16-byte loads at
    3200000), so the resample re-reads two steps of the target's chunk."""
    _compare(dsa, orc, *_case(74, 2, 2, 800001, temp_q=2.0))
    _compare(dsa, orc, *_case(75, 1, 2, 3200000, temp_q=2.0))
