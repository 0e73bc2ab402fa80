"""Parity at the workloads' full sizes, in the launch configuration the benchmark times.

Inputs are generated on the device by the seeded fill kernels; the oracle gets the same
values regenerated on the host (bit-identical by construction, see test_synth.py) for
sampled sequences / query rows, and recomputes those outputs one by one:
  - the index list of every sampled row must equal the oracle's bit for bit;
  - the attention output of sampled (row, layer) pairs must be within the tolerance.
"""
import numpy as np
import pytest

import synth
import synth.device as sd
from gpu_util import assert_close, host
from synth import configs as C

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def dsa():
    import sparse_long_context_score_b200 as m
    from sparse_long_context_score_b200 import build
    build.build()
    m.lib()
    return m


def device_group(w, group=0, step=0, L=None):
    """The group's inputs in HBM, filled on the device."""
    import torch
    L = w.L if L is None else L
    bf = torch.bfloat16
    iq = sd.int17_bf16(torch.empty(w.B, w.T, 32, 128, dtype=bf, device="cuda"), w.key(synth.KIND_IQ, group, 0, step))
    wt = sd.pow2_f32(torch.empty(w.B, w.T, 32, dtype=torch.float32, device="cuda"), w.key(synth.KIND_W, group, 0, step))
    ik = sd.int17_bf16(torch.empty(w.B, w.N, 128, dtype=bf, device="cuda"), w.key(synth.KIND_IK, group))
    qs = [sd.normal_bf16(torch.empty(w.B, w.T, w.H, 576, dtype=bf, device="cuda"), w.key(synth.KIND_Q, group, l, step))
          for l in range(L)]
    kvs = [sd.normal_bf16(torch.empty(w.B, w.N, 576, dtype=bf, device="cuda"), w.key(synth.KIND_KV, group, l))
           for l in range(L)]
    return iq, wt, ik, qs, kvs


def oracle_row(orc, w, b, t, group=0, step=0):
    """Oracle index list of query (b, t) from host-regenerated inputs."""
    row = b * w.T + t
    iq = synth.int17_bf16(w.key(synth.KIND_IQ, group, 0, step),
                          index=synth.rows_index(np.array([row]), 32 * 128)).reshape(1, 1, 32, 128)
    wt = synth.pow2_f32(w.key(synth.KIND_W, group, 0, step),
                        index=synth.rows_index(np.array([row]), 32)).reshape(1, 1, 32)
    vis = min(w.N, w.q_pos0 + t + 1)
    ik = synth.int17_bf16(w.key(synth.KIND_IK, group),
                          index=synth.rows_index(np.arange(b * w.N, b * w.N + vis), 128)).reshape(1, vis, 128)
    sc = orc.index_score(iq, wt, ik, vis - 1).astype(np.float32)
    return orc.topk(sc, vis - 1, w.k)[0, 0]


def oracle_attn(orc, w, b, t, layer, idx_row, group=0, step=0):
    """Oracle attention output of (b, t, layer) over the oracle's own index list."""
    row = b * w.T + t
    q = synth.normal_bf16(w.key(synth.KIND_Q, group, layer, step),
                          index=synth.rows_index(np.array([row]), w.H * 576)).reshape(1, 1, w.H, 576)
    sel = idx_row[idx_row >= 0].astype(np.uint64)
    kv = synth.normal_bf16(w.key(synth.KIND_KV, group, layer),
                           index=synth.rows_index(np.uint64(b * w.N) + sel, 576)).reshape(1, len(sel), 576)
    local = np.full((1, 1, w.k), -1, np.int32)
    local[0, 0, :len(sel)] = np.arange(len(sel))
    return orc.sparse_attn(q, kv, local, C.SCALE)[0, 0]


def run_and_check(dsa, orc, w, samples, layers_checked, group=0):
    import torch
    iq, wt, ik, qs, kvs = device_group(w, group)
    idx, outs = dsa.dsa_group_forward(iq, wt, ik, qs, kvs, w.q_pos0, w.k, C.SCALE)
    torch.cuda.synchronize()
    assert dsa.dsa_device_error() == 0
    got_idx = host(idx)
    for (b, t) in samples:
        want = oracle_row(orc, w, b, t, group)
        assert np.array_equal(got_idx[b, t], want), f"{w.name} group {group} row ({b},{t})"
        for layer in layers_checked:
            ref = oracle_attn(orc, w, b, t, layer, want, group)
            assert_close(host(outs[layer][b, t]), ref, f"{w.name} ({b},{t}) layer {layer}")
    del iq, wt, ik, qs, kvs, idx, outs
    torch.cuda.empty_cache()


def test_decode128k_full(dsa, orc):
    w = C.WORKLOADS["decode128k"]
    run_and_check(dsa, orc, w, samples=[(0, 0), (5, 0), (7, 0)], layers_checked=[0, 3])


def test_decode1m_full_one_group(dsa, orc):
    w = C.WORKLOADS["decode1m"]
    run_and_check(dsa, orc, w, samples=[(0, 0), (1, 0)], layers_checked=[1], group=5)


def test_prefill_full(dsa, orc):
    w = C.WORKLOADS["prefill"]
    run_and_check(dsa, orc, w, samples=[(0, 0), (0, 1029), (0, 4095)], layers_checked=[0, 2])


def test_mtp_full(dsa, orc):
    """MTP drafting at full size: step 1 computes the list over the target cache (the draft
    rows after it are invisible), steps 2..7 reuse it with new queries (KV share)."""
    import torch
    w = C.WORKLOADS["mtp"]
    iq, wt, ik, qs, kvs = device_group(w, L=1)
    kv = kvs[0]
    idx = None
    samples = [(0, 0), (11, 0)]
    wants = {b: oracle_row(orc, w, b, 0) for b, _ in samples}
    for step in range(w.steps):
        q = sd.normal_bf16(torch.empty(w.B, 1, w.H, 576, dtype=torch.bfloat16, device="cuda"),
                           w.key(synth.KIND_Q, 0, 0, step))
        if step == 0:
            idx, outs = dsa.dsa_group_forward(iq, wt, ik, [q], [kv], w.q_pos0, w.k, C.SCALE)
            saved = idx.clone()
        else:
            _, outs = dsa.dsa_group_forward(None, None, None, [q], [kv], w.q_pos0, w.k, C.SCALE,
                                            compute_indices=False, idx_shared=idx)
        torch.cuda.synchronize()
        assert torch.equal(idx, saved)
        got = host(idx)
        assert got.max() < w.q_pos0 + 1  # no draft row can be selected
        for b, _ in samples:
            assert np.array_equal(got[b, 0], wants[b])
            if step in (0, 6):
                ref = oracle_attn(orc, w, b, 0, 0, wants[b], step=step)
                assert_close(host(outs[0][b, 0]), ref, f"mtp step {step + 1} seq {b}")
    assert dsa.dsa_device_error() == 0
