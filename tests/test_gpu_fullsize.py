"""Parity at the workloads' full sizes, in the launch configuration the benchmark times.

Inputs are generated on the device by the seeded fill kernels (the generator shared with
the host side, bit-identical to it: test_synth.py).  The index keys of the rows the oracle
recomputes are copied to the host before the library runs; query rows and the selected
compressed rows are regenerated on the host.  The oracle then recomputes, one by one and
in parallel threads (its C calls release the GIL):
  - the index list of every sampled query row, which must equal the GPU's bit for bit;
  - the attention output of sampled (row, layer) pairs, within the tolerance.
Samples: decode128k all 8 rows x 4 layers; decode1m both rows of all 8 groups, attention
in one layer per group; MTP all 16 rows at every draft step, attention at steps 1, 4, 7;
prefill 72 rows: the first and last query groups and the query groups where the
indexer's per-CTA item ranges begin, attention on 2 layers.
"""
import concurrent.futures as cf
import os

import numpy as np
import pytest

import synth
import synth.device as sd
from gpu_util import assert_close, host
from synth import configs as C

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

POOL = cf.ThreadPoolExecutor(max_workers=max(1, min(32, os.cpu_count() or 1)))


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


def host_indexer_inputs(iq, wt, ik, seqs):
    """Host copies of the indexer inputs of the given sequences (taken before any library
    call touches the device tensors)."""
    import torch
    torch.cuda.synchronize()
    return host(iq), host(wt), {b: host(ik[b]) for b in seqs}


def oracle_row(orc, w, hiq, hwt, hik, b, t):
    """Oracle index list of query (b, t)."""
    vis = min(w.N, w.q_pos0 + t + 1)
    sc = orc.index_score(hiq[b:b + 1, t:t + 1], hwt[b:b + 1, t:t + 1], hik[b][None, :vis], vis - 1)
    return orc.topk(sc.astype(np.float32), vis - 1, w.k)[0, 0]


def oracle_attn(orc, w, b, t, layer, idx_row, group=0, step=0):
    """Oracle attention output of (b, t, layer) over the oracle's own index list; the query
    row and the selected compressed rows are regenerated on the host."""
    row = b * w.T + t
    q = synth.normal_bf16(w.key(synth.KIND_Q, group, layer, step),
                          index=synth.rows_index(np.array([row]), w.H * 576)).reshape(1, 1, w.H, 576)
    sel = idx_row[idx_row >= 0].astype(np.uint64)
    kv = synth.normal_bf16(w.key(synth.KIND_KV, group, layer),
                           index=synth.rows_index(np.uint64(b * w.N) + sel, 576)).reshape(1, len(sel), 576)
    local = np.full((1, 1, w.k), -1, np.int32)
    local[0, 0, :len(sel)] = np.arange(len(sel))
    return orc.sparse_attn(q, kv, local, C.SCALE)[0, 0]


def check(dsa, orc, w, got_idx, outs, samples, layers, hiq, hwt, hik, group=0, step=0, label=""):
    """Compare the GPU's index lists (all samples) and attention outputs (samples x layers)
    with the oracle's, computed in parallel."""
    want = dict(zip(samples, POOL.map(lambda bt: oracle_row(orc, w, hiq, hwt, hik, *bt), samples)))
    for (b, t) in samples:
        assert np.array_equal(got_idx[b, t], want[(b, t)]), f"{label} row ({b},{t})"
    jobs = [(b, t, l) for (b, t) in samples for l in layers]
    refs = POOL.map(lambda j: oracle_attn(orc, w, j[0], j[1], j[2], want[(j[0], j[1])], group, step), jobs)
    for (b, t, l), ref in zip(jobs, refs):
        assert_close(outs[l][b, t], ref, f"{label} ({b},{t}) layer {l}")
    return want


def run_group(dsa, w, group=0):
    import torch
    iq, wt, ik, qs, kvs = device_group(w, group)
    hiq, hwt, hik = host_indexer_inputs(iq, wt, ik, range(w.B))
    idx, outs = dsa.dsa_group_forward(iq, wt, ik, qs, kvs, w.q_pos0, w.k, C.SCALE)
    torch.cuda.synchronize()
    assert dsa.dsa_check_device_status() == 0
    res = host(idx), [host(o) for o in outs], (hiq, hwt, hik)
    del iq, wt, ik, qs, kvs, idx, outs
    torch.cuda.empty_cache()
    return res


def test_decode128k_full(dsa, orc):
    w = C.WORKLOADS["decode128k"]
    got, outs, hin = run_group(dsa, w)
    check(dsa, orc, w, got, outs, [(b, 0) for b in range(w.B)], range(w.L), *hin, label="decode128k")


def test_decode1m_full_every_group(dsa, orc):
    w = C.WORKLOADS["decode1m"]
    for g in range(w.groups):
        got, outs, hin = run_group(dsa, w, group=g)
        check(dsa, orc, w, got, outs, [(0, 0), (1, 0)], [g % w.L], *hin, group=g, label=f"decode1m group {g}")


def prefill_sample_rows(w, sms):
    """Query rows of the first and last query groups of 8, and of the query groups in which
    the indexer's contiguous per-CTA ranges of (query group, 128-key tile) items begin (the
    same partition as the launch: one CTA per SM)."""
    qg_tiles = []
    for g in range((w.T + 7) // 8):
        t_last = min(8 * g + 8, w.T) - 1
        qg_tiles.append((min(w.N, w.q_pos0 + t_last + 1) + 127) // 128)
    total = sum(qg_tiles)
    grid = min(total, sms)
    per, extra = divmod(total, grid)
    starts = [c * per + min(c, extra) for c in range(grid)]
    groups, acc, g = set(), 0, 0
    bounds = iter(sorted(starts))
    nxt = next(bounds)
    for g, n in enumerate(qg_tiles):
        while nxt is not None and nxt < acc + n:
            groups.add(g)
            nxt = next(bounds, None)
        acc += n
    picked = sorted(groups)
    # spread over the boundaries: about 7 query groups, plus the first and the last
    chosen = {0, len(qg_tiles) - 1} | set(picked[::max(1, len(picked) // 7)])
    return sorted(t for g in chosen for t in range(8 * g, min(8 * g + 8, w.T)))


def test_prefill_full(dsa, orc):
    import torch
    w = C.WORKLOADS["prefill"]
    rows = prefill_sample_rows(w, torch.cuda.get_device_properties(0).multi_processor_count)
    assert len(rows) >= 64 and 0 in rows and w.T - 1 in rows
    got, outs, hin = run_group(dsa, w)
    check(dsa, orc, w, got, outs, [(0, t) for t in rows], [0, 2], *hin, label="prefill")


def test_mtp_full(dsa, orc):
    """MTP drafting at full size: step 1 computes the list over the target cache (the draft
    rows after it are invisible), steps 2..7 reuse it with new queries (KV share)."""
    import torch
    w = C.WORKLOADS["mtp"]
    iq, wt, ik, qs, kvs = device_group(w, L=1)
    hiq, hwt, hik = host_indexer_inputs(iq, wt, ik, range(w.B))
    kv = kvs[0]
    samples = [(b, 0) for b in range(w.B)]
    want = None
    idx = None
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
        assert torch.equal(idx, saved)  # the step-1 list is never rewritten
        got = host(idx)
        assert got.max() < w.q_pos0 + 1  # no draft row can be selected
        layers = [0] if step in (0, 3, 6) else []
        if step == 0:
            want = check(dsa, orc, w, got, [host(outs[0])], samples, layers, hiq, hwt, hik, step=step,
                         label=f"mtp step {step + 1}")
        else:
            for b, t in samples:
                assert np.array_equal(got[b, t], want[(b, t)])
            out = host(outs[0])
            jobs = samples if layers else []
            refs = POOL.map(lambda bt: oracle_attn(orc, w, bt[0], 0, 0, want[bt], step=step), jobs)
            for (b, _), ref in zip(jobs, refs):
                assert_close(out[b, 0], ref, f"mtp step {step + 1} seq {b}")
    assert dsa.dsa_check_device_status() == 0
