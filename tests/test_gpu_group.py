"""Parity of the IndexShare group driver (and the MTP reuse) against the CPU oracle."""
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


def run_group(dsa, w, group=0, step=0):
    iq, wt, ik, qs, kvs = C.host_group_inputs(w, group, step)
    idx, outs = dsa.dsa_group_forward(dev_bf16(iq), dev(wt), dev_bf16(ik), [dev_bf16(x) for x in qs],
                                      [dev_bf16(x) for x in kvs], w.q_pos0, w.k, C.SCALE)
    return (iq, wt, ik, qs, kvs), host(idx), [host(o) for o in outs]


@pytest.mark.parametrize("name,kw", [
    ("tiny", {}),
    ("decode128k", dict(B=2, N=20000, q_pos0=19999)),
    ("prefill", dict(T=48, N=6000, q_pos0=6000 - 48)),
    ("decode1m", dict(B=1, N=9000, q_pos0=8999, groups=1)),
])
def test_group_matches_oracle(dsa, orc, name, kw):
    w = C.scaled(C.WORKLOADS[name], **kw)
    (iq, wt, ik, qs, kvs), idx, outs = run_group(dsa, w)
    ridx, routs = orc.group_forward(iq, wt, ik, qs, kvs, w.q_pos0, w.k, C.SCALE)
    assert np.array_equal(idx, ridx)
    for l in range(w.L):
        assert_close(outs[l], routs[l], f"{name} layer {l}")
    for t in range(w.T):
        assert np.all(idx[:, t][idx[:, t] >= 0] <= w.q_pos0 + t)


@pytest.mark.parametrize("kw", [dict(T=24, N=4000, q_pos0=4000 - 24), dict(B=2, T=19, N=3000, q_pos0=3000 - 19)])
def test_prefill_chunked_score_plane_matches_oracle(dsa, orc, kw):
    """A workspace smaller than dsa_workspace_size: the query rows are scored and selected
    in chunks (8 rows at dsa_workspace_size_min, more with more bytes; ragged last chunks,
    two sequences), with the same index lists and outputs as the oracle."""
    w = C.scaled(C.WORKLOADS["prefill"], **kw)
    iq, wt, ik, qs, kvs = C.host_group_inputs(w)
    ridx, routs = orc.group_forward(iq, wt, ik, qs, kvs, w.q_pos0, w.k, C.SCALE)
    n_min = dsa.dsa_workspace_size_min(w.B, w.T, w.N, w.k, w.H, w.L)
    n_all = dsa.dsa_workspace_size(w.B, w.T, w.N, w.k, w.H, w.L)
    assert n_min < n_all
    dq, dkv = [dev_bf16(x) for x in qs], [dev_bf16(x) for x in kvs]
    for nbytes in (n_min, n_min + 8 * w.N * 4 + 65536):
        ws = dsa.workspace(w.B, w.T, w.N, w.k, w.H, w.L, nbytes=nbytes)
        idx, outs = dsa.dsa_group_forward(dev_bf16(iq), dev(wt), dev_bf16(ik), dq, dkv, w.q_pos0, w.k, C.SCALE, ws=ws)
        assert np.array_equal(host(idx), ridx), f"workspace {nbytes}"
        for l in range(w.L):
            assert_close(host(outs[l]), routs[l], f"chunked layer {l}, workspace {nbytes}")
    with pytest.raises(dsa.DsaError):
        ws = dsa.workspace(w.B, w.T, w.N, w.k, w.H, w.L, nbytes=n_min - 256)
        dsa.dsa_group_forward(dev_bf16(iq), dev(wt), dev_bf16(ik), dq, dkv, w.q_pos0, w.k, C.SCALE, ws=ws)
    assert dsa.dsa_check_device_status() == 0


def test_index_list_is_shared_and_unchanged(dsa):
    """compute_indices=0 reads idx_shared without writing it, and gives the same outputs
    as the computing call for every layer."""
    import torch
    w = C.scaled(C.WORKLOADS["decode128k"], B=2, N=5000, q_pos0=4999)
    iq, wt, ik, qs, kvs = C.host_group_inputs(w)
    dq, dkv = [dev_bf16(x) for x in qs], [dev_bf16(x) for x in kvs]
    idx, outs = dsa.dsa_group_forward(dev_bf16(iq), dev(wt), dev_bf16(ik), dq, dkv, w.q_pos0, w.k, C.SCALE)
    before = idx.clone()
    _, outs2 = dsa.dsa_group_forward(None, None, None, dq, dkv, w.q_pos0, w.k, C.SCALE, compute_indices=False,
                                     idx_shared=idx)
    torch.cuda.synchronize()
    assert torch.equal(before, idx)
    for a, b in zip(outs, outs2):
        assert torch.equal(a, b)


def test_mtp_draft_steps_reuse_step1_indices(dsa, orc):
    """MTP drafting: step 1 runs the indexer over the target cache (the query sits at the
    last target position, so the appended draft rows are invisible); steps 2.. reuse the
    step-1 list unchanged, with a new query each step, on the same target cache."""
    import torch
    w = C.scaled(C.WORKLOADS["mtp"], B=3, N=4000 + 7, q_pos0=3999, k=256, steps=7)
    iq, wt, ik, _, kvs = C.host_group_inputs(w)
    kv = kvs[0]
    dkv = dev_bf16(kv)
    idx = None
    for step in range(w.steps):
        q = synth.normal_bf16(w.key(synth.KIND_Q, 0, 0, step), (w.B, 1, w.H, 576))
        if step == 0:
            didx, outs = dsa.dsa_group_forward(dev_bf16(iq), dev(wt), dev_bf16(ik), [dev_bf16(q)], [dkv], w.q_pos0,
                                               w.k, C.SCALE)
            idx = host(didx)
            ridx, routs = orc.group_forward(iq, wt, ik, [q], [kv], w.q_pos0, w.k, C.SCALE)
            assert np.array_equal(idx, ridx)
            saved = didx.clone()
        else:
            _, outs = dsa.dsa_group_forward(None, None, None, [dev_bf16(q)], [dkv], w.q_pos0, w.k, C.SCALE,
                                            compute_indices=False, idx_shared=didx)
            _, routs = orc.group_forward(iq, wt, ik, [q], [kv], w.q_pos0, w.k, C.SCALE, compute_indices=False,
                                         idx_shared=idx)
            torch.cuda.synchronize()
            assert torch.equal(didx, saved)
        assert np.all(idx < 4000)
        assert_close(host(outs[0]), routs[0], f"mtp step {step + 1}")


@pytest.mark.parametrize("B,G,in_order", [(3, 2, False), (2, 3, False), (1, 2, False), (8, 1, False),
                                          (3, 2, True)])
def test_decode_step_matches_oracle(dsa, orc, B, G, in_order):
    """dsa_decode_step (two micro-batches on two streams, indexers taking turns) gives every
    group the oracle's index list bit for bit and its attention within the tolerance."""
    import torch
    w = C.scaled(C.WORKLOADS["decode1m"], B=B, N=9000, q_pos0=8999, groups=G)
    groups, ref = [], []
    for g in range(G):
        iq, wt, ik, qs, kvs = C.host_group_inputs(w, g)
        ref.append(orc.group_forward(iq, wt, ik, qs, kvs, w.q_pos0, w.k, C.SCALE))
        groups.append(dict(iq=dev_bf16(iq), w=dev(wt), ik=dev_bf16(ik), qs=[dev_bf16(x) for x in qs],
                           kvs=[dev_bf16(x) for x in kvs],
                           idx=torch.empty(B, 1, w.k, dtype=torch.int32, device="cuda"),
                           outs=[torch.empty(B, 1, w.H, 512, dtype=torch.float32, device="cuda") for _ in range(w.L)]))
    stream = torch.cuda.current_stream()
    # in order: side == stream runs the whole batch's groups on one stream
    dsa.dsa_decode_step(groups, w.k, C.SCALE, stream=stream, side=stream if in_order else None)
    torch.cuda.synchronize()
    assert dsa.dsa_check_device_status() == 0
    for g in range(G):
        ridx, routs = ref[g]
        assert np.array_equal(host(groups[g]["idx"]), ridx), f"group {g}"
        for l in range(w.L):
            assert_close(host(groups[g]["outs"][l]), routs[l], f"group {g} layer {l}")


@pytest.mark.parametrize("case", ["flat_rows", "short_rows_padded", "mixed"])
def test_decode_select_edge_rows(dsa, orc, case):
    """Decode groups with degenerate rows: every score equal (all-zero keys: the threshold
    bin is the whole row, ties to the lower positions), rows shorter than k (kept whole,
    padded), and one flat row among ordinary ones.  The index lists equal the oracle's."""
    N = {"flat_rows": 20000, "short_rows_padded": 1500, "mixed": 12000}[case]
    w = C.scaled(C.WORKLOADS["decode128k"], B=3, N=N, q_pos0=N - 1)
    iq, wt, ik, qs, kvs = C.host_group_inputs(w)
    if case == "flat_rows":
        ik = np.zeros_like(ik)
    if case == "mixed":
        ik[1] = 0                                     # one flat row among ordinary ones
    idx, outs = dsa.dsa_group_forward(dev_bf16(iq), dev(wt), dev_bf16(ik), [dev_bf16(x) for x in qs],
                                      [dev_bf16(x) for x in kvs], w.q_pos0, w.k, C.SCALE)
    ridx, routs = orc.group_forward(iq, wt, ik, qs, kvs, w.q_pos0, w.k, C.SCALE)
    assert np.array_equal(host(idx), ridx)
    assert_close(host(outs[0]), routs[0], f"{case} layer 0")
    assert dsa.dsa_check_device_status() == 0
