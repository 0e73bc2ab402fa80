"""dsa_topk_noalloc: the top-k select for callers that cannot allocate device memory when
they run it (an engine plugin whose enqueue step must not allocate, a serving loop held
to a fixed memory plan, a latency-critical thread that must not call cudaMalloc).  Its
scratch is a fixed array inside libdsa instead of a caller workspace.

Shapes whose rows fit one cluster of CTAs need no scratch; the others take the scan
kernels, which keep their histograms, candidate lists and per-chunk counters in that
array.  The cases below take the scan kernels, so they read and write the array: they are
called back to back with different score data (the array keeps the previous call's
contents, and the parts that must start at zero are cleared by each call), and every
result must equal the CPU oracle's selection bit for bit and dsa_topk's output.

This file is collected last on purpose so that a run stopping at the first failure has
already run every other test."""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import sparse_long_context_score_b200 as m
    from sparse_long_context_score_b200 import build
    build.build()
    m.lib()
    return m


def _scores(seed, B, T, N, levels):
    key = synth.stream_key(seed, synth.tensor_id(synth.KIND_SCORES))
    u = synth.unit_f32(key, (B, T, N)).astype(np.float64) + 0.5
    return (np.floor(u * levels) / 64.0).astype(np.float32)


# (B, T, N, q_pos0, k, levels); every shape takes the scan kernels and fits the array
SCAN_CASES = [
    (2, 1, 1 << 20, (1 << 20) - 1, 2048, 1 << 20),  # rows too long for one cluster
    (20, 1, 200000, 199999, 2048, 7),               # more rows than one wave of clusters;
                                                    # the threshold bin overflows the candidate list
    (3, 1, 300000, 299999, 2048, 5000),             # long rows with many ties
    (1, 20, 200000, 199980, 2048, 1 << 16),         # causal rows of one sequence
]


def test_noalloc_scan_route_matches_oracle_on_consecutive_calls(dsa, orc):
    import torch
    host = [_scores(31 + i, B, T, N, lv) for i, (B, T, N, _, _, lv) in enumerate(SCAN_CASES)]
    want = [orc.topk(sc, c[3], c[4]) for sc, c in zip(host, SCAN_CASES)]
    # two rounds: in the second every call finds the array as the previous shape left it
    for rnd in range(2):
        for i, (B, T, N, q_pos0, k, lv) in enumerate(SCAN_CASES):
            sc = torch.from_numpy(host[i]).cuda()
            got = dsa.dsa_topk_noalloc(sc, q_pos0, k)
            torch.cuda.synchronize()
            assert np.array_equal(got.cpu().numpy(), want[i]), f"round {rnd} case {i}"
            assert torch.equal(got, dsa.dsa_topk(sc, q_pos0, k)), f"round {rnd} case {i} vs dsa_topk"


def test_noalloc_cluster_route_needs_no_scratch(dsa, orc):
    """Many short rows: one cluster per row, no scratch, so the row count is not bounded
    by the array (the scan route would need ~11 MB here)."""
    import torch
    B, T, N, k = 120, 1, 4096, 256
    sc = _scores(77, B, T, N, 300)
    got = dsa.dsa_topk_noalloc(torch.from_numpy(sc).cuda(), N - 1, k)
    torch.cuda.synchronize()
    assert np.array_equal(got.cpu().numpy(), orc.topk(sc, N - 1, k))


def test_noalloc_refuses_sizes_beyond_its_scratch(dsa):
    import torch
    sc = torch.zeros((64, 1, 1 << 20), dtype=torch.float32, device="cuda")
    with pytest.raises(dsa.DsaError) as err:
        dsa.dsa_topk_noalloc(sc, (1 << 20) - 1, 2048)
    assert err.value.status == -3  # DSA_ERR_WORKSPACE
