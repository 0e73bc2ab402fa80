"""dsa_topk_noalloc: the top-k select for callers that cannot allocate device memory
(an engine plugin's enqueue step, a serving loop held to a fixed memory plan, code being
recorded into a CUDA graph).  Its scratch is a fixed array inside libdsa, so its output
must equal dsa_topk's (bit-exact, as every top-k test here requires) on consecutive calls
that reuse that array, and sizes beyond the array must be refused.

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


def test_noalloc_matches_workspace_topk_on_consecutive_calls(dsa):
    import torch
    cases = [  # (B, T, N, q_pos0, k, levels)
        (4, 1, 131072, 131071, 2048, 5000),   # decode rows with many ties
        (2, 3, 50000, 20000, 300, 1 << 20),   # causal prefill rows, fewer visible than N
    ]
    for seed, (B, T, N, q_pos0, k, levels) in enumerate(cases):
        sc = torch.from_numpy(_scores(seed + 11, B, T, N, levels)).cuda()
        want = dsa.dsa_topk(sc, q_pos0, k)
        got = dsa.dsa_topk_noalloc(sc, q_pos0, k)
        torch.cuda.synchronize()
        assert torch.equal(got, want), f"case {seed}"


def test_noalloc_refuses_sizes_beyond_its_scratch(dsa):
    import torch
    sc = torch.zeros((64, 1, 1 << 20), dtype=torch.float32, device="cuda")
    with pytest.raises(dsa.DsaError) as err:
        dsa.dsa_topk_noalloc(sc, (1 << 20) - 1, 2048)
    assert err.value.status == -3  # DSA_ERR_WORKSPACE
