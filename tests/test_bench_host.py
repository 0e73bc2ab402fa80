"""Host-side helpers of bench.py, on CPU: the packed per-step buffers and the launch count
the benchmark line claims."""
import sys

import pytest
import torch

sys.argv = sys.argv[:1]
import bench  # noqa: E402
from synth import configs as C  # noqa: E402


def test_packed_views_are_aligned_disjoint_and_typed():
    specs = [((3, 5, 7), torch.bfloat16), ((2, 9), torch.float32), ((4, 1, 11), torch.int32), ((1,), torch.bfloat16)]
    buf, views = bench._packed(specs, "cpu")
    spans = []
    for (shape, dt), v in zip(specs, views):
        assert tuple(v.shape) == shape and v.dtype == dt and v.is_contiguous()
        off = v.data_ptr() - buf.data_ptr()
        assert off % 256 == 0
        spans.append((off, off + v.numel() * v.element_size()))
    spans.sort()
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
    assert spans[-1][1] <= buf.numel()
    # writing through one view changes only its own bytes
    buf.zero_()
    views[1].fill_(1.5)
    assert float(views[1].sum()) == 1.5 * 18
    assert float(views[0].float().abs().sum()) == 0.0 and int(views[2].abs().sum()) == 0
    assert float(views[3].float().abs().sum()) == 0.0


@pytest.mark.parametrize("name,expected", [("decode128k", 4), ("mtp", 4), ("tiny", 4), ("decode1m", 4), ("prefill", 5)])
def test_launches_per_group(name, expected):
    # indexer + top-k (one kernel for decode-shaped rows and for long rows that fit the GPU
    # at once; else select + compact, plus a histogram kernel when the indexer does not
    # count the first digit) + the attention (and its split combine when few (row, layer)
    # units split their keys over several CTAs: every decode shape, not the prefill)
    assert bench.launches_per_group(C.WORKLOADS[name]) == expected


def test_step_launches():
    # decode128k micro-batched: two halves of 4 sequences, each indexer + cluster top-k +
    # attention + split combine
    assert bench.step_launches(C.WORKLOADS["decode128k"], True) == 8
    assert bench.step_launches(C.WORKLOADS["decode128k"], False) == 4
    # decode1m: two halves of one 1M-token sequence, 8 groups: indexer + one-launch top-k +
    # attention + split combine
    assert bench.step_launches(C.WORKLOADS["decode1m"], True) == 64
    # MTP: one group, 7 draft steps: indexer + top-k + 7 x (attention + split combine)
    assert bench.step_launches(C.WORKLOADS["mtp"], False) == 16


def test_auto_schedule():
    # two micro-batches only for decode steps whose rows take the long-row select
    W = C.WORKLOADS
    assert bench.use_micro("auto", W["decode1m"])
    assert not bench.use_micro("auto", W["decode128k"])
    assert not bench.use_micro("auto", W["decode128k_fp8"])
    assert not bench.use_micro("auto", W["mtp"])        # draft steps: not a plain decode step
    assert not bench.use_micro("auto", W["prefill"])
    assert not bench.use_micro("auto", C.scaled(W["decode1m"], B=1))
    assert bench.use_micro("micro", W["decode128k"]) and not bench.use_micro("sequential", W["decode1m"])


def test_reference_arm_json_line():
    """bench.py --impl reference (the CPU oracle on the bench's workload, no GPU needed)
    prints one JSON line with the contract's keys."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "1"], cwd=root, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 1 and d["value"] > 0
    assert d["config"]["workload"] == "decode128k"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
