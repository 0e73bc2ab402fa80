"""The seeded input generator: distributions, determinism, and host == device."""
import numpy as np
import pytest

import synth
from synth import configs as C


def test_int17_values_and_determinism():
    key = synth.stream_key(1234, synth.tensor_id(synth.KIND_IK))
    a = synth.int17_bf16(key, (1000, 128))
    v = synth.bf16_bits_to_f32(a)
    assert set(np.unique(v).tolist()) == set(range(-8, 9))
    assert np.array_equal(a, synth.int17_bf16(key, (1000, 128)))
    assert abs(v.mean()) < 0.05
    other = synth.int17_bf16(synth.stream_key(1235, synth.tensor_id(synth.KIND_IK)), (1000, 128))
    assert not np.array_equal(a, other)


def test_index_form_matches_full_tensor():
    key = synth.stream_key(7, synth.tensor_id(synth.KIND_KV, 0, 2))
    full = synth.normal_bf16(key, (50, 576))
    rows = np.array([3, 17, 49])
    part = synth.normal_bf16(key, index=synth.rows_index(rows, 576)).reshape(3, 576)
    assert np.array_equal(part, full[rows])


def test_pow2_weights():
    key = synth.stream_key(9, synth.tensor_id(synth.KIND_W))
    w = synth.pow2_f32(key, (4000,))
    assert set(np.unique(w).tolist()) == {2.0 ** -e for e in range(1, 7)}


def test_normal_moments_and_bf16_rounding():
    key = synth.stream_key(11, synth.tensor_id(synth.KIND_Q))
    x = synth.bf16_bits_to_f32(synth.normal_bf16(key, (200000,))).astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    assert np.abs(x).max() < 6.0


def test_bf16_round_to_nearest_even():
    vals = np.array([1.0, 1.00390625, 1.01171875, -1.00390625, 3.0e-3, 0.0], np.float32)
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties go to the even significand (1.0)
    got = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(vals))
    assert got[0] == 1.0 and got[1] == 1.0 and got[2] == 1.015625 and got[3] == -1.0
    u = np.array([0x3F808000, 0x3F818000], dtype=np.uint32).view(np.float32)
    assert synth.f32_to_bf16_bits(u).tolist() == [0x3F80, 0x3F82]


def test_workload_seeds_are_distinct():
    """Every workload draws its own tensors, except that the E4M3 variant of a workload
    reuses that workload's seed on purpose (the same integers in the other format)."""
    seen = set()
    for w in C.WORKLOADS.values():
        if w.index_fp8:
            base = [v for v in C.WORKLOADS.values() if v.number == w.number and not v.index_fp8]
            assert len(base) == 1 and base[0].B == w.B and base[0].N == w.N
            continue
        for kind in (synth.KIND_IQ, synth.KIND_W, synth.KIND_IK, synth.KIND_Q, synth.KIND_KV):
            for layer in range(w.L):
                k = w.key(kind, 0, layer)
                assert k not in seen
                seen.add(k)


@pytest.mark.gpu
def test_device_fill_matches_host():
    import torch
    import synth.device as dev
    key = synth.stream_key(99, synth.tensor_id(synth.KIND_KV, 1, 3))
    for fill, host, dtype, n, off in [
        (dev.int17_bf16, synth.int17_bf16, torch.bfloat16, 70001, 5),
        (dev.int17_e4m3, synth.int17_e4m3, torch.uint8, 70003, 11),
        (dev.normal_bf16, synth.normal_bf16, torch.bfloat16, 65537, 123456789),
        (dev.pow2_f32, synth.pow2_f32, torch.float32, 4099, 0),
        (dev.unit_f32, synth.unit_f32, torch.float32, 5000, 77),
    ]:
        t = torch.empty(n, dtype=dtype, device="cuda")
        fill(t, key, off)
        torch.cuda.synchronize()
        want = host(key, index=np.arange(off, off + n, dtype=np.uint64))
        got = t.cpu().view(torch.int16).numpy().view(np.uint16) if dtype == torch.bfloat16 else t.cpu().numpy()
        assert np.array_equal(got.view(np.uint8), np.ascontiguousarray(want).view(np.uint8)), fill.__name__
