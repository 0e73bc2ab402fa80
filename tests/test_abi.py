"""The C-ABI library loads, exports every symbol include/dsa.h declares, and rejects bad
arguments before launching anything.  CPU only: no call here reaches a kernel launch."""
import ctypes
import os
import re

import pytest

import sparse_long_context_score_b200 as dsa

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "dsa.h")


@pytest.fixture(scope="module")
def L():
    from sparse_long_context_score_b200 import build
    build.build()
    return dsa.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(dsa.EXPORTS)


def test_every_declared_symbol_is_exported(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings_and_version(L):
    for code, name in dsa.STATUS.items():
        assert L.dsa_status_string(code).decode() == name
    assert L.dsa_version() >= 10000


def test_workspace_size(L):
    assert L.dsa_workspace_size(8, 1, 131072, 2048, 64, 4) > 8 * 131072 * 4
    assert L.dsa_workspace_size(0, 1, 10, 10, 64, 4) == 0
    assert L.dsa_workspace_size(1, 1, 10, 4096, 64, 4) == 0      # k above index_topk
    assert L.dsa_workspace_size(1, 1, 10, 16, 64, 9) == 0        # too many layers
    big = L.dsa_workspace_size(1, 4096, 131072, 2048, 64, 4)
    assert big >= 4096 * 131072 * 4                                 # the prefill score plane
    # the smallest workspace: the prefill's plane in chunks of 8 query rows; decode has no
    # smaller form
    small = L.dsa_workspace_size_min(1, 4096, 131072, 2048, 64, 4)
    assert 8 * 131072 * 4 <= small < big // 100
    assert L.dsa_workspace_size_min(8, 1, 131072, 2048, 64, 4) == L.dsa_workspace_size(8, 1, 131072, 2048, 64, 4)
    assert L.dsa_workspace_size_min(1, 5, 1000, 64, 64, 1) == L.dsa_workspace_size(1, 5, 1000, 64, 64, 1)  # T < 8
    assert L.dsa_workspace_size_min(0, 8, 10, 10, 64, 4) == 0


FAKE = ctypes.c_void_p(1 << 20)  # aligned, never dereferenced: every call below fails validation


def test_index_score_rejects(L):
    assert L.dsa_index_score(None, FAKE, FAKE, 1, 1, 16, 15, FAKE, None) == -1
    assert L.dsa_index_score(FAKE, FAKE, FAKE, 0, 1, 16, 15, FAKE, None) == -1
    assert L.dsa_index_score(FAKE, FAKE, FAKE, 1, 1, 0, 15, FAKE, None) == -1
    assert L.dsa_index_score(ctypes.c_void_p((1 << 20) + 2), FAKE, FAKE, 1, 1, 16, 15, FAKE, None) == -1


def test_topk_rejects(L):
    assert L.dsa_topk(None, 1, 1, 16, 15, 4, FAKE, FAKE, 1 << 30, None) == -1
    assert L.dsa_topk(FAKE, 1, 1, 16, 15, 0, FAKE, FAKE, 1 << 30, None) == -1
    assert L.dsa_topk(FAKE, 1, 1, 16, 15, 4096, FAKE, FAKE, 1 << 30, None) == -2
    assert L.dsa_topk(FAKE, 1, 1, 16, 15, 4, FAKE, FAKE, 8, None) == -3
    assert L.dsa_topk(FAKE, 1, 1, 16, 15, 4, FAKE, None, 1 << 30, None) == -3


def test_sparse_attn_rejects(L):
    assert L.dsa_sparse_attn(None, FAKE, FAKE, 1, 1, 16, 64, 4, 0.1, FAKE, FAKE, 1 << 30, None) == -1
    assert L.dsa_sparse_attn(FAKE, FAKE, FAKE, 1, 1, 16, 20, 4, 0.1, FAKE, FAKE, 1 << 30, None) == -2
    assert L.dsa_sparse_attn(FAKE, FAKE, FAKE, 1, 1, 16, 64, 4096, 0.1, FAKE, FAKE, 1 << 30, None) == -2
    # unaligned output
    assert L.dsa_sparse_attn(FAKE, FAKE, FAKE, 4, 1, 16, 64, 2048, 0.1, ctypes.c_void_p((1 << 20) + 4), None, 0,
                             None) == -1


def test_group_forward_rejects(L):
    arr = (ctypes.c_void_p * 2)(FAKE.value, FAKE.value)
    nul = (ctypes.c_void_p * 2)(FAKE.value, None)
    a = ctypes.addressof(arr)
    # missing indexer inputs with compute_indices=1
    assert L.dsa_group_forward(None, None, None, a, a, 2, 1, 1, 64, 63, 64, 8, 0.1, 1, FAKE, a, FAKE, 1 << 30, None) == -1
    # a null layer pointer
    assert L.dsa_group_forward(None, None, None, ctypes.addressof(nul), a, 2, 1, 1, 64, 63, 64, 8, 0.1, 0, FAKE, a,
                               FAKE, 1 << 30, None) == -1
    # too many layers, unsupported heads
    assert L.dsa_group_forward(None, None, None, a, a, 9, 1, 1, 64, 63, 64, 8, 0.1, 0, FAKE, a, FAKE, 1 << 30, None) == -2
    assert L.dsa_group_forward(None, None, None, a, a, 2, 1, 1, 64, 63, 24, 8, 0.1, 0, FAKE, a, FAKE, 1 << 30, None) == -2
    # workspace too small
    assert L.dsa_group_forward(FAKE, FAKE, FAKE, a, a, 2, 1, 1, 64, 63, 64, 8, 0.1, 1, FAKE, a, FAKE, 16, None) == -3
    # a prefill-shaped call (T = 64 queries over 100000 keys): one byte short of the smallest
    # chunked workspace is refused before anything is enqueued
    n_min = L.dsa_workspace_size_min(1, 64, 100000, 2048, 64, 2)
    assert 0 < n_min < L.dsa_workspace_size(1, 64, 100000, 2048, 64, 2)
    assert L.dsa_group_forward(FAKE, FAKE, FAKE, a, a, 2, 1, 64, 100000, 99936, 64, 2048, 0.1, 1, FAKE, a, FAKE,
                               n_min - 1, None) == -3


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises((ValueError, ImportError)):
        dsa.dsa_index_score(torch.zeros(1, 1, 32, 128, dtype=torch.bfloat16), torch.zeros(1, 1, 32),
                            torch.zeros(1, 8, 128, dtype=torch.bfloat16), 7, scores=torch.zeros(1, 1, 8))


def test_last_cuda_error_starts_clear_and_names_codes(L):
    # argument errors are returned before any CUDA call, so they never set it
    assert L.dsa_topk(None, 1, 1, 16, 15, 4, FAKE, FAKE, 1 << 30, None) == -1
    assert L.dsa_last_cuda_error() == 0
    assert L.dsa_cuda_error_string(0) == b"no error"
    assert L.dsa_cuda_error_string(1)  # cudaErrorInvalidValue has a description
