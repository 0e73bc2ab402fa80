"""Device fill of the seeded synthetic inputs (same values as the host generator).

Built from synth_fill.cu into libsynth.so next to this file.  Used by the GPU tests and
the benchmark to fill large caches in HBM without a host round trip."""
from __future__ import annotations

import ctypes
import os
import subprocess

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth_fill.cu")
_LIB = os.path.join(_HERE, "libsynth.so")
NVCC_ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        nvcc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call([nvcc, *NVCC_ARCH, "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
                               "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        for name in ("synth_fill_int17_bf16", "synth_fill_int17_e4m3", "synth_fill_pow2_f32", "synth_fill_normal_bf16",
                     "synth_fill_unit_f32"):
            fn = getattr(_lib, name)
            fn.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64, ctypes.c_int64,
                           ctypes.c_void_p]
            fn.restype = ctypes.c_int
    return _lib


def _fill(name, tensor, key, offset=0):
    import torch
    assert tensor.is_cuda and tensor.is_contiguous()
    stream = torch.cuda.current_stream(tensor.device).cuda_stream
    rc = getattr(lib(), name)(tensor.data_ptr(), tensor.numel(), key, offset, stream)
    if rc != 0:
        raise RuntimeError(f"{name} failed with CUDA error {rc}")
    return tensor


def int17_bf16(tensor, key, offset=0):
    """tensor: contiguous torch.bfloat16 (or int16) CUDA tensor, filled in place."""
    return _fill("synth_fill_int17_bf16", tensor, key, offset)


def int17_e4m3(tensor, key, offset=0):
    """tensor: contiguous torch.uint8 CUDA tensor, filled in place with the integers of
    int17_bf16 (same key, same draws) as E4M3 bytes."""
    return _fill("synth_fill_int17_e4m3", tensor, key, offset)


def pow2_f32(tensor, key, offset=0):
    return _fill("synth_fill_pow2_f32", tensor, key, offset)


def normal_bf16(tensor, key, offset=0):
    return _fill("synth_fill_normal_bf16", tensor, key, offset)


def unit_f32(tensor, key, offset=0):
    return _fill("synth_fill_unit_f32", tensor, key, offset)
