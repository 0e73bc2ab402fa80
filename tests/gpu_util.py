"""Helpers for the GPU parity tests: host (numpy) <-> device (torch) marshalling and the
tolerance the attention outputs are held to."""
from __future__ import annotations

import numpy as np

TOL_REL = 2e-3   # max|gpu - oracle| <= TOL_REL * max|oracle| + TOL_ABS   (f32 outputs,
TOL_ABS = 1e-3   # bf16 operands, f32 accumulation; the oracle is exact in f64)


def dev_bf16(a: np.ndarray):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def dev(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t) -> np.ndarray:
    import torch
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def assert_close(got: np.ndarray, ref: np.ndarray, what: str = "") -> float:
    err = float(np.abs(got.astype(np.float64) - ref).max()) if ref.size else 0.0
    bound = TOL_REL * float(np.abs(ref).max() if ref.size else 0.0) + TOL_ABS
    assert err <= bound, f"{what}: max|diff| {err:.3e} > {bound:.3e}"
    return err
