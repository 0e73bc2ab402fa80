"""Python binding of libdsa (argument marshalling only).

Every step of the DSA hot path runs in the CUDA kernels of ``libdsa.so``; this module
checks tensor dtypes, shapes and devices, passes raw device pointers and the current
CUDA stream through ctypes, and raises ``DsaError`` on a non-OK status.  PyTorch is used
only for device memory and streams.  There is no fallback: if ``libdsa.so`` is missing
or no CUDA device is present, the calls raise.

Names and argument order follow the C ABI in ``include/dsa.h``.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsa.so")

INDEX_HEADS = 32
INDEX_DIM = 128
DQK = 576
DV = 512
MAX_TOPK = 2048
MAX_LAYERS = 8

DSA_OK = 0
STATUS = {0: "DSA_OK", -1: "DSA_ERR_INVALID_ARG", -2: "DSA_ERR_UNSUPPORTED", -3: "DSA_ERR_WORKSPACE",
          -4: "DSA_ERR_CUDA", -5: "DSA_ERR_TIMEOUT", -6: "DSA_ERR_DEVICE"}

# every symbol include/dsa.h declares
EXPORTS = ("dsa_status_string", "dsa_version", "dsa_workspace_size", "dsa_workspace_size_min", "dsa_index_score",
           "dsa_index_score_e4m3",
           "dsa_sparse_attn_shard", "dsa_shard_candidates", "dsa_merge_candidates", "dsa_merge_partials",
           "dsa_topk",
           "dsa_sparse_attn", "dsa_group_forward", "dsa_topk_noalloc", "dsa_device_error",
           "dsa_check_device_status", "dsa_last_cuda_error", "dsa_cuda_error_string", "dsa_verify",
           "dsa_decode_workspace_size", "dsa_decode_step")


class GroupIO(ctypes.Structure):
    """dsa_group_io: one IndexShare group's tensors for dsa_decode_step."""
    _fields_ = [("iq", ctypes.c_void_p), ("ik", ctypes.c_void_p), ("w", ctypes.c_void_p),
                ("q", ctypes.c_void_p * MAX_LAYERS), ("kv", ctypes.c_void_p * MAX_LAYERS), ("idx", ctypes.c_void_p),
                ("out", ctypes.c_void_p * MAX_LAYERS), ("index_format", ctypes.c_int)]


class DsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load libdsa.so (built in-tree by ``python -m sparse_long_context_score_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is not built; run python -m sparse_long_context_score_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        P, I, LL, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float, ctypes.c_size_t
        L.dsa_status_string.argtypes = [I]
        L.dsa_status_string.restype = ctypes.c_char_p
        L.dsa_version.argtypes = []
        L.dsa_version.restype = I
        L.dsa_workspace_size.argtypes = [I, I, I, I, I, I]
        L.dsa_workspace_size.restype = S
        L.dsa_workspace_size_min.argtypes = [I, I, I, I, I, I]
        L.dsa_workspace_size_min.restype = S
        L.dsa_index_score.argtypes = [P, P, P, I, I, I, LL, P, P]
        L.dsa_index_score_e4m3.argtypes = [P, P, P, I, I, I, LL, P, P]
        L.dsa_sparse_attn_shard.argtypes = [P, P, P, I, I, I, LL, I, I, F, P, P, P, S, P]
        L.dsa_shard_candidates.argtypes = [P, P, I, I, I, I, LL, P, P, P]
        L.dsa_merge_candidates.argtypes = [P, P, I, I, I, I, I, P, P]
        L.dsa_merge_partials.argtypes = [P, P, I, I, I, I, P, P]
        L.dsa_topk.argtypes = [P, I, I, I, LL, I, P, P, S, P]
        L.dsa_sparse_attn.argtypes = [P, P, P, I, I, I, I, I, F, P, P, S, P]
        L.dsa_group_forward.argtypes = [P, P, P, P, P, I, I, I, I, LL, I, I, F, I, P, P, P, S, P]
        L.dsa_topk_noalloc.argtypes = [P, I, I, I, LL, I, P, P]
        L.dsa_device_error.argtypes = [ctypes.POINTER(I), I]
        L.dsa_device_error.restype = I
        L.dsa_check_device_status.argtypes = [P]
        L.dsa_check_device_status.restype = I
        L.dsa_last_cuda_error.argtypes = []
        L.dsa_last_cuda_error.restype = I
        L.dsa_cuda_error_string.argtypes = [I]
        L.dsa_cuda_error_string.restype = ctypes.c_char_p
        L.dsa_verify.argtypes = [P, P, P, P, P, I, I, I, P, P, P, P, P]
        L.dsa_decode_workspace_size.argtypes = [I, I, I, I, I]
        L.dsa_decode_workspace_size.restype = S
        L.dsa_decode_step.argtypes = [P, I, I, I, I, I, I, F, P, S, P, P]
        L.dsa_decode_step.restype = I
        for f in ("dsa_index_score", "dsa_index_score_e4m3", "dsa_sparse_attn_shard", "dsa_shard_candidates",
                  "dsa_merge_candidates", "dsa_merge_partials", "dsa_topk", "dsa_sparse_attn", "dsa_group_forward", "dsa_topk_noalloc",
                  "dsa_verify"):
            getattr(L, f).restype = I
        _lib = L
    return _lib


def _torch():
    import torch
    return torch


def _stream(stream) -> int:
    torch = _torch()
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t, dtypes, name, shape=None):
    torch = _torch()
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t.data_ptr()


def _bf16_types():
    torch = _torch()
    return (torch.bfloat16, torch.int16, torch.uint16)


def _check(rc: int, where: str) -> None:
    if rc != DSA_OK:
        if rc == -4:  # DSA_ERR_CUDA: name the CUDA error behind it
            code = lib().dsa_last_cuda_error()
            where = f"{where} (CUDA error {code}: {lib().dsa_cuda_error_string(code).decode()})"
        raise DsaError(rc, where)


def dsa_device_error(clear: bool = False) -> int:
    """Device error word of the tensor-core kernels' bounded waits (0 = none); syncs."""
    code = ctypes.c_int(0)
    rc = lib().dsa_device_error(ctypes.byref(code), int(bool(clear)))
    if rc not in (DSA_OK, -5):
        raise DsaError(rc, "dsa_device_error")
    return code.value


def dsa_check_device_status(stream=None) -> int:
    """Synchronise `stream` and return the device-side status of the work on it (0 = OK,
    -5 a bounded wait ran out, -6 a top-k invariant failed); resets the error words."""
    return int(lib().dsa_check_device_status(_stream(stream)))


def dsa_workspace_size(B: int, T: int, N: int, k: int, H: int, L: int) -> int:
    return int(lib().dsa_workspace_size(B, T, N, k, H, L))


def dsa_workspace_size_min(B: int, T: int, N: int, k: int, H: int, L: int) -> int:
    return int(lib().dsa_workspace_size_min(B, T, N, k, H, L))


def workspace(B: int, T: int, N: int, k: int, H: int, L: int, device=None, nbytes=None):
    """Allocate a workspace tensor (torch allocation): dsa_workspace_size bytes, or
    `nbytes` (down to dsa_workspace_size_min: a group call then scores and selects the query
    rows in chunks)."""
    torch = _torch()
    n = dsa_workspace_size(B, T, N, k, H, L) if nbytes is None else int(nbytes)
    if n == 0:
        raise ValueError("invalid sizes for dsa_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def dsa_index_score(q, w, k, q_pos0: int, scores=None, stream=None):
    """q [B,T,32,128] bf16, w [B,T,32] f32, k [B,N,128] bf16 -> scores [B,T,N] f32."""
    torch = _torch()
    B, T = q.shape[0], q.shape[1]
    N = k.shape[1]
    if scores is None:
        scores = torch.empty((B, T, N), dtype=torch.float32, device=q.device)
    rc = lib().dsa_index_score(_ptr(q, _bf16_types(), "q", (B, T, INDEX_HEADS, INDEX_DIM)),
                               _ptr(w, (torch.float32,), "w", (B, T, INDEX_HEADS)),
                               _ptr(k, _bf16_types(), "k", (B, N, INDEX_DIM)), B, T, N, int(q_pos0),
                               _ptr(scores, (torch.float32,), "scores", (B, T, N)), _stream(stream))
    _check(rc, "dsa_index_score")
    return scores


def dsa_index_score_e4m3(q, w, k, q_pos0: int, scores=None, stream=None):
    """q [B,T,32,128] E4M3 bytes (uint8), w [B,T,32] f32, k [B,N,128] E4M3 bytes -> scores
    [B,T,N] f32."""
    torch = _torch()
    B, T = q.shape[0], q.shape[1]
    N = k.shape[1]
    if scores is None:
        scores = torch.empty((B, T, N), dtype=torch.float32, device=q.device)
    rc = lib().dsa_index_score_e4m3(_ptr(q, (torch.uint8,), "q", (B, T, INDEX_HEADS, INDEX_DIM)),
                                    _ptr(w, (torch.float32,), "w", (B, T, INDEX_HEADS)),
                                    _ptr(k, (torch.uint8,), "k", (B, N, INDEX_DIM)), B, T, N, int(q_pos0),
                                    _ptr(scores, (torch.float32,), "scores", (B, T, N)), _stream(stream))
    _check(rc, "dsa_index_score_e4m3")
    return scores


def dsa_topk(scores, q_pos0: int, k: int, idx=None, ws=None, stream=None):
    """scores [B,T,N] f32 -> idx [B,T,k] int32 (ascending, -1 padding)."""
    torch = _torch()
    B, T, N = scores.shape
    if idx is None:
        idx = torch.empty((B, T, k), dtype=torch.int32, device=scores.device)
    if ws is None:
        ws = workspace(B, T, N, k, 16, 1, scores.device)
    rc = lib().dsa_topk(_ptr(scores, (torch.float32,), "scores"), B, T, N, int(q_pos0), int(k),
                        _ptr(idx, (torch.int32,), "idx", (B, T, k)), _ptr(ws, (torch.uint8,), "workspace"),
                        ws.numel(), _stream(stream))
    _check(rc, "dsa_topk")
    return idx


def dsa_sparse_attn(q, kv, idx, scale: float, out=None, ws=None, stream=None):
    """q [B,T,H,576] bf16, kv [B,N,576] bf16, idx [B,T,k] int32 -> out [B,T,H,512] f32."""
    torch = _torch()
    B, T, H, _ = q.shape
    N = kv.shape[1]
    k = idx.shape[2]
    if out is None:
        out = torch.empty((B, T, H, DV), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(B, T, N, k, H, 1, q.device)
    rc = lib().dsa_sparse_attn(_ptr(q, _bf16_types(), "q", (B, T, H, DQK)),
                               _ptr(kv, _bf16_types(), "kv", (B, N, DQK)),
                               _ptr(idx, (torch.int32,), "idx", (B, T, k)), B, T, N, H, k, float(scale),
                               _ptr(out, (torch.float32,), "out", (B, T, H, DV)),
                               _ptr(ws, (torch.uint8,), "workspace"), ws.numel(), _stream(stream))
    _check(rc, "dsa_sparse_attn")
    return out


def dsa_sparse_attn_shard(q, kv, idx, offset: int, scale: float, out=None, lse=None, ws=None, stream=None):
    """Attention over the selected rows one context shard holds (kv: global positions
    [offset, offset + N)): q [B,T,H,576] bf16, kv [B,N,576] bf16, idx [B,T,k] int32 global
    positions -> (out [B,T,H,512] f32, lse [B,T,H] f32)."""
    torch = _torch()
    B, T, H, _ = q.shape
    N = kv.shape[1]
    k = idx.shape[2]
    if out is None:
        out = torch.empty((B, T, H, DV), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, T, H), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(B, T, N, k, H, 1, q.device)
    rc = lib().dsa_sparse_attn_shard(_ptr(q, _bf16_types(), "q", (B, T, H, DQK)),
                                     _ptr(kv, _bf16_types(), "kv", (B, N, DQK)),
                                     _ptr(idx, (torch.int32,), "idx", (B, T, k)), B, T, N, int(offset), H, k,
                                     float(scale), _ptr(out, (torch.float32,), "out", (B, T, H, DV)),
                                     _ptr(lse, (torch.float32,), "lse", (B, T, H)),
                                     _ptr(ws, (torch.uint8,), "workspace"), ws.numel(), _stream(stream))
    _check(rc, "dsa_sparse_attn_shard")
    return out, lse


def dsa_shard_candidates(scores, idx, offset: int, cand_score=None, cand_pos=None, stream=None):
    """scores [B,T,N] f32 and the shard's top-k idx [B,T,k] int32 -> (cand_score [B,T,k] f32,
    cand_pos [B,T,k] int32 global positions)."""
    torch = _torch()
    B, T, N = scores.shape
    k = idx.shape[2]
    if cand_score is None:
        cand_score = torch.empty((B, T, k), dtype=torch.float32, device=scores.device)
    if cand_pos is None:
        cand_pos = torch.empty((B, T, k), dtype=torch.int32, device=scores.device)
    rc = lib().dsa_shard_candidates(_ptr(scores, (torch.float32,), "scores", (B, T, N)),
                                    _ptr(idx, (torch.int32,), "idx", (B, T, k)), B, T, N, k, int(offset),
                                    _ptr(cand_score, (torch.float32,), "cand_score", (B, T, k)),
                                    _ptr(cand_pos, (torch.int32,), "cand_pos", (B, T, k)), _stream(stream))
    _check(rc, "dsa_shard_candidates")
    return cand_score, cand_pos


def dsa_merge_candidates(cand_score, cand_pos, k: int, idx=None, stream=None):
    """cand_score [W,B,T,kc] f32, cand_pos [W,B,T,kc] int32 (shard-major, shards in position
    order) -> idx [B,T,k] int32: the k best, ascending, -1 padding."""
    torch = _torch()
    W, B, T, kc = cand_score.shape
    if idx is None:
        idx = torch.empty((B, T, k), dtype=torch.int32, device=cand_score.device)
    rc = lib().dsa_merge_candidates(_ptr(cand_score, (torch.float32,), "cand_score", (W, B, T, kc)),
                                    _ptr(cand_pos, (torch.int32,), "cand_pos", (W, B, T, kc)), W, B, T, kc, int(k),
                                    _ptr(idx, (torch.int32,), "idx", (B, T, k)), _stream(stream))
    _check(rc, "dsa_merge_candidates")
    return idx


def dsa_merge_partials(outs, lses, out=None, stream=None):
    """outs [W,B,T,H,512] f32, lses [W,B,T,H] f32 -> out [B,T,H,512] f32."""
    torch = _torch()
    W, B, T, H, _ = outs.shape
    if out is None:
        out = torch.empty((B, T, H, DV), dtype=torch.float32, device=outs.device)
    rc = lib().dsa_merge_partials(_ptr(outs, (torch.float32,), "outs", (W, B, T, H, DV)),
                                  _ptr(lses, (torch.float32,), "lses", (W, B, T, H)), W, B, T, H,
                                  _ptr(out, (torch.float32,), "out", (B, T, H, DV)), _stream(stream))
    _check(rc, "dsa_merge_partials")
    return out


def dsa_group_forward(iq, w, ik, qs, kvs, q_pos0: int, k: int, scale: float, compute_indices: bool = True,
                      idx_shared=None, outs=None, ws=None, stream=None):
    """One IndexShare group (or MTP draft step): indexer + top-k once when
    compute_indices, then sparse attention for each of the L layers with the same index
    list.  Returns (idx_shared, [out_l])."""
    torch = _torch()
    L = len(qs)
    if L < 1 or L > MAX_LAYERS or len(kvs) != L:
        raise ValueError("need 1..8 layers with one q and one kv each")
    B, T, H, _ = qs[0].shape
    N = kvs[0].shape[1]
    dev = qs[0].device
    if idx_shared is None:
        if not compute_indices:
            raise ValueError("idx_shared is required when compute_indices is False")
        idx_shared = torch.empty((B, T, k), dtype=torch.int32, device=dev)
    if outs is None:
        outs = [torch.empty((B, T, H, DV), dtype=torch.float32, device=dev) for _ in range(L)]
    if ws is None:
        ws = workspace(B, T, N, k, H, L, dev)
    qp = (ctypes.c_void_p * L)(*[_ptr(x, _bf16_types(), "q[l]", (B, T, H, DQK)) for x in qs])
    kp = (ctypes.c_void_p * L)(*[_ptr(x, _bf16_types(), "kv[l]", (B, N, DQK)) for x in kvs])
    op = (ctypes.c_void_p * L)(*[_ptr(x, (torch.float32,), "out[l]", (B, T, H, DV)) for x in outs])
    ci = bool(compute_indices)
    rc = lib().dsa_group_forward(
        _ptr(iq, _bf16_types(), "iq", (B, T, INDEX_HEADS, INDEX_DIM)) if ci else None,
        _ptr(w, (torch.float32,), "w", (B, T, INDEX_HEADS)) if ci else None,
        _ptr(ik, _bf16_types(), "ik", (B, N, INDEX_DIM)) if ci else None,
        ctypes.addressof(qp), ctypes.addressof(kp), L, B, T, N, int(q_pos0), H, int(k), float(scale), int(ci),
        _ptr(idx_shared, (torch.int32,), "idx_shared", (B, T, k)), ctypes.addressof(op),
        _ptr(ws, (torch.uint8,), "workspace"), ws.numel(), _stream(stream))
    _check(rc, "dsa_group_forward")
    return idx_shared, outs


def dsa_topk_noalloc(scores, q_pos0: int, k: int, idx=None, stream=None):
    """dsa_topk for callers that cannot allocate device memory: the select's scratch is a
    fixed array inside libdsa (see include/dsa.h), so no workspace is passed.  Calls that
    overlap on the GPU share that array and must not be issued."""
    torch = _torch()
    B, T, N = scores.shape
    if idx is None:
        idx = torch.empty((B, T, k), dtype=torch.int32, device=scores.device)
    rc = lib().dsa_topk_noalloc(_ptr(scores, (torch.float32,), "scores"), B, T, N, int(q_pos0), int(k),
                                _ptr(idx, (torch.int32,), "idx", (B, T, k)), _stream(stream))
    _check(rc, "dsa_topk_noalloc")
    return idx


def dsa_verify(p, q, draft, u, u2, stream=None):
    """MTP verify step.  p, q [B,S,V] f32 probabilities; draft [B,S] int32; u, u2 [B,S] f32.
    Returns (alpha [B,S] f32, accept [B,S] int32, token [B,S] int32, accepted_len [B] int32)."""
    torch = _torch()
    B, S, V = p.shape
    dev = p.device
    alpha = torch.empty((B, S), dtype=torch.float32, device=dev)
    accept = torch.empty((B, S), dtype=torch.int32, device=dev)
    token = torch.empty((B, S), dtype=torch.int32, device=dev)
    alen = torch.empty((B,), dtype=torch.int32, device=dev)
    rc = lib().dsa_verify(_ptr(p, (torch.float32,), "p", (B, S, V)), _ptr(q, (torch.float32,), "q", (B, S, V)),
                          _ptr(draft, (torch.int32,), "draft", (B, S)), _ptr(u, (torch.float32,), "u", (B, S)),
                          _ptr(u2, (torch.float32,), "u2", (B, S)), B, S, V, _ptr(alpha, (torch.float32,), "alpha"),
                          _ptr(accept, (torch.int32,), "accept"), _ptr(token, (torch.int32,), "token"),
                          _ptr(alen, (torch.int32,), "accepted_len"), _stream(stream))
    _check(rc, "dsa_verify")
    return alpha, accept, token, alen


def decode_workspace(B: int, N: int, k: int, H: int, L: int, device=None):
    """A workspace tensor of dsa_decode_workspace_size bytes (torch allocation)."""
    torch = _torch()
    n = int(lib().dsa_decode_workspace_size(B, N, k, H, L))
    if n == 0:
        raise ValueError("invalid sizes for dsa_decode_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def dsa_decode_step(groups, k: int, scale: float, ws=None, stream=None, side=None):
    """A micro-batched decode step over IndexShare groups (see include/dsa.h).  `groups` is
    a list of dicts with iq, w, ik, qs (L tensors), kvs (L tensors), idx, outs (L tensors);
    iq and ik are bf16, or uint8 holding E4M3 bytes (the index format is taken from their
    dtype); `side` a second CUDA stream (created when None), or `stream` itself to run the
    whole batch's groups in order on one stream."""
    torch = _torch()
    G = len(groups)
    L = len(groups[0]["qs"])
    B, _, H, _ = groups[0]["qs"][0].shape
    N = groups[0]["kvs"][0].shape[1]
    if ws is None:
        ws = decode_workspace(B, N, k, H, L, groups[0]["qs"][0].device)
    if side is None:
        side = torch.cuda.Stream(groups[0]["qs"][0].device)
    arr = (GroupIO * G)()
    for g, d in enumerate(groups):
        io = arr[g]
        f8 = d["ik"].dtype == torch.uint8
        itypes = (torch.uint8,) if f8 else _bf16_types()
        io.index_format = 1 if f8 else 0
        io.iq = _ptr(d["iq"], itypes, "iq", (B, 1, INDEX_HEADS, INDEX_DIM))
        io.w = _ptr(d["w"], (torch.float32,), "w", (B, 1, INDEX_HEADS))
        io.ik = _ptr(d["ik"], itypes, "ik", (B, N, INDEX_DIM))
        io.idx = _ptr(d["idx"], (torch.int32,), "idx", (B, 1, k))
        if len(d["qs"]) != L or len(d["kvs"]) != L or len(d["outs"]) != L:
            raise ValueError("every group needs L queries, caches and outputs")
        for l in range(L):
            io.q[l] = _ptr(d["qs"][l], _bf16_types(), "q[l]", (B, 1, H, DQK))
            io.kv[l] = _ptr(d["kvs"][l], _bf16_types(), "kv[l]", (B, N, DQK))
            io.out[l] = _ptr(d["outs"][l], (torch.float32,), "out[l]", (B, 1, H, DV))
    rc = lib().dsa_decode_step(ctypes.addressof(arr), G, L, B, N, H, int(k), float(scale),
                               _ptr(ws, (torch.uint8,), "workspace"), ws.numel(), _stream(stream), _stream(side))
    _check(rc, "dsa_decode_step")
