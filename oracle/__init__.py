"""CPU oracle for the DSA + IndexShare hot path (test infrastructure only).

This package is the slow, obviously-correct reference the CUDA library is checked
against.  Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import it; the product path never does.  It shares no code with the
CUDA library: the arithmetic lives in ``dsa_oracle.c`` (plain C11, double precision,
single threaded), and this module only marshals numpy arrays into it.

Page citations (title, section) are in ``dsa_oracle.c`` next to each function.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRCS = [os.path.join(_HERE, "dsa_oracle.c"), os.path.join(_HERE, "verify_oracle.c"),
         os.path.join(_HERE, "fp8_oracle.c"), os.path.join(_HERE, "shard_oracle.c")]
_LIB = os.path.join(_HERE, "liboracle.so")

OR_OK = 0
OR_ERR_ARG = -1
OR_ERR_NOMEM = -2
OR_ERR_INVARIANT = -3


def compile_c(srcs, out: str) -> str:
    """gcc -O2 (no fast-math) of the oracle sources into one shared library."""
    srcs = [srcs] if isinstance(srcs, str) else list(srcs)
    tmp = out + ".tmp%d" % os.getpid()
    subprocess.check_call(["gcc", "-O2", "-std=gnu11", "-Wall", "-Wextra", "-fPIC", "-shared",
                           "-o", tmp, *srcs, "-lm"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile the oracle sources into liboracle.so next to them (rebuilt when a source is
    newer)."""
    newest = max(os.path.getmtime(x) for x in _SRCS)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        compile_c(_SRCS, _LIB)
    return _LIB


class Oracle:
    """ctypes view of one compiled copy of dsa_oracle.c."""

    def __init__(self, so_path: str):
        self.so_path = so_path
        L = ctypes.CDLL(so_path)
        P, I, Lg, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_long, ctypes.c_double
        L.oracle_index_score.argtypes = [P, P, P, I, I, I, I, I, Lg, P]
        L.oracle_topk.argtypes = [P, I, I, I, Lg, I, P]
        L.oracle_sparse_attn.argtypes = [P, P, P, I, I, I, I, I, I, I, D, P]
        L.oracle_dense_masked_attn.argtypes = [P, P, P, I, I, I, I, I, I, I, D, P]
        L.oracle_group_forward.argtypes = [P, P, P, P, P, I, I, I, I, I, I, Lg, I, I, I, I, D, I, P, P]
        L.oracle_verify.argtypes = [P, P, P, P, P, I, I, I, P, P, P, P]
        L.oracle_index_score_e4m3.argtypes = [P, P, P, I, I, I, I, I, Lg, P]
        L.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_to_double.restype = D
        L.oracle_sparse_attn_partial.argtypes = [P, P, P, I, I, I, Lg, I, I, I, I, D, P, P]
        L.oracle_merge_partials.argtypes = [P, P, I, Lg, I, P]
        L.oracle_merge_candidates.argtypes = [P, P, Lg, I, I, P]
        for f in ("oracle_index_score", "oracle_topk", "oracle_sparse_attn",
                  "oracle_dense_masked_attn", "oracle_group_forward", "oracle_verify", "oracle_index_score_e4m3",
                  "oracle_sparse_attn_partial", "oracle_merge_partials", "oracle_merge_candidates"):
            getattr(L, f).restype = I
        self.L = L

    def index_score(self, q: np.ndarray, w: np.ndarray, k: np.ndarray, q_pos0: int) -> np.ndarray:
        """q [B,T,nh,hd] bf16 bits, w [B,T,nh] f32, k [B,N,hd] bf16 bits -> scores [B,T,N] f64
        (-inf where the position is not visible to the query)."""
        q = _bf16(q)
        k = _bf16(k)
        w = np.ascontiguousarray(w, dtype=np.float32)
        B, T, nh, hd = q.shape
        N = k.shape[1]
        assert w.shape == (B, T, nh) and k.shape == (B, N, hd)
        out = np.empty((B, T, N), dtype=np.float64)
        _check(self.L.oracle_index_score(_ptr(q), _ptr(w), _ptr(k), B, T, N, nh, hd, q_pos0,
                                         _ptr(out)), "oracle_index_score")
        return out

    def topk(self, scores: np.ndarray, q_pos0: int, k: int) -> np.ndarray:
        """scores [B,T,N] f32 -> idx [B,T,k] int32 (ascending token order, -1 padding)."""
        scores = np.ascontiguousarray(scores, dtype=np.float32)
        B, T, N = scores.shape
        idx = np.empty((B, T, k), dtype=np.int32)
        _check(self.L.oracle_topk(_ptr(scores), B, T, N, q_pos0, k, _ptr(idx)), "oracle_topk")
        return idx

    def sparse_attn(self, q: np.ndarray, kv: np.ndarray, idx: np.ndarray, scale: float,
                    dv: int = 512, dense_masked: bool = False) -> np.ndarray:
        """q [B,T,H,dqk], kv [B,N,dqk] bf16 bits; idx [B,T,k] -> out [B,T,H,dv] f64."""
        q = _bf16(q)
        kv = _bf16(kv)
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        B, T, H, dqk = q.shape
        N = kv.shape[1]
        k = idx.shape[2]
        assert kv.shape == (B, N, dqk) and idx.shape[:2] == (B, T)
        out = np.empty((B, T, H, dv), dtype=np.float64)
        fn = self.L.oracle_dense_masked_attn if dense_masked else self.L.oracle_sparse_attn
        _check(fn(_ptr(q), _ptr(kv), _ptr(idx), B, T, N, H, k, dqk, dv, float(scale), _ptr(out)),
               "oracle attention")
        return out

    def group_forward(self, iq, w, ik, qs, kvs, q_pos0, k, scale, compute_indices=True,
                      idx_shared=None, dv=512):
        """One IndexShare group: indexer + top-k once (unless compute_indices is False and
        idx_shared is given), then sparse attention for every layer with the same indices.
        Returns (idx [B,T,k] int32, [out_l [B,T,H,dv] f64 for each layer])."""
        iq = _bf16(iq)
        ik = _bf16(ik)
        w = np.ascontiguousarray(w, dtype=np.float32)
        qs = [_bf16(x) for x in qs]
        kvs = [_bf16(x) for x in kvs]
        L = len(qs)
        B, T, nh, hd = iq.shape
        N = ik.shape[1]
        H, dqk = qs[0].shape[2], qs[0].shape[3]
        if idx_shared is None:
            idx_shared = np.full((B, T, k), -1, dtype=np.int32)
        idx_shared = np.ascontiguousarray(idx_shared, dtype=np.int32)
        outs = [np.empty((B, T, H, dv), dtype=np.float64) for _ in range(L)]
        qp = (ctypes.c_void_p * L)(*[_ptr(x) for x in qs])
        kp = (ctypes.c_void_p * L)(*[_ptr(x) for x in kvs])
        op = (ctypes.c_void_p * L)(*[_ptr(x) for x in outs])
        _check(self.L.oracle_group_forward(_ptr(iq), _ptr(w), _ptr(ik), ctypes.addressof(qp),
                                           ctypes.addressof(kp), L, B, T, N, nh, hd, q_pos0, H,
                                           k, dqk, dv, float(scale), int(bool(compute_indices)),
                                           _ptr(idx_shared), ctypes.addressof(op)),
               "oracle_group_forward")
        return idx_shared, outs


    def e4m3_to_double(self, b: int) -> float:
        """One E4M3 byte decoded (fp8_oracle.c)."""
        return float(self.L.oracle_e4m3_to_double(int(b)))

    def index_score_e4m3(self, q: np.ndarray, w: np.ndarray, k: np.ndarray, q_pos0: int) -> np.ndarray:
        """q [B,T,nh,hd] E4M3 bytes, w [B,T,nh] f32, k [B,N,hd] E4M3 bytes -> scores [B,T,N]
        f64 (-inf where the position is not visible to the query)."""
        q = np.ascontiguousarray(q, dtype=np.uint8)
        k = np.ascontiguousarray(k, dtype=np.uint8)
        w = np.ascontiguousarray(w, dtype=np.float32)
        B, T, nh, hd = q.shape
        N = k.shape[1]
        out = np.empty((B, T, N), dtype=np.float64)
        _check(self.L.oracle_index_score_e4m3(_ptr(q), _ptr(w), _ptr(k), B, T, N, nh, hd, q_pos0, _ptr(out)),
               "oracle_index_score_e4m3")
        return out

    def sparse_attn_partial(self, q, kv, idx, offset: int, scale: float, dv: int = 512):
        """Attention over the selected rows of one context shard (shard_oracle.c): kv holds
        global positions [offset, offset + Ns).  Returns (out [B,T,H,dv] f64, lse [B,T,H] f64)."""
        q = _bf16(q)
        kv = _bf16(kv)
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        B, T, H, dqk = q.shape
        Ns = kv.shape[1]
        k = idx.shape[2]
        out = np.empty((B, T, H, dv), np.float64)
        lse = np.empty((B, T, H), np.float64)
        _check(self.L.oracle_sparse_attn_partial(_ptr(q), _ptr(kv), _ptr(idx), B, T, Ns, int(offset), H, k, dqk, dv,
                                                 float(scale), _ptr(out), _ptr(lse)), "oracle_sparse_attn_partial")
        return out, lse

    def merge_partials(self, outs, lses):
        """outs [W, ..., dv], lses [W, ...] -> out [..., dv] (shard_oracle.c)."""
        outs = np.ascontiguousarray(outs, dtype=np.float64)
        lses = np.ascontiguousarray(lses, dtype=np.float64)
        W, dv = outs.shape[0], outs.shape[-1]
        R = lses[0].size
        out = np.empty(outs.shape[1:], np.float64)
        _check(self.L.oracle_merge_partials(_ptr(outs), _ptr(lses), W, R, dv, _ptr(out)), "oracle_merge_partials")
        return out

    def merge_candidates(self, score, pos, k: int):
        """score [..., M] f32, pos [..., M] i32 (< 0: none) -> idx [..., k] (shard_oracle.c)."""
        score = np.ascontiguousarray(score, dtype=np.float32)
        pos = np.ascontiguousarray(pos, dtype=np.int32)
        M = score.shape[-1]
        R = score.size // M if M else 0
        idx = np.empty(score.shape[:-1] + (k,), np.int32)
        _check(self.L.oracle_merge_candidates(_ptr(score), _ptr(pos), R, M, int(k), _ptr(idx)),
               "oracle_merge_candidates")
        return idx

    def verify(self, p: np.ndarray, q: np.ndarray, draft: np.ndarray, u: np.ndarray, u2: np.ndarray):
        """MTP verify step (rejection sampling), verify_oracle.c.  p, q [B, S, V] float32
        target / draft probabilities; draft, u, u2 [B, S].  Returns (alpha [B,S] f64,
        accept [B,S] i32, token [B,S] i32, accepted_len [B] i32)."""
        p = np.ascontiguousarray(p, dtype=np.float32)
        q = np.ascontiguousarray(q, dtype=np.float32)
        B, S, V = p.shape
        assert q.shape == p.shape
        draft = np.ascontiguousarray(draft, dtype=np.int32).reshape(B, S)
        u = np.ascontiguousarray(u, dtype=np.float32).reshape(B, S)
        u2 = np.ascontiguousarray(u2, dtype=np.float32).reshape(B, S)
        alpha = np.empty((B, S), np.float64)
        accept = np.empty((B, S), np.int32)
        token = np.empty((B, S), np.int32)
        alen = np.empty((B,), np.int32)
        _check(self.L.oracle_verify(_ptr(p), _ptr(q), _ptr(draft), _ptr(u), _ptr(u2), B, S, V, _ptr(alpha),
                                    _ptr(accept), _ptr(token), _ptr(alen)), "oracle_verify")
        return alpha, accept, token, alen


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _check(rc: int, what: str) -> None:
    if rc != OR_OK:
        raise RuntimeError(f"{what} failed with oracle status {rc}")


def _bf16(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 tensors are passed as uint16 bit patterns")
    return a


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def index_score(*a, **kw):
    return default().index_score(*a, **kw)


def topk(*a, **kw):
    return default().topk(*a, **kw)


def sparse_attn(*a, **kw):
    return default().sparse_attn(*a, **kw)


def group_forward(*a, **kw):
    return default().group_forward(*a, **kw)


def verify(*a, **kw):
    return default().verify(*a, **kw)


def sparse_attn_partial(*a, **kw):
    return default().sparse_attn_partial(*a, **kw)


def merge_partials(*a, **kw):
    return default().merge_partials(*a, **kw)


def merge_candidates(*a, **kw):
    return default().merge_candidates(*a, **kw)
