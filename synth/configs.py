"""The five DSA group workloads (shapes, seeds and tensor ids) and their host inputs.

Sizes follow the GLM-5.2 configuration the pages quote (index_n_heads 32,
index_head_dim 128, index_topk 2048, index_topk_freq 4, kv_lora_rank 512, 64 attention
heads); the compressed row is 576 wide (512 latent + 64 rope) with the value in its
first 512 entries and softmax scale 1/sqrt(576).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

from . import (KIND_IK, KIND_IQ, KIND_KV, KIND_Q, KIND_W, int17_bf16, normal_bf16, pow2_f32,
               stream_key, tensor_id)

INDEX_HEADS = 32
INDEX_DIM = 128
DQK = 576
DV = 512
SCALE = 1.0 / math.sqrt(576.0)
BASE_SEED = 0x5EEDD5A0


@dataclass(frozen=True)
class Workload:
    name: str
    number: int          # 1-based, used in the seed
    B: int               # sequences
    T: int               # query tokens per sequence
    N: int               # cached rows per sequence (index keys and compressed rows)
    q_pos0: int          # position of query 0; query t sees s <= q_pos0 + t
    k: int               # top-k
    H: int               # attention heads
    L: int               # layers per IndexShare group (attention calls per index list)
    groups: int = 1      # IndexShare groups run in sequence
    steps: int = 1       # MTP draft steps (steps 2.. reuse the step-1 indices)
    index_fp8: bool = False  # index keys and indexer queries as E4M3 bytes instead of bf16
    note: str = ""

    @property
    def seed(self) -> int:
        return BASE_SEED + self.number

    def key(self, kind: int, group: int = 0, layer: int = 0, step: int = 0) -> int:
        return stream_key(self.seed, tensor_id(kind, group, layer, step))

    @property
    def visible_max(self) -> int:
        return min(self.N, self.q_pos0 + self.T)


WORKLOADS = {
    "tiny": Workload("tiny", 1, B=1, T=1, N=4096, q_pos0=4095, k=256, H=16, L=4,
                     note="tiny decode, 1 group of 4 layers"),
    "decode128k": Workload("decode128k", 2, B=8, T=1, N=131072, q_pos0=131071, k=2048, H=64, L=4,
                           note="decode at 128K, 1 group of 4 layers"),
    "prefill": Workload("prefill", 3, B=1, T=4096, N=131072, q_pos0=126976, k=2048, H=64, L=4,
                        note="chunked prefill, 4096 queries after 126976 cached tokens, causal"),
    "decode1m": Workload("decode1m", 4, B=2, T=1, N=1048576, q_pos0=1048575, k=2048, H=64, L=4,
                         groups=8, note="decode at 1M, 8 IndexShare groups (32 layers)"),
    # MTP: 262144 target tokens plus room for the 7 draft rows that the draft steps append;
    # the step-1 query sits at the last target position, so the draft rows are never visible.
    "mtp": Workload("mtp", 5, B=16, T=1, N=262144 + 7, q_pos0=262143, k=2048, H=64, L=1,
                    steps=7, note="MTP drafting, 1 layer, 7 draft steps reusing step-1 indices"),
    # decode at 128K over an FP8 (E4M3) index-key cache: the same integers as decode128k
    "decode128k_fp8": Workload("decode128k_fp8", 2, B=8, T=1, N=131072, q_pos0=131071, k=2048, H=64, L=4,
                               index_fp8=True, note="decode at 128K, E4M3 index keys and queries"),
}


def scaled(w: Workload, **kw) -> Workload:
    """A smaller workload with the same structure (for oracle-sized parity cases)."""
    d = dict(w.__dict__)
    d.update(kw)
    return Workload(**d)


def host_group_inputs(w: Workload, group: int = 0, step: int = 0, with_attention: bool = True):
    """All inputs of one group (or one MTP step) generated on the host."""
    iq = int17_bf16(w.key(KIND_IQ, group, 0, step), (w.B, w.T, INDEX_HEADS, INDEX_DIM))
    wt = pow2_f32(w.key(KIND_W, group, 0, step), (w.B, w.T, INDEX_HEADS))
    ik = int17_bf16(w.key(KIND_IK, group), (w.B, w.N, INDEX_DIM))
    qs, kvs = [], []
    if with_attention:
        for layer in range(w.L):
            qs.append(normal_bf16(w.key(KIND_Q, group, layer, step), (w.B, w.T, w.H, DQK)))
            kvs.append(normal_bf16(w.key(KIND_KV, group, layer), (w.B, w.N, DQK)))
    return iq, wt, ik, qs, kvs
