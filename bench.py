"""Benchmark of the DSA IndexShare group decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode128k]
    python bench.py --impl reference ...        # the CPU oracle, timed on a bounded sample

One step = one pass of the whole hot path over one batch: the indexer over the index-key
cache, the top-k select, and sparse MLA attention for the 4 layers of the group (all
IndexShare groups of the workload in sequence).  Inputs are seeded synthetic tensors
generated in HBM before timing; the step is captured once in a CUDA graph and replayed.
L2 is flushed (a 512 MiB write, then a 512 MiB read that evicts the dirty lines) before
every timed step and the step alone is timed with
CUDA events on the launching stream.  Under torchrun every rank runs its own batch
(weak scaling, no data-path collective) and rank 0 reports the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

INDEXER_BYTES_PER_KEY = 128 * 2                  # one index key read per visible token
INDEXER_BYTES_PER_QUERY = 32 * 128 * 2 + 32 * 4  # indexer query + head weights
SCORE_BYTES_PER_KEY = 4                          # score write: reported, not algorithmic
ROW_BYTES = 576 * 2                              # one gathered compressed row


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default="decode128k")
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--cpu-sample", type=int, default=2, help="sequences in the CPU-oracle sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-extra", action="store_true", help="skip the 1M / MTP / prefill workloads")
    p.add_argument("--shard", default="batch", choices=["batch", "context"],
                   help="multi-GPU: each rank its own batch (weak scaling), or every sequence's context "
                        "spread over the ranks (strong scaling; sparse_long_context_score_b200.sharded)")
    p.add_argument("--schedule", default="auto", choices=["auto", "micro", "sequential"],
                   help="decode workloads through dsa_decode_step: the groups in order on one stream, or "
                        "two micro-batches on two streams (the indexer of one beside the top-k and "
                        "attention of the other); auto: micro-batches when the rows are longer than a "
                        "cluster's select holds (N > 262144, as at 1M contexts), in order otherwise")
    p.add_argument("--ncu-case", choices=["indexer", "topk", "attn", "indexer_prefill", "attn_mtp", "topk_1m",
                                          "indexer_fp8", "verify"],
                   help="run one kernel of the decode step a few times on a profiler-sized case and exit "
                        "(for ncu captures; prints no benchmark line)")
    return p.parse_args()


def algorithmic(w):
    """Algorithmic HBM bytes of one step and of one indexer launch: the indexer reads the
    visible index keys of each sequence once, plus its queries and head weights; the
    attention gathers k compressed rows per (query, layer, draft step) and reads the
    queries and writes the outputs; the index list is written once.  The score write
    (4 B per visible key, L2-resident) is not algorithmic: it is returned separately."""
    vis = min(w.N, w.q_pos0 + w.T)
    esz = 1 if w.index_fp8 else 2  # E4M3 or bf16 index keys and indexer queries
    per_query = INDEXER_BYTES_PER_QUERY - 32 * 128 * (2 - esz)
    idx_launch = w.B * w.T * per_query + w.B * vis * INDEXER_BYTES_PER_KEY * esz // 2
    attn = w.B * w.T * w.L * w.steps * (w.k * ROW_BYTES + w.H * 576 * 2 + w.H * 512 * 4)
    scores = w.B * w.T * vis * SCORE_BYTES_PER_KEY
    return w.groups * (idx_launch + attn + w.B * w.T * w.k * 4), idx_launch, scores


def prefill_indexer_flops(w):
    """Tensor FLOPs of the prefill indexer: 2 * 32 heads * 128 dims per (query, visible key)."""
    pairs = sum(min(w.N, w.q_pos0 + t + 1) for t in range(w.T))
    return w.B * pairs * 2 * 32 * 128


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            m = json.load(fh)
        return float(m["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def _bf16_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            return float(json.load(fh)["bf16_tflops"])
    except Exception:
        return 1590.0


def profiled_traffic(kernel_src: str, workload: str):
    """Per-launch DRAM bytes of the indexer from the committed ncu summary, if it was taken
    on the current kernel source; None otherwise."""
    path = os.path.join(ROOT, "profiles", f"indexer_{workload}.md")
    src = os.path.join(ROOT, "sparse_long_context_score_b200", "csrc", kernel_src)
    try:
        text = open(path).read()
        digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        m = re.search(r"traffic_bytes_per_launch:\s*(\d+)\s*\(source sha256 ([0-9a-f]{16})\)", text)
        if m and m.group(2) == digest:
            return int(m.group(1))
    except OSError:
        pass
    return None


class ClockSampler:
    """nvidia-smi clock and throttle-reason samples during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            out, _ = self.proc.communicate(timeout=10)
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        rows = []
        for l in self.lines:
            parts = [x.strip() for x in l.split(",")]
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[2:]))
            except (ValueError, IndexError):
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower() == "active"})
        sms = sorted(r[0] for r in rows)
        return {"sm_mhz": sms[len(sms) // 2], "sm_max_mhz": rows[0][1], "reasons": reasons, "samples": len(rows)}


def rank_key(key: int, rank: int) -> int:
    """Each rank decodes its own batch (weak scaling): its inputs use the workload's keys
    XOR the rank, so no two ranks see the same tensors."""
    return key ^ rank


def max_over_ranks(values, world: int, device=None):
    """Element-wise max of a list of floats over all ranks (the slowest rank sets the step
    time).  Uses the initialised process group; a no-op for a single process."""
    import torch
    if world <= 1:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def job_throughput(units_per_rank: int, world: int, max_ms: float) -> float:
    """Whole-job units per second: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / (max_ms * 1e-3)


def _packed(specs, device):
    """One device byte buffer holding tensors of the given (shape, dtype) at 256-byte
    aligned offsets, and the tensors as views of it: a step's query-side inputs (and its
    outputs) then cross PCIe in one copy each."""
    import torch
    offs, total = [], 0
    for shape, dt in specs:
        offs.append(total)
        n = torch.tensor([], dtype=dt).element_size()
        for d in shape:
            n *= d
        total = (total + n + 255) & ~255
    buf = torch.empty(total, dtype=torch.uint8, device=device)
    views = []
    for (shape, dt), o in zip(specs, offs):
        n = torch.tensor([], dtype=dt).element_size()
        for d in shape:
            n *= d
        views.append(buf[o:o + n].view(dt).view(shape))
    return buf, views


def make_inputs(w, device, rank):
    """Seeded synthetic inputs of every group.  The caches live in their own tensors; the
    per-step query-side inputs of all groups (indexer queries, head weights, attention
    queries, MTP draft queries) share one buffer, and so do the outputs (index lists and
    attention outputs) -- groups[0]["in_buf"] / ["out_buf"]."""
    import torch
    import synth
    import synth.device as sd
    bf = torch.bfloat16
    f32 = torch.float32
    ins, outs_spec = [], []
    ixt = torch.uint8 if w.index_fp8 else bf
    fill_index = sd.int17_e4m3 if w.index_fp8 else sd.int17_bf16
    for g in range(w.groups):
        ins += [((w.B, w.T, 32, 128), ixt), ((w.B, w.T, 32), f32)]
        ins += [((w.B, w.T, w.H, 576), bf)] * (w.L + max(0, w.steps - 1))
        outs_spec += [((w.B, w.T, w.k), torch.int32)] + [((w.B, w.T, w.H, 512), f32)] * w.L
    in_buf, in_views = _packed(ins, device)
    out_buf, out_views = _packed(outs_spec, device)
    groups = []
    for g in range(w.groups):
        ik = torch.empty(w.B, w.N, 128, dtype=ixt, device=device)
        fill_index(ik, rank_key(w.key(synth.KIND_IK, g), rank))
        kvs = []
        for l in range(w.L):
            kv = torch.empty(w.B, w.N, 576, dtype=bf, device=device)
            sd.normal_bf16(kv, rank_key(w.key(synth.KIND_KV, g, l), rank))
            kvs.append(kv)
        iq, wt = in_views.pop(0), in_views.pop(0)
        fill_index(iq, rank_key(w.key(synth.KIND_IQ, g), rank))
        sd.pow2_f32(wt, rank_key(w.key(synth.KIND_W, g), rank))
        qs = []
        for l in range(w.L):
            q = in_views.pop(0)
            sd.normal_bf16(q, rank_key(w.key(synth.KIND_Q, g, l), rank))
            qs.append(q)
        draft_qs = []
        for st in range(1, w.steps):
            qd = in_views.pop(0)
            sd.normal_bf16(qd, rank_key(w.key(synth.KIND_Q, g, 0, st), rank))
            draft_qs.append(qd)
        idx = out_views.pop(0)
        outs = [out_views.pop(0) for _ in range(w.L)]
        groups.append(dict(ik=ik, kvs=kvs, iq=iq, wt=wt, qs=qs, idx=idx, outs=outs, draft_qs=draft_qs))
    groups[0]["in_buf"], groups[0]["out_buf"] = in_buf, out_buf
    return groups


# Rows longer than this take the long-row select (one cooperative launch with row barriers),
# whose latency two micro-batches hide behind the other half's indexer (measured on B200:
# 1M contexts 1056 -> 871 us per step, 512K 725 -> 654 us; at 128K-256K in order is faster).
CLUSTER_MAX_ROW = 8 * 1024 * 32


def use_micro(schedule: str, w) -> bool:
    """Whether the decode step of workload w runs as two micro-batches."""
    if not (w.T == 1 and w.steps == 1 and w.B >= 2):
        return False
    return schedule == "micro" or (schedule == "auto" and min(w.N, w.q_pos0 + 1) > CLUSTER_MAX_ROW)


def run_ours(args, rank, world, device, w=None, e2e=True):
    """Times the workload's step on this rank's GPU.  Returns a dict: the step time (graph
    replay, inputs resident in HBM), the indexer launch time, the end-to-end times (eager
    and graph) with their host<->device bytes, and the clock record."""
    import torch
    import sparse_long_context_score_b200 as dsa
    from synth import configs as C

    w = w or C.WORKLOADS[args.workload]
    torch.cuda.set_device(device)
    dsa.lib()
    groups = make_inputs(w, device, rank)
    micro = use_micro(args.schedule, w)
    # a decode step (one query per sequence, no draft steps) runs through dsa_decode_step, in
    # order (side = stream) unless micro-batched; MTP drafting and prefill through
    # dsa_group_forward
    use_step = micro or (w.T == 1 and w.steps == 1)
    if w.index_fp8 and not use_step:
        raise ValueError("the E4M3 index format runs through the decode step only")
    ws = dsa.decode_workspace(w.B, w.N, w.k, w.H, w.L, device) if use_step else \
        dsa.workspace(w.B, w.T, w.N, w.k, w.H, w.L, device)
    stream = torch.cuda.Stream(device)
    side = torch.cuda.Stream(device)
    dgroups = [dict(iq=g["iq"], w=g["wt"], ik=g["ik"], qs=g["qs"], kvs=g["kvs"], idx=g["idx"], outs=g["outs"])
               for g in groups]
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    flush_rd = torch.zeros(512 << 20, dtype=torch.uint8, device=device)

    def flush_l2():
        # write a buffer larger than L2, then read another: the dirty lines of the write are
        # evicted (written back) by the read, before the timed region, not during it
        flush.zero_()
        flush_rd.view(torch.int64).sum()

    def step():
        if use_step:
            dsa.dsa_decode_step(dgroups, w.k, C.SCALE, ws=ws, stream=stream, side=side if micro else stream)
            return
        for g in groups:
            dsa.dsa_group_forward(g["iq"], g["wt"], g["ik"], g["qs"], g["kvs"], w.q_pos0, w.k, C.SCALE,
                                  idx_shared=g["idx"], outs=g["outs"], ws=ws, stream=stream)
            # MTP draft steps 2..: the step-1 index list and the target cache are reused
            for qd in g.get("draft_qs", []):
                dsa.dsa_group_forward(None, None, None, [qd], g["kvs"], w.q_pos0, w.k, C.SCALE,
                                      compute_indices=False, idx_shared=g["idx"], outs=g["outs"], ws=ws,
                                      stream=stream)

    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        step()  # eager once (sets kernel attributes) before capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    torch.cuda.synchronize()

    def timed(fn, K, W, host_in_region=False):
        """K timed runs of fn after W warm-up runs, L2 flushed before each; CUDA events on
        the launching stream.  With host_in_region the device is idle when the start event
        is recorded, so the host's enqueue work of fn is inside the measured interval."""
        with torch.cuda.stream(stream):
            for _ in range(W):
                flush_l2()
                fn()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        with torch.cuda.stream(stream):
            for a, b in ev:
                flush_l2()
                if host_in_region:
                    torch.cuda.synchronize()
                a.record(stream)
                fn()
                b.record(stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in ev]

    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        times = timed(graph.replay, args.steps, args.warmup)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    res = {"step_ms": sum(times) / len(times), "clocks": clk.summary(),
           "schedule": "two micro-batches (dsa_decode_step)" if micro else
           "groups in order (dsa_decode_step, side = stream)" if use_step else "groups in order (dsa_group_forward)"}

    # the dominant kernel alone: the indexer over the first group's cache, same launch shape
    g0 = groups[0]
    scores = torch.empty(w.B, w.T, w.N, dtype=torch.float32, device=device)
    # captured in a graph like the step, so the host-side set-up of a launch (tensor-map
    # encoding) is not inside the timed region
    index_score = dsa.dsa_index_score_e4m3 if w.index_fp8 else dsa.dsa_index_score
    with torch.cuda.stream(stream):
        index_score(g0["iq"], g0["wt"], g0["ik"], w.q_pos0, scores=scores, stream=stream)
    torch.cuda.synchronize()
    igraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(igraph, stream=stream):
        index_score(g0["iq"], g0["wt"], g0["ik"], w.q_pos0, scores=scores, stream=stream)
    torch.cuda.synchronize()
    idx_times = timed(igraph.replay, args.steps, args.warmup)
    res["idx_ms"] = sum(idx_times) / len(idx_times)
    status = dsa.dsa_check_device_status(stream)
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed runs")

    if e2e:
        # end to end through the public API with host buffers: per step, the step's
        # query-side inputs (one packed buffer) go host -> device from pinned memory, the
        # library calls run, and the outputs (index lists and attention outputs, one packed
        # buffer) come back.  "eager" calls the C ABI per step (its host-side work included);
        # "graph" replays the captured step between the two copies.
        in_buf, out_buf = groups[0]["in_buf"], groups[0]["out_buf"]
        pinned_in = in_buf.cpu().pin_memory()
        pinned_out = torch.empty_like(out_buf, device="cpu").pin_memory()

        def e2e_eager():
            in_buf.copy_(pinned_in, non_blocking=True)
            step()
            pinned_out.copy_(out_buf, non_blocking=True)

        def e2e_graph():
            in_buf.copy_(pinned_in, non_blocking=True)
            graph.replay()
            pinned_out.copy_(out_buf, non_blocking=True)

        eager = timed(e2e_eager, args.steps, args.warmup, host_in_region=True)
        gr = timed(e2e_graph, args.steps, args.warmup, host_in_region=True)
        res.update(e2e_ms=sum(eager) / len(eager), e2e_graph_ms=sum(gr) / len(gr), h2d=in_buf.numel(),
                   d2h=out_buf.numel())
        keys = ["step_ms", "idx_ms", "e2e_ms", "e2e_graph_ms"]
    else:
        keys = ["step_ms", "idx_ms"]
    for k, v in zip(keys, max_over_ranks([res[k] for k in keys], world, device)):
        res[k] = v
    del groups, dgroups, ws, flush, flush_rd, scores, graph, igraph
    torch.cuda.empty_cache()
    return w, res


VERIFY_VOCAB = 151552  # a GLM-sized vocabulary (the pages do not fix it)


def run_verify(args, device, peak):
    """The MTP verify step (dsa_verify) for the mtp workload's 16 sequences x 7 draft
    positions over a 151552-entry vocabulary: graph-captured, L2 flushed before each of
    K timed runs; HBM-bound (8 B read per vocabulary entry and position)."""
    import torch
    import sparse_long_context_score_b200 as dsa
    import synth
    import synth.device as sd
    from synth import configs as C
    w = C.WORKLOADS["mtp"]
    B, S, V = w.B, w.steps, VERIFY_VOCAB
    torch.cuda.set_device(device)
    zp = sd.normal_bf16(torch.empty(B, S, V, dtype=torch.bfloat16, device=device), w.key(synth.KIND_Q, 1, 0))
    zq = sd.normal_bf16(torch.empty(B, S, V, dtype=torch.bfloat16, device=device), w.key(synth.KIND_Q, 1, 1))
    p = torch.softmax(zp.float() * 2.0, dim=-1).contiguous()
    q = torch.softmax(zq.float() * 2.6 + zp.float(), dim=-1).contiguous()
    draft = torch.argmax(q, dim=-1).to(torch.int32).contiguous()
    u = sd.unit_f32(torch.empty(B, S, dtype=torch.float32, device=device), w.key(synth.KIND_SCORES, 1, 0)) + 0.5
    u2 = sd.unit_f32(torch.empty(B, S, dtype=torch.float32, device=device), w.key(synth.KIND_SCORES, 1, 1)) + 0.5
    stream = torch.cuda.Stream(device)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    flush_rd = torch.zeros(512 << 20, dtype=torch.uint8, device=device)
    with torch.cuda.stream(stream):
        dsa.dsa_verify(p, q, draft, u, u2, stream=stream)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        dsa.dsa_verify(p, q, draft, u, u2, stream=stream)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            flush.zero_()
            flush_rd.view(torch.int64).sum()
            graph.replay()
        for a, b in ev:
            flush.zero_()
            flush_rd.view(torch.int64).sum()
            a.record(stream)
            graph.replay()
            b.record(stream)
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in ev) / len(ev)
    nbytes = 2 * B * S * V * 4
    del zp, zq, p, q, flush, flush_rd, graph
    torch.cuda.empty_cache()
    return {"B": B, "draft_steps": S, "vocab": V, "us_per_step": ms * 1e3, "hbm_gbs": nbytes / (ms * 1e-3) / 1e9,
            "roofline_frac": nbytes / (ms * 1e-3) / 1e9 / peak, "algorithmic_bytes": nbytes}


def host_cpu() -> dict:
    """The host CPU the oracle runs on: model name and logical core count."""
    model = None
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    import platform
    return {"model": model or platform.processor() or "unknown", "logical_cores": os.cpu_count()}


def oracle_sequence(w, b, o):
    """The oracle over sequence b of the workload: for every IndexShare group the indexer
    over its N keys, the top-k, and the attention of its L layers (and of every MTP draft
    step, on the step-1 index list).  The inputs of each call are generated before it;
    returns the seconds spent inside the oracle calls."""
    import numpy as np
    import synth
    from synth import configs as C
    elapsed = 0.0
    for g in range(w.groups):
        iq = synth.int17_bf16(w.key(synth.KIND_IQ, g), (w.B, w.T, 32, 128))[b:b + 1]
        wt = synth.pow2_f32(w.key(synth.KIND_W, g), (w.B, w.T, 32))[b:b + 1]
        ik = synth.int17_bf16(w.key(synth.KIND_IK, g), index=synth.rows_index(
            np.arange(b * w.N, (b + 1) * w.N), 128)).reshape(1, w.N, 128)
        t0 = time.perf_counter()
        sc = o.index_score(iq, wt, ik, w.q_pos0).astype(np.float32)
        idx = o.topk(sc, w.q_pos0, w.k)
        elapsed += time.perf_counter() - t0
        for t in range(w.T):
            rows = idx[0, t][idx[0, t] >= 0]
            local = np.full((1, 1, w.k), -1, np.int32)
            local[0, 0, :len(rows)] = np.arange(len(rows))
            for l in range(w.L):
                kv = synth.normal_bf16(w.key(synth.KIND_KV, g, l), index=synth.rows_index(
                    b * w.N + rows.astype(np.uint64), 576)).reshape(1, len(rows), 576)
                for st in range(w.steps):
                    q = synth.normal_bf16(w.key(synth.KIND_Q, g, l, st), index=synth.rows_index(
                        np.array([b * w.T + t]), w.H * 576)).reshape(1, 1, w.H, 576)
                    t0 = time.perf_counter()
                    o.sparse_attn(q, kv, local, C.SCALE)
                    elapsed += time.perf_counter() - t0
    return elapsed


def cpu_baseline(w, n_seq):
    """The oracle as it stands on n_seq whole sequences of the workload (every group,
    layer and draft step), timed on this host with one thread; tokens/s."""
    import oracle
    o = oracle.default()
    n_seq = max(1, min(n_seq, w.B))
    elapsed = sum(oracle_sequence(w, b, o) for b in range(n_seq))
    tokens = n_seq * w.T * w.steps
    cpu = host_cpu()
    return {"value": tokens / elapsed, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "host_cpu": cpu["model"], "host_logical_cores": cpu["logical_cores"],
            "sample": f"{n_seq} of {w.B} sequences of {w.name}, whole (all {w.groups} IndexShare group(s): "
                      f"indexer over {w.N} keys, top-{w.k}, {w.L} attention layer(s) x {w.steps} step(s)); "
                      f"single-threaded C oracle in double precision; inputs generated outside the timed "
                      f"region; {tokens} token(s) in {elapsed:.1f} s"}


def workload_config(w, world: int) -> dict:
    """The `config` object of the bench line: the workload and how it is run (the same in
    both arms)."""
    return {"workload": w.name, "B": w.B, "T": w.T, "N": w.N, "k": w.k, "H": w.H, "L": w.L, "groups": w.groups,
            "draft_steps": w.steps, "index_keys": "e4m3" if w.index_fp8 else "bf16", "parallelism": f"dp{world}" if world > 1 else "single GPU",
            "l2": "flushed before every timed step (512 MiB write, then a 512 MiB read so the write-back is not timed)"}


def launches_per_group(w, sms: int = 148, long_per_sm: int = 4) -> int:
    """libdsa kernels one dsa_group_forward launches: the indexer, the top-k and the
    attention of all layers (one launch, plus the split combine when it splits keys).  The top-k is one kernel for rows a cluster holds
    (decode shapes) and for long rows whose CTAs (one per 8192 scores) all fit the GPU at
    once (a cooperative launch: `long_per_sm` of them per SM); otherwise a select and a
    compact kernel, plus a histogram kernel when the indexer does not count the first
    digit.  Mirrors the shape rules of the library (topk_cluster_plan, launch_topk)."""
    rows = w.B * w.T
    vmax = min(w.N, w.q_pos0 + w.T)
    cluster = False
    for c in (1, 2, 4, 8):
        per = -(-vmax // (c * 1024))
        kp = 4 if per <= 4 else 8 if per <= 8 else 16 if per <= 16 else 32 if per <= 32 else 0
        if kp == 0 or (kp == 32 and c < 8):
            continue
        cluster = rows * c <= sms
        break
    nchunks = -(-w.N // 8192)
    long_rows = nchunks <= 512 and rows * nchunks <= long_per_sm * sms
    fused_hist = w.T == 1 and w.B <= sms
    topk = 1 if (cluster or long_rows) else (2 if fused_hist else 3)
    return 1 + topk + attn_launches(w, sms)


def attn_launches(w, sms: int = 148) -> int:
    """Launches of one attention call over the group's L layers: the attention kernel, and
    the split combine when the (row, layer) units are few enough for their keys to be split
    over several CTAs (mirrors attn_num_splits: at most one CTA per SM in all)."""
    units = w.B * w.T * w.L
    return 2 if (w.k > 64 and 2 * units <= sms) else 1


def step_launches(w, micro: bool) -> int:
    """libdsa kernels of one step: per group, per micro-batch (two halves of the batch when
    the step is micro-batched), launches_per_group of that micro-batch; every MTP draft
    step after the first adds one attention call (L = 1)."""
    from synth import configs as C
    if not micro:
        return (launches_per_group(w) + (w.steps - 1) * attn_launches(C.scaled(w, L=1))) * w.groups
    b0 = (w.B + 1) // 2
    halves = [C.scaled(w, B=b0), C.scaled(w, B=w.B - b0)]
    return sum(launches_per_group(h, sms=148 // 4) for h in halves if h.B > 0) * w.groups


def ncu_case(kind: str) -> None:
    """A few launches of one kernel, sized for an ncu capture (a few GB on the device):
      indexer, topk   the decode128k shapes (268 MB of keys, 4 MB of scores);
      indexer_fp8     the decode128k indexer over E4M3 keys and queries (134 MB of keys);
      attn            32 (row, layer) units as in the decode128k step (4 key splits each)
                      over caches of 65536 rows (2.4 GB, larger than L2);
      attn_mtp        16 units as in an MTP draft step, run once first so that the 37.7 MB
                      of selected rows are in L2, as in draft steps 2..7;
      indexer_prefill 512 prefill queries (causal, after 126976 cached tokens) over the
                      131072-token key cache, QG = 8 tensor-core tiles;
      topk_1m         the decode1m select: 2 rows of 1,048,576 scores, first digit counted
                      by the indexer as in the step;
      verify          the MTP verify step: 16 x 7 draft positions over a 151552-token
                      vocabulary (136 MB of p and q)."""
    import torch
    import synth
    import synth.device as sd
    import sparse_long_context_score_b200 as dsa
    from synth import configs as C
    w = C.WORKLOADS["decode128k"]
    bf = torch.bfloat16
    launches = 3
    if kind in ("indexer", "topk"):
        iq = sd.int17_bf16(torch.empty(w.B, 1, 32, 128, dtype=bf, device="cuda"), w.key(synth.KIND_IQ))
        wt = sd.pow2_f32(torch.empty(w.B, 1, 32, dtype=torch.float32, device="cuda"), w.key(synth.KIND_W))
        ik = sd.int17_bf16(torch.empty(w.B, w.N, 128, dtype=bf, device="cuda"), w.key(synth.KIND_IK))
        sc = torch.empty(w.B, 1, w.N, dtype=torch.float32, device="cuda")
        idx = torch.empty(w.B, 1, w.k, dtype=torch.int32, device="cuda")
        ws = dsa.workspace(w.B, 1, w.N, w.k, w.H, w.L)
        dsa.dsa_index_score(iq, wt, ik, w.q_pos0, scores=sc)
        for _ in range(launches):
            if kind == "indexer":
                dsa.dsa_index_score(iq, wt, ik, w.q_pos0, scores=sc)
            else:
                dsa.dsa_topk(sc, w.q_pos0, w.k, idx=idx, ws=ws)
    elif kind == "indexer_fp8":
        iq = sd.int17_e4m3(torch.empty(w.B, 1, 32, 128, dtype=torch.uint8, device="cuda"), w.key(synth.KIND_IQ))
        wt = sd.pow2_f32(torch.empty(w.B, 1, 32, dtype=torch.float32, device="cuda"), w.key(synth.KIND_W))
        ik = sd.int17_e4m3(torch.empty(w.B, w.N, 128, dtype=torch.uint8, device="cuda"), w.key(synth.KIND_IK))
        sc = torch.empty(w.B, 1, w.N, dtype=torch.float32, device="cuda")
        for _ in range(launches + 1):
            dsa.dsa_index_score_e4m3(iq, wt, ik, w.q_pos0, scores=sc)
    elif kind == "indexer_prefill":
        wp = C.WORKLOADS["prefill"]
        T = 512
        iq = sd.int17_bf16(torch.empty(1, T, 32, 128, dtype=bf, device="cuda"), wp.key(synth.KIND_IQ))
        wt = sd.pow2_f32(torch.empty(1, T, 32, dtype=torch.float32, device="cuda"), wp.key(synth.KIND_W))
        ik = sd.int17_bf16(torch.empty(1, wp.N, 128, dtype=bf, device="cuda"), wp.key(synth.KIND_IK))
        sc = torch.empty(1, T, wp.N, dtype=torch.float32, device="cuda")
        for _ in range(launches):
            dsa.dsa_index_score(iq, wt, ik, wp.q_pos0, scores=sc)
    elif kind == "topk_1m":
        w1 = C.WORKLOADS["decode1m"]
        iq = sd.int17_bf16(torch.empty(w1.B, 1, 32, 128, dtype=bf, device="cuda"), w1.key(synth.KIND_IQ))
        wt = sd.pow2_f32(torch.empty(w1.B, 1, 32, dtype=torch.float32, device="cuda"), w1.key(synth.KIND_W))
        ik = sd.int17_bf16(torch.empty(w1.B, w1.N, 128, dtype=bf, device="cuda"), w1.key(synth.KIND_IK))
        q = sd.normal_bf16(torch.empty(w1.B, 1, w1.H, 576, dtype=bf, device="cuda"), w1.key(synth.KIND_Q))
        kv = sd.normal_bf16(torch.empty(w1.B, w1.N, 576, dtype=bf, device="cuda"), w1.key(synth.KIND_KV))
        ws = dsa.workspace(w1.B, 1, w1.N, w1.k, w1.H, 1)
        for _ in range(launches):  # the group call: indexer (with the first digit) -> top-k -> attention
            dsa.dsa_group_forward(iq, wt, ik, [q], [kv], w1.q_pos0, w1.k, C.SCALE, ws=ws)
    elif kind == "verify":
        wm = C.WORKLOADS["mtp"]
        B, S, V = wm.B, wm.steps, VERIFY_VOCAB
        zp = sd.normal_bf16(torch.empty(B, S, V, dtype=bf, device="cuda"), wm.key(synth.KIND_Q, 1, 0))
        zq = sd.normal_bf16(torch.empty(B, S, V, dtype=bf, device="cuda"), wm.key(synth.KIND_Q, 1, 1))
        pr = torch.softmax(zp.float() * 2.0, dim=-1).contiguous()
        qr = torch.softmax(zq.float() * 2.6 + zp.float(), dim=-1).contiguous()
        draft = torch.argmax(qr, dim=-1).to(torch.int32).contiguous()
        u = sd.unit_f32(torch.empty(B, S, dtype=torch.float32, device="cuda"), wm.key(synth.KIND_SCORES, 1, 0)) + 0.5
        u2 = sd.unit_f32(torch.empty(B, S, dtype=torch.float32, device="cuda"), wm.key(synth.KIND_SCORES, 1, 1)) + 0.5
        for _ in range(launches):
            dsa.dsa_verify(pr, qr, draft, u, u2)
    else:
        rows, n = (32, 65536) if kind == "attn" else (16, 262151)
        q = sd.normal_bf16(torch.empty(rows, 1, w.H, 576, dtype=bf, device="cuda"), w.key(synth.KIND_Q))
        kv = sd.normal_bf16(torch.empty(rows, n, 576, dtype=bf, device="cuda"), w.key(synth.KIND_KV))
        g = torch.Generator(device="cpu").manual_seed(w.key(synth.KIND_SCORES) & 0x7FFFFFFF)
        idx = torch.stack([torch.sort(torch.randperm(n - 7, generator=g)[:w.k]).values for _ in range(rows)])
        idx = idx.view(rows, 1, w.k).to(torch.int32).cuda()
        out = torch.empty(rows, 1, w.H, 512, dtype=torch.float32, device="cuda")
        ws = dsa.workspace(rows, 1, n, w.k, w.H, 1)
        for _ in range(launches):
            dsa.dsa_sparse_attn(q, kv, idx, C.SCALE, out=out, ws=ws)
    torch.cuda.synchronize()
    err = dsa.dsa_device_error()
    print(f"ncu case {kind}: {launches} launches, device error word {err}")
    if err:
        sys.exit(1)


def run_context_sharded(args, rank, world, device, w):
    """The decode step of `w` with every sequence's cached tokens spread over the ranks
    (contiguous shards): per group, the sharded group of sparse_long_context_score_b200.sharded
    (local indexer and top-k, candidate all-gather and merge, local attention, partial
    all-gather and merge).  Eager calls (NCCL collectives between the kernels), L2 flushed
    before every step, CUDA events on the stream, the max over ranks.  Returns (ms per
    step, clock record)."""
    import torch
    import synth
    import synth.device as sd
    from sparse_long_context_score_b200 import sharded
    from synth import configs as C
    torch.cuda.set_device(device)
    offset, n = sharded.shard_bounds(w.N, world)[rank]
    bf = torch.bfloat16
    groups = []
    for g in range(w.groups):
        # the shard of each cache: positions [offset, offset + n) of the same seeded tensors
        ik = torch.empty(w.B, n, 128, dtype=bf, device=device)
        kvs = [torch.empty(w.B, n, 576, dtype=bf, device=device) for _ in range(w.L)]
        for b in range(w.B):
            sd.int17_bf16(ik[b], w.key(synth.KIND_IK, g), offset=(b * w.N + offset) * 128)
            for l in range(w.L):
                sd.normal_bf16(kvs[l][b], w.key(synth.KIND_KV, g, l), offset=(b * w.N + offset) * 576)
        iq = sd.int17_bf16(torch.empty(w.B, 1, 32, 128, dtype=bf, device=device), w.key(synth.KIND_IQ, g))
        wt = sd.pow2_f32(torch.empty(w.B, 1, 32, dtype=torch.float32, device=device), w.key(synth.KIND_W, g))
        qs = [sd.normal_bf16(torch.empty(w.B, 1, w.H, 576, dtype=bf, device=device), w.key(synth.KIND_Q, g, l))
              for l in range(w.L)]
        groups.append((iq, wt, ik, qs, kvs))
    comm = sharded.TorchComm() if world > 1 else None
    ops = sharded.cuda_ops()

    class _Self:  # one rank: the all-gather of a tensor is that tensor with a leading axis
        @staticmethod
        def all_gather(t):
            return t.unsqueeze(0)
    comm = comm or _Self()
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    flush_rd = torch.zeros(512 << 20, dtype=torch.uint8, device=device)

    def step():
        for iq, wt, ik, qs, kvs in groups:
            sharded.sharded_group_forward(comm, ops, iq, wt, ik, qs, kvs, w.q_pos0, offset, w.k, C.SCALE)

    times = []
    with ClockSampler(torch.cuda.current_device()) as clk:
        for i in range(args.warmup + args.steps):
            flush.zero_()
            flush_rd.view(torch.int64).sum()
            if world > 1:
                torch.distributed.barrier()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            step()
            b.record()
            torch.cuda.synchronize()
            if i >= args.warmup:
                times.append(a.elapsed_time(b))
    import sparse_long_context_score_b200 as dsa
    if dsa.dsa_check_device_status() != 0:
        raise RuntimeError("device status after the context-sharded steps")
    ms = max_over_ranks([sum(times) / len(times)], world, device)[0]
    return ms, clk.summary()


def main():
    args = parse()
    if args.ncu_case:
        ncu_case(args.ncu_case)
        return
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    from synth import configs as C
    w = C.WORKLOADS[args.workload]
    metric = "DSA group decode tokens/s"
    if args.impl == "reference":
        if rank == 0:
            import oracle
            o = oracle.default()
            times = []
            for step in range(args.warmup + args.steps):
                dt = oracle_sequence(w, step % w.B, o)
                if step >= args.warmup:
                    times.append(dt)
            step_s = sum(times) / len(times)
            v = w.T * w.steps / step_s
            cpu = host_cpu()
            print(json.dumps({"impl": "reference", "metric": metric, "value": v, "unit": "tokens/s",
                              "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                              "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
                              "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                              "config": workload_config(w, args.gpus),
                              "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                               "host_cpu": cpu["model"], "host_logical_cores": cpu["logical_cores"],
                                               "sample": f"each step is one whole sequence of {w.name} (sequence "
                                                         f"step mod {w.B}), the single-threaded C oracle in double "
                                                         f"precision; inputs generated outside the timed region"},
                              "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                                      "d2h_bytes_per_step": 0}}))
        return

    import torch
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    device = torch.device("cuda", local)
    if args.shard == "context":
        wc = C.WORKLOADS[args.workload if args.workload != "decode128k" else "decode1m"]
        ms, clocks = run_context_sharded(args, rank, world, device, wc)
        if rank == 0:
            tokens = wc.B * wc.T
            cfg = workload_config(wc, world)
            cfg["parallelism"] = f"context shards x{world}" if world > 1 else "single GPU (one context shard)"
            print(json.dumps({"metric": metric, "value": tokens / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world,
                              "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                              "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
                              "data": "synthetic", "config": cfg, "clocks": clocks,
                              "mode": "context-sharded decode (eager calls, NCCL all-gathers between kernels)"}))
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        return
    w, r = run_ours(args, rank, world, device)
    step_bytes, idx_bytes, score_bytes = algorithmic(w)
    tokens = w.B * w.T * w.steps * world
    value = job_throughput(w.B * w.T * w.steps, world, r["step_ms"])
    peak, peak_kind = peaks()
    achieved = idx_bytes / (r["idx_ms"] * 1e-3) / 1e9
    step_gbs = step_bytes / (r["step_ms"] * 1e-3) / 1e9
    line = {
        "metric": metric, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r["step_ms"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(w, world),
        "clocks": r["clocks"],
        "e2e": {"value": tokens / (r["e2e_ms"] * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": r["h2d"],
                "d2h_bytes_per_step": r["d2h"], "calls": "eager: the C ABI called per step",
                "graph_replay_value": tokens / (r["e2e_graph_ms"] * 1e-3)},
        "gpu_launches": step_launches(w, r["schedule"].startswith("two")) * args.steps,
        "roofline": {"kernel": "indexer", "bound": "hbm", "achieved": achieved, "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": profiled_traffic("indexer_tc.cu", w.name), "launch_us": r["idx_ms"] * 1e3,
                     "algorithmic_bytes_per_launch": idx_bytes, "score_write_bytes_per_launch": score_bytes},
        "step": {"hbm_gbs": step_gbs, "roofline_frac": step_gbs / peak, "algorithmic_bytes": step_bytes,
                 "schedule": r["schedule"]},
    }
    if not args.no_extra and args.workload == "decode128k":
        extra = {"mtp_verify": run_verify(args, device, peak)}
        for name in ("decode1m", "mtp", "prefill", "decode128k_fp8"):
            we, r2 = run_ours(args, rank, world, device, w=C.WORKLOADS[name], e2e=False)
            b2, ib2, _ = algorithmic(we)
            ms, ims = r2["step_ms"], r2["idx_ms"]
            toks = we.B * we.T * we.steps * world
            ent = {"tokens_per_s": toks / (ms * 1e-3), "ms_per_step": ms, "step_hbm_gbs": b2 / (ms * 1e-3) / 1e9,
                   "step_roofline_frac": b2 / (ms * 1e-3) / 1e9 / peak, "indexer_launch_us": ims * 1e3,
                   "indexer_hbm_gbs": ib2 / (ims * 1e-3) / 1e9, "schedule": r2["schedule"],
                   "clocks_sm_mhz": r2["clocks"].get("sm_mhz"),
                   "clock_reasons": r2["clocks"].get("reasons")}
            if name == "prefill":
                fl = prefill_indexer_flops(we)
                ent["indexer_tflops"] = fl / (ims * 1e-3) / 1e12
                ent["indexer_tflops_frac_of_bf16_peak"] = ent["indexer_tflops"] / _bf16_peak()
            extra[name] = ent
        line["other_workloads"] = extra
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_sample)
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
