#!/usr/bin/env python
"""Throughput of the MISA token indexer on B200 (one JSON line on rank 0).

Workload (N = 1): DeepSeek-V3.2-shaped indexer decode -- 32 sequences x 1
query, L = 32768 bf16 keys each, d = 128, H = 64 indexer heads of which h = 8
are routed per query from B = 128 mean-pooled key blocks, top-k = 2048.  One
step is the whole per-query path: router, routed token scoring, top-k (the
block statistics are per-cache state maintained on KV append; they are timed
separately).  The metric is indexed q.k pairs per second = sum over queries of
the keys each query's top-k decision covers, divided by the step time.

Multi-GPU (torchrun): every rank runs its own batch of the same shape (weak
scaling, no collective on the data path); the step time is the max over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--quick]

`--impl reference` times the fp64 CPU oracle (this repository's reference
implementation of the same path) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import make_workload  # noqa: E402

WORKLOAD = "dsv32_decode_L32768"
METRIC = "indexed q.k pairs/s (top-k=2048, L=32K, MISA h=8 of H=64)"
UNIT = "pairs/s"
L2_FLUSH_BYTES = 256 << 20
SCORE_SOURCES = ["sparse_attention_token_misa_b200/csrc/score_tc.cu",
                 "sparse_attention_token_misa_b200/csrc/misa_device.cuh"]


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def bench_config(wl, ws_n: int) -> dict:
    """The `config` object both arms print (identical keys and values)."""
    return {"workload": WORKLOAD, "queries": wl.T, "L": wl.L, "H": wl.H, "h": wl.h, "B": wl.B, "k": wl.k, "d": 128,
            "parallelism": f"dp{ws_n} (independent batches)",
            "l2": "not flushed between steps: the keys (T x L x 256 B = 268 MB) exceed L2 (126 MB); "
                  "detail.*_l2_flushed_ms repeat the timings with a 256 MiB write before every step"}


def decode_step_bytes(T: int, L: int, H: int, h: int, B: int, k: int) -> int:
    """Algorithmic HBM bytes of one MISA decode step (router + routed scoring +
    top-k), each byte the method must move once: the keys, the bf16 hi/lo block
    means and all heads' query rows the router reads, the head weights, the
    fp32 score rows written by the scoring and read back by the top-k, the
    indices written (the routed heads and rows re-read from L2 are not
    counted)."""
    M = (L + B - 1) // B
    return (T * L * 256 + T * M * 128 * 2 * 2 + T * H * 256 + T * H * 4 + 2 * T * L * 4 + T * k * 4)


def fused_kernel_bytes(T: int, L: int, H: int, h: int, B: int) -> int:
    """Algorithmic HBM bytes of the router + scoring kernel of the decode step:
    the keys, the bf16 hi/lo block means, all heads' query rows and weights,
    the fp32 score rows written, the heads and importances written."""
    M = (L + B - 1) // B
    return T * L * 256 + T * M * 128 * 2 * 2 + T * H * 256 + T * H * 4 + T * L * 4 + T * h * 4 + T * H * 4


def dagger_step_bytes(T: int, L: int, H: int, B: int, kp: int, k: int) -> int:
    """MISA-dagger decode step: the routed coarse pass (as decode_step_bytes with
    k' outputs), the k' candidate ids read back, the gathered candidate key rows,
    the k' rerank scores written and read, the final indices."""
    return (decode_step_bytes(T, L, H, 8, B, kp) + T * kp * 4 + T * kp * 256 + 2 * T * kp * 4 + T * k * 4)


def hisa_step_bytes(T: int, L: int, H: int, B: int, m: int, k: int) -> int:
    """HISA decode step: bf16 hi/lo block means and the query rows (block
    filter), block scores written and read, the candidate list written and read
    twice (scoring, top-k id map), the candidate key rows, their scores written
    and read, the indices."""
    M = (L + B - 1) // B
    n = m * B
    return (T * M * 128 * 2 * 2 + T * H * 256 + T * H * 4 + 2 * T * M * 4 + 3 * T * n * 4 + T * n * 256
            + 2 * T * n * 4 + T * k * 4)


def router_flops(wl) -> float:
    """Tensor-core flops of the router: for every query and every block visible
    to its routing decision, H dot products of 128 against the block mean's bf16
    hi and lo halves (2 flops per multiply-add)."""
    pl = wl.prefix_len.numpy().astype(np.int64)
    first = pl[(np.arange(wl.T) // wl.q_block) * wl.q_block]
    M = (wl.L + wl.B - 1) // wl.B
    vis = np.where(first >= wl.L, M, first // wl.B)
    return float(vis.sum()) * wl.H * 128 * 2 * 2


def _source_hash(paths) -> str:
    h = hashlib.sha256()
    for rel in paths:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _traffic_for(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel)
    if not e or e.get("workload") != workload or e.get("source_sha256_16") != _source_hash(e.get("sources", [])):
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        if not self.lines:
            return None
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        under_load = [s for s in sm if s > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(under_load), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def rank_batch(rank: int):
    """The batch rank `rank` indexes: the bench workload's shape on every rank
    (weak scaling, no data shared between ranks); rank 0 is the named workload,
    rank r > 0 the same shape drawn with seed 2 + 1000 r."""
    if rank == 0:
        return make_workload(WORKLOAD)
    from workloads import make_decode
    return make_decode(WORKLOAD, 2 + 1000 * rank, T=32, L=32768, H=64, h=8, B=128, k=2048, n_planted=16)


def reduce_max(x: float, dist, device) -> float:
    """Max of a per-rank time over all ranks (identity without a process group)."""
    if not dist:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def selection_agreement(a, b):
    """(mean IoU, mean recovery |a & b| / |b|) over the rows of two [T, k]
    index arrays (-1: empty slot); informational, computed on the host."""
    a = np.asarray(a.cpu() if hasattr(a, "cpu") else a)
    b = np.asarray(b.cpu() if hasattr(b, "cpu") else b)
    ious, recs = [], []
    for ra, rb in zip(a, b):
        sa, sb = set(ra[ra >= 0].tolist()), set(rb[rb >= 0].tolist())
        inter, uni = len(sa & sb), len(sa | sb)
        ious.append(inter / uni if uni else 1.0)
        recs.append(inter / len(sb) if sb else 1.0)
    return float(np.mean(ious)), float(np.mean(recs))


def planted_recall(idx, planted):
    """Fraction of the planted key positions that the indices select."""
    idx = np.asarray(idx.cpu() if hasattr(idx, "cpu") else idx)
    planted = np.asarray(planted)
    if planted.size == 0:
        return None
    hits = sum(len(set(planted[t].tolist()) & set(idx[t].tolist())) for t in range(planted.shape[0]))
    return hits / planted.size


def _time_steps(step, steps, flush, stream, marks=None, after=None):
    """Per-step CUDA-event timing with an untimed L2 flush before every step.
    marks: optional list of names; step(ev) records intermediate events.
    after: called after every step (its events have completed)."""
    tot = 0.0
    marks = list(marks or [])
    parts = {m: 0.0 for m in marks}
    n_ev = max(2, len(marks) + 1)  # start, one event between consecutive parts, end
    for _ in range(steps):
        flush()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
        evs[0].record(stream)
        step(evs[1:-1])
        evs[-1].record(stream)
        torch.cuda.synchronize()
        tot += evs[0].elapsed_time(evs[-1])
        for i, m in enumerate(marks):
            parts[m] += evs[i].elapsed_time(evs[i + 1])
        if after:
            after()
    return tot, parts


def run_cuda(args):
    import sparse_attention_token_misa_b200 as misa

    ws_n, rank, local = _dist()
    torch.cuda.set_device(local)
    dist = None
    if ws_n > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()

    wl = rank_batch(rank)
    q, w, keys = wl.q.to(dev), wl.w.to(dev), wl.keys.to(dev)
    seq_of, plen = wl.seq_of.to(dev), wl.prefix_len.to(dev)
    T, H, h, L, B, k = wl.T, wl.H, wl.h, wl.L, wl.B, wl.k
    pairs = int(wl.prefix_len.sum())

    means = misa.block_stats(keys, B, split=True)
    ixf = misa.MisaIndexer(T, H, h, L, B, k, q_block=1, device=dev, fused=True)
    ix = misa.MisaIndexer(T, H, h, L, B, k, q_block=1, device=dev)
    dense = misa.DenseIndexer(T, H, L, k, device=dev)
    flush_buf = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def flush():
        flush_buf.fill_(1.0)

    def no_flush():
        pass

    # warm-up (eager), then every variant as one CUDA graph
    from sparse_attention_token_misa_b200.indexer import capture_graph
    for _ in range(args.warmup):
        ixf.run(q, w, keys, means, seq_of, plen)
        ix.run(q, w, keys, means, seq_of, plen)
        dense.run(q, w, keys, seq_of, plen)
    torch.cuda.synchronize()
    inner = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)]

    def misa_graph_body():
        inner[0].record()
        ix.route(q, w, means, seq_of, plen)
        inner[1].record()
        ix.score(q, w, keys, seq_of, plen)
        inner[2].record()
        ix.select(plen)
        inner[3].record()

    # the timed step: misa_index_decode (router + scoring kernel, the top-k
    # behind it), one graph; beside it the same without the top-k (the fused
    # kernel alone, for its roofline) and the three separate calls (route,
    # score, top-k), whose per-kernel split comes from a graph with timing
    # events recorded between the stages
    g_step = capture_graph(lambda: ixf.run(q, w, keys, means, seq_of, plen))
    g_rs = capture_graph(lambda: ixf.route_score(q, w, keys, means, seq_of, plen))
    ix.capture(q, w, keys, means, seq_of, plen)
    g_split = capture_graph(misa_graph_body)
    dense.capture(q, w, keys, seq_of, plen)
    for _ in range(args.warmup):
        g_step.replay()
        g_rs.replay()
        ix.g_step.replay()
        g_split.replay()
    torch.cuda.synchronize()
    for ws_ in (ixf.ws_decode, ix.ws, ix.ws_route):
        misa.error_reset(ws_)

    parts = {"route": 0.0, "score": 0.0, "topk": 0.0}

    def after_split():
        parts["route"] += inner[0].elapsed_time(inner[1])
        parts["score"] += inner[1].elapsed_time(inner[2])
        parts["topk"] += inner[2].elapsed_time(inner[3])

    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t0 = time.perf_counter()
        tot_ms, _ = _time_steps(lambda evs: g_step.replay(), args.steps, no_flush, stream)
        wall = time.perf_counter() - t0
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    ms_step = reduce_max(tot_ms / args.steps, dist, dev)
    rs_ms = _time_steps(lambda evs: g_rs.replay(), args.steps, no_flush, stream)[0] / args.steps
    flushed_ms = _time_steps(lambda evs: g_step.replay(), args.steps, flush, stream)[0] / args.steps
    three_ms = _time_steps(lambda evs: ix.g_step.replay(), args.steps, no_flush, stream)[0] / args.steps
    three_flushed_ms = _time_steps(lambda evs: ix.g_step.replay(), args.steps, flush, stream)[0] / args.steps
    split_ms, _ = _time_steps(lambda evs: g_split.replay(), args.steps, no_flush, stream, after=after_split)
    dev_err = misa.error_query(ixf.ws_decode) | misa.error_query(ix.ws) | misa.error_query(ix.ws_route)
    if dev_err:
        raise RuntimeError(f"device error word {dev_err:#x}")
    if not torch.equal(ixf.idx, ix.idx) and torch.equal(ixf.heads, ix.heads):
        raise RuntimeError("fused and three-call indices differ on equal heads")

    # the dense 64-head indexer and the block statistics on the same batch
    # (same protocol)
    dense_ms, dparts = _time_steps(lambda evs: (dense.g_score.replay(), evs[0].record(stream),
                                                dense.g_select.replay()), args.steps, no_flush, stream,
                                   marks=["score", "topk"])
    dense_one_ms, _ = _time_steps(lambda evs: dense.g_step.replay(), args.steps, no_flush, stream)
    stats_ms, _ = _time_steps(lambda evs: misa.block_stats(keys, B, out=means[0], out_hi=means[1], out_lo=means[2]),
                              args.steps, no_flush, stream)
    dense_ms /= args.steps
    dense_one_ms /= args.steps
    stats_ms /= args.steps

    # e2e through the public API: the step's inputs (q, w, seq_of, prefix_len)
    # packed in one pinned host buffer and copied in one transfer, the indexer
    # on device views of the copy, the indices copied back -- one graph
    e2e_parts = [wl.q, wl.w, wl.seq_of, wl.prefix_len]
    offs, nbytes = [], 0
    for t_ in e2e_parts:
        offs.append(nbytes)
        nbytes += (t_.numel() * t_.element_size() + 255) // 256 * 256
    stage_h = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    stage_d = torch.empty(nbytes, dtype=torch.uint8, device=dev)

    def _view(buf, i):
        t_ = e2e_parts[i]
        n_ = t_.numel() * t_.element_size()
        return buf[offs[i]:offs[i] + n_].view(t_.dtype).view(t_.shape)

    for i, t_ in enumerate(e2e_parts):
        _view(stage_h, i).copy_(t_)
    q_d, w_d, so_d, pl_d = (_view(stage_d, i) for i in range(4))
    idx_h = torch.empty((T, k), dtype=torch.int32).pin_memory()
    ix_e = misa.MisaIndexer(T, H, h, L, B, k, q_block=1, device=dev, fused=True)

    def e2e_eager():
        stage_d.copy_(stage_h, non_blocking=True)
        out = ix_e.run(q_d, w_d, keys, means, so_d, pl_d)
        idx_h.copy_(out, non_blocking=True)

    g_e2e = capture_graph(e2e_eager)
    for _ in range(3):
        g_e2e.replay()
    torch.cuda.synchronize()
    e2e_ms, _ = _time_steps(lambda evs: g_e2e.replay(), args.steps, no_flush, stream)
    e2e_ms = reduce_max(e2e_ms / args.steps, dist, dev)
    e2e_eager_ms, _ = _time_steps(lambda evs: e2e_eager(), args.steps, no_flush, stream)
    e2e_eager_ms /= args.steps
    if not torch.equal(idx_h.cuda(dev), ixf.idx):
        raise RuntimeError("e2e indices differ from the device-timed step")
    h2d = stage_h.numel()   # q, w, seq_of, prefix_len, each padded to 256 bytes
    d2h = idx_h.numel() * 4
    # selection agreement with the dense indexer on the same batch (for information)
    sel_iou, sel_rec = selection_agreement(ixf.idx, dense.idx)
    selection = {"misa8_iou_vs_dense64": sel_iou, "misa8_recovery_of_dense64": sel_rec,
                 "misa8_planted_recall": planted_recall(ixf.idx, wl.planted),
                 "dense64_planted_recall": planted_recall(dense.idx, wl.planted)}

    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    hbm_gbs, tc_tflops, peak_kind = _peaks()
    score_ms = parts["score"] / args.steps
    # algorithmic bytes of one launch of the router + scoring kernel
    fk_bytes = fused_kernel_bytes(T, L, H, h, B)
    achieved = fk_bytes / (rs_ms * 1e-3) / 1e9
    traffic = _traffic_for("decode_fused_kernel", WORKLOAD)
    # the three-call path's scoring kernel: K once, the routed query rows and
    # weights, the fp32 score rows written
    score_bytes = T * L * 128 * 2 + T * h * (128 * 2 + 4 + 4) + T * L * 4
    step_bytes = decode_step_bytes(T, L, H, h, B, k)
    value = pairs * ws_n / (ms_step * 1e-3)
    line = {
        "metric": METRIC,
        "value": value,
        "unit": UNIT,
        "n_gpus": ws_n,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; shapes of the DeepSeek-V3.2 indexer decode)",
        "config": bench_config(wl, ws_n),
        "queries_per_s": T * ws_n / (ms_step * 1e-3),
        # the work actually done: q.k products over the routed heads (MISA-8),
        # and over all heads for the dense indexer on the same batch
        "scored_head_pairs_per_s": pairs * h * ws_n / (ms_step * 1e-3),
        "dense64_scored_head_pairs_per_s": pairs * H * ws_n / (dense_one_ms * 1e-3),
        "gpu_launches": 2 * args.steps,  # router + scoring kernel, top-k kernel per step
        "timing": "CUDA events on the launching stream around one graph replay per step of misa_index_decode "
                  "(router + scoring kernel, the top-k kernel behind it); the fused kernel alone from a graph of "
                  "the same call without the top-k (detail.fused_kernel_ms); the three separate calls in "
                  "detail.three_call_* (per-kernel split from a graph with timing events between the stages)",
        "roofline": {"bound": "hbm", "kernel": "decode_fused_kernel (misa_index_decode without its top-k)",
                     "achieved": achieved, "peak": hbm_gbs, "peak_kind": f"{peak_kind} hbm copy GB/s (burst)",
                     "unit": "GB/s", "frac": achieved / hbm_gbs, "traffic": traffic,
                     "algorithmic_bytes_per_launch": fk_bytes, "launch_ms": rs_ms},
        "step_roofline": {"bound": "hbm", "what": "whole step (router + scoring kernel, top-k), one graph replay",
                          "algorithmic_bytes_per_step": step_bytes,
                          "achieved": step_bytes / (ms_step * 1e-3) / 1e9, "peak": hbm_gbs, "unit": "GB/s",
                          "frac": step_bytes / (ms_step * 1e-3) / 1e9 / hbm_gbs,
                          "frac_of_8TBps": step_bytes / (ms_step * 1e-3) / 8e12},
        "e2e": {"value": pairs * ws_n / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "how": "q/w/seq_of/prefix_len packed in one pinned host buffer -> device in one copy, "
                       "misa_index_decode on device views of it, idx -> pinned host; one CUDA graph replay per step",
                "eager_ms_per_step": e2e_eager_ms},
        "selection": selection,
        "detail": {"misa8_ms": ms_step, "misa8_l2_flushed_ms": flushed_ms, "fused_kernel_ms": rs_ms,
                   "topk_tail_ms": ms_step - rs_ms,
                   "three_call_ms": three_ms, "three_call_l2_flushed_ms": three_flushed_ms,
                   "three_call_split_ms": split_ms / args.steps,
                   "three_call_route_ms": parts["route"] / args.steps, "three_call_score_ms": score_ms,
                   "three_call_topk_ms": parts["topk"] / args.steps,
                   "three_call_score_GBps": score_bytes / (score_ms * 1e-3) / 1e9,
                   "dense64_ms": dense_one_ms, "dense64_score_ms": dparts["score"] / args.steps,
                   "dense64_topk_ms": dparts["topk"] / args.steps, "dense64_over_misa8": dense_one_ms / ms_step,
                   "block_stats_ms": stats_ms,
                   "block_stats_GBps": (T * L * 128 * 2 + T * (L // B) * 128 * 8) / (stats_ms * 1e-3) / 1e9,
                   "wall_s_timed_region": wall},
    }
    summ = clk.summary()
    if summ:
        line["clocks"] = summ
    if not args.quick and ws_n == 1:
        line["other_workloads"] = other_workloads(misa, dev, stream, flush, max(3, min(args.steps, 10)))
        del flush_buf
    if ws_n == 1:
        line["cpu_baseline"] = cpu_baseline(wl, budget_s=args.cpu_budget)
        if not args.quick and args.cpu_budget > 0:
            line["cpu_baseline"]["other_workloads"] = cpu_baselines()
    print(json.dumps(line), flush=True)


def other_workloads(misa, dev, stream, flush, steps, only=None):
    """The other four workloads through their indexers (same timing protocol)."""
    out = {}

    from sparse_attention_token_misa_b200.indexer import capture_graph

    def timed(fn):
        g = capture_graph(lambda: fn([]))
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        ms, _ = _time_steps(lambda evs: g.replay(), steps, flush, stream)
        return ms / steps

    if only in (None, "prefill"):
        out.update(_prefill(misa, dev, stream, flush, steps))
    if only in (None, "dagger"):
        out.update(_dagger(misa, dev, stream, flush, steps, timed))
        out.update(_dagger_prefill(misa, dev, stream, flush, steps, timed))
    if only in (None, "hisa"):
        out.update(_hisa(misa, dev, stream, flush, steps, timed))
    if only in (None, "quality"):
        out["selection_quality_local_inputs"] = _selection_quality(misa, dev)
    if only in (None, "attn"):
        out.update(_sparse_attention(misa, dev, stream, flush, steps, timed))
    return out


def _prefill(misa, dev, stream, flush, steps):
    out = {}
    wl = make_workload("prefill_L131072")
    q, w, keys, so, pl = (x.to(dev) for x in (wl.q, wl.w, wl.keys, wl.seq_of, wl.prefix_len))
    means = misa.block_stats(keys, wl.B, split=True)
    ix = misa.MisaIndexer(wl.T, wl.H, wl.h, wl.L, wl.B, wl.k, wl.q_block, device=dev)
    pairs = int(wl.prefix_len.sum())

    from sparse_attention_token_misa_b200.indexer import capture_graph
    inner = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)]

    def body():
        inner[0].record()
        ix.route(q, w, means, so, pl)
        inner[1].record()
        ix.score(q, w, keys, so, pl)
        inner[2].record()
        ix.select(pl)
        inner[3].record()

    g = capture_graph(body)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    parts = {"route": 0.0, "score": 0.0, "topk": 0.0}

    def after():
        parts["route"] += inner[0].elapsed_time(inner[1])
        parts["score"] += inner[1].elapsed_time(inner[2])
        parts["topk"] += inner[2].elapsed_time(inner[3])

    ms, _ = _time_steps(lambda evs: g.replay(), steps, flush, stream, after=after)
    g_step = capture_graph(lambda: ix.run(q, w, keys, means, so, pl))
    for _ in range(2):
        g_step.replay()
    torch.cuda.synchronize()
    step_ms, _ = _time_steps(lambda evs: g_step.replay(), steps, flush, stream)
    step_ms /= steps
    score_ms = parts["score"] / steps
    route_ms = parts["route"] / steps
    topk_ms = parts["topk"] / steps
    flops = 2.0 * 128 * wl.h * pairs
    rflops = router_flops(wl)
    topk_bytes = pairs * 4 + wl.T * wl.k * 4      # the visible scores read once, the indices written
    hbm, tc, kind = _peaks()
    misa_idx = ix.idx.clone()
    del ix, g, g_step
    torch.cuda.empty_cache()

    # the dense 64-head indexer on the same prefill chunk (every head scores every visible pair)
    dx = misa.DenseIndexer(wl.T, wl.H, wl.L, wl.k, device=dev)
    dx.capture(q, w, keys, so, pl)
    for _ in range(2):
        dx.g_step.replay()
    torch.cuda.synchronize()
    d_ms, dparts = _time_steps(lambda evs: (dx.g_score.replay(), evs[0].record(stream), dx.g_select.replay()),
                               steps, flush, stream, marks=["score", "topk"])
    d_one, _ = _time_steps(lambda evs: dx.g_step.replay(), steps, flush, stream)
    d_one /= steps
    d_score = dparts["score"] / steps
    dflops = 2.0 * 128 * wl.H * pairs
    iou, rec = selection_agreement(misa_idx, dx.idx)
    del dx
    torch.cuda.empty_cache()
    out["prefill_L131072"] = {
        "ms_per_step": step_ms, "pairs_per_s": pairs / (step_ms * 1e-3),
        "split_ms": ms / steps, "route_ms": route_ms, "score_ms": score_ms, "topk_ms": topk_ms,
        "score_tflops": flops / (score_ms * 1e-3) / 1e12,
        "score_frac_of_bf16_peak": flops / (score_ms * 1e-3) / 1e12 / tc,
        "route_tflops": rflops / (route_ms * 1e-3) / 1e12,
        "route_frac_of_bf16_peak": rflops / (route_ms * 1e-3) / 1e12 / tc,
        "topk_GBps": topk_bytes / (topk_ms * 1e-3) / 1e9,
        "topk_frac_of_hbm": topk_bytes / (topk_ms * 1e-3) / 1e9 / hbm,
        "step_frac_of_bf16_peak": (flops + rflops) / (step_ms * 1e-3) / 1e12 / tc,
        "algorithmic": {"score_flops": flops, "route_flops": rflops, "topk_bytes": topk_bytes,
                        "peaks": f"{kind}: {hbm} GB/s, {tc} TFLOP/s bf16 (burst)"},
        "dense64_ms": d_one, "dense64_score_ms": d_score, "dense64_topk_ms": dparts["topk"] / steps,
        "dense64_score_tflops": dflops / (d_score * 1e-3) / 1e12,
        "dense64_score_frac_of_bf16_peak": dflops / (d_score * 1e-3) / 1e12 / tc,
        "dense64_over_misa8": d_one / step_ms,
        "dense64_score_over_misa8_score": d_score / score_ms,
        "misa8_iou_vs_dense64": iou, "misa8_recovery_of_dense64": rec}
    return out


def _dagger_prefill(misa, dev, stream, flush, steps, timed):
    """MISA-dagger on the causal 128K prefill: coarse top-8192 of the routed
    scores, all-head rerank of the candidates, top-2048."""
    out = {}
    wl = make_workload("prefill_L131072")
    q, w, keys, so, pl = (x.to(dev) for x in (wl.q, wl.w, wl.keys, wl.seq_of, wl.prefix_len))
    means = misa.block_stats(keys, wl.B, split=True)
    dg = misa.MisaDaggerIndexer(wl.T, wl.H, wl.h, wl.L, wl.B, 8192, wl.k, wl.q_block, device=dev)
    ms = timed(lambda evs: dg.run(q, w, keys, means, so, pl))
    out["prefill_L131072_dagger_kp8192"] = {"ms_per_step": ms, "pairs_per_s": int(wl.prefix_len.sum()) / (ms * 1e-3)}
    return out


def _dagger(misa, dev, stream, flush, steps, timed):
    out = {}
    wl = make_workload("glm5_dagger_decode_L65536")
    q, w, keys, so, pl = (x.to(dev) for x in (wl.q, wl.w, wl.keys, wl.seq_of, wl.prefix_len))
    means = misa.block_stats(keys, wl.B, split=True)
    dg3 = misa.MisaDaggerIndexer(wl.T, wl.H, wl.h, wl.L, wl.B, wl.kp, wl.k, device=dev)
    ms3 = timed(lambda evs: dg3.run(q, w, keys, means, so, pl))
    dg = misa.MisaDaggerIndexer(wl.T, wl.H, wl.h, wl.L, wl.B, wl.kp, wl.k, device=dev, fused=True)
    ms = timed(lambda evs: dg.run(q, w, keys, means, so, pl))
    dx = misa.DenseIndexer(wl.T, wl.H, wl.L, wl.k, device=dev)
    dx.run(q, w, keys, so, pl)
    torch.cuda.synchronize()
    iou, rec = selection_agreement(dg.idx, dx.idx)
    hbm, _, _ = _peaks()
    nb = dagger_step_bytes(wl.T, wl.L, wl.H, wl.B, wl.kp, wl.k)
    out["glm5_dagger_decode_L65536"] = {"ms_per_step": ms, "pairs_per_s": int(wl.prefix_len.sum()) / (ms * 1e-3),
                                        "roofline": {"bound": "hbm", "algorithmic_bytes_per_step": nb,
                                                     "achieved": nb / (ms * 1e-3) / 1e9, "peak": hbm,
                                                     "unit": "GB/s", "frac": nb / (ms * 1e-3) / 1e9 / hbm},
                                        "coarse_stage": "misa_index_decode (router + scoring kernel, top-k')",
                                        "three_call_coarse_ms_per_step": ms3,
                                        "iou_vs_dense32": iou, "recovery_of_dense32": rec,
                                        "planted_recall": planted_recall(dg.idx, wl.planted),
                                        "dense32_planted_recall": planted_recall(dx.idx, wl.planted)}
    return out


def _hisa(misa, dev, stream, flush, steps, timed):
    out = {}
    wl = make_workload("hisa_decode_L131072")
    q, w, keys, so, pl = (x.to(dev) for x in (wl.q, wl.w, wl.keys, wl.seq_of, wl.prefix_len))
    dx = misa.DenseIndexer(wl.T, wl.H, wl.L, wl.k, device=dev)
    dense_idx = dx.run(q, w, keys, so, pl).clone()
    for B, m in ((128, 64), (64, 128)):
        means = misa.block_stats(keys, B, split=True)
        hx = misa.HisaIndexer(wl.T, wl.H, wl.L, B, m, wl.k, device=dev)
        ms = timed(lambda evs: hx.run(q, w, keys, means, so, pl))
        iou, rec = selection_agreement(hx.idx, dense_idx)
        hbm, _, _ = _peaks()
        nb = hisa_step_bytes(wl.T, wl.L, wl.H, B, m, wl.k)
        out[f"hisa_decode_L131072_B{B}_m{m}"] = {"ms_per_step": ms,
                                                 "pairs_per_s": int(wl.prefix_len.sum()) / (ms * 1e-3),
                                                 "roofline": {"bound": "hbm (latency-dominated)",
                                                              "algorithmic_bytes_per_step": nb,
                                                              "achieved": nb / (ms * 1e-3) / 1e9, "peak": hbm,
                                                              "unit": "GB/s", "frac": nb / (ms * 1e-3) / 1e9 / hbm},
                                                 "iou_vs_dense64": iou, "recovery_of_dense64": rec,
                                                 "needle_recall": planted_recall(hx.idx, wl.planted)}
    # the block statistics the HISA page names as improvements (section 七): max
    # pooling, and half-overlapping windows (stride 64)
    for tag, B, S, m, pool in (("max", 128, 128, 64, "max"), ("overlap_S64", 128, 64, 64, "mean")):
        means = misa.block_stats(keys, B, split=True, stride=S, pool=pool)
        hx = misa.HisaIndexer(wl.T, wl.H, wl.L, B, m, wl.k, device=dev, stride=S)
        ms = timed(lambda evs: hx.run(q, w, keys, means, so, pl))
        iou, rec = selection_agreement(hx.idx, dense_idx)
        hbm, _, _ = _peaks()
        M = misa.num_windows(wl.L, B, S)
        nb = hisa_step_bytes(wl.T, wl.L, wl.H, B, m, wl.k) + wl.T * (M - (wl.L + B - 1) // B) * 128 * 4
        out[f"hisa_decode_L131072_B{B}_m{m}_{tag}"] = {
            "ms_per_step": ms, "pairs_per_s": int(wl.prefix_len.sum()) / (ms * 1e-3), "windows": M,
            "roofline": {"bound": "hbm (latency-dominated)", "algorithmic_bytes_per_step": nb,
                         "achieved": nb / (ms * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
                         "frac": nb / (ms * 1e-3) / 1e9 / hbm},
            "iou_vs_dense64": iou, "recovery_of_dense64": rec, "needle_recall": planted_recall(hx.idx, wl.planted)}
    ms = timed(lambda evs: dx.run(q, w, keys, so, pl))
    out["hisa_decode_L131072_dense64"] = {"ms_per_step": ms, "pairs_per_s": int(wl.prefix_len.sum()) / (ms * 1e-3),
                                          "needle_recall": planted_recall(dense_idx, wl.planted)}
    # causal prefill: every query keeps the block its prefix cuts
    wp = make_workload("prefill_L131072")
    q, w, keys, so, pl = (x.to(dev) for x in (wp.q, wp.w, wp.keys, wp.seq_of, wp.prefix_len))
    means = misa.block_stats(keys, 128, split=True)
    hx = misa.HisaIndexer(wp.T, wp.H, wp.L, 128, 64, wp.k, device=dev)
    ms = timed(lambda evs: hx.run(q, w, keys, means, so, pl))
    out["prefill_L131072_hisa_B128_m64"] = {"ms_per_step": ms, "pairs_per_s": int(wp.prefix_len.sum()) / (ms * 1e-3)}
    return out


def _selection_quality(misa, dev):
    """Selection agreement with the dense 64-head indexer on inputs with
    locality (keys in contiguous regions around their own centroids, needles
    aligned with the positively weighted heads' query rows): the HISA decode
    shape (16 x 131072 keys, k = 2048) through MISA-8, MISA-dagger (k' = 8192)
    and HISA with mean-pooled blocks, max-pooled blocks and half-overlapping
    windows.  Information only: the pages' figures come from real text."""
    from workloads import make_local_decode
    wl = make_local_decode("local_decode_L131072", 6, T=16, L=131072, H=64, h=8, B=128, k=2048, n_planted=8,
                           planted_range=(0.4, 0.6))
    q, w, keys, so, pl = (x.to(dev) for x in (wl.q, wl.w, wl.keys, wl.seq_of, wl.prefix_len))
    dx = misa.DenseIndexer(wl.T, wl.H, wl.L, wl.k, device=dev)
    dense_idx = dx.run(q, w, keys, so, pl).clone()
    out = {"inputs": "16 caches of 131072 keys in regions of 256-4096 tokens around their own centroid "
                     "(k = c + 0.3 eps), 8 needles per query aligned with sum_h max(w_h, 0) q_h, in [0.4 L, 0.6 L)",
           "dense64_needle_recall": planted_recall(dense_idx, wl.planted)}
    means = misa.block_stats(keys, wl.B, split=True)
    ix = misa.MisaIndexer(wl.T, wl.H, wl.h, wl.L, wl.B, wl.k, device=dev)
    ix.run(q, w, keys, means, so, pl)
    dg = misa.MisaDaggerIndexer(wl.T, wl.H, wl.h, wl.L, wl.B, 8192, wl.k, device=dev)
    dg.run(q, w, keys, means, so, pl)
    runs = {"misa8": ix.idx, "misa_dagger_kp8192": dg.idx}
    for tag, S, pool in (("hisa_B128_m64_mean", 128, "mean"), ("hisa_B128_m64_max", 128, "max"),
                         ("hisa_B128_m64_overlap_S64", 64, "mean")):
        st = misa.block_stats(keys, 128, split=True, stride=S, pool=pool)
        hx = misa.HisaIndexer(wl.T, wl.H, wl.L, 128, 64, wl.k, device=dev, stride=S)
        runs[tag] = hx.run(q, w, keys, st, so, pl).clone()
    torch.cuda.synchronize()
    for tag, idx in runs.items():
        iou, rec = selection_agreement(idx, dense_idx)
        out[tag] = {"iou_vs_dense64": iou, "recovery_of_dense64": rec,
                    "needle_recall": planted_recall(idx, wl.planted)}
    del keys
    torch.cuda.empty_cache()
    return out


def _latent_cache(dev, seed: int, nseq: int, L: int) -> torch.Tensor:
    """Seeded synthetic latent KV rows [nseq, L, 576] bf16 ~ N(0, 1), drawn on the
    device (timing only; the parity tests draw theirs on the host)."""
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    kv = torch.empty((nseq, L, 576), dtype=torch.bfloat16, device=dev)
    for b in range(nseq):
        kv[b] = torch.randn((L, 576), generator=g, device=dev).to(torch.bfloat16)
    return kv


def _sparse_attention(misa, dev, stream, flush, steps, timed):
    """Sparse attention (128 heads over one 576-entry latent row per token, values
    = its first 512 entries) over the k = 2048 tokens the indexer selected, and
    the indexer's share of indexer + attention, at 32K and 128K."""
    out = {}
    scale = 192 ** -0.5
    cases = (("dsv32_decode_L32768", "misa8", lambda wl, B: misa.MisaIndexer(wl.T, wl.H, wl.h, wl.L, B, wl.k,
                                                                               device=dev)),
             ("hisa_decode_L131072", "hisa_B128_m64", lambda wl, B: misa.HisaIndexer(wl.T, wl.H, wl.L, B, 64, wl.k,
                                                                                       device=dev)))
    for name, tag, make_ix in cases:
        wl = make_workload(name)
        q, w, keys, so, pl = (x.to(dev) for x in (wl.q, wl.w, wl.keys, wl.seq_of, wl.prefix_len))
        means = misa.block_stats(keys, wl.B, split=True)
        ix = make_ix(wl, wl.B)
        dx = misa.DenseIndexer(wl.T, wl.H, wl.L, wl.k, device=dev)
        kv = _latent_cache(dev, 11, wl.nseq, wl.L)
        g = torch.Generator(device=dev)
        g.manual_seed(12)
        qa = torch.randn((wl.T, 128, 576), generator=g, device=dev).to(torch.bfloat16)
        o = torch.empty((wl.T, 128, 512), dtype=torch.bfloat16, device=dev)
        ws = misa.alloc_workspace(misa.workspace_bytes(misa._native.OP_SPARSE_MLA, wl.T, 128, 0, 0, wl.k), dev)
        idx = ix.run(q, w, keys, means, so, pl)
        attn = lambda evs: misa.sparse_mla(qa, kv, so, idx, scale, out=o, workspace=ws)
        ms_attn = timed(attn)
        ms_ix = timed(lambda evs: ix.run(q, w, keys, means, so, pl))
        ms_dense = timed(lambda evs: dx.run(q, w, keys, so, pl))
        ms_both = timed(lambda evs: (ix.run(q, w, keys, means, so, pl), attn(evs)))
        if misa.error_query(ws) != 0:
            raise RuntimeError("sparse attention recorded a device error")
        gathered = wl.T * wl.k * 576 * 2
        moved = gathered + wl.T * 128 * (576 + 512) * 2          # + q rows and the bf16 output
        flops = 2.0 * wl.T * 128 * wl.k * (576 + 512)
        hbm, tc, kind = _peaks()
        out[f"{name}_sparse_mla_k2048"] = {
            "attention_ms": ms_attn, "attention_GBps_unique_rows": gathered / (ms_attn * 1e-3) / 1e9,
            "attention_TFLOPs": flops / (ms_attn * 1e-3) / 1e12,
            "attention_roofline": {"bound": "hbm", "achieved": moved / (ms_attn * 1e-3) / 1e9, "peak": hbm,
                                   "unit": "GB/s", "frac": moved / (ms_attn * 1e-3) / 1e9 / hbm,
                                   "tensor_frac": flops / (ms_attn * 1e-3) / 1e12 / tc, "peaks": kind},
            f"{tag}_indexer_ms": ms_ix, f"{tag}_plus_attention_ms": ms_both,
            f"{tag}_share_of_indexer_plus_attention": ms_ix / (ms_ix + ms_attn),
            "dense64_indexer_ms": ms_dense, "dense64_share_of_indexer_plus_attention": ms_dense / (ms_dense + ms_attn)}
        del kv, keys
        torch.cuda.empty_cache()
    return out


def _blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:  # noqa: BLE001
        return 1


def cpu_baseline(wl, budget_s: float = 15.0, max_queries: int | None = None):
    """The fp64 oracle on whole queries of the workload until ~budget_s of CPU
    work; pairs/s over the queries done."""
    import oracle

    done, pairs, t_used = 0, 0, 0.0
    limit = max_queries or 64 * wl.T  # passes over the batch until the budget is spent
    for i in range(limit):
        t = i % wl.T
        sub_q = wl.q[t:t + 1].to(torch.float64).numpy()
        sub_w = wl.w[t:t + 1].numpy().astype(np.float64)
        keys = wl.keys[int(wl.seq_of[t]):int(wl.seq_of[t]) + 1].to(torch.float64).numpy()
        plen = wl.prefix_len[t:t + 1].numpy().astype(np.int64)
        t0 = time.perf_counter()
        oracle.misa_indexer(sub_q, sub_w, keys, np.zeros(1, np.int64), plen, wl.B, 1, wl.h, wl.k)
        t_used += time.perf_counter() - t0
        done += 1
        pairs += int(plen[0])
        if t_used >= budget_s:
            break
    return {"value": pairs / t_used, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{done} queries (cycling over the {wl.T} of {wl.name}; full route+score+top-k each), "
                      f"{t_used:.1f} s", **_host()}


def _cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _host():
    return {"cores_used": _blas_threads(), "host_cpus": os.cpu_count(), "cpu_model": _cpu_model(),
            "note": "numpy fp64; matrix products use the BLAS threads, the rest runs on one core"}


def cpu_baselines(budget_s: float = 20.0):
    """The fp64 oracle on the other workloads, each step of the path timed on
    the host (the block means, which the GPU path keeps as cache state, are
    computed before the clock starts): the tiny decode, the GLM-5-shaped
    MISA-dagger decode and the HISA decode in full, the 128K prefill on a
    seeded subsample of 8 of its 64 query blocks (the first and the last among
    them), labelled as such.  Value = indexed pairs / oracle seconds."""
    import oracle

    out = {}

    def per_query(wl, run_one, label):
        t_used, pairs, done = 0.0, 0, 0
        for t in range(wl.T):
            b = int(wl.seq_of[t])
            keys = wl.keys[b:b + 1].to(torch.float64).numpy()
            means = np.stack([oracle.block_means(keys[0], wl.B)])
            a = dict(q=wl.q[t:t + 1].to(torch.float64).numpy(), w=wl.w[t:t + 1].numpy().astype(np.float64),
                     keys=keys, seq_of=np.zeros(1, np.int64),
                     prefix_len=wl.prefix_len[t:t + 1].numpy().astype(np.int64), means=means)
            t0 = time.perf_counter()
            run_one(a)
            t_used += time.perf_counter() - t0
            pairs += int(wl.prefix_len[t])
            done += 1
            if t_used > budget_s:
                break
        full = done == wl.T
        out[wl.name] = {"value": pairs / t_used, "unit": UNIT, "queries": done, "seconds": t_used,
                        "sample": ("full batch" if full else f"first {done} of {wl.T} queries") + f"; {label}"}

    wl = make_workload("tiny_decode_L4096")
    k64 = wl.keys.to(torch.float64).numpy()
    means = np.stack([oracle.block_means(k64[0], wl.B)])
    t0 = time.perf_counter()
    oracle.misa_indexer(wl.q.to(torch.float64).numpy(), wl.w.numpy().astype(np.float64), k64,
                        wl.seq_of.numpy().astype(np.int64), wl.prefix_len.numpy().astype(np.int64), wl.B, 1, wl.h,
                        wl.k, means=means)
    dt = time.perf_counter() - t0
    out[wl.name] = {"value": int(wl.prefix_len.sum()) / dt, "unit": UNIT, "queries": wl.T, "seconds": dt,
                    "sample": "full batch; MISA route + score + top-k"}

    wl = make_workload("glm5_dagger_decode_L65536")
    per_query(wl, lambda a: oracle.misa_dagger_indexer(a["q"], a["w"], a["keys"], a["seq_of"], a["prefix_len"],
                                                       wl.B, 1, wl.h, wl.kp, wl.k, means=a["means"]),
              "MISA-dagger route + coarse score + top-k' + rerank + top-k")
    wl = make_workload("hisa_decode_L131072")
    per_query(wl, lambda a: oracle.hisa_indexer(a["q"], a["w"], a["keys"], a["seq_of"], a["prefix_len"],
                                                wl.B, wl.m, wl.k, means=a["means"]),
              "HISA block filter + candidate scoring + top-k (B=128, m=64)")

    wl = make_workload("prefill_L131072")
    k64 = wl.keys.to(torch.float64).numpy()
    means = np.stack([oracle.block_means(k64[0], wl.B)])
    n_blk = wl.T // wl.q_block
    rng = np.random.default_rng(33)
    chosen = sorted({0, n_blk - 1} | set(rng.choice(np.arange(1, n_blk - 1), size=6, replace=False).tolist()))
    t_used, pairs, done = 0.0, 0, []
    for gblk in chosen:
        sl = slice(gblk * wl.q_block, (gblk + 1) * wl.q_block)
        q = wl.q[sl].to(torch.float64).numpy()
        wv = wl.w[sl].numpy().astype(np.float64)
        pl = wl.prefix_len[sl].numpy().astype(np.int64)
        t0 = time.perf_counter()
        oracle.misa_indexer(q, wv, k64, np.zeros(q.shape[0], np.int64), pl, wl.B, wl.q_block, wl.h, wl.k,
                            means=means)
        t_used += time.perf_counter() - t0
        pairs += int(pl.sum())
        done.append(gblk)
        if t_used > budget_s:
            break
    out[wl.name] = {"value": pairs / t_used, "unit": UNIT, "queries": len(done) * wl.q_block, "seconds": t_used,
                    "sample": f"subsample: query blocks {done} of {n_blk} (64 queries each, seed 33; first and "
                              f"last always included); MISA route + score + top-k; not extrapolated"}
    return out


def run_reference(args):
    ws_n, rank, _ = _dist()
    if rank != 0:
        return
    wl = make_workload(WORKLOAD)
    # one query per step (its whole path); warm-up steps untimed
    for i in range(args.warmup):
        cpu_baseline(wl, budget_s=0.0, max_queries=1)
    t0 = time.perf_counter()
    res = [cpu_baseline(wl, budget_s=0.0, max_queries=1) for _ in range(args.steps)]
    wall = time.perf_counter() - t0
    value = statistics.median(r["value"] for r in res)
    line = {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws_n, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": wall / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(wl, ws_n),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
                         "sample": "1 query of the batch per step (route + score + top-k in fp64 numpy)",
                         **_host()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--quick", action="store_true", help="skip the other four workloads")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--only", choices=["prefill", "dagger", "hisa", "attn", "quality"], default=None,
                    help="time one of the other workloads alone (for profiler captures); prints its own JSON")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.only:
        import sparse_attention_token_misa_b200 as misa
        dev = torch.device("cuda", 0)
        flush_buf = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        res = other_workloads(misa, dev, torch.cuda.current_stream(), lambda: flush_buf.fill_(1.0),
                              max(3, args.steps), only=args.only)
        print(json.dumps({"only": args.only, "results": res}), flush=True)
    else:
        run_cuda(args)


if __name__ == "__main__":
    main()
