"""Benchmark of the hybrid compressed attention core on B200: one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

A step is one pass of the whole hot path over one batch of synthetic input: for the
default CSA prefill workload (B=1, S=8192, 64 heads, head_dim 512, m=4, top-512,
window 128) that is compress(kv) + compress(kI) + indexer/top-k + sparse attention.
Other workloads: HCA and DSA prefill, CSA decode over a pre-filled cache, a
sliding-window layer (RoPE of the K=V rows + window attention) and the decode-cache
append of one token per sequence (timed with L2 flushed between steps, since its
inputs fit in L2).
``value`` is whole-job tokens/s with inputs resident in HBM (device time, CUDA events,
max over ranks); ``e2e`` is the same metric through the layer entry point with pinned
host inputs copied in and the output copied back every step.  With N > 1 every rank
runs its own batch (independent sequences, no data-path collective): weak scaling.
``--impl reference`` times the fp64 CPU oracle on a bounded sample of query rows.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "CSA/HCA layer prefill tokens/s and decode µs/step on 1 B200; % of roofline"


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def _visible(w, q_index):
    t = q_index.reshape(-1).astype(np.int64)
    return np.minimum((t + 1) // w.m, w.P_cap)


def attn_keys_per_query(w, q_index):
    """Keys each query attends: window tokens plus min(topk, visible) pool entries."""
    t = q_index.reshape(-1).astype(np.int64)
    win = np.minimum(w.n_win, t + 1) if w.n_win > 0 else np.zeros_like(t)
    vis = _visible(w, q_index)
    pool = np.minimum(vis, w.topk) if w.kind != "hca" else vis
    return win + pool


def part_work(w, q_index):
    """Algorithmic (FLOPs, HBM bytes) of one launch of each part of a step.

    attention: H x keys x (D + dv) x 2 FLOPs; bytes = q + out + index lists + the K=V rows
      each sequence needs once (prefill: every rotated token row and pool entry; decode:
      the gathered rows of its one query); when the attention selects the index lists itself
      (CSA prefill, dsv4_sparse_mqa_attn_scores) also the fp32 score rows it reads, and there
      is no topk part.
    indexer_scores: visible entries x nI x cI x 2 FLOPs; bytes = the indexer pool once per
      sequence + qI + wI + the fp32 score rows written.
    indexer_topk (decode: scores and selection in one kernel): the same FLOPs; bytes = the
      indexer pool once per sequence + qI + wI + the index rows written.
    topk: no FLOPs; bytes = the fp32 score rows read + the index rows written.
    compress: bytes = token rows (kv and kI) and their logits (m > 1) read, pools and the
      rotated K=V rows written.
    append: bytes per sequence and stream of c channels: the new row and its logits read and
      written to the buffer (+ its position), the rotated window row (K=V stream); when the
      token closes a block, the Lw buffered rows and logits read and the entry written.
    out_proj: 2 T (H dv dg + g dg hidden) FLOPs (the g group products, then o_b_proj); bytes =
      o, both weights, the bf16 intermediate written and read back, and y.
    """
    e = 2 if w.dtype == "bf16" else 4
    if w.kind == "outproj":
        T = w.B * w.Sq
        inner = w.o_groups * w.o_rank
        flops = 2.0 * T * (w.H * w.dv * w.o_rank + inner * w.hidden)
        nbytes = e * (T * w.H * w.dv + inner * (w.H // w.o_groups) * w.dv + w.hidden * inner
                      + 2 * T * inner + T * w.hidden)
        return {"out_proj": (flops, nbytes)}
    if w.kind == "append":
        lw = 2 * w.m if w.overlap else w.m
        t = q_index.reshape(-1).astype(np.int64)
        closing = float(((t + 1) % w.m == 0).sum())
        nbytes = 0.0
        for c, window in ((w.D, True), (w.cI, False)):
            nbytes += w.B * (4 * c * e + 8 + (c * e if window else 0))
            nbytes += closing * (2 * lw * c * e + lw * c * 4 + c * e)
        return {"append": (0.0, nbytes)}
    nq = w.B * w.Sq
    keys = float(attn_keys_per_query(w, q_index).sum())
    vis = _visible(w, q_index).astype(np.float64)
    if w.kind == "decode":
        kv_bytes = keys * w.D * e
    else:
        kv_bytes = w.B * (w.S + w.P_cap) * w.D * e
    # the attention selects the lists itself (dsv4_sparse_mqa_attn_scores' fused condition, the
    # same test as harness.selects_in_attention)
    selects = w.kind == "csa" and w.dtype == "bf16" and 0 < w.P_cap <= 2048 and 0 < w.topk <= 512
    work = {"attention": (keys * w.H * (w.D + w.dv) * 2.0,
                          nq * w.H * (w.D + w.dv) * e + kv_bytes + (nq * w.topk * 4 if w.topk else 0)
                          + (vis.sum() * 4 if selects else 0.0))}
    if w.nI > 0:
        pool_once = float(w.B) * float(vis.reshape(w.B, -1).max(axis=1).mean()) * w.cI * e
        if w.kind == "decode":
            # one kernel: the indexer pool once, qI and wI in, the index rows out
            work["indexer_topk"] = (vis.sum() * w.nI * w.cI * 2.0,
                                    pool_once + nq * w.nI * (w.cI * e + 4) + nq * w.topk * 4)
        else:
            work["indexer_scores"] = (vis.sum() * w.nI * w.cI * 2.0,
                                      pool_once + nq * w.nI * (w.cI * e + 4) + vis.sum() * 4)
            if not selects:
                work["topk"] = (0.0, vis.sum() * 4 + nq * w.topk * 4)
    if w.kind != "decode":
        ch = w.D + (w.cI if w.nI else 0)
        rows_in = w.B * w.S * ch * e * (2 if w.m > 1 else 1)
        work["compress"] = (0.0, rows_in + w.B * w.P_cap * ch * e + w.B * w.S * w.D * e)
    return work


def tensor_peak_kind(timed_ms: float, clocks: dict) -> str:
    """Which measured bf16 peak a tensor-bound kernel is held to: the burst figure when the
    timed region is short (under a second) or the sampled SM clock stayed at its maximum,
    the sustained (power-capped) figure for a long region that ran below the maximum clock."""
    sm, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    if timed_ms < 1000.0 or (sm and mx and sm >= 0.97 * mx):
        return "burst"
    return "sustained"


def roofline_of(name, flops, nbytes, ms, peaks, peak_src, kind="burst"):
    """Roofline entry of one kernel: bound = the larger of its tensor time and HBM time at
    the measured peaks; achieved = its algorithmic work / its CUDA-event time.  A tensor
    bound is held to the burst or the sustained bf16 peak (``kind``); the other fraction is
    reported beside it."""
    pk_burst = peaks["bf16_tflops"]
    pk_sus = peaks.get("bf16_tflops_sustained", pk_burst)
    pk_t = pk_burst if kind == "burst" else pk_sus
    pk_b = peaks["hbm_gbs"]
    t_tensor = flops / (pk_t * 1e12)
    t_hbm = nbytes / (pk_b * 1e9)
    if t_tensor >= t_hbm:
        ach = flops / (ms / 1e3) / 1e12
        return {"bound": "tensor", "achieved": ach, "peak": pk_t, "unit": "TFLOP/s", "frac": ach / pk_t,
                "frac_of_burst": ach / pk_burst, "frac_of_sustained": ach / pk_sus,
                "kernel": name, "kernel_ms": ms, "algorithmic_flops": flops,
                "peak_source": f"{peak_src} bf16_tflops ({kind})"}
    ach = nbytes / (ms / 1e3) / 1e9
    return {"bound": "hbm", "achieved": ach, "peak": pk_b, "unit": "GB/s", "frac": ach / pk_b,
            "kernel": name, "kernel_ms": ms, "algorithmic_bytes": nbytes, "peak_source": f"{peak_src} hbm_gbs"}


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per launch of a part's main
# kernel, from one ncu capture of that kernel on that workload.  Each record carries the
# SHA-256 of the source that makes up the kernel at capture time (its file up to the end of
# the kernel definition, and the headers it includes): once any of it changes, traffic reads
# null until the kernel is captured again.  Values: (source segments, sha256, bytes per launch).
_ATTN_SOURCE = (("attn_tc.cu", "\ntypedef CUresult (*EncodeTiledFn)"), ("tc_ptx.cuh", None), ("common.cuh", None),
                ("internal.h", None), ("select.cuh", None))
_INDEXER_SOURCE = (("indexer_tc.cu", "\n}  // namespace\n\nbool indexer_tc_supported"), ("tc_ptx.cuh", None),
                   ("common.cuh", None), ("internal.h", None), ("select.cuh", None))
_OUT_PROJ_SOURCE = (("out_proj.cu", "\ntypedef CUresult (*EncodeTiledFn)"), ("tc_ptx.cuh", None), ("internal.h", None))
NCU_TRAFFIC = {
    # ncu --set full, one launch of the CSA prefill step (B=1, S=8192, H=64, D=dv=512, top-512,
    # window 128; the kernel selects each query's index list from its score row):
    # dram__bytes_read.sum 579.6 MB + dram__bytes_write.sum 511.7 MB.  (Re-keyed when the hash
    # took in select.cuh, which attn_tc.cu includes; it has not changed since the capture.)
    ("csa_prefill_bf16", "attention"): (_ATTN_SOURCE, "c39ebe7dad0102f834d73fa380b0cf0c41b674c81b356b8a5dadc60a1abe8bde", 1091308544),
    # ncu --set full, one launch of the CSA decode step (64 queries, pool 32768, top-2048): the fused
    # scores + top-k kernel, dram__bytes_read.sum 535.8 MB + dram__bytes_write.sum 3.8 MB (taken with
    # the split selection over per-warp lists).
    ("csa_decode_bf16", "indexer_topk"): (_INDEXER_SOURCE, "10a99b0b9836b53ff66523ba51d13f9a831cec632672ea4f7b5f1b954f4a39a2", 539641344),
    # ncu --set full, both launches of one output-projection step (o_a_proj, then o_b_proj; the
    # part is the two launches): 608.2 + 117.7 + 604.0 + 61.5 MB.  (Re-keyed when internal.h gained
    # the attention's score-row fields; nothing this kernel compiles changed.)
    ("out_proj_bf16", "out_proj"): (_OUT_PROJ_SOURCE, "46c2805ba7084d9716b7a12a62394346cdbf6c5ee751bba21f79f340f4959c99", 1391330304),
}


def kernel_source_sha(segments) -> str | None:
    """SHA-256 over the kernel's source segments (a file up to an end marker, or whole)."""
    import hashlib
    h = hashlib.sha256()
    for name, end in segments:
        try:
            text = open(os.path.join(ROOT, "sparse_long_context_csa_b200", "csrc", name)).read()
        except OSError:
            return None
        if end is not None:
            k = text.find(end)
            if k < 0:
                return None
            text = text[:k]
        h.update(text.encode())
    return h.hexdigest()


def ncu_traffic(workload: str, part: str):
    rec = NCU_TRAFFIC.get((workload, part))
    if rec is None:
        return None
    return rec[2] if kernel_source_sha(rec[0]) == rec[1] else None


class ClockSampler:
    """nvidia-smi SM clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), [x.strip() for x in line.split(",")]))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        rows = [s for (ts, s) in self.samples if t0 <= ts <= t1] or [s for _, s in self.samples]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if len(r) > 5 + i and "Active" in r[5 + i]
                          and "Not" not in r[5 + i]})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def cpu_oracle_rate(w, budget_s: float, host=None):
    """Time the fp64 oracle on a bounded, time-limited sample of the workload's query rows.

    Returns (tokens_per_s, rows_done, seconds, description).  The sample starts with the
    compression of the whole sequence (for prefill workloads) and then runs indexer + top-k
    + attention row by row over a strided sample of query rows until `budget_s` elapses.
    """
    from oracle import dsv4_oracle as O
    if host is None:
        host = synth.make_inputs(w) if w.kind != "decode" else None
    t0 = time.perf_counter()
    if w.kind == "decode":
        sp = synth.cache_specs(w)
        specs = synth.tensor_specs(w)
        qi, qpos = synth.positions(w)
        done = 0
        for b in range(w.B):
            pool = sp["pool"].rows(b * w.P_cap, (b + 1) * w.P_cap)[None]
            poolI = sp["poolI"].rows(b * w.P_cap, (b + 1) * w.P_cap)[None]
            win = sp["win"].rows(b * w.win_ring, (b + 1) * w.win_ring)[None]
            q = specs["q"].rows(b, b + 1).reshape(1, 1, w.H, w.D)
            qI = specs["qI"].rows(b, b + 1).reshape(1, 1, w.nI, w.cI)
            wI = specs["wI"].rows(b, b + 1).reshape(1, 1, w.nI)
            sink = specs["sink"].full()
            idx = O.indexer_topk(qI, wI, poolI, qi[b:b + 1], m=w.m, topk=w.topk, P_cap=w.P_cap)
            O.sparse_mqa_attention(q, win, pool, idx, sink, qpos[b:b + 1], qi[b:b + 1], n_win=w.n_win, m=w.m,
                                   scale=w.scale, dv=w.dv, R=w.R, theta=w.theta, rope_q=True,
                                   rotate_out=w.rotate_out, win_ring=w.win_ring, P_cap=w.P_cap)
            done += 1
            if time.perf_counter() - t0 > budget_s:
                break
        dt = time.perf_counter() - t0
        return done / dt, done, dt, f"{done} of {w.B} decode sequences (indexer + top-k + attention)"
    if w.kind == "outproj":
        # blocks of 16 tokens through both projections until the budget is spent
        done = 0
        T = w.B * w.Sq
        while done < T and time.perf_counter() - t0 < budget_s:
            O.grouped_out_proj(host["o"][done:done + 16], host["wa"], host["wb"])
            done = min(T, done + 16)
        dt = time.perf_counter() - t0
        return done / dt, done, dt, f"{done} of {T} tokens through o_a_proj (8 groups) and o_b_proj"
    if w.kind == "append":
        # per sequence: the Lw-1 earlier tokens are appended untimed, the step's token timed
        lw = host["kv"].shape[0]
        done, dt = 0, 0.0
        for b in range(w.B):
            caches = [(O.new_decode_cache(w.D, m=w.m, overlap=w.overlap, P_cap=w.P_cap, win_ring=w.win_ring),
                       "kv", "z", "bias", True),
                      (O.new_decode_cache(w.cI, m=w.m, overlap=w.overlap, P_cap=w.P_cap), "kI", "zI", "biasI", False)]
            for k in range(lw):
                if k == lw - 1:
                    t1 = time.perf_counter()
                for cache, xk, zk, bk, rope in caches:
                    O.decode_append(cache, host[xk][k, b], host[zk][k, b], int(host["pos_hist"][k, b]),
                                    int(host["t_hist"][k, b]), m=w.m, overlap=w.overlap, bias=host[bk],
                                    apply_rope=rope, R=w.R, theta=w.theta)
            dt += time.perf_counter() - t1
            done += 1
            if time.perf_counter() - t0 > budget_s:
                break
        return done / dt, done, time.perf_counter() - t0, (
            f"{done} of {w.B} sequences: one token appended to the K=V and indexer-key caches "
            f"(the {lw - 1} tokens before it appended untimed)")
    kw = dict(m=w.m, n_win=w.n_win, scale=w.scale, dv=w.dv, R=w.R, theta=w.theta, rotate_out=w.rotate_out)
    if w.kind == "swa":
        pool = np.zeros((w.B, 0, w.D))
        kw["P_cap"] = 0
    else:
        pool = O.compress(host["kv"], host.get("z"), host.get("bias"), host["pos"], m=w.m, overlap=w.overlap,
                          apply_rope=True, R=w.R, theta=w.theta)
    kv_rot = O.rope_rotate(host["kv"], host["pos"], w.R, w.theta)
    poolI = O.compress(host["kI"], host.get("zI"), host.get("biasI"), host["pos"], m=w.m,
                       overlap=w.overlap, apply_rope=False) if w.nI > 0 else None
    t_comp = time.perf_counter() - t0
    order = np.random.default_rng(0).permutation(w.S)
    done = 0
    t1 = time.perf_counter()
    qi = np.tile(np.arange(w.S), (w.B, 1))
    for s in order:
        rows = [(0, int(s))]
        idx = O.indexer_topk(host["qI"], host["wI"], poolI, qi, m=w.m, topk=w.topk, rows=rows) \
            if w.nI > 0 else None
        O.sparse_mqa_attention(host["q"], kv_rot, pool, idx, host["sink"], host["pos"], qi, rope_q=True,
                               rows=rows, **{k: v for k, v in kw.items()})
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    t_rows = time.perf_counter() - t1
    per_row = t_rows / max(done, 1)
    total = t_comp + per_row * w.S * w.B
    first = "RoPE of all" if w.kind == "swa" else "compression of all"
    return (w.S * w.B) / total, done, t_comp + t_rows, (
        f"{first} {w.S} tokens ({t_comp:.2f} s) + {done} random query rows "
        f"({per_row * 1e3:.1f} ms/row), extrapolated to {w.S} rows")


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    host = synth.make_inputs(w) if w.kind != "decode" else None
    per_step = []
    desc = ""
    # each step is a bounded sample; the whole run stays within a few minutes
    budget = min(args.ref_budget, max(1.5, 150.0 / max(1, args.warmup + args.steps)))
    for i in range(args.warmup + args.steps):
        rate, rows, secs, desc = cpu_oracle_rate(w, budget, host)
        if i >= args.warmup:
            per_step.append(rate)
    if per_step_kind(w) == "us/step":
        value = 1e6 / float(np.mean(per_step)) * w.B  # us per step of all B sequences
        unit = "us/step"
    else:
        value = float(np.mean(per_step))
        unit = "tokens/s"
    cores = blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": unit == "tokens/s",
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w),
            "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def reduce_max(v: float, world: int, device: str) -> float:
    """The maximum of `v` over all ranks (every rank must call it, in the same order)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def per_step_kind(w) -> str:
    """Decode workloads (one token per sequence) report us/step, prefill ones tokens/s."""
    return "us/step" if w.kind in ("decode", "append") else "tokens/s"


def job_value(kind: str, world: int, tokens_per_rank: int, steps: int, ms_max: float):
    """Whole-job metric from the slowest rank's time for `steps` steps: decode reports
    microseconds per step; prefill reports the tokens of all ranks per second."""
    if kind in ("decode", "append"):
        return ms_max / steps * 1e3, "us/step", False
    return world * tokens_per_rank * steps / (ms_max / 1e3), "tokens/s", True


def l2_flush_needed(w) -> bool:
    """True when a step's inputs fit in the 126 MB L2: such steps are timed with L2 flushed."""
    if w.kind == "append":
        return True
    if w.kind == "outproj":
        return w.B * w.Sq * w.H * w.dv * 2 <= (126 << 20)
    if w.kind == "decode":
        return w.B * w.P_cap * (w.D + w.cI) * 2 <= (126 << 20)
    return w.B * w.Sq * w.H * w.D * 2 <= (126 << 20)


def config_of(w):
    c = {"workload": w.name, "B": w.B, "S": w.S, "Sq": w.Sq, "H": w.H, "head_dim": w.D, "rope_dim": w.R,
         "dv": w.dv, "sliding_window": w.n_win, "m": w.m, "overlap": w.overlap, "pool_cap": w.P_cap}
    if w.nI:
        c.update({"index_n_heads": w.nI, "index_head_dim": w.cI, "index_topk": w.topk})
    if w.kind == "append":
        c = {"workload": w.name, "B": w.B, "cache_tokens": w.S, "head_dim": w.D, "rope_dim": w.R, "m": w.m,
             "overlap": w.overlap, "buffer_rows": 2 * w.m if w.overlap else w.m, "window_ring": w.win_ring,
             "pool_cap": w.P_cap, "index_head_dim": w.cI}
    if w.kind == "outproj":
        c = {"workload": w.name, "tokens": w.B * w.Sq, "H": w.H, "dv": w.dv, "o_groups": w.o_groups,
             "o_lora_rank": w.o_rank, "hidden_size": w.hidden}
    if l2_flush_needed(w):
        c["l2"] = "L2 flushed between steps (a 256 MiB buffer written outside the timed events)"
    elif w.kind == "decode":
        c["l2"] = "inputs larger than L2 (pools 2.5 GB)"
    else:
        c["l2"] = "inputs larger than L2 (q and out are each > 126 MB)"
    return c


EXTRA_WORKLOADS = ("hca_prefill_bf16", "csa_decode_bf16", "dsa_prefill_bf16", "out_proj_bf16")


class Runner:
    """One rank's device state for timing workloads (the process group, if any, is set up)."""

    def __init__(self, args, world, rank, local):
        import torch
        from sparse_long_context_csa_b200 import abi, harness
        self.torch, self.abi, self.harness = torch, abi, harness
        self.args, self.world, self.rank, self.local = args, world, rank, local
        self.sampler = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                                    else local)
        if not args.profile_run:
            self.sampler.start()
        abi.load()

    def barrier(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()

    def max_over_ranks(self, v: float) -> float:
        return reduce_max(v, self.world, "cuda")

    def device_check(self, what: str):
        """Every bounded wait in the kernels must have ended in time: a CTA that gave one up
        returned early with invalid output, so its step must not count as a timed step."""
        try:
            self.abi.dsv4_device_check()
        except self.abi.Dsv4Error as e:
            raise SystemExit(f"bench: device-side check failed after {what}: {e}")

    def setup(self, w):
        torch, harness = self.torch, self.harness
        host = synth.make_inputs(w)
        params = harness.params_for(w)
        x = harness.to_device(w, host)
        o = harness.make_outputs(w, params, scores=True)
        return {"w": w, "host": host, "params": params, "x": x, "o": o, "stream": torch.cuda.current_stream()}

    def measure(self, st, steps: int, warmup: int):
        """W untimed warm-up steps, then K timed steps (CUDA events on the launching stream,
        every part bracketed by its own events); returns the max-over-ranks times."""
        torch, harness, abi = self.torch, self.harness, self.abi
        w, params, x, o, stream = st["w"], st["params"], st["x"], st["o"], st["stream"]
        q_index = st["host"]["q_index"]
        parts = [p for p in harness.PARTS if p in part_work(w, q_index)]

        def step(events=None):
            harness.step_parts(w, params, x, o, stream, events=events)

        if w.kind == "append":
            harness.append_prefill(w, params, x, o, stream)  # the cache just before the step's token
        flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda") if l2_flush_needed(w) else None
        for _ in range(warmup):
            step()
        torch.cuda.synchronize()
        t_w = time.time()
        while not self.args.profile_run and time.time() - t_w < 1.0:  # the clock sampler settles
            step()
            torch.cuda.synchronize()
        self.device_check(f"the warm-up of {w.name}")
        evs = [{p: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for p in parts}
               for _ in range(steps)]
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(steps)] if flush is not None else None
        self.barrier()
        torch.cuda.synchronize()
        n0 = abi.dsv4_launch_count()
        wall0 = time.time()
        start.record(stream)
        for i in range(steps):
            if flush is not None:
                flush.fill_(i & 255)  # evicts the previous step's lines from L2; not inside the step's events
                step_ev[i][0].record(stream)
            step(evs[i])
            if flush is not None:
                step_ev[i][1].record(stream)
        end.record(stream)
        torch.cuda.synchronize()
        wall1 = time.time()
        n1 = abi.dsv4_launch_count()
        self.device_check(f"the timed steps of {w.name}")
        self.barrier()
        total_ms = start.elapsed_time(end) if flush is None else sum(a.elapsed_time(b) for a, b in step_ev)
        ms = self.max_over_ranks(total_ms)
        part_ms = {p: self.max_over_ranks(float(np.mean([e[p][0].elapsed_time(e[p][1]) for e in evs])))
                   for p in parts}
        return {"ms": ms, "part_ms": part_ms, "parts": parts, "launches": int(n1 - n0),
                "clocks": self.sampler.summary(wall0, wall1)}

    def roofline(self, w, q_index, m):
        peaks, peak_src = _peaks()
        work = part_work(w, q_index)
        parts, part_ms = m["parts"], m["part_ms"]
        kind = tensor_peak_kind(m["ms"], m["clocks"])
        dom = max(parts, key=lambda p: part_ms[p])
        roof = roofline_of(dom, work[dom][0], work[dom][1], part_ms[dom], peaks, peak_src, kind)
        roof["traffic"] = ncu_traffic(w.name, dom)
        roof["parts_ms"] = part_ms
        roof["others"] = {p: {k: v for k, v in roofline_of(p, work[p][0], work[p][1], part_ms[p], peaks, peak_src,
                                                           kind).items()
                              if k in ("bound", "achieved", "unit", "frac")} for p in parts if p != dom}
        return roof

    def e2e(self, st, steps: int):
        """The same metric through the layer entry point: every step copies its activations in
        from pinned host memory and its output back.  Steps are pipelined over two buffer sets:
        step i's inputs go in on one copy stream while step i-1 computes and its output goes
        out on a second copy stream (the decode append, whose result is cache state, runs
        serially).  Returns (ms per step, h2d bytes, d2h bytes)."""
        torch, harness = self.torch, self.harness
        w, params, x, o, stream, host = st["w"], st["params"], st["x"], st["o"], st["stream"], st["host"]
        keys = [k for k in harness.step_input_keys(w) if k in x]
        host_t = harness.to_device(w, {k: host[k] for k in keys}, device=None, pin=True)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if w.kind == "append":
            last = host["kv"].shape[0] - 1
            pairs = [(x[k][last], host_t[k][last]) for k in keys]
            result = o["buf_pos"]   # the buffer's position record (the rows stay on the device)
            out_host = torch.empty(result.shape, dtype=result.dtype, pin_memory=True)
            h2d = sum(t.numel() * t.element_size() for _, t in pairs)
            d2h = out_host.numel() * out_host.element_size()

            def e2e_run(n):
                for _ in range(n):
                    for dst, src in pairs:
                        dst.copy_(src, non_blocking=True)
                    harness.step(w, params, x, o, stream)
                    out_host.copy_(result, non_blocking=True)

            e2e_run(1)
            torch.cuda.synchronize()
            self.barrier()
            e0.record(stream)
            e2e_run(steps)
            e1.record(stream)
        else:
            sets = [x, {**x, **{k: torch.empty_like(x[k]) for k in keys}}]
            outs = [o, {**o, "out": torch.empty_like(o["out"])}]
            out_host = [torch.empty(o["out"].shape, dtype=o["out"].dtype, pin_memory=True) for _ in range(2)]
            h2d = sum(host_t[k].numel() * host_t[k].element_size() for k in keys)
            d2h = out_host[0].numel() * out_host[0].element_size()
            s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
            in_ready, in_free, out_ready, out_free = ([torch.cuda.Event() for _ in range(2)] for _ in range(4))

            def e2e_run(n):
                for i in range(n):
                    b = i % 2
                    s_in.wait_event(in_free[b])        # the step two back has read this input set
                    with torch.cuda.stream(s_in):
                        for k in keys:
                            sets[b][k].copy_(host_t[k], non_blocking=True)
                    in_ready[b].record(s_in)
                    stream.wait_event(in_ready[b])
                    stream.wait_event(out_free[b])     # this output buffer has been copied out
                    harness.step(w, params, sets[b], outs[b], stream)
                    in_free[b].record(stream)
                    out_ready[b].record(stream)
                    s_out.wait_event(out_ready[b])
                    with torch.cuda.stream(s_out):
                        out_host[b].copy_(outs[b]["out"], non_blocking=True)
                    out_free[b].record(s_out)

            e2e_run(2)
            torch.cuda.synchronize()
            self.barrier()
            e0.record(s_in)
            e2e_run(steps)
            e1.record(s_out)
        torch.cuda.synchronize()
        self.device_check(f"the end-to-end steps of {w.name}")
        return self.max_over_ranks(e0.elapsed_time(e1)) / steps, h2d, d2h


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=None, choices=sorted(synth.WORKLOADS),
                    help="time this workload alone (default: CSA prefill as the headline, then the "
                         "HCA prefill, CSA decode and DSA prefill workloads under \"workloads\")")
    ap.add_argument("--ref-budget", type=float, default=12.0,
                    help="at most this many seconds of oracle work per reference step (fewer when "
                         "warm-up + steps would make the run longer than ~150 s)")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-run", action="store_true",
                    help="for profilers: only the warm-up and timed steps (no clock sampler, e2e or cpu_baseline)")
    args = ap.parse_args()
    w = synth.WORKLOADS[args.workload or "csa_prefill_bf16"]
    extras = [] if (args.workload or args.profile_run) else list(EXTRA_WORKLOADS)
    if args.impl == "reference":
        return run_reference(args, w)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    run = Runner(args, world, rank, local)
    st = run.setup(w)
    m = run.measure(st, args.steps, args.warmup)
    ms = m["ms"]
    if args.profile_run:
        if rank == 0:
            print(json.dumps({"profile_run": True, "ms_per_step": ms / args.steps, "part_ms": m["part_ms"]}),
                  flush=True)
        return

    e2e_ms, h2d, d2h = run.e2e(st, max(3, min(args.steps, 10)))
    tokens = w.B * w.Sq
    value, unit, hib = job_value(w.kind, world, tokens, args.steps, ms)
    e2e_val = job_value(w.kind, world, tokens, 1, e2e_ms)[0]
    roof = run.roofline(w, st["host"]["q_index"], m)
    line = {"metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": hib, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded N(0,1)/sqrt(d) inputs, no weights)",
            "config": config_of(w), "parallelism": f"replicas x{world} (independent sequences)",
            "gpu_launches": m["launches"], "clocks": m["clocks"], "roofline": roof,
            "e2e": {"value": e2e_val, "unit": unit, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, rows, secs, desc = cpu_oracle_rate(w, args.cpu_budget, st["host"])
        cv = (1e6 / rate * w.B) if per_step_kind(w) == "us/step" else rate
        line["cpu_baseline"] = {"value": cv, "unit": unit, "cores": blas_threads(), "kind": "oracle",
                                "sample": desc, "seconds": round(secs, 2)}
    del st
    # the other configurations the metric names, each its own timed region on the same rank(s)
    others = {}
    for name in extras:
        wx = synth.WORKLOADS[name]
        torch.cuda.empty_cache()
        sx = run.setup(wx)
        k = max(3, min(args.steps, 10))
        mx = run.measure(sx, k, max(3, min(args.warmup, 5)))
        vx, ux, hx = job_value(wx.kind, world, wx.B * wx.Sq, k, mx["ms"])
        others[name] = {"value": vx, "unit": ux, "higher_is_better": hx, "steps": k,
                        "ms_per_step": mx["ms"] / k, "gpu_launches": mx["launches"], "clocks": mx["clocks"],
                        "config": config_of(wx), "roofline": run.roofline(wx, sx["host"]["q_index"], mx)}
        del sx
    if others:
        line["workloads"] = others
    run.sampler.stop()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
