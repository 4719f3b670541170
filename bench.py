"""Benchmark of the sparse index attention decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload: the bf16 decode batch -- 64 sequences with contexts uniform in [8192, 32768], one query
token each, a 64-head x 128-dim indexer, Top-2048, sparse MLA with 128 heads over a paged
latent cache of 512 + 64 dims (page 64), softmax scale 1/sqrt(576).  Synthetic seeded inputs,
resident in HBM before the timed region.

One step = one pass of the whole path over the batch: hsa_fused_decode (index score -> Top-K
-> sparse MLA) on one stream.  The same call with an auxiliary stream (second half of the batch
overlapping the first half's attention) is timed as well and reported under "two_stream"; on
this workload the attention is bound by per-row pipeline latency, so splitting the batch only
serializes the halves and the single-stream call is the faster one.  L2 is flushed before every
timed step by writing a 256 MiB buffer and then reading it back (so that L2 holds clean lines
and no write-back of the flush itself lands inside the timed step); each step is timed with
CUDA events on the launching stream, the time reported is the sum over the K steps (max over
ranks when N > 1).
Multi-GPU runs are independent replicas (the decode batch shards by sequence; no collective is
on the data path): every rank runs the full batch on its own GPU.

The JSON line also carries: the roofline of the dominant kernel (per-kernel CUDA-event times
from a second timed loop that issues the three C-ABI calls separately on one stream), the
end-to-end throughput through the C ABI with host buffers (H2D of the step's query inputs and
D2H of its output inside the timed region), the oracle timed on a bounded sample on the host
cores, the SM clocks sampled during the timed region, and (one GPU) "other_workloads": the FP8
and MXFP8 decode batches, the draft-verify batch, the KV quantizer, the bf16 causal prefill of
16384 tokens and the 131072-token zigzag prefill with FP8 index keys (each prefill with its
per-kernel times), each with its roofline fraction.

--impl reference runs the float64 CPU oracle (the only reference implementation of this path)
on the same workload, as many query rows per step as the oracle has threads (--ref-rows), and
prints the same JSON line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_index_attention_b200 import workloads  # noqa: E402

METRIC = "decode & prefill tokens/s on 1 B200; % of HBM / tensor-core roofline"
UNIT = "tokens/s"
WORKLOAD = "decode_bf16"
FLUSH_BYTES = 256 << 20


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def workload_config(wl):
    lens = wl.seq_lens.tolist()
    return {"workload": WORKLOAD, "B": wl.B, "context_min": min(lens), "context_max": max(lens),
            "context_mean": round(sum(lens) / len(lens), 1), "query_rows": wl.T_q,
            "index_heads": wl.H_I, "index_dim": wl.D_I, "top_k": wl.K, "heads": wl.H,
            "latent_dim": wl.D_v, "rope_dim": wl.D_rope, "page_size": wl.page_size,
            "softmax_scale": wl.softmax_scale, "seed": wl.seed,
            "l2": "flushed before every timed step (256 MiB written, then read back)"}


def algorithmic_work(wl):
    """Bytes (and flops) each kernel must move, from the workload's shape (per launch over the
    whole batch).  Index score: 256 B per key read + 4 B score written per key, plus q_I and w;
    Top-K: 4 B per score read + 4 B per index written; attention: 1152 B per selected latent
    row + q and output."""
    n = (wl.q_pos.long() + 1).cpu()
    sel = torch.clamp(n, max=wl.K)
    esz = 2
    idx_bytes = int(n.sum()) * (wl.D_I * esz + 4) + wl.T_q * wl.H_I * (wl.D_I * esz + 4)
    topk_bytes = int(n.sum()) * 4 + wl.T_q * wl.K * 4
    attn_bytes = int(sel.sum()) * wl.D_qk * esz + wl.T_q * wl.H * (wl.D_qk + wl.D_v) * esz + \
        wl.T_q * wl.K * 4 + wl.T_q * wl.H * 4
    idx_flops = int(n.sum()) * wl.H_I * wl.D_I * 2
    attn_flops = int(sel.sum()) * wl.H * (wl.D_qk + wl.D_v) * 2
    return {"index_score": {"bytes": idx_bytes, "flops": idx_flops},
            "topk": {"bytes": topk_bytes, "flops": 0},
            "sparse_mla": {"bytes": attn_bytes, "flops": attn_flops}}


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.02):
        self.samples, self.reasons = [], set()
        self.period = period_s
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.nv = None
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                mask = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if mask & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._t:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def cpu_baseline(wl, rows, timer_label="oracle"):
    """The float64 oracle (as it is) on a sample of query rows: index score -> Top-K -> sparse
    MLA for those rows over their full contexts.  Returns (tokens/s, seconds, threads)."""
    import oracle
    pg = oracle.Paging(wl.seq_lens, wl.block_table, wl.page_size, wl.num_pages, wl.q_seq, wl.q_pos)
    k = wl.k_I.float().cpu().numpy().astype(np.float64)
    kv = wl.kv.float().cpu().numpy().astype(np.float64)
    qI, w, q = wl.q_I[rows].cpu(), wl.w[rows].cpu(), wl.q[rows].cpu()
    t0 = time.perf_counter()
    oracle.sparse_index_attention(pg.subset(rows), qI, w, k, q, kv, wl.K, wl.D_v, wl.softmax_scale)
    dt = time.perf_counter() - t0
    return len(rows) / dt, dt, min(oracle.num_threads(), len(rows))


def run_reference(args, rank, world):
    if rank != 0:
        return
    import oracle
    wl = workloads.make(WORKLOAD, "cpu")
    pg = oracle.Paging(wl.seq_lens, wl.block_table, wl.page_size, wl.num_pages, wl.q_seq, wl.q_pos)
    k = wl.k_I.float().numpy().astype(np.float64)
    kv = wl.kv.float().numpy().astype(np.float64)

    rows_per_step = args.ref_rows or max(1, oracle.num_threads())

    def step(i):
        r0 = (i * rows_per_step) % wl.T_q
        rows = [(r0 + j) % wl.T_q for j in range(rows_per_step)]
        oracle.sparse_index_attention(pg.subset(rows), wl.q_I[rows], wl.w[rows], k, wl.q[rows], kv,
                                      wl.K, wl.D_v, wl.softmax_scale)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    dt = time.perf_counter() - t0
    value = args.steps * rows_per_step / dt
    threads = min(oracle.num_threads(), rows_per_step)   # OpenMP spreads a step's rows
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(wl),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": f"{rows_per_step} query rows per step (index score over "
                                       "each whole context, Top-2048, 128-head sparse MLA), the "
                                       "batch's rows in turn"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def rank_ops(dist, dev):
    """(barrier, max_over_ranks) over the process group `dist` (the torch.distributed module after
    init_process_group, or None for one process).  Every rank calls both at the same points."""
    def barrier():
        if dist is not None:
            dist.barrier()

    def max_over_ranks(x: float) -> float:
        if dist is None:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())
    return barrier, max_over_ranks


def replica_throughput(world: int, rows_per_step: int, steps: int, t_ms_max: float) -> float:
    """Whole-job rows/s of `world` replicas that each ran `steps` steps of `rows_per_step` query
    rows, from the slowest rank's time (ms)."""
    return world * rows_per_step * steps / (t_ms_max * 1e-3)


def _timed(fn, reps, flush_l2, main):
    """Median of `reps` CUDA-event timings (ms) of fn() on `main`, L2 flushed before each."""
    ts = []
    for _ in range(reps):
        flush_l2()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(main)
        fn()
        b.record(main)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.median(ts)


def stage_times(calls, names, reps, flush_l2, main):
    """Mean CUDA-event time (ms) of each call, the calls issued in turn on `main` with events
    between them, L2 flushed before each round."""
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)] for _ in range(reps)]
    for i in range(reps):
        flush_l2()
        ev[i][0].record(main)
        for j, c in enumerate(calls):
            c()
            ev[i][j + 1].record(main)
    torch.cuda.synchronize()
    return {n: {"ms": round(statistics.mean(e[j].elapsed_time(e[j + 1]) for e in ev), 4)}
            for j, n in enumerate(names)}


def block_aligned(dev, flush_l2, main, peaks, reps):
    """Block-aligned selection on the bf16 decode batch (blocks of one cache page, 64 positions):
    the selection kernel, and the attention over whole-page selections beside the attention over
    the position selection of the same scores (both gather 2048 rows per query row)."""
    import sparse_index_attention_b200 as hsa
    wl = workloads.make(WORKLOAD, dev)
    seq = hsa.PagedSeq(wl.seq_lens, wl.block_table, wl.page_size, wl.num_pages, wl.q_seq, wl.q_pos,
                       q_run=wl.q_run)
    sc = hsa.hsa_index_score(seq, wl.q_I, wl.w, wl.k_I)
    idx_p = hsa.hsa_topk(seq, sc, wl.K)
    idx_b = hsa.hsa_topk_blocks(seq, sc, wl.K, wl.page_size)
    o = torch.empty((wl.T_q, wl.H, wl.D_v), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((wl.T_q, wl.H), dtype=torch.float32, device=dev)
    ws = torch.zeros(max(1, hsa.hsa_sparse_mla_workspace_size(seq, wl.H, wl.D_qk, wl.D_v, wl.K)),
                     dtype=torch.uint8, device=dev)
    for _ in range(3):
        hsa.hsa_sparse_mla_attn(seq, wl.q, wl.kv, idx_b, wl.D_v, wl.softmax_scale, out=o, lse=lse, ws=ws, stream=main)
    st = stage_times(
        [lambda: hsa.hsa_topk(seq, sc, wl.K, idx=idx_p, stream=main),
         lambda: hsa.hsa_topk_blocks(seq, sc, wl.K, wl.page_size, idx=idx_b, stream=main),
         lambda: hsa.hsa_sparse_mla_attn(seq, wl.q, wl.kv, idx_p, wl.D_v, wl.softmax_scale, out=o,
                                         lse=lse, ws=ws, stream=main),
         lambda: hsa.hsa_sparse_mla_attn(seq, wl.q, wl.kv, idx_b, wl.D_v, wl.softmax_scale, out=o,
                                         lse=lse, ws=ws, stream=main)],
        ["topk_positions", "topk_blocks", "sparse_mla_positions", "sparse_mla_blocks"], reps,
        flush_l2, main)
    rows = int((idx_b >= 0).sum())
    byt = rows * wl.D_qk * 2 + wl.T_q * wl.H * (wl.D_qk + wl.D_v) * 2
    res = {"workload": "the bf16 decode batch, selection of whole cache pages (64 positions): the "
                       "32 pages with the highest page maximum per row",
           "stages": st, "rows_gathered": rows,
           "attention_frac_blocks": round(byt / (st["sparse_mla_blocks"]["ms"] * 1e-3) / (peaks["hbm_gbs"] * 1e9), 4)}
    del wl, seq, sc, idx_p, idx_b, o, lse, ws
    torch.cuda.empty_cache()
    return res


def secondary(dev, flush_l2, main, peaks, reps):
    """The path's other workloads, each measured once per bench run (rank 0, one GPU): the FP8
    decode batch (fp32 and MXFP8 index scales), the draft-verify decode batch, the bf16 causal
    prefill and the KV-cache quantizer.  Each entry gives tokens/s and the fraction of the bound that applies to it (HBM
    bytes, or bf16 tensor flops for prefill; algorithmic counts from the shapes)."""
    import sparse_index_attention_b200 as hsa
    out = {}
    hbm = peaks["hbm_gbs"] * 1e9

    # FP8 decode: 128 sequences x 65536 keys, FP8 index keys and FP8 latent cache
    wl = workloads.make("decode_fp8", dev)
    k8, ks = hsa.hsa_quantize_index(wl.k_I, wl.D_I)
    kv8, kvs, rope = hsa.hsa_quantize_kv(wl.kv, wl.D_v, wl.D_v)
    ks, kvs = ks.view(-1), kvs.view(-1)
    seq = hsa.PagedSeq(wl.seq_lens, wl.block_table, wl.page_size, wl.num_pages, wl.q_seq, wl.q_pos,
                       q_run=wl.q_run)
    sc = torch.empty((wl.T_q, seq.max_seq_len), dtype=torch.float32, device=dev)
    idx = torch.empty((wl.T_q, wl.K), dtype=torch.int32, device=dev)
    o = torch.empty((wl.T_q, wl.H, wl.D_v), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((wl.T_q, wl.H), dtype=torch.float32, device=dev)
    ws = torch.zeros(max(1, hsa.hsa_fused_decode_workspace_size(seq, wl.q, kv8, wl.D_v, wl.K)),
                     dtype=torch.uint8, device=dev)

    def fp8_step():
        hsa.hsa_fused_decode(seq, wl.q_I, wl.w, k8, ks, wl.q, kv8, kvs, rope, wl.K, wl.D_v,
                             wl.softmax_scale, scores=sc, idx=idx, out=o, lse=lse, ws=ws, stream=main)
    for _ in range(3):
        fp8_step()
    ms = _timed(fp8_step, reps, flush_l2, main)
    n = (wl.q_pos.long() + 1).cpu()
    sel = int(torch.clamp(n, max=wl.K).sum())
    byt = int(n.sum()) * (wl.D_I + 4 + 4) + sel * (wl.D_v + 4 + 2 * (wl.D_qk - wl.D_v)) + \
        wl.T_q * wl.H * (wl.D_qk + wl.D_v) * 2 + wl.T_q * wl.H_I * (wl.D_I * 2 + 4)
    stage = stage_times(
        [lambda: hsa.hsa_index_score(seq, wl.q_I, wl.w, k8, ks, scores=sc, stream=main),
         lambda: hsa.hsa_topk(seq, sc, wl.K, idx=idx, stream=main),
         lambda: hsa.hsa_sparse_mla_attn(seq, wl.q, kv8, idx, wl.D_v, wl.softmax_scale, kv_scale=kvs,
                                         kv_rope=rope, out=o, lse=lse, ws=ws, stream=main)],
        ["index_score", "topk", "sparse_mla"], reps, flush_l2, main)
    idx_bytes = int(n.sum()) * (wl.D_I + 4 + 4) + wl.T_q * wl.H_I * (wl.D_I * 2 + 4)
    attn_bytes = sel * (wl.D_v + 4 + 2 * (wl.D_qk - wl.D_v)) + wl.T_q * wl.H * (wl.D_qk + wl.D_v) * 2
    stage["index_score"]["frac"] = round(idx_bytes / (stage["index_score"]["ms"] * 1e-3) / hbm, 4)
    stage["sparse_mla"]["frac"] = round(attn_bytes / (stage["sparse_mla"]["ms"] * 1e-3) / hbm, 4)
    out["decode_fp8"] = {"workload": "128 sequences x 65536 keys, FP8 index keys (fp32 scale per key), "
                                     "FP8 latent (fp32 scale per token) + bf16 rope, Top-2048, 128 heads",
                         "ms_per_step": round(ms, 4), "value": wl.T_q / (ms * 1e-3), "unit": UNIT,
                         "bound": "hbm", "bytes": byt,
                         "frac": round(byt / (ms * 1e-3) / hbm, 4), "stages": stage}
    # the same batch with the index queries and keys in MXFP8 (one E8M0 byte per 32 dims): the
    # step quantizes q_I to MX codes and scales (hsa_quantize_mx, one kernel) and scores them
    # against the MX key cache with the block-scaled MMA (hsa_index_score_mx inside the step)
    kmx, kmx_e = hsa.hsa_quantize_mx(wl.k_I)
    qI_flat = wl.q_I.view(-1, wl.D_I)
    q_codes = torch.empty(qI_flat.shape, dtype=torch.uint8, device=dev)
    q_e = torch.empty((qI_flat.shape[0], wl.D_I // 32), dtype=torch.uint8, device=dev)

    def mx_step():
        hsa.hsa_quantize_mx(qI_flat, codes=q_codes, scales=q_e, stream=main)
        hsa.hsa_fused_decode(seq, q_codes.view(wl.q_I.shape), wl.w, kmx, kmx_e, wl.q, kv8, kvs, rope,
                             wl.K, wl.D_v, wl.softmax_scale, scores=sc, idx=idx, out=o, lse=lse,
                             ws=ws, stream=main, q_I_scale=q_e)
    for _ in range(3):
        mx_step()
    ms = _timed(mx_step, reps, flush_l2, main)
    n_q = wl.T_q * wl.H_I
    # the index kernel reads codes + scale words instead of bf16 queries; the quantizer reads the
    # bf16 queries and writes codes and scales
    byt_mx = byt - n_q * wl.D_I * 2 + n_q * (wl.D_I + 4) + n_q * (wl.D_I * 2 + wl.D_I + 4)
    stage_mx = stage_times(
        [lambda: hsa.hsa_quantize_mx(qI_flat, codes=q_codes, scales=q_e, stream=main),
         lambda: hsa.hsa_index_score(seq, q_codes.view(wl.q_I.shape), wl.w, kmx, kmx_e, scores=sc,
                                     stream=main, q_scale=q_e)],
        ["quantize_q", "index_score_mx"], reps, flush_l2, main)
    idx_mx_bytes = int(n.sum()) * (wl.D_I + 4 + 4) + n_q * (wl.D_I + 4 + 4)
    stage_mx["index_score_mx"]["frac"] = round(idx_mx_bytes / (stage_mx["index_score_mx"]["ms"] * 1e-3) / hbm, 4)
    out["decode_mxfp8"] = {"workload": "the FP8 decode batch with MXFP8 index queries and keys "
                                       "(E8M0 scale per 32 dims, block-scaled MMA on the codes), "
                                       "quantization of q_I included",
                           "ms_per_step": round(ms, 4), "value": wl.T_q / (ms * 1e-3), "unit": UNIT,
                           "bound": "hbm", "bytes": byt_mx,
                           "frac": round(byt_mx / (ms * 1e-3) / hbm, 4), "stages": stage_mx}
    del kmx, kmx_e, q_codes, q_e
    # KV-cache quantizer on the same cache (8.4 M rows): read 1152 B, write 512 + 4 + 128 B per row
    nrow = wl.kv.shape[0]

    def quant():
        hsa.hsa_quantize_kv(wl.kv, wl.D_v, wl.D_v, codes=kv8, scales=kvs.view(-1, 1), rope_cache=rope,
                            stream=main)
    quant()
    ms = _timed(quant, reps, flush_l2, main)
    byt = nrow * (wl.D_qk * 2 + wl.D_v + 4 + 2 * (wl.D_qk - wl.D_v))
    out["quantize_kv"] = {"workload": f"{nrow} cache rows of 512 latent + 64 rope bf16",
                          "ms": round(ms, 4), "value": nrow / (ms * 1e-3), "unit": "rows/s",
                          "bound": "hbm", "bytes": byt, "frac": round(byt / (ms * 1e-3) / hbm, 4)}
    del wl, k8, ks, kv8, kvs, rope, sc, idx, o, lse, ws, seq
    torch.cuda.empty_cache()

    # draft-verify decode: the bf16 decode batch with 4 query rows per sequence (the last 4
    # positions).  The four rows of a sequence share one pass over its index keys; the bytes
    # counted are the keys once per sequence plus the distinct cache rows the four selections
    # name (measured from the step's own idx), q, q_I, w and the outputs.
    wl = workloads.make("decode_draft_bf16", dev)
    seq = hsa.PagedSeq(wl.seq_lens, wl.block_table, wl.page_size, wl.num_pages, wl.q_seq, wl.q_pos,
                       q_run=wl.q_run)
    sc = torch.empty((wl.T_q, seq.max_seq_len), dtype=torch.float32, device=dev)
    idx = torch.empty((wl.T_q, wl.K), dtype=torch.int32, device=dev)
    o = torch.empty((wl.T_q, wl.H, wl.D_v), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((wl.T_q, wl.H), dtype=torch.float32, device=dev)
    ws = torch.zeros(max(1, hsa.hsa_fused_decode_workspace_size(seq, wl.q, wl.kv, wl.D_v, wl.K)),
                     dtype=torch.uint8, device=dev)

    def draft_step():
        hsa.hsa_fused_decode(seq, wl.q_I, wl.w, wl.k_I, None, wl.q, wl.kv, None, None, wl.K,
                             wl.D_v, wl.softmax_scale, scores=sc, idx=idx, out=o, lse=lse, ws=ws,
                             stream=main)
    for _ in range(3):
        draft_step()
    ms = _timed(draft_step, reps, flush_l2, main)
    main.synchronize()
    rows_read = 0
    for b in range(wl.B):
        sel = idx[b * wl.q_run:(b + 1) * wl.q_run]
        rows_read += int(torch.unique(sel[sel >= 0]).numel())
    byt = int(wl.seq_lens.long().sum()) * wl.D_I * 2 + rows_read * wl.D_qk * 2 + \
        wl.T_q * wl.H * (wl.D_qk + wl.D_v) * 2 + wl.T_q * wl.H_I * (wl.D_I * 2 + 4)
    out["decode_draft_bf16"] = {
        "workload": f"{wl.B} sequences x 8192..32768 keys, {wl.q_run} draft rows per sequence "
                    "(draft-verify), bf16 caches, Top-2048, 128 heads",
        "ms_per_step": round(ms, 4), "value": wl.T_q / (ms * 1e-3), "unit": UNIT,
        "bound": "hbm", "bytes": byt, "distinct_rows_gathered": rows_read,
        "frac": round(byt / (ms * 1e-3) / hbm, 4)}
    del wl, sc, idx, o, lse, ws, seq
    torch.cuda.empty_cache()

    out["decode_bf16_block_aligned"] = block_aligned(dev, flush_l2, main, peaks, reps)

    # causal prefill: the bf16 16384-token workload (4 chunks of 4096 in zigzag pairs) and the
    # 131072-token workload with FP8 index keys (32 chunks of 4096 in zigzag pairs)
    out["prefill_bf16"] = prefill_measure("prefill_bf16", dev, flush_l2, main, peaks, 4, reps)
    out["prefill_long_zigzag"] = prefill_measure("prefill_long_zigzag", dev, flush_l2, main, peaks,
                                                 None, 2)
    return out


def prefill_measure(name, dev, flush_l2, main, peaks, n_chunks, reps):
    """One causal prefill workload: the whole pass (hsa_prefill_chunked, chunk pairs on two
    streams, caller-owned score buffers) timed with CUDA events, plus the time of each kernel
    (index score, Top-K, sparse MLA) from a second pass that issues every chunk's three calls on
    one stream with events between them.  Fractions are of the burst bf16 tensor peak (the calls
    are sub-second, not the seconds-long loop the sustained figure describes)."""
    import sparse_index_attention_b200 as hsa
    wl = workloads.make(name, dev)
    chunks = wl.chunks if n_chunks is None else workloads.zigzag_chunks(wl.T_q, n_chunks)
    k, ks = wl.k_I, None
    if wl.index_fp8:
        k, ks = hsa.hsa_quantize_index(wl.k_I, wl.D_I)
        ks = ks.view(-1)
    seq = hsa.PagedSeq(wl.seq_lens, wl.block_table, wl.page_size, wl.num_pages, wl.q_seq, wl.q_pos,
                       q_run=wl.q_run)
    o = torch.empty((wl.T_q, wl.H, wl.D_v), dtype=torch.bfloat16, device=dev)
    idx = torch.empty((wl.T_q, wl.K), dtype=torch.int32, device=dev)
    streams = (torch.cuda.Stream(), torch.cuda.Stream())
    bufs = hsa.prefill_score_buffers(seq, chunks, dev)

    def prefill():
        hsa.hsa_prefill_chunked(seq, wl.q_I, wl.w, k, ks, wl.q, wl.kv, None, None, wl.K,
                                wl.D_v, wl.softmax_scale, chunks, out=o, lse=False, idx=idx,
                                streams=streams, score_bufs=bufs)
    prefill()
    ms = _timed(prefill, max(2, reps), flush_l2, main)
    # per-kernel times: every chunk's calls on `main`, events around each call
    names = ["index_score", "topk", "sparse_mla"]
    tot = {n: 0.0 for n in names}
    flush_l2()
    evs = []
    for r0, r1 in chunks:
        part = seq.rows(r0, r1, q_run=min(seq.q_run, r1 - r0))
        sc = bufs[0][:r1 - r0]
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        e[0].record(main)
        hsa.hsa_index_score(part, wl.q_I[r0:r1], wl.w[r0:r1], k, ks, scores=sc, stream=main)
        e[1].record(main)
        hsa.hsa_topk(part, sc, wl.K, idx=idx[r0:r1], stream=main)
        e[2].record(main)
        hsa.hsa_sparse_mla_attn(part, wl.q[r0:r1], wl.kv, idx[r0:r1], wl.D_v, wl.softmax_scale,
                                out=o[r0:r1], lse=False, stream=main)
        e[3].record(main)
        evs.append(e)
    torch.cuda.synchronize()
    for e in evs:
        for j, n in enumerate(names):
            tot[n] += e[j].elapsed_time(e[j + 1])
    n = (wl.q_pos.long() + 1).cpu()
    idx_flops = int(n.sum()) * wl.H_I * wl.D_I * 2
    attn_flops = int(torch.clamp(n, max=wl.K).sum()) * wl.H * (wl.D_qk + wl.D_v) * 2
    flops = idx_flops + attn_flops
    peak = peaks["bf16_tflops"] * 1e12
    stage = {
        "index_score": {"ms": round(tot["index_score"], 3), "flops": idx_flops,
                        "TFLOP/s": round(idx_flops / (tot["index_score"] * 1e-3) / 1e12, 1),
                        "frac": round(idx_flops / (tot["index_score"] * 1e-3) / peak, 4)},
        "topk": {"ms": round(tot["topk"], 3)},
        "sparse_mla": {"ms": round(tot["sparse_mla"], 3), "flops": attn_flops,
                       "TFLOP/s": round(attn_flops / (tot["sparse_mla"] * 1e-3) / 1e12, 1),
                       "frac": round(attn_flops / (tot["sparse_mla"] * 1e-3) / peak, 4)},
    }
    desc = (f"one sequence of {wl.T_q} tokens, every token a query, Top-{wl.K}, "
            f"{len(chunks)} chunks of {chunks[0][1] - chunks[0][0]} in zigzag pairs on two streams"
            + (", FP8 index keys (fp32 scale per key)" if wl.index_fp8 else ", bf16 caches"))
    res = {"workload": desc, "ms_per_step": round(ms, 3), "value": wl.T_q / (ms * 1e-3), "unit": UNIT,
           "bound": "tensor", "flops": flops, "frac": round(flops / (ms * 1e-3) / peak, 4),
           "peak": f"bf16_tflops {peaks['bf16_tflops']} (burst, MEASURED_PEAKS.json)",
           "stages_one_stream": stage}
    del wl, seq, o, idx, bufs, k, ks
    torch.cuda.empty_cache()
    return res


def run_ours(args, rank, world, local_rank):
    import sparse_index_attention_b200 as hsa
    dist = None
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))

    wl = workloads.make(WORKLOAD, dev)
    seq = hsa.PagedSeq(wl.seq_lens, wl.block_table, wl.page_size, wl.num_pages, wl.q_seq, wl.q_pos,
                       q_run=wl.q_run)
    ld = seq.max_seq_len
    scores = torch.empty((wl.T_q, ld), dtype=torch.float32, device=dev)
    idx = torch.empty((wl.T_q, wl.K), dtype=torch.int32, device=dev)
    out = torch.empty((wl.T_q, wl.H, wl.D_v), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((wl.T_q, wl.H), dtype=torch.float32, device=dev)
    ws = torch.zeros(max(1, hsa.hsa_fused_decode_workspace_size(seq, wl.q, wl.kv, wl.D_v, wl.K)),
                     dtype=torch.uint8, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def flush_l2():
        flush.zero_()
        flush.view(torch.float32).sum()
    main = torch.cuda.current_stream()
    aux = torch.cuda.Stream()

    def step(q_I=wl.q_I, w=wl.w, q=wl.q, aux_stream=None, out_t=None):
        hsa.hsa_fused_decode(seq, q_I, w, wl.k_I, None, q, wl.kv, None, None, wl.K, wl.D_v,
                             wl.softmax_scale, scores=scores, idx=idx,
                             out=out if out_t is None else out_t, lse=lse, ws=ws,
                             stream=main, aux_stream=aux_stream)

    barrier, max_over_ranks = rank_ops(dist, dev)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # ---- timed region: K fused steps, L2 flushed before each ----
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    launches0 = hsa.hsa_launch_count()
    wall0 = time.perf_counter()
    with ClockSampler(local_rank) as clocks:
        for i in range(args.steps):
            flush_l2()
            starts[i].record(main)
            step()
            ends[i].record(main)
        torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    barrier()
    launches = hsa.hsa_launch_count() - launches0
    t_ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    t_ms = max_over_ranks(t_ms)
    value = replica_throughput(world, wl.T_q, args.steps, t_ms)

    # ---- the same step on two streams (hsa_fused_decode with an auxiliary stream)
    reps2 = max(3, min(args.steps, 50))
    ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps2)]
    for i in range(reps2):
        flush_l2()
        ev2[i][0].record(main)
        step(aux_stream=aux)
        ev2[i][1].record(main)
    torch.cuda.synchronize()
    two_ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in ev2))

    # ---- per-kernel times: the three C-ABI calls on one stream, events between them ----
    reps = max(3, min(args.steps, 50))
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(reps)]
    for i in range(reps):
        flush_l2()
        ev[i][0].record(main)
        hsa.hsa_index_score(seq, wl.q_I, wl.w, wl.k_I, None, scores=scores, stream=main)
        ev[i][1].record(main)
        hsa.hsa_topk(seq, scores, wl.K, idx=idx, stream=main)
        ev[i][2].record(main)
        hsa.hsa_sparse_mla_attn(seq, wl.q, wl.kv, idx, wl.D_v, wl.softmax_scale, out=out, lse=lse,
                                ws=ws, stream=main)
        ev[i][3].record(main)
    torch.cuda.synchronize()
    names = ["index_score", "topk", "sparse_mla"]
    stage_ms = {n: statistics.mean(e[j].elapsed_time(e[j + 1]) for e in ev) for j, n in enumerate(names)}
    work = algorithmic_work(wl)
    peaks = load_peaks()
    stages = {}
    for n in names:
        ms = stage_ms[n]
        stages[n] = {"ms": round(ms, 4), "GB/s": round(work[n]["bytes"] / (ms * 1e-3) / 1e9, 1),
                     "TFLOP/s": round(work[n]["flops"] / (ms * 1e-3) / 1e12, 2),
                     "bytes": work[n]["bytes"], "flops": work[n]["flops"]}
    dom = max(names, key=lambda n: stage_ms[n])
    achieved = work[dom]["bytes"] / (stage_ms[dom] * 1e-3) / 1e9
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "dram_traffic_decode_bf16.json")
    try:
        import hashlib
        rec = json.load(open(tpath))["kernels"][dom]
        cur = hashlib.sha256(open(os.path.join(ROOT, rec["source"]), "rb").read()).hexdigest()[:16]
        if cur == rec["source_sha256_16"]:       # counters taken on this very kernel source
            traffic = rec["traffic_bytes"]
    except Exception:
        traffic = None
    roofline = {"kernel": dom, "bound": "hbm", "achieved": round(achieved, 1),
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": traffic, "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json hbm_gbs)"
                if peaks["source"] == "measured" else "fallback 6.65 TB/s"}

    # ---- end to end through the C ABI with host buffers: every step copies its query inputs in
    # from pinned host memory and its output back out.  The copies run on their own streams with
    # double-buffered device tensors, so that step i+1's inputs and step i-1's output cross PCIe
    # while step i computes, as a serving loop would run it. ----
    h_qI = torch.empty_like(wl.q_I, device="cpu").pin_memory()
    h_w = torch.empty_like(wl.w, device="cpu").pin_memory()
    h_q = torch.empty_like(wl.q, device="cpu").pin_memory()
    h_qI.copy_(wl.q_I)
    h_w.copy_(wl.w)
    h_q.copy_(wl.q)
    h_out = [torch.empty_like(out, device="cpu").pin_memory() for _ in range(2)]
    dbuf = [(torch.empty_like(wl.q_I), torch.empty_like(wl.w), torch.empty_like(wl.q), torch.empty_like(out))
            for _ in range(2)]
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs landed
    ev_comp = [torch.cuda.Event() for _ in range(2)]   # step done: inputs free, output ready
    ev_out = [torch.cuda.Event() for _ in range(2)]    # output copied out: buffer free
    e_steps = max(3, min(args.steps, 50))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier()
    e0.record(main)
    h2d_s.wait_event(e0)
    d2h_s.wait_event(e0)
    for i in range(e_steps):
        b = i % 2
        d_qI, d_w, d_q, d_out = dbuf[b]
        if i >= 2:
            h2d_s.wait_event(ev_comp[b])      # step i-2 has finished reading these inputs
        with torch.cuda.stream(h2d_s):
            d_qI.copy_(h_qI, non_blocking=True)
            d_w.copy_(h_w, non_blocking=True)
            d_q.copy_(h_q, non_blocking=True)
        ev_in[b].record(h2d_s)
        main.wait_event(ev_in[b])
        if i >= 2:
            main.wait_event(ev_out[b])        # step i-2's output has left this buffer
        step(d_qI, d_w, d_q, out_t=d_out)
        ev_comp[b].record(main)
        d2h_s.wait_event(ev_comp[b])
        with torch.cuda.stream(d2h_s):
            h_out[b].copy_(d_out, non_blocking=True)
        ev_out[b].record(d2h_s)
    main.wait_stream(h2d_s)
    main.wait_stream(d2h_s)
    e1.record(main)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1))
    h2d = h_qI.numel() * h_qI.element_size() + h_w.numel() * 4 + h_q.numel() * h_q.element_size()
    d2h = h_out[0].numel() * h_out[0].element_size()
    e2e = {"value": world * wl.T_q * e_steps / (e2e_ms * 1e-3), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e_steps,
           "note": "copies on their own streams, double-buffered, overlapping the neighbouring "
                   "steps' compute; L2 not flushed between end-to-end steps"}

    other = None
    if rank == 0 and world == 1 and not args.no_secondary:
        other = secondary(dev, flush_l2, main, load_peaks(), reps=max(3, min(args.steps, 10)))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rows = list(range(args.cpu_rows))
        v, secs, threads = cpu_baseline(wl, rows)
        cpu = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"{len(rows)} query rows of the batch (index score over each full context, "
                         f"Top-2048, 128-head sparse MLA), {secs:.1f} s"}

    if dist is not None:
        dist.barrier()
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_ms / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic", "config": workload_config(wl),
                "parallelism": f"replicas x{world} (independent decode batches, no collective on the data path)",
                "roofline": roofline, "stages": stages,
                "two_stream": {"ms_per_step": round(two_ms, 4),
                               "value": world * wl.T_q / (two_ms * 1e-3), "unit": UNIT},
                "cpu_baseline": cpu, "e2e": e2e, "other_workloads": other,
                "gpu_launches": launches, "clocks": clocks.summary(),
                "wall_s_timed_region": round(wall, 3)}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def run_profile_case(args):
    """A small causal prefill (prefill_bf16 shapes, --profile-rows query rows of one sequence):
    index score, Top-K and sparse MLA, each called three times on one stream, nothing timed.
    For one-kernel ncu captures of the prefill kernels at a size whose capture ends quickly."""
    import sparse_index_attention_b200 as hsa
    dev = "cuda"
    wl = workloads.make("prefill_bf16", dev, T=args.profile_rows)
    seq = hsa.PagedSeq(wl.seq_lens, wl.block_table, wl.page_size, wl.num_pages, wl.q_seq, wl.q_pos,
                       q_run=wl.q_run)
    sc = hsa.hsa_index_score(seq, wl.q_I, wl.w, wl.k_I)
    idx = hsa.hsa_topk(seq, sc, wl.K)
    out, _ = hsa.hsa_sparse_mla_attn(seq, wl.q, wl.kv, idx, wl.D_v, wl.softmax_scale, lse=False)
    for _ in range(2):
        hsa.hsa_index_score(seq, wl.q_I, wl.w, wl.k_I, scores=sc)
        hsa.hsa_topk(seq, sc, wl.K, idx=idx)
        hsa.hsa_sparse_mla_attn(seq, wl.q, wl.kv, idx, wl.D_v, wl.softmax_scale, out=out, lse=False)
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": "prefill_bf16", "rows": wl.T_q, "launches_per_kernel": 3}))


def run_profile_decode_fp8(args):
    """The FP8 decode batch's shapes with --profile-fp8-seqs sequences of 65536 keys (E4M3 index
    keys with fp32 scales, FP8 latent cache): index score, Top-K and sparse MLA, each called
    three times on one stream, nothing timed.  For one-kernel ncu captures."""
    import sparse_index_attention_b200 as hsa
    dev = "cuda"
    wl = workloads.make("decode_fp8", dev, B=args.profile_fp8_seqs)
    seq = hsa.PagedSeq(wl.seq_lens, wl.block_table, wl.page_size, wl.num_pages, wl.q_seq, wl.q_pos,
                       q_run=wl.q_run)
    k8, ks = hsa.hsa_quantize_index(wl.k_I, wl.D_I)
    ks = ks.view(-1)
    kv8, kvs, rope = hsa.hsa_quantize_kv(wl.kv, wl.D_v, wl.D_v)
    kvs = kvs.view(-1)
    sc = hsa.hsa_index_score(seq, wl.q_I, wl.w, k8, ks)
    idx = hsa.hsa_topk(seq, sc, wl.K)
    out, lse = hsa.hsa_sparse_mla_attn(seq, wl.q, kv8, idx, wl.D_v, wl.softmax_scale, kv_scale=kvs,
                                       kv_rope=rope)
    for _ in range(2):
        hsa.hsa_index_score(seq, wl.q_I, wl.w, k8, ks, scores=sc)
        hsa.hsa_topk(seq, sc, wl.K, idx=idx)
        hsa.hsa_sparse_mla_attn(seq, wl.q, kv8, idx, wl.D_v, wl.softmax_scale, kv_scale=kvs,
                                kv_rope=rope, out=out, lse=lse)
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": "decode_fp8", "sequences": wl.B, "launches_per_kernel": 3}))


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-rows", type=int, default=16, help="query rows for the oracle baseline")
    ap.add_argument("--ref-rows", type=int, default=0,
                    help="query rows per step of the reference arm (default: the oracle's threads)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the FP8 decode, prefill and quantizer measurements")
    ap.add_argument("--profile-rows", type=int, default=0,
                    help="only run a small prefill of this many rows (three calls of each kernel, "
                         "for ncu captures) and exit")
    ap.add_argument("--profile-fp8-seqs", type=int, default=0,
                    help="only run the FP8 decode kernels on this many 65536-key sequences (three "
                         "calls each, for ncu captures) and exit")
    args = ap.parse_args()
    if args.profile_rows > 0:
        run_profile_case(args)
        return
    if args.profile_fp8_seqs > 0:
        run_profile_decode_fp8(args)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
