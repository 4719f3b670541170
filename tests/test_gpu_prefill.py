"""GPU parity of the prefill workloads at their full sizes (sampled rows against the oracle,
Top-K bit-exact on the GPU's own scores for every row) and of the zigzag chunk schedule
(bitwise equal to the sequential schedule: the pages state that the layout does not change the
semantics -- "Inference Adaptation and Performance Optimization for a Domestically Developed
LLM's New Architecture", 5.2)."""
import numpy as np
import pytest
import torch

import oracle
import sparse_index_attention_b200 as hsa
from sparse_index_attention_b200 import workloads

from helpers import (GpuCaches, OracleCaches, attention_vs_oracle, check_selection_vs_oracle,
                     check_status, compact_workload, index_tolerance_ok, oracle_paging, paged_seq)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def stable_topk_batched(scores, q_pos, K):
    """Reference selection on the same fp32 scores for all rows at once (torch stable sort)."""
    T, ld = scores.shape
    pos = q_pos.long().to(scores.device)
    col = torch.arange(ld, device=scores.device)
    sc = scores.clone()
    sc[sc == 0] = 0.0                                  # -0.0 == +0.0
    sc[col[None, :] > pos[:, None]] = -float("inf")
    order = torch.sort(sc, dim=1, descending=True, stable=True).indices[:, :K]
    sel = order.sort(dim=1).values.to(torch.int32)
    n = pos + 1
    short = n <= K
    if short.any():
        ar = torch.arange(K, device=scores.device)
        pad = torch.where(ar[None, :] < n[short][:, None], ar[None, :], torch.full_like(ar[None, :], -1))
        sel[short] = pad.to(torch.int32)
    return sel


def check_rows(wl_full, rows, sc, idx, out, tol):
    """Index tolerance, oracle-selection agreement with the near-tie check on every mismatch,
    and attention tolerance on the GPU's own selection, for the sampled rows (sc / idx / out
    hold those rows' GPU results, in order)."""
    wl = compact_workload(wl_full, rows)
    labels = list(rows)
    rows = list(range(wl.T_q))
    oc = OracleCaches(wl)
    pg = oracle_paging(wl)
    qI, w = oc.q_I, wl.w
    ld = sc.shape[1]
    ref_sc = oracle.index_score(pg, qI, w, oc.k, ld=ld)
    mag = oracle.index_score(pg, qI, w.abs(), oc.k, ld=ld)
    got = sc.cpu().numpy()
    n_valid = (wl.q_pos[rows] + 1).cpu().numpy().astype(np.int32)
    for i in range(len(rows)):
        n = n_valid[i]
        ok, worst = index_tolerance_ok(got[i, :n], ref_sc[i, :n], mag[i, :n])
        assert ok, ("index", labels[i], worst)
    gidx = idx.cpu().numpy()
    ref_idx = check_selection_vs_oracle(ref_sc, mag, gidx, n_valid, wl.K, labels)
    e2e = attention_vs_oracle(pg, wl.q, oc.kv, gidx, ref_idx, wl.D_v, wl.softmax_scale, out, tol)
    print(f"{wl.name}: end-to-end attention difference over {len(rows)} rows {e2e:.3g}")


def run_prefill(wl, chunks=None):
    gc = GpuCaches(wl)
    seq = paged_seq(wl)
    chunks = chunks or [(0, wl.T_q)]
    out, lse, idx = hsa.hsa_prefill_chunked(seq, wl.q_I, wl.w, gc.k, gc.k_scale, wl.q, gc.kv,
                                            gc.kv_scale, gc.kv_rope, wl.K, wl.D_v,
                                            wl.softmax_scale, chunks)
    check_status(seq)
    return gc, seq, out, lse, idx


def test_prefill_bf16_full_size():
    """16384-token causal prefill, every token a query, Top-2048 (rows t < 2048 select all)."""
    wl = workloads.make("prefill_bf16", DEV)
    gc = GpuCaches(wl)
    seq = paged_seq(wl)
    sc = hsa.hsa_index_score(seq, wl.q_I, wl.w, gc.k)
    idx = hsa.hsa_topk(seq, sc, wl.K)
    out, lse = hsa.hsa_sparse_mla_attn(seq, wl.q, gc.kv, idx, wl.D_v, wl.softmax_scale)
    check_status(seq)
    assert torch.equal(idx, stable_topk_batched(sc, wl.q_pos, wl.K))
    rows = workloads.sample_rows(wl.T_q, 1024, extra=(2046, 2047, 2048, 2049))
    check_rows(wl, rows, sc[rows], idx[rows], out[rows], 2e-2)


def test_zigzag_equals_sequential():
    wl = workloads.make("prefill_long_zigzag", DEV, T=8192, n_chunks=8)
    _, _, out_z, lse_z, idx_z = run_prefill(wl, wl.chunks)
    seq_order = sorted(wl.chunks)
    _, _, out_s, lse_s, idx_s = run_prefill(wl, seq_order)
    assert torch.equal(idx_z, idx_s) and torch.equal(out_z, out_s) and torch.equal(lse_z, lse_s)
    # one call over all rows gives the same bits as well
    _, _, out_1, lse_1, idx_1 = run_prefill(wl, [(0, wl.T_q)])
    assert torch.equal(idx_z, idx_1) and torch.equal(out_z, out_1)


def test_prefill_long_zigzag_full_size():
    """131072 tokens, 32 chunks of 4096 issued as zigzag pairs, FP8 index keys."""
    wl = workloads.make("prefill_long_zigzag", DEV)
    gc, seq, out, lse, idx = run_prefill(wl, wl.chunks)
    rows = workloads.sample_rows(wl.T_q, 16384, wl.chunks, extra=(2047, 2048))
    # Top-K bit-exact on the GPU's own scores for the sampled rows (scores recomputed per row:
    # the tile order of a key does not depend on the launch, so they are the scores the chunked
    # run selected from)
    part_scores = []
    for r in rows:
        s1 = hsa.hsa_index_score(seq.rows(r, r + 1, q_run=1), wl.q_I[r:r + 1], wl.w[r:r + 1], gc.k,
                                 gc.k_scale)
        part_scores.append(s1)
    sc_rows = torch.cat(part_scores)
    assert torch.equal(idx[rows], stable_topk_batched(sc_rows, wl.q_pos[rows], wl.K))
    check_rows(wl, rows, sc_rows, idx[rows], out[rows], 2e-2)


def test_decode_fp8_full_size_sampled():
    """128 sequences of 65536 tokens, FP8 index keys and FP8 latent cache."""
    wl = workloads.make("decode_fp8", DEV)
    gc = GpuCaches(wl)
    seq = paged_seq(wl)
    out, lse, idx, sc = hsa.hsa_fused_decode(seq, wl.q_I, wl.w, gc.k, gc.k_scale, wl.q, gc.kv,
                                             gc.kv_scale, gc.kv_rope, wl.K, wl.D_v,
                                             wl.softmax_scale)
    check_status(seq)
    assert torch.equal(idx, stable_topk_batched(sc, wl.q_pos, wl.K))
    rows = [0, 77, 127]
    check_rows(wl, rows, sc[rows], idx[rows], out[rows], 6e-2)


def test_zigzag_cp_single_rank_equals_chunked_prefill():
    """The context-parallel prefill on one NCCL rank (segments 0 and 1 of 2, the cache gathered
    from itself and read through the rebuilt block table) gives the same bits as the chunked
    prefill over the workload's own paging: the whole host path down to the library kernels."""
    import datetime
    import socket
    import torch.distributed as dist
    from sparse_index_attention_b200 import cp
    wl = workloads.make("prefill_bf16", DEV, T=2048)
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device(DEV, 0))
    try:
        pos = cp.rank_positions(wl.T_q, 1, 0).to(DEV).long()
        slot = wl.block_table[0].long()[pos // wl.page_size] * wl.page_size + pos % wl.page_size
        out_c, lse_c, idx_c = cp.prefill_zigzag_cp(
            wl.T_q, wl.page_size, wl.q_I[pos], wl.w[pos], wl.q[pos], wl.k_I[slot], wl.kv[slot], wl.K,
            wl.D_v, wl.softmax_scale, gather_outputs=True)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    gc, seq, out, lse, idx = run_prefill(wl, [(0, 1024), (1024, 2048)])
    assert torch.equal(idx_c, idx) and torch.equal(out_c, out) and torch.equal(lse_c, lse)
    # the context-parallel result against the oracle on sampled rows (scores recomputed per row)
    rows = workloads.sample_rows(wl.T_q, 256, extra=(1023, 1024, 2047))
    sc_rows = torch.cat([hsa.hsa_index_score(seq.rows(r, r + 1, q_run=1), wl.q_I[r:r + 1],
                                             wl.w[r:r + 1], gc.k) for r in rows])
    check_rows(wl, rows, sc_rows, idx_c[rows], out_c[rows], 2e-2)
