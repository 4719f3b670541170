"""GPU parity of the whole path (index score -> Top-K -> sparse MLA) against the oracle, run end
to end on both sides from the same seeded inputs, plus the fused/two-stream invariants.

Checks per the path's contract:
  (i)   Top-K bit-exact against a reference selection (torch stable sort) on the GPU's own scores;
  (ii)  the oracle's own float64 selection agrees on >= 99.9% of positions, and every position in
        the symmetric difference is a near tie of the oracle's K-th score within the index-score
        tolerance;
  (iii) index scores within 1e-3 (|I_ref| + M); attention outputs within 2e-2 abs/rel (bf16),
        6e-2 (FP8 caches), 1e-4 (fp32) of the oracle's attention over the GPU's own selection
        (the end-to-end difference, over the oracle's own selection, is printed);
  (iv)  fused == unfused bitwise; two-stream == one-stream bitwise for scores and selections,
        and within rounding for attention (the halves cut rows between clusters elsewhere).
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_index_attention_b200 as hsa
from sparse_index_attention_b200 import workloads

from helpers import (GpuCaches, OracleCaches, attention_vs_oracle, check_selection_vs_oracle,
                     check_status, compact_workload, index_tolerance_ok, oracle_paging, paged_seq,
                     stable_topk_reference)

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = {"f32": 1e-4, "bf16": 2e-2}


def run_fused(wl, gc, aux=False):
    seq = paged_seq(wl)
    aux_stream = torch.cuda.Stream() if aux else None
    out, lse, idx, sc = hsa.hsa_fused_decode(seq, gc.q_I, wl.w, gc.k, gc.k_scale, wl.q, gc.kv,
                                             gc.kv_scale, gc.kv_rope, wl.K, wl.D_v,
                                             wl.softmax_scale, aux_stream=aux_stream)
    check_status(seq)
    return out, lse, idx, sc


def check_against_oracle(wl, rows, sc, idx, out):
    """(i)-(iii) on the sampled rows."""
    K = wl.K
    ref_sel = stable_topk_reference(sc[rows], wl.q_pos[rows], K)
    assert torch.equal(idx[rows], ref_sel), "Top-K differs from the stable-sort selection"
    oc = OracleCaches(wl)
    pg = oracle_paging(wl, rows)
    qI, w = oc.q_I[rows], wl.w[rows].cpu()
    ld = sc.shape[1]
    ref_sc = oracle.index_score(pg, qI, w, oc.k, ld=ld)
    mag = oracle.index_score(pg, qI, w.abs(), oc.k, ld=ld)
    got_sc = sc[rows].cpu().numpy()
    n_valid = (wl.q_pos[rows] + 1).cpu().numpy().astype(np.int32)
    for i in range(len(rows)):
        n = n_valid[i]
        ok, worst = index_tolerance_ok(got_sc[i, :n], ref_sc[i, :n], mag[i, :n])
        assert ok, ("index score", rows[i], worst)
    gidx = idx[rows].cpu().numpy()
    ref_idx = check_selection_vs_oracle(ref_sc, mag, gidx, n_valid, K, rows)
    tol = 6e-2 if (wl.kv_fp8 or wl.index_fp8) else TOL[wl.dtype]
    e2e = attention_vs_oracle(pg, wl.q[rows].cpu(), oc.kv, gidx, ref_idx, wl.D_v, wl.softmax_scale,
                              out[rows], tol)
    print(f"{wl.name}: end-to-end attention difference over {len(rows)} rows {e2e:.3g}")


@pytest.mark.parametrize("name,kw", [
    ("tiny_decode_fp32", {}),
    ("decode_bf16", dict(B=8, L_min=1500, L_max=5000)),
    ("decode_fp8", dict(B=4, L=4500)),
    ("decode_mxfp8", dict(B=4, L=4500)),
    ("decode_draft_bf16", dict(B=5, L_min=1500, L_max=5000)),
    ("decode_draft_bf16", dict(B=3, n_draft=2, L_min=2040, L_max=2052)),
])
def test_pipeline_vs_oracle_small(name, kw):
    wl = workloads.make(name, DEV, **kw)
    gc = GpuCaches(wl)
    out, lse, idx, sc = run_fused(wl, gc)
    check_against_oracle(wl, list(range(wl.T_q)), sc, idx, out)


@pytest.mark.parametrize("name,kw,kv_group", [
    ("tiny_decode_fp32", {}, None),
    ("decode_bf16", dict(B=8, L_min=1500, L_max=5000), None),
    ("decode_fp8", dict(B=6, L=3000), None),
    ("decode_fp8", dict(B=6, L=3000), 128),
    ("decode_draft_bf16", dict(B=6, L_min=1500, L_max=5000), None),
    ("decode_mxfp8", dict(B=6, L=3000), 128),
])
def test_fused_equals_unfused_and_two_streams(name, kw, kv_group):
    wl = workloads.make(name, DEV, **kw)
    gc = GpuCaches(wl, kv_group)
    out1, lse1, idx1, sc1 = run_fused(wl, gc, aux=False)
    out2, lse2, idx2, sc2 = run_fused(wl, gc, aux=True)
    seq = paged_seq(wl)
    sc3 = hsa.hsa_index_score(seq, gc.q_I, wl.w, gc.k, gc.k_scale)
    idx3 = hsa.hsa_topk(seq, sc3, wl.K)
    out3, lse3 = hsa.hsa_sparse_mla_attn(seq, wl.q, gc.kv, idx3, wl.D_v, wl.softmax_scale,
                                         kv_scale=gc.kv_scale, kv_rope=gc.kv_rope)
    torch.cuda.synchronize()
    for t in range(wl.T_q):
        n = int(wl.q_pos[t]) + 1
        assert torch.equal(sc1[t, :n], sc2[t, :n]) and torch.equal(sc1[t, :n], sc3[t, :n])
    assert torch.equal(idx1, idx2) and torch.equal(idx1, idx3)
    assert torch.equal(out1, out3) and torch.equal(lse1, lse3)
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2)


def test_decode_bf16_full_size_sampled():
    """The benchmark's workload and launch configuration (64 sequences, contexts 8192..32768,
    Top-2048, 128 heads, latent 512 + rope 64, two streams): Top-K bit-exact on every row,
    oracle checks on sampled rows."""
    wl = workloads.make("decode_bf16", DEV)
    gc = GpuCaches(wl)
    out, lse, idx, sc = run_fused(wl, gc, aux=True)
    ref_sel = stable_topk_reference(sc, wl.q_pos, wl.K)
    assert torch.equal(idx, ref_sel)
    rows = [0, 17, 40, 63]
    check_against_oracle(wl, rows, sc, idx, out)


def test_decode_draft_full_size_sampled():
    """Draft-verify decode at full size (64 sequences, contexts 8192..32768, four query rows per
    sequence at its last four positions, Top-2048, 128 heads): the four rows of a sequence share
    one pass over its index keys.  Top-K bit-exact on every row; oracle checks on all four rows
    of three sequences."""
    wl = workloads.make("decode_draft_bf16", DEV)
    gc = GpuCaches(wl)
    out, lse, idx, sc = run_fused(wl, gc)
    ref_sel = stable_topk_reference(sc, wl.q_pos, wl.K)
    assert torch.equal(idx, ref_sel)
    rows = [r for b in (0, 29, 63) for r in range(4 * b, 4 * b + 4)]
    check_against_oracle(wl, rows, sc, idx, out)


def test_decode_mxfp8_full_size_sampled():
    """The tiered-quantization decode at full size (128 sequences x 65536 keys, Top-2048) with
    the index queries and keys in MXFP8 and the latent cache in FP8: Top-K bit-exact on every
    row, oracle checks on three rows."""
    wl = workloads.make("decode_mxfp8", DEV)
    gc = GpuCaches(wl)
    out, lse, idx, sc = run_fused(wl, gc)
    ref_sel = stable_topk_reference(sc, wl.q_pos, wl.K)
    assert torch.equal(idx, ref_sel)
    rows = [0, 77, 127]
    small = compact_workload(wl, rows)    # the oracle quantizes only these rows' pages
    del gc
    check_against_oracle(small, list(range(len(rows))), sc[rows], idx[rows], out[rows])


def test_draft_verify_with_mxfp8_index_and_fp8_latent():
    """Draft-verify rows (four per sequence, scored four to an MMA tile) over the tiered caches:
    MXFP8 index queries and keys, FP8 latent cache with a scale per token; all rows against the
    oracle, and the fused call equal to the three calls in sequence."""
    wl = workloads.make("decode_draft_bf16", DEV, B=6, L_min=1500, L_max=5000)
    wl.index_fp8 = wl.index_mx = wl.kv_fp8 = True
    gc = GpuCaches(wl)
    out, lse, idx, sc = run_fused(wl, gc)
    check_against_oracle(wl, list(range(wl.T_q)), sc, idx, out)
    seq = paged_seq(wl)
    sc3 = hsa.hsa_index_score(seq, gc.q_I, wl.w, gc.k, gc.k_scale)
    idx3 = hsa.hsa_topk(seq, sc3, wl.K)
    out3, lse3 = hsa.hsa_sparse_mla_attn(seq, wl.q, gc.kv, idx3, wl.D_v, wl.softmax_scale,
                                         kv_scale=gc.kv_scale, kv_rope=gc.kv_rope)
    assert torch.equal(idx, idx3) and torch.equal(out, out3) and torch.equal(lse, lse3)


@pytest.mark.parametrize("mx", [True, False])
def test_decode_prolog_three_streams_equals_one_shot_caches(mx):
    """The decode prolog writes the newest token of every sequence into caches that hold the
    rest (index keys MXFP8 or E4M3, latent FP8 per token, rope bf16) and rounds q_I onto the
    MX grid, on three streams.  Caches and queries must equal, bit for bit, those written by
    one quantizer call over all rows, and so must the decode step that follows."""
    wl = workloads.make("decode_fp8", DEV, B=4, L=3000)
    n = wl.num_slots
    last = torch.tensor([int(wl.block_table[b, (int(wl.seq_lens[b]) - 1) // wl.page_size]) * wl.page_size
                         + (int(wl.seq_lens[b]) - 1) % wl.page_size for b in range(wl.B)],
                        dtype=torch.int64, device=DEV)
    if mx:
        k_ref, ks_ref = hsa.hsa_quantize_mx(wl.k_I)
    else:
        k_ref, ks_ref = hsa.hsa_quantize_index(wl.k_I, wl.D_I)
        ks_ref = ks_ref.view(-1)
    kv_ref, kvs_ref, rope_ref = hsa.hsa_quantize_kv(wl.kv, wl.D_v, wl.D_v)
    kvs_ref = kvs_ref.view(-1)
    k, ks, kv, kvs, rope = (t.clone() for t in (k_ref, ks_ref, kv_ref, kvs_ref, rope_ref))
    for t in (k, ks, kv, kvs, rope):
        t[last] = 0
    q_out = torch.empty_like(wl.q_I)
    q_codes = torch.empty(wl.q_I.shape, dtype=torch.uint8, device=DEV) if mx else None
    q_sc = torch.empty((wl.T_q, wl.H_I, wl.D_I // 32), dtype=torch.uint8, device=DEV) if mx else None
    hsa.hsa_decode_prolog(wl.k_I[last], wl.kv[last], last, k, ks, kv, kvs, rope, wl.q_I, q_out, wl.D_v,
                          q_codes_out=q_codes, q_scale_out=q_sc)
    torch.cuda.synchronize()
    for got, ref in ((k, k_ref), (ks, ks_ref), (kv, kv_ref), (kvs, kvs_ref), (rope, rope_ref)):
        assert torch.equal(got, ref)
    assert torch.equal(q_out, hsa.mx_round(wl.q_I))
    # the rows the prolog wrote, against the oracle's own quantizers of the same source rows
    src_k = wl.k_I[last].float().cpu()
    if mx:
        rc, rs = oracle.mx_quantize_rows(src_k)
        assert np.array_equal(k[last].cpu().numpy(), rc) and np.array_equal(ks[last].cpu().numpy(), rs)
    else:
        rc, rs = oracle.quantize_rows(src_k, wl.D_I)
        assert np.array_equal(k[last].cpu().numpy(), rc)
        assert np.array_equal(ks[last].cpu().numpy(), rs[:, 0])
    rc, rs = oracle.quantize_rows(wl.kv[last][:, :wl.D_v].float().cpu(), wl.D_v)
    assert np.array_equal(kv[last].cpu().numpy(), rc) and np.array_equal(kvs[last].cpu().numpy(), rs[:, 0])
    assert torch.equal(rope[last], wl.kv[last][:, wl.D_v:])
    # q_I on the MX grid: the oracle's quantize-then-dequantize, rounded to bf16 (exact here:
    # every block exponent of N(0, 1) data is far above the bf16 subnormal range)
    qf = wl.q_I.float().cpu().reshape(-1, wl.D_I)
    qc_ref, qs_ref = oracle.mx_quantize_rows(qf)
    q_ref = oracle.mx_dequantize_rows(qc_ref, qs_ref)
    assert np.array_equal(q_out.float().cpu().numpy().reshape(q_ref.shape), q_ref)
    if mx:   # the queries' MXFP8 codes and scales for the block-scaled index path
        assert np.array_equal(q_codes.cpu().numpy().reshape(qc_ref.shape), qc_ref)
        assert np.array_equal(q_sc.cpu().numpy().reshape(qs_ref.shape), qs_ref)
    seq = paged_seq(wl)
    a = hsa.hsa_fused_decode(seq, q_out, wl.w, k, ks, wl.q, kv, kvs, rope, wl.K, wl.D_v,
                             wl.softmax_scale)
    b = hsa.hsa_fused_decode(seq, hsa.mx_round(wl.q_I), wl.w, k_ref, ks_ref, wl.q, kv_ref, kvs_ref,
                             rope_ref, wl.K, wl.D_v, wl.softmax_scale)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    if mx:
        # the step on the codes (block-scaled MMA): same scores up to the index tolerance
        c = hsa.hsa_fused_decode(seq, q_codes, wl.w, k, ks, wl.q, kv, kvs, rope, wl.K, wl.D_v,
                                 wl.softmax_scale, q_I_scale=q_sc)
        mag = hsa.hsa_index_score(seq, q_out, wl.w.abs(), k, ks)
        for t in range(wl.T_q):
            n = int(wl.q_pos[t]) + 1
            ok, worst = index_tolerance_ok(c[3][t, :n].cpu().numpy(), a[3][t, :n].cpu().numpy().astype(np.float64),
                                           mag[t, :n].cpu().numpy().astype(np.float64))
            assert ok, (t, worst)


@pytest.mark.parametrize("aux", [False, True])
def test_decode_graph_replays_bitwise(aux):
    """The fused decode step captured as a CUDA graph equals the direct call bitwise, and a
    replay after new query rows are written into the captured inputs follows them."""
    wl = workloads.make("decode_bf16", DEV, B=8, L_min=1500, L_max=5000)
    gc = GpuCaches(wl)
    seq = paged_seq(wl)
    g = hsa.DecodeGraph(seq, wl.q_I, wl.w, gc.k, gc.k_scale, wl.q, gc.kv, gc.kv_scale, gc.kv_rope,
                        wl.K, wl.D_v, wl.softmax_scale, aux=aux)
    for it in range(2):
        if it == 1:                                  # next step's queries, same buffers
            wl.q.mul_(-1.0)
            wl.q_I.copy_(torch.roll(wl.q_I, 1, dims=0))
        out_g, lse_g, idx_g, _ = (t.clone() for t in g.replay())
        torch.cuda.synchronize()
        out_d, lse_d, idx_d, _ = hsa.hsa_fused_decode(seq, wl.q_I, wl.w, gc.k, gc.k_scale, wl.q, gc.kv,
                                                      gc.kv_scale, gc.kv_rope, wl.K, wl.D_v,
                                                      wl.softmax_scale)
        torch.cuda.synchronize()
        assert torch.equal(idx_g, idx_d) and torch.equal(out_g, out_d) and torch.equal(lse_g, lse_d)
        # the replayed step against the oracle on this step's inputs
        check_against_oracle(wl, [0, 3, 7], g.scores, idx_g, out_g)
    check_status(seq)


def _growing_decode(wl, steps):
    """A decode loop's state before its first step: every sequence holds `steps` tokens fewer
    than the workload, each crosses into a new cache page during the loop, the caches hold no
    rows for the missing tokens yet (zeroed slots) and the block table has no entries for the
    pages still to come (an out-of-range page id, which a kernel would report as a bad page if
    it read one)."""
    P = wl.page_size
    final = wl.seq_lens.tolist()
    len0 = []
    for b, L in enumerate(final):
        m = (L - steps + 1) // P
        len0.append(P * m - 1 - (b % 2))
    len0_t = torch.tensor(len0, dtype=torch.int32, device=DEV)
    bt_true = wl.block_table.clone()
    bt = bt_true.clone()
    for b, n0 in enumerate(len0):
        bt[b, (n0 + P - 1) // P:] = wl.num_pages + 7
    return len0, len0_t, bt_true, bt


def _slot_of(bt_true, P, b, pos):
    return int(bt_true[b, pos // P]) * P + pos % P


@pytest.mark.parametrize("graph", [False, True])
def test_decode_loop_descriptors_advanced_on_device(graph):
    """A decode loop that advances the row descriptors on the device, on the launching stream,
    right before each step: seq_lens and q_pos grow by one, the block table gains the page of
    the new position when it starts one, and the decode prolog writes the new token's MXFP8
    index key, FP8 latent row and rope into the caches and rounds q_I onto the MX grid.  Each
    step (the fused call, or a replay of the captured step) must see all of it: it is compared
    with the oracle on the state of that step, and no device check may fire."""
    steps = 3
    wl = workloads.make("decode_mxfp8", DEV, B=4, L=2600)
    P = wl.page_size
    len0, _, bt_true, bt = _growing_decode(wl, steps)
    k_full, ks_full = hsa.hsa_quantize_mx(wl.k_I)
    kv_full, kvs_full, rope_full = hsa.hsa_quantize_kv(wl.kv, wl.D_v, wl.D_v)
    k, ks, kv, kvs, rope = (t.clone() for t in (k_full, ks_full, kv_full, kvs_full.view(-1), rope_full))
    for b, n0 in enumerate(len0):
        for pos in range(n0, int(wl.seq_lens[b])):
            s = _slot_of(bt_true, P, b, pos)
            for t in (k, ks, kv, kvs, rope):
                t[s] = 0
    seq_lens = torch.tensor(len0, dtype=torch.int32, device=DEV)
    q_pos = seq_lens - 1
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    seq = hsa.PagedSeq(seq_lens, bt, P, wl.num_pages, wl.q_seq, q_pos,
                       max_seq_len=int(wl.seq_lens.max()), q_run=1, status=status)
    assert seq.seq_lens.data_ptr() == seq_lens.data_ptr() and seq.block_table.data_ptr() == bt.data_ptr()
    q_out = hsa.mx_round(wl.q_I)
    g = None
    if graph:
        g = hsa.DecodeGraph(seq, q_out, wl.w, k, ks, wl.q, kv, kvs, rope, wl.K, wl.D_v,
                            wl.softmax_scale, aux=True)
    main = torch.cuda.current_stream()
    rows = list(range(wl.T_q))
    ar = torch.arange(wl.B, device=DEV)
    for i in range(steps):
        # ---- the loop's own device work, on the launching stream, before the step
        pos = [n0 + i for n0 in len0]
        slots = torch.tensor([_slot_of(bt_true, P, b, p) for b, p in enumerate(pos)], dtype=torch.int64,
                             device=DEV)
        seq_lens.add_(1)
        q_pos.add_(1)
        lp = (q_pos // P).long()
        bt[ar, lp] = bt_true[ar, lp]
        hsa.hsa_decode_prolog(wl.k_I[slots], wl.kv[slots], slots, k, ks, kv, kvs, rope, wl.q_I,
                              q_out, wl.D_v, stream=main)
        if graph:
            out, lse, idx, sc = (t.clone() for t in g.replay())
        else:
            out, lse, idx, sc = hsa.hsa_fused_decode(seq, q_out, wl.w, k, ks, wl.q, kv, kvs, rope,
                                                     wl.K, wl.D_v, wl.softmax_scale, stream=main)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"device status {int(status.item()):#x} at step {i}"
        import dataclasses
        state = dataclasses.replace(wl, seq_lens=seq_lens.clone(), q_pos=q_pos.clone(),
                                    block_table=bt_true)
        check_against_oracle(state, rows, sc, idx, out)
