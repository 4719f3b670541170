"""Shared test plumbing: turn a seeded workload into library descriptors / oracle inputs, and the
tolerance checks the parity tests use.  No method arithmetic lives here: scores, selections and
attention come from the library (GPU side) or from ``oracle`` (reference side)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import sparse_index_attention_b200 as hsa
from sparse_index_attention_b200 import workloads


def paged_seq(wl: workloads.Workload, status=None) -> hsa.PagedSeq:
    """Descriptor of the workload's rows.  Unless a status tensor is given, a fresh one is
    attached so that check_status() can assert that no device-side check fired."""
    if status is None and wl.seq_lens.is_cuda:
        status = torch.zeros(1, dtype=torch.int32, device=wl.seq_lens.device)
    return hsa.PagedSeq(wl.seq_lens, wl.block_table, wl.page_size, wl.num_pages, wl.q_seq, wl.q_pos,
                        max_seq_len=int(wl.seq_lens.max().item()), q_run=wl.q_run, status=status)


def check_status(seq: hsa.PagedSeq):
    """No device-side check (bad page / position / grouping, or a pipeline wait that gave up)
    fired during the calls made with this descriptor."""
    if seq.status is not None:
        torch.cuda.synchronize()
        v = int(seq.status.item())
        assert v == 0, f"device status bits {v:#x}"


def oracle_paging(wl: workloads.Workload, rows=None) -> oracle.Paging:
    pg = oracle.Paging(wl.seq_lens, wl.block_table, wl.page_size, wl.num_pages, wl.q_seq, wl.q_pos)
    return pg if rows is None else pg.subset(rows)


class GpuCaches:
    """The caches the GPU path reads, written by the library's own quantizers when FP8
    (latent scales per token, or per `kv_group` latent dims)."""

    def __init__(self, wl: workloads.Workload, kv_group=None):
        self.k_scale = None
        self.kv_scale = None
        self.kv_rope = None
        self.q_I = wl.q_I
        if wl.index_mx:
            self.k, self.k_scale = hsa.hsa_quantize_mx(wl.k_I)
            self.q_I = hsa.mx_round(wl.q_I)
        elif wl.index_fp8:
            self.k, sc = hsa.hsa_quantize_index(wl.k_I, wl.D_I)
            self.k_scale = sc.view(-1)
        else:
            self.k = wl.k_I
        if wl.kv_fp8:
            self.kv, sc, self.kv_rope = hsa.hsa_quantize_kv(wl.kv, wl.D_v, kv_group or wl.D_v)
            self.kv_scale = sc if kv_group else sc.view(-1)
        else:
            self.kv = wl.kv


class OracleCaches:
    """Exact values of the caches (and of the index queries) as the oracle reads them: its own
    quantizers for FP8 and MXFP8."""

    def __init__(self, wl: workloads.Workload, need_kv: bool = True, kv_group=None):
        self.q_I = wl.q_I.cpu()
        if wl.index_mx:
            self.k = oracle.mx_dequantize_rows(*oracle.mx_quantize_rows(wl.k_I.float().cpu()))
            q = wl.q_I.float().cpu().reshape(-1, wl.D_I)
            self.q_I = oracle.mx_dequantize_rows(*oracle.mx_quantize_rows(q)).reshape(wl.q_I.shape)
        elif wl.index_fp8:
            codes, sc = oracle.quantize_rows(wl.k_I.float().cpu(), wl.D_I)
            self.k = oracle.dequantize_rows(codes, sc, wl.D_I)
        else:
            self.k = wl.k_I.cpu()
        if need_kv:
            kv = wl.kv.float().cpu().numpy().astype(np.float64)
            if wl.kv_fp8:
                grp = kv_group or wl.D_v
                codes, sc = oracle.quantize_rows(wl.kv[:, :wl.D_v].float().cpu(), grp)
                kv[:, :wl.D_v] = oracle.dequantize_rows(codes, sc, grp)
            self.kv = kv


def index_tolerance_ok(gpu, ref, mag, rel=1e-3):
    """|I_gpu - I_ref| <= rel * (|I_ref| + M) elementwise, M = sum_j |w_j| ReLU(q_j . k_s)."""
    gpu = np.asarray(gpu, dtype=np.float64)
    err = np.abs(gpu - ref)
    bound = rel * (np.abs(ref) + mag)
    return bool(np.all(err <= bound)), float(np.max(err / np.maximum(bound, 1e-300)))


def attn_close(gpu, ref, tol):
    gpu = np.asarray(gpu, dtype=np.float64)
    err = np.abs(gpu - ref)
    ok = err <= tol + tol * np.abs(ref)
    return bool(np.all(ok)), float(err.max())


def check_selection_vs_oracle(ref_sc, mag, gidx, n_valid, K, labels=None, rel=1e-3):
    """Oracle-score agreement of the GPU selection, per the path's contract: the float64-score
    selection (oracle Top-K) agrees on >= 99.9 % of positions summed over the rows, and every
    position in the symmetric difference of a row is a near tie of the oracle's K-th score,
    |I_ref(s) - I_ref(kth)| <= rel (|I_ref(kth)| + M) with M the larger magnitude sum of the two
    positions.  Rows with n <= K must agree exactly.  Returns the oracle selection."""
    ref_idx = oracle.topk(ref_sc, n_valid, K)
    agree = total = 0
    for i in range(len(gidx)):
        a = set(gidx[i][gidx[i] >= 0].tolist())
        b = set(ref_idx[i][ref_idx[i] >= 0].tolist())
        total += len(b)
        agree += len(a & b)
        n = int(n_valid[i])
        label = labels[i] if labels is not None else i
        if n <= K:
            assert a == b, ("short row selects every position", label)
            continue
        row = ref_sc[i, :n]
        kth = -np.partition(-row, K - 1)[K - 1]
        m_kth = mag[i, :n][row == kth].max()
        for s in a ^ b:
            m = max(mag[i, s], m_kth)
            assert abs(row[s] - kth) <= rel * (abs(kth) + m), ("not a near tie", label, s)
    assert agree >= 0.999 * total, (agree, total)
    return ref_idx


def attention_vs_oracle(pg, q, kv, gidx, ref_idx, D_v, scale, out, tol):
    """Attention of the GPU's own selection against the oracle's attention over that same
    selection (gated at `tol`), so that a near-tie swap in the index is not charged to the
    attention kernel.  The end-to-end comparison (oracle attention over the oracle's own
    selection) is returned as a reported number: a swapped near tie of the index score may carry
    any attention weight."""
    ref_out, _ = oracle.sparse_mla(pg, q, kv, gidx, D_v, scale)
    got = out.float().cpu().numpy()
    ok, worst = attn_close(got, ref_out, tol)
    assert ok, ("attention on the GPU's selection", worst)
    e2e_out, _ = oracle.sparse_mla(pg, q, kv, ref_idx, D_v, scale)
    return float(np.abs(got - e2e_out).max())


def stable_topk_reference(scores: torch.Tensor, q_pos: torch.Tensor, K: int) -> torch.Tensor:
    """Selection from the same fp32 scores with torch's stable sort (descending score, ties by
    position), re-sorted ascending: the reference for the bit-exact Top-K check."""
    T, ld = scores.shape
    out = torch.full((T, K), -1, dtype=torch.int32, device=scores.device)
    pos = q_pos.tolist()
    for t in range(T):
        n = pos[t] + 1
        if n <= K:
            out[t, :n] = torch.arange(n, dtype=torch.int32, device=scores.device)
            continue
        row = scores[t, :n].clone()
        row[row == 0] = 0.0                          # -0.0 == +0.0
        order = torch.sort(row, descending=True, stable=True).indices[:K]
        out[t] = order.sort().values.to(torch.int32)
    return out


def compact_workload(wl: workloads.Workload, rows) -> workloads.Workload:
    """A copy of the workload reduced to the given query rows and the pages of their sequences
    (pages renumbered consecutively, contents copied).  Rows' results are unchanged: every cache
    row is read through the block table and FP8 quantization is per row."""
    import dataclasses
    import math
    rows = list(rows)
    q_seq = wl.q_seq[rows].tolist()
    seqs = sorted(set(q_seq))
    pages_of = []
    for b in seqs:
        n = math.ceil(int(wl.seq_lens[b]) / wl.page_size)
        pages_of.append(wl.block_table[b, :n].long())
    old = torch.cat(pages_of)
    P = old.numel()
    maxp = max(p.numel() for p in pages_of)
    bt = torch.zeros((len(seqs), maxp), dtype=torch.int32)
    off = 0
    for i, p in enumerate(pages_of):
        bt[i, :p.numel()] = torch.arange(off, off + p.numel(), dtype=torch.int32)
        off += p.numel()
    def pages(x):
        return x.view(wl.num_pages, wl.page_size, -1)[old.to(x.device)].reshape(P * wl.page_size, -1).cpu()
    remap = {b: i for i, b in enumerate(seqs)}
    return dataclasses.replace(
        wl, B=len(seqs), seq_lens=wl.seq_lens[seqs].cpu(), block_table=bt, num_pages=P,
        T_q=len(rows), q_seq=torch.tensor([remap[b] for b in q_seq], dtype=torch.int32),
        q_pos=wl.q_pos[rows].cpu(), q_I=wl.q_I[rows].cpu(), w=wl.w[rows].cpu(), k_I=pages(wl.k_I),
        q=wl.q[rows].cpu(), kv=pages(wl.kv), q_run=1)
