"""Pins for the oracle's sparse MLA attention and the whole-path composition (CPU only).

Sparse attention over the selected latent rows ("Day 0 Inference Adaptation and Optimization
for Hybrid Attention Models", "Sparse Attention Pipeline Optimization"; "Day-One Inference
Adaptation for Very Large Hybrid-Attention Models", 3.2).  Pinned by: pure-Python brute force on
a tiny case, torch's scaled_dot_product_attention (float64) when every causal position is
selected, closed forms (q = 0 gives the mean of the selected values; one dominant logit gives
that row's value; uniform logits give lse = log n), paging invariance, and the zigzag schedule's
closed-form load balance.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from sparse_index_attention_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _tiny():
    wl = workloads.make("tiny_decode_fp32")
    pg = oracle.Paging(wl.seq_lens, wl.block_table, wl.page_size, wl.num_pages, wl.q_seq, wl.q_pos)
    return wl, pg


def _slot(wl, b, s):
    return int(wl.block_table[b, s // wl.page_size]) * wl.page_size + s % wl.page_size


def test_brute_force_pure_python():
    wl, pg = _tiny()
    idx = workloads.random_selection(wl.q_pos, wl.K, seed=3)
    out, lse = oracle.sparse_mla(pg, wl.q, wl.kv, idx, wl.D_v, wl.softmax_scale)
    q = wl.q.tolist()
    kv = wl.kv.tolist()
    for t in range(wl.T_q):
        for h in (0, 5, wl.H - 1):
            rows = [kv[_slot(wl, 0, n)] for n in idx[t].tolist() if n != -1]
            z = [wl.softmax_scale * sum(a * b for a, b in zip(q[t][h], r)) for r in rows]
            m = max(z)
            e = [math.exp(v - m) for v in z]
            den = sum(e)
            o = [sum(e[i] * rows[i][d] for i in range(len(rows))) / den for d in range(wl.D_v)]
            np.testing.assert_allclose(out[t, h], o, rtol=1e-11, atol=1e-12)
            assert lse[t, h] == pytest.approx(m + math.log(den), rel=1e-12)


def test_full_selection_equals_dense_and_torch_sdpa():
    wl, pg = _tiny()
    K = 256  # >= context length: every causal position is selected
    n = wl.q_pos + 1
    idx = torch.full((wl.T_q, K), -1, dtype=torch.int32)
    for t in range(wl.T_q):
        idx[t, :n[t]] = torch.arange(int(n[t]), dtype=torch.int32)
    out, lse = oracle.sparse_mla(pg, wl.q, wl.kv, idx, wl.D_v, wl.softmax_scale)
    dout, dlse = oracle.dense_attn(pg, wl.q, wl.kv, wl.D_v, wl.softmax_scale)
    np.testing.assert_allclose(out, dout, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, dlse, rtol=1e-12)
    # library routine: torch SDPA in float64 over the de-paged cache with a causal mask
    slots = torch.tensor([_slot(wl, 0, s) for s in range(256)])
    kvc = wl.kv.double()[slots]                                   # [256, D_qk] in position order
    q = wl.q.double().permute(1, 0, 2)                            # [H, T, D_qk]
    k = kvc[None].expand(wl.H, -1, -1)
    v = kvc[None, :, :wl.D_v].expand(wl.H, -1, -1)
    mask = torch.arange(256)[None, :] <= wl.q_pos.long()[:, None]  # [T, 256]
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask,
                                                           scale=wl.softmax_scale)
    np.testing.assert_allclose(out, ref.permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)


def test_closed_forms():
    wl, pg = _tiny()
    idx = workloads.random_selection(wl.q_pos, wl.K, seed=4)
    # q = 0: uniform weights -> mean of the selected value rows, lse = log(count)
    out, lse = oracle.sparse_mla(pg, torch.zeros_like(wl.q), wl.kv, idx, wl.D_v, wl.softmax_scale)
    for t in range(wl.T_q):
        sel = [_slot(wl, 0, n) for n in idx[t].tolist() if n != -1]
        mean = wl.kv.double()[sel, :wl.D_v].mean(0).numpy()
        for h in range(wl.H):
            np.testing.assert_allclose(out[t, h], mean, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse[t], math.log(len(sel)), rtol=1e-13)
    # one selected row 40 nats above every other: output is that row's value part
    kv = wl.kv.double().clone() * 1e-3
    t, star = 2, int(idx[2, 7])
    qv = wl.q.double()[t]                                        # [H, D_qk]
    q = torch.zeros_like(wl.q.double())
    q[t] = qv
    u = torch.randn(wl.D_qk, generator=torch.Generator().manual_seed(0), dtype=torch.float64)
    kv[_slot(wl, 0, star)] = u
    for h in range(wl.H):
        q[t, h] = u * (60.0 / (wl.softmax_scale * float(u @ u)))   # logit 60 on the star row
    out2, _ = oracle.sparse_mla(pg, q, kv, idx, wl.D_v, wl.softmax_scale)
    for h in range(wl.H):
        np.testing.assert_allclose(out2[t, h], u[:wl.D_v].numpy(), rtol=1e-9, atol=1e-9)


def test_empty_selection_and_paging_invariance():
    wl, pg = _tiny()
    idx = workloads.random_selection(wl.q_pos, wl.K, seed=5)
    idx[1] = -1
    out, lse = oracle.sparse_mla(pg, wl.q, wl.kv, idx, wl.D_v, wl.softmax_scale)
    assert np.all(out[1] == 0) and np.all(np.isneginf(lse[1]))
    # duplicate the cache into a bigger pool under a different page placement
    rng = np.random.default_rng(6)
    new_np = wl.num_pages * 2
    perm = rng.permutation(new_np)[:wl.num_pages]
    pool = torch.randn(new_np * wl.page_size, wl.D_qk, dtype=torch.float64)
    for p in range(wl.num_pages):
        pool[perm[p] * wl.page_size:(perm[p] + 1) * wl.page_size] = \
            wl.kv.double()[p * wl.page_size:(p + 1) * wl.page_size]
    bt = perm[wl.block_table.numpy()]
    pg2 = oracle.Paging(wl.seq_lens, bt, wl.page_size, new_np, wl.q_seq, wl.q_pos)
    out2, lse2 = oracle.sparse_mla(pg2, wl.q, pool, idx, wl.D_v, wl.softmax_scale)
    assert np.array_equal(out2, out) and np.array_equal(lse2, lse)


def test_whole_path_with_large_k_is_dense_attention():
    wl, pg = _tiny()
    sc, idx, out, lse = oracle.sparse_index_attention(pg, wl.q_I, wl.w, wl.k_I, wl.q, wl.kv,
                                                      512, wl.D_v, wl.softmax_scale)
    dout, dlse = oracle.dense_attn(pg, wl.q, wl.kv, wl.D_v, wl.softmax_scale)
    np.testing.assert_allclose(out, dout, rtol=1e-12, atol=1e-13)
    # with the workload's K the selection is the K best causal positions of each row
    sc, idx, out, lse = oracle.sparse_index_attention(pg, wl.q_I, wl.w, wl.k_I, wl.q, wl.kv,
                                                      wl.K, wl.D_v, wl.softmax_scale)
    for t in range(wl.T_q):
        p = int(wl.q_pos[t])
        kth = np.sort(sc[t, :p + 1])[::-1][wl.K - 1]
        assert np.all(sc[t, idx[t]] >= kth) and len(set(idx[t].tolist())) == wl.K


def test_zigzag_rule_and_balanced_load():
    spec = {}
    for line in open(os.path.join(GOLDEN, "zigzag_rule.txt")):
        line = line.split("#")[0].strip()
        if line:
            k, *v = line.split()
            spec[k] = v
    T, n_chunks = int(spec["T"][0]), int(spec["chunks"][0])
    pairs = [tuple(map(int, p.split(":"))) for p in spec["pairs"]]
    order = workloads.zigzag_chunks(T, n_chunks)
    c = T // n_chunks
    got_pairs = [(order[2 * i][0] // c, order[2 * i + 1][0] // c) for i in range(n_chunks // 2)]
    assert got_pairs == pairs
    assert sorted(a for a, _ in order) == list(range(0, T, c))       # each chunk exactly once
    loads = []
    for i in range(n_chunks // 2):
        (a0, a1), (b0, b1) = order[2 * i], order[2 * i + 1]
        # causal pairs of a query chunk [a0, a1): sum_{t} (t + 1), counted by brute force sum
        loads.append(sum(range(a0 + 1, a1 + 1)) + sum(range(b0 + 1, b1 + 1)))
    assert set(loads) == {int(spec["pairs_per_pair"][0])}


def test_draft_rows_see_only_their_own_prefix():
    """Draft-verify decode (several query rows per sequence at its last positions): each row's
    result equals a one-row decode of the same sequence cut after that row's position, so no
    row reads a key past its own position, and the rows of a sequence differ."""
    kw = dict(B=3, n_draft=3, L_min=40, L_max=90, page_size=16, H_I=4, D_I=32, H=8, D_v=64,
              D_rope=16, K=16)
    wl = workloads.make("decode_draft_bf16", **kw)
    assert wl.T_q == 9 and wl.q_run == 3
    for b in range(wl.B):
        L = int(wl.seq_lens[b])
        assert wl.q_seq[3 * b:3 * b + 3].tolist() == [b] * 3
        assert wl.q_pos[3 * b:3 * b + 3].tolist() == [L - 3, L - 2, L - 1]
    pg = oracle.Paging(wl.seq_lens, wl.block_table, wl.page_size, wl.num_pages, wl.q_seq, wl.q_pos)
    sc, idx, out, lse = oracle.sparse_index_attention(pg, wl.q_I, wl.w, wl.k_I, wl.q, wl.kv,
                                                      wl.K, wl.D_v, wl.softmax_scale)
    for t in range(wl.T_q):
        b, p = int(wl.q_seq[t]), int(wl.q_pos[t])
        assert idx[t].max() <= p
        lens = wl.seq_lens.clone()
        lens[b] = p + 1
        one = oracle.Paging(lens, wl.block_table, wl.page_size, wl.num_pages,
                            wl.q_seq[t:t + 1], wl.q_pos[t:t + 1])
        sc1, idx1, out1, lse1 = oracle.sparse_index_attention(
            one, wl.q_I[t:t + 1], wl.w[t:t + 1], wl.k_I, wl.q[t:t + 1], wl.kv, wl.K, wl.D_v,
            wl.softmax_scale)
        assert np.array_equal(idx1[0], idx[t])
        np.testing.assert_array_equal(sc1[0, :p + 1], sc[t, :p + 1])
        np.testing.assert_array_equal(out1[0], out[t])
        np.testing.assert_array_equal(lse1[0], lse[t])
    assert not np.array_equal(out[0], out[1])
