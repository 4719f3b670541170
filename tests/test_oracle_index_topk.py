"""Pins for the oracle's index score and Top-K (CPU only).

Index score I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j] . k_I[s]) over causal positions s <= p_t
("Day 0 Inference Adaptation and Optimization for Hybrid Attention Models", "Sparse Attention
Pipeline Optimization": per-head scores over the paged K cache, summed with per-head weights).
Pinned by: a one-head special case against numpy's matmul, linearity in w with one-hot weights
(head indexing), exact integer arithmetic, sign/causal special cases, paging invariance and
positive homogeneity (the FP8 scale factoring).

Top-K: pinned against a full lexicographic sort (numpy lexsort) and constructed rows.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_index_attention_b200 import workloads


def _contiguous_to_paged(keys: np.ndarray, page: int, rng):
    """Scatter contiguous per-position rows into a randomly permuted page pool and return
    (pool, block_table row)."""
    L, D = keys.shape
    n_pages = -(-L // page)
    perm = rng.permutation(n_pages)
    pool = rng.standard_normal((n_pages * page, D))  # junk in unused slots
    for p in range(n_pages):
        rows = keys[p * page:(p + 1) * page]
        pool[perm[p] * page: perm[p] * page + len(rows)] = rows
    return pool, perm.astype(np.int32)[None, :], n_pages


def _pg(L, bt, n_pages, page, q_pos):
    T = len(q_pos)
    return oracle.Paging([L], bt, page, n_pages, [0] * T, q_pos)


def test_one_head_unit_weight_is_relu_of_matmul():
    rng = np.random.default_rng(1)
    L, D, page = 100, 16, 8
    keys = rng.standard_normal((L, D))
    pool, bt, npg = _contiguous_to_paged(keys, page, rng)
    q_pos = [99, 57, 0, 8]
    q = rng.standard_normal((4, 1, D))
    w = np.ones((4, 1))
    sc = oracle.index_score(_pg(L, bt, npg, page, q_pos), q, w, pool, ld=L)
    for t, p in enumerate(q_pos):
        ref = np.maximum(keys[:p + 1] @ q[t, 0], 0.0)
        np.testing.assert_allclose(sc[t, :p + 1], ref, rtol=1e-13, atol=1e-13)
        assert np.all(np.isnan(sc[t, p + 1:]))           # non-causal entries untouched


def test_linear_in_head_weights_one_hot():
    rng = np.random.default_rng(2)
    L, D, H, page = 70, 8, 5, 16
    keys = rng.standard_normal((L, D))
    pool, bt, npg = _contiguous_to_paged(keys, page, rng)
    q = rng.standard_normal((2, H, D))
    w = rng.standard_normal((2, H))
    pg = _pg(L, bt, npg, page, [69, 33])
    full = oracle.index_score(pg, q, w, pool, ld=L)
    acc = np.zeros_like(full)
    for j in range(H):
        oh = np.zeros_like(w)
        oh[:, j] = w[:, j]
        part = oracle.index_score(pg, q, oh, pool, ld=L)
        # head j alone: w_j * ReLU(q_j . k)
        for t, p in enumerate([69, 33]):
            np.testing.assert_allclose(part[t, :p + 1], w[t, j] * np.maximum(keys[:p + 1] @ q[t, j], 0),
                                       rtol=1e-12, atol=1e-12)
        acc = np.where(np.isnan(part), np.nan, np.nan_to_num(acc) + np.nan_to_num(part))
    np.testing.assert_allclose(acc, full, rtol=1e-12, atol=1e-12)


def test_integer_inputs_exact():
    rng = np.random.default_rng(3)
    L, D, H, page = 64, 32, 4, 16
    keys = rng.integers(-2, 3, (L, D)).astype(np.float64)
    pool, bt, npg = _contiguous_to_paged(keys, page, rng)
    q = rng.integers(-2, 3, (3, H, D)).astype(np.float64)
    w = (2.0 ** rng.integers(-3, 4, (3, H))) * rng.choice([-1, 1], (3, H))
    pos = [63, 20, 41]
    sc = oracle.index_score(_pg(L, bt, npg, page, pos), q, w, pool, ld=L)
    ki = keys.astype(np.int64)
    for t, p in enumerate(pos):
        dots = ki[:p + 1] @ q[t].astype(np.int64).T                 # exact integers [p+1, H]
        ref = (np.maximum(dots, 0) * w[t][None, :]).sum(axis=1)      # dyadic, exact in double
        assert np.array_equal(sc[t, :p + 1], ref)


def test_sign_and_causal_special_cases():
    rng = np.random.default_rng(4)
    L, D, H, page = 40, 8, 3, 8
    keys = np.abs(rng.standard_normal((L, D)))
    pool, bt, npg = _contiguous_to_paged(keys, page, rng)
    q = -np.abs(rng.standard_normal((1, H, D)))      # every dot product negative
    w = rng.standard_normal((1, H))
    sc = oracle.index_score(_pg(L, bt, npg, page, [39]), q, w, pool, ld=L)
    assert np.all(sc[0] == 0.0)
    # the query's own position p is part of its history: a key equal to q only at s = p
    keys2 = np.zeros((L, D))
    qv = rng.standard_normal(D)
    keys2[17] = qv
    pool2, bt2, npg2 = _contiguous_to_paged(keys2, page, rng)
    sc2 = oracle.index_score(_pg(L, bt2, npg2, page, [17]), qv[None, None, :], np.ones((1, 1)),
                             pool2, ld=L)
    assert sc2[0, 17] == pytest.approx(float(qv @ qv), rel=1e-14)
    assert np.all(sc2[0, :17] == 0) and np.all(np.isnan(sc2[0, 18:]))


def test_paging_invariance_and_positive_homogeneity():
    wl = workloads.make("tiny_decode_fp32")
    pg = oracle.Paging(wl.seq_lens, wl.block_table, wl.page_size, wl.num_pages, wl.q_seq, wl.q_pos)
    base = oracle.index_score(pg, wl.q_I, wl.w, wl.k_I)
    # move every page to a new physical location
    rng = np.random.default_rng(5)
    perm = rng.permutation(wl.num_pages)
    k = wl.k_I.numpy()
    moved = np.zeros_like(k)
    for p in range(wl.num_pages):
        moved[perm[p] * wl.page_size:(perm[p] + 1) * wl.page_size] = k[p * wl.page_size:(p + 1) * wl.page_size]
    bt = perm[wl.block_table.numpy()]
    pg2 = oracle.Paging(wl.seq_lens, bt, wl.page_size, wl.num_pages, wl.q_seq, wl.q_pos)
    assert np.array_equal(oracle.index_score(pg2, wl.q_I, wl.w, moved), base, equal_nan=True)
    # scaling every key by a positive power of two scales every score by it exactly
    np.testing.assert_array_equal(oracle.index_score(pg, wl.q_I, wl.w, k.astype(np.float64) * 8.0),
                                  base * 8.0)


def _lexsort_topk(row: np.ndarray, K: int) -> np.ndarray:
    n = len(row)
    if n <= K:
        return np.concatenate([np.arange(n), -np.ones(K - n, dtype=int)])
    order = np.lexsort((np.arange(n), -row))      # primary: score desc; secondary: position asc
    return np.sort(order[:K])


@pytest.mark.parametrize("ties", [False, True])
def test_topk_matches_full_sort(ties):
    T, ld, K = 24, 300, 37
    sc = workloads.random_scores(T, ld, seed=9, ties=ties).numpy().astype(np.float64)
    n_valid = np.array([1, 2, 36, 37, 38, 39, 300, 299, 150, 74, 75, 100] * 2, dtype=np.int32)
    idx = oracle.topk(sc, n_valid, K)
    for t in range(T):
        assert np.array_equal(idx[t], _lexsort_topk(sc[t, :n_valid[t]], K)), t


def test_topk_constructed_rows():
    K, n = 16, 50
    rows = np.stack([np.full(n, 3.5), -np.arange(n, dtype=np.float64), np.arange(n, dtype=np.float64),
                     np.where(np.arange(n) % 2 == 0, 0.0, -0.0)])
    idx = oracle.topk(rows, [n] * 4, K)
    assert np.array_equal(idx[0], np.arange(K))          # all equal -> lowest positions
    assert np.array_equal(idx[1], np.arange(K))          # decreasing -> first K
    assert np.array_equal(idx[2], np.arange(n - K, n))   # increasing -> last K
    assert np.array_equal(idx[3], np.arange(K))          # +0 and -0 tie
    short = oracle.topk(rows[:1, :10], [10], K)
    assert np.array_equal(short[0], np.concatenate([np.arange(10), -np.ones(6, dtype=int)]))


def test_topk_rejects_non_finite():
    with pytest.raises(oracle.OracleError):
        oracle.topk(np.array([[1.0, np.nan, 2.0]]), [3], 1)


# ----------------------------------------------------------------- block-aligned selection
def _blocks_brute(row, n, K, B):
    """Independent restatement: block maxima over the causal prefix, blocks ordered by (max
    descending, block ascending) with numpy's lexsort, the first K / B blocks kept whole."""
    if n <= K:
        return [i for i in range(n)] + [-1] * (K - n)
    nb = -(-n // B)
    bmax = np.full(nb, -np.inf)
    for b in range(nb):
        bmax[b] = np.max(row[b * B:min(n, (b + 1) * B)])
    order = np.lexsort((np.arange(nb), -bmax))[:K // B]
    keep = sorted(order.tolist())
    out = [s for b in keep for s in range(b * B, min(n, (b + 1) * B))]
    return out + [-1] * (K - len(out))


@pytest.mark.parametrize("B", [1, 4, 16, 64])
def test_topk_blocks_matches_brute_force(B):
    rng = np.random.default_rng(31 + B)
    K = 64
    T, ld = 40, 700
    sc = rng.integers(-6, 7, size=(T, ld)).astype(np.float64)      # heavy ties
    sc[::3] = rng.standard_normal((len(sc[::3]), ld))
    n_valid = rng.integers(1, ld + 1, size=T).astype(np.int32)
    n_valid[:3] = [K, K + 1, 1]
    got = oracle.topk_blocks(sc, n_valid, K, B)
    for t in range(T):
        assert got[t].tolist() == _blocks_brute(sc[t], int(n_valid[t]), K, B), (t, B)


def test_topk_blocks_with_unit_blocks_is_topk():
    rng = np.random.default_rng(5)
    sc = rng.integers(-3, 4, size=(25, 300)).astype(np.float64)
    n_valid = rng.integers(1, 301, size=25).astype(np.int32)
    assert np.array_equal(oracle.topk_blocks(sc, n_valid, 32, 1), oracle.topk(sc, n_valid, 32))


def test_topk_blocks_constructed_row():
    """Block 3 holds one very high score among low ones: it is kept whole, and the block of the
    next-highest maxima follow; a position Top-K would instead take scattered positions."""
    B, K = 8, 16
    row = np.zeros(100)
    row[:] = -np.arange(100) / 1000.0          # decreasing: block 0 has the best maximum
    row[27] = 50.0                              # block 3 (positions 24..31)
    got = oracle.topk_blocks(row[None], np.array([100], np.int32), K, B)[0].tolist()
    assert got == list(range(0, 8)) + list(range(24, 32))
    # a partial last block counts with its causal positions only
    row2 = np.zeros(20)
    row2[17] = 9.0                              # block 2 = positions 16..19 (n = 20)
    got2 = oracle.topk_blocks(row2[None], np.array([20], np.int32), 8, 4)[0].tolist()
    assert got2 == [0, 1, 2, 3, 16, 17, 18, 19]


def test_topk_blocks_invariants():
    rng = np.random.default_rng(9)
    B, K = 16, 128
    sc = rng.standard_normal((30, 2000))
    n_valid = rng.integers(129, 2001, size=30).astype(np.int32)
    got = oracle.topk_blocks(sc, n_valid, K, B)
    for t in range(30):
        n = int(n_valid[t])
        sel = got[t][got[t] >= 0]
        assert np.all(np.diff(sel) > 0)                          # ascending, distinct
        blocks = sorted(set((sel // B).tolist()))
        assert len(blocks) == K // B
        for b in blocks:                                          # whole causal blocks
            assert set(range(b * B, min(n, (b + 1) * B))) <= set(sel.tolist())
        bmax = np.array([sc[t, b * B:min(n, (b + 1) * B)].max() for b in range(-(-n // B))])
        kept = np.array(blocks)
        dropped = np.setdiff1d(np.arange(len(bmax)), kept)
        if len(dropped):
            assert bmax[kept].min() >= bmax[dropped].max()       # no dropped block beats a kept one


def test_topk_blocks_rejects_bad_arguments():
    with pytest.raises(oracle.OracleError):
        oracle.topk_blocks(np.zeros((1, 10)), np.array([10], np.int32), 12, 8)   # 8 does not divide 12
