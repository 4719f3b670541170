"""GPU parity: every C-ABI entry point against the float64 oracle on seeded inputs that span
several tiles and a ragged tail.  Tolerances (written here, per element):
  index score    |I_gpu - I_ref| <= 1e-3 (|I_ref| + M),  M = sum_j |w_j| ReLU(q_j . k_s)
  Top-K          bit-exact (same fp32 scores on both sides)
  attention      |o_gpu - o_ref| <= 2e-2 + 2e-2 |o_ref| (bf16), 6e-2 for FP8 caches, 1e-4 fp32
  quantizers     bit-exact codes and scales
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_index_attention_b200 as hsa
from sparse_index_attention_b200 import workloads

from helpers import (GpuCaches, OracleCaches, attn_close, check_status, index_tolerance_ok,
                     oracle_paging, paged_seq, stable_topk_reference)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _index_vs_oracle(wl, rows=None):
    gc = GpuCaches(wl)
    seq = paged_seq(wl)
    sc = hsa.hsa_index_score(seq, gc.q_I, wl.w, gc.k, gc.k_scale)
    check_status(seq)
    rows = list(range(wl.T_q)) if rows is None else rows
    oc = OracleCaches(wl, need_kv=False)
    pg = oracle_paging(wl, rows)
    qI, w = oc.q_I[rows], wl.w[rows].cpu()
    ref = oracle.index_score(pg, qI, w, oc.k, ld=sc.shape[1])
    mag = oracle.index_score(pg, qI, w.abs(), oc.k, ld=sc.shape[1])
    got = sc[rows].cpu().numpy()
    for i, t in enumerate(rows):
        n = int(wl.q_pos[t]) + 1
        ok, worst = index_tolerance_ok(got[i, :n], ref[i, :n], mag[i, :n])
        assert ok, (wl.name, t, worst)
    return sc


@pytest.mark.parametrize("name,kw", [
    ("tiny_decode_fp32", {}),
    ("decode_bf16", dict(B=6, L_min=100, L_max=1500)),
    ("decode_fp8", dict(B=3, L=700)),
    ("prefill_bf16", dict(T=700)),
    ("prefill_long_zigzag", dict(T=1024, n_chunks=4)),
])
def test_index_score_vs_oracle(name, kw):
    _index_vs_oracle(workloads.make(name, DEV, **kw))


@pytest.mark.parametrize("name,kw", [
    ("tiny_decode_fp32", {}),                       # CUDA-core kernel (4 x 32 indexer)
    ("decode_bf16", dict(B=5, L_min=100, L_max=1500)),   # tensor-core kernel, one row per tile
    ("prefill_bf16", dict(T=700)),                  # tensor-core kernel, four rows per tile
])
def test_index_score_mxfp8_vs_oracle(name, kw):
    """MXFP8 index queries and keys (E8M0 scale per 32 dims) on both index kernels, against the
    oracle's own MX quantizer and the float64 score of the dequantized values."""
    wl = workloads.make(name, DEV, **kw)
    wl.index_fp8 = wl.index_mx = True
    _index_vs_oracle(wl)


@pytest.mark.parametrize("name,kw", [
    ("decode_bf16", dict(B=5, L_min=100, L_max=1500)),                   # one query row per tile
    ("decode_draft_bf16", dict(B=4, n_draft=2, L_min=300, L_max=1400)),  # row pairs: two per tile
    ("prefill_bf16", dict(T=700)),                                      # two rows per tile
    ("prefill_bf16", dict(T=301)),                                      # odd run: one row per tile
])
def test_index_score_mx_block_scaled_vs_oracle(name, kw):
    """MXFP8 queries and keys as codes + E8M0 scales (hsa_index_score_mx: the block-scaled MMA on
    the codes), against the float64 score of the oracle's own MX quantization of both, and
    against the bf16-query MX path on the same rounded queries."""
    _index_mx_bs_vs_oracle(name, kw)


def _index_mx_bs_vs_oracle(name, kw):
    wl = workloads.make(name, DEV, **kw)
    wl.index_fp8 = wl.index_mx = True
    seq = paged_seq(wl)
    k, ks = hsa.hsa_quantize_mx(wl.k_I)
    qc, qs = hsa.hsa_quantize_mx(wl.q_I.reshape(-1, wl.D_I))
    sc = hsa.hsa_index_score(seq, qc.view(wl.q_I.shape), wl.w, k, ks,
                             q_scale=qs.view(wl.T_q, wl.H_I, wl.D_I // 32))
    check_status(seq)
    # the same scores through the bf16-query MX path (queries rounded onto the MX grid)
    sc_bf = hsa.hsa_index_score(seq, hsa.mx_round(wl.q_I), wl.w, k, ks)
    oc = OracleCaches(wl, need_kv=False)
    rows = list(range(wl.T_q))
    pg = oracle_paging(wl, rows)
    ref = oracle.index_score(pg, oc.q_I, wl.w.cpu(), oc.k, ld=sc.shape[1])
    mag = oracle.index_score(pg, oc.q_I, wl.w.cpu().abs(), oc.k, ld=sc.shape[1])
    got, got_bf = sc.cpu().numpy(), sc_bf.cpu().numpy()
    for t in rows:
        n = int(wl.q_pos[t]) + 1
        ok, worst = index_tolerance_ok(got[t, :n], ref[t, :n], mag[t, :n])
        assert ok, (name, t, worst)
        ok, worst = index_tolerance_ok(got[t, :n], got_bf[t, :n], mag[t, :n])
        assert ok, (name, t, worst)


def test_index_score_mx_block_scaled_every_code():
    """Every finite E4M3 key code through the block-scaled MMA, with four different block
    exponents per key (as in the MXFP8 key-path test) and MXFP8 queries +1 / -1 at dim 32b of
    block b: the score is sum_b decode(code) 2^(E_b - 127), bit for bit wherever that is a normal
    fp32 number; below 2^-126 the tensor core may flush to zero, which is all that is allowed."""
    wl = workloads.make("decode_fp8", DEV, B=1, L=1536)
    slots = wl.num_pages * wl.page_size
    code_of_slot = torch.arange(slots, dtype=torch.int64) % 256
    code_of_slot[(code_of_slot & 0x7F) == 0x7F] = 0
    k8 = code_of_slot.to(torch.uint8)[:, None].expand(slots, wl.D_I).contiguous().to(DEV)
    bases = torch.tensor([0, 1, 60, 127, 200, 240])
    sl = torch.arange(slots)
    base = bases[(sl // 256) % len(bases)]
    E = torch.stack([base + (sl + 3 * b) % 4 for b in range(4)], dim=1).to(torch.uint8)
    q = torch.zeros((1, wl.H_I, wl.D_I), dtype=torch.bfloat16)
    w = torch.zeros((1, wl.H_I), dtype=torch.float32)
    for b in range(4):
        q[0, b, 32 * b], q[0, 4 + b, 32 * b] = 1.0, -1.0
        w[0, b], w[0, 4 + b] = 1.0, -1.0
    qc, qs = hsa.hsa_quantize_mx(q.reshape(-1, wl.D_I).to(DEV))
    seq = hsa.PagedSeq(wl.seq_lens, wl.block_table, wl.page_size, wl.num_pages,
                       wl.q_seq[:1], wl.q_pos[:1], max_seq_len=int(wl.seq_lens.max()),
                       status=torch.zeros(1, dtype=torch.int32, device=DEV))
    sc = hsa.hsa_index_score(seq, qc.view(1, wl.H_I, wl.D_I), w.to(DEV), k8, E.contiguous().to(DEV),
                             q_scale=qs.view(1, wl.H_I, wl.D_I // 32))
    check_status(seq)
    n = int(wl.q_pos[0]) + 1
    bt = wl.block_table[0].cpu().long()
    pos = torch.arange(n)
    slot = bt[pos // wl.page_size] * wl.page_size + pos % wl.page_size
    codes = code_of_slot[slot].numpy().astype(np.uint8)
    vals = oracle.e4m3_decode(codes)
    ref = sum(vals * np.exp2(E[slot, b].double().numpy() - 127) for b in range(4))
    assert len(set(codes.tolist())) == 254
    got = sc[0, :n].cpu().numpy().astype(np.float64)
    normal = np.abs(ref) >= 2.0 ** -126
    assert np.array_equal(got[normal], ref[normal])
    assert np.all((got[~normal] == ref[~normal]) | (got[~normal] == 0.0))


@pytest.mark.parametrize("q_run,T", [(1, 2500), (2, 600), (4, 300)])
def test_index_score_row_groupings(q_run, T):
    """The tensor-core kernel groups q_run-aligned rows (1, 2 or 4 per MMA tile) and splits
    launches past its group limit; every grouping must give the same per-row contract."""
    wl = workloads.make("prefill_bf16", DEV, T=T)
    wl.q_run = q_run
    _index_vs_oracle(wl, rows=sorted(set(range(0, T, 7)) | {T - 1}))


@pytest.mark.parametrize("page_size", [16, 128, 256, 384])
def test_index_score_page_sizes(page_size):
    """Page sizes below, at and above the 128-key tile (384: not a power of two, so the kernel's
    page arithmetic takes its division path), for bf16, E4M3 and block-scaled MXFP8 keys."""
    _index_vs_oracle(workloads.make("decode_bf16", DEV, B=4, L_min=200, L_max=1300, page_size=page_size))
    _index_vs_oracle(workloads.make("decode_fp8", DEV, B=2, L=900, page_size=page_size))
    _index_mx_bs_vs_oracle("decode_bf16", dict(B=3, L_min=300, L_max=1200, page_size=page_size))


def test_index_score_integer_inputs_bit_exact():
    wl = workloads.make("decode_bf16", DEV, B=3, L_min=200, L_max=900)
    g = torch.Generator(device=DEV).manual_seed(77)
    wl.q_I = torch.randint(-2, 3, wl.q_I.shape, generator=g, device=DEV).to(torch.bfloat16)
    wl.k_I = torch.randint(-2, 3, wl.k_I.shape, generator=g, device=DEV).to(torch.bfloat16)
    e = torch.randint(-3, 4, wl.w.shape, generator=g, device=DEV).float()
    wl.w = torch.exp2(e) * torch.where(torch.rand(wl.w.shape, generator=g, device=DEV) < 0.5, -1.0, 1.0)
    sc = hsa.hsa_index_score(paged_seq(wl), wl.q_I, wl.w, wl.k_I)
    ref = oracle.index_score(oracle_paging(wl), wl.q_I.cpu(), wl.w.cpu(), wl.k_I.cpu(), ld=sc.shape[1])
    got = sc.cpu().numpy()
    for t in range(wl.T_q):
        n = int(wl.q_pos[t]) + 1
        assert np.array_equal(got[t, :n].astype(np.float64), ref[t, :n]), t


def test_index_score_fp8_every_code_bit_exact():
    """Every finite E4M3 code through the FP8 key path: key s holds one code in all 128 dims, and
    two index heads read dim 0 with q = +1 and -1 and weights +1 and -1, so the score is exactly
    decode(code) x scale (scales are powers of two).  Pins the kernel's widening of the codes,
    subnormals and signed zero included, bit for bit against the E4M3 definition."""
    wl = workloads.make("decode_fp8", DEV, B=1, L=1024)
    slots = wl.num_pages * wl.page_size
    code_of_slot = torch.arange(slots, dtype=torch.int64) % 256
    code_of_slot[(code_of_slot & 0x7F) == 0x7F] = 0           # NaN codes are outside the contract
    k8 = code_of_slot.to(torch.uint8)[:, None].expand(slots, wl.D_I).contiguous().to(DEV)
    scale = torch.exp2(-(torch.arange(slots) % 5).float()).to(DEV)
    q = torch.zeros((1, wl.H_I, wl.D_I), dtype=torch.bfloat16)
    q[0, 0, 0], q[0, 1, 0] = 1.0, -1.0
    w = torch.zeros((1, wl.H_I), dtype=torch.float32)
    w[0, 0], w[0, 1] = 1.0, -1.0
    seq = hsa.PagedSeq(wl.seq_lens, wl.block_table, wl.page_size, wl.num_pages,
                       wl.q_seq[:1], wl.q_pos[:1], max_seq_len=int(wl.seq_lens.max()),
                       status=torch.zeros(1, dtype=torch.int32, device=DEV))
    sc = hsa.hsa_index_score(seq, q.to(DEV), w.to(DEV), k8, scale)
    check_status(seq)
    n = int(wl.q_pos[0]) + 1
    bt = wl.block_table[0].cpu().long()
    pos = torch.arange(n)
    slot = bt[pos // wl.page_size] * wl.page_size + pos % wl.page_size
    codes = code_of_slot[slot].numpy().astype(np.uint8)
    ref = (oracle.e4m3_decode(codes) * scale.cpu()[slot].double().numpy()).astype(np.float32)
    assert len(set(codes.tolist())) == 254                   # every finite code is exercised
    assert np.array_equal(sc[0, :n].cpu().numpy(), ref)


@pytest.mark.parametrize("name,kw,q_run", [
    ("decode_fp8", dict(B=3, L=900), 1),                      # one query row per tile
    ("prefill_long_zigzag", dict(T=700, n_chunks=4), 2),      # two rows per tile
    ("prefill_long_zigzag", dict(T=700, n_chunks=4), 4),      # four rows per tile
])
def test_index_score_fp8_integer_inputs_bit_exact_both_paths(name, kw, q_run):
    """E4M3 keys holding small integers with power-of-two scales, integer bf16 queries and
    power-of-two weights: every product and partial sum is exact in fp32 in any order, so the
    score must equal the float64 oracle bit for bit.  Through the 8-bit MMAs on split queries
    (hi + lo; the scale array 16-byte aligned) and through the widening path (the same scales
    one float off 16-byte alignment), for one, two and four query rows per tile."""
    wl = workloads.make(name, DEV, **kw)
    wl.q_run = q_run
    g = torch.Generator(device=DEV).manual_seed(78)
    slots = wl.num_pages * wl.page_size
    q = torch.randint(-31, 32, wl.q_I.shape, generator=g, device=DEV).to(torch.bfloat16)
    kint = torch.randint(-4, 5, (slots, wl.D_I), generator=g, device=DEV)
    lut = torch.from_numpy(oracle.e4m3_encode(np.arange(-4, 5)).astype(np.uint8)).to(DEV)
    k8 = lut[kint + 4].contiguous()
    scale = torch.exp2(torch.randint(0, 2, (slots,), generator=g, device=DEV).float())
    e = torch.randint(-2, 1, wl.w.shape, generator=g, device=DEV).float()
    w = torch.exp2(e) * torch.where(torch.rand(wl.w.shape, generator=g, device=DEV) < 0.5, -1.0, 1.0)
    seq = paged_seq(wl)
    k_exact = oracle.e4m3_decode(k8.cpu().numpy()) * scale.cpu().double().numpy()[:, None]
    off = torch.zeros(slots + 1, dtype=torch.float32, device=DEV)
    off[1:] = scale
    for ks in (scale, off[1:]):
        assert (ks.data_ptr() % 16 == 0) == (ks is scale)
        sc = hsa.hsa_index_score(seq, q, w, k8, ks)
        check_status(seq)
        ref = oracle.index_score(oracle_paging(wl), q.cpu(), w.cpu(), k_exact, ld=sc.shape[1])
        got = sc.cpu().numpy()
        for t in range(wl.T_q):
            n = int(wl.q_pos[t]) + 1
            assert np.array_equal(got[t, :n].astype(np.float64), ref[t, :n]), t


def test_index_score_mxfp8_every_code_bit_exact():
    """Every finite E4M3 code through the MXFP8 key path of the tensor-core kernel, with the four
    block exponents of a key all different and the largest one in any of the four blocks.  Key s
    holds one code in all 128 dims; index heads 0-3 read dim 32b of block b with q = +1 and heads
    4-7 with q = -1, weights +1 and -1, so the score is exactly sum_b decode(code) 2^(E_b - 127):
    the converters' per-block rescale and the epilogue's 2^(E_max - 127) must recombine bit for
    bit, down to scale byte 0 (2^-127) and up to 2^117."""
    wl = workloads.make("decode_fp8", DEV, B=1, L=1536)
    slots = wl.num_pages * wl.page_size
    code_of_slot = torch.arange(slots, dtype=torch.int64) % 256
    code_of_slot[(code_of_slot & 0x7F) == 0x7F] = 0
    k8 = code_of_slot.to(torch.uint8)[:, None].expand(slots, wl.D_I).contiguous().to(DEV)
    bases = torch.tensor([0, 1, 60, 127, 200, 240])
    sl = torch.arange(slots)
    base = bases[(sl // 256) % len(bases)]
    E = torch.stack([base + (sl + 3 * b) % 4 for b in range(4)], dim=1).to(torch.uint8)
    q = torch.zeros((1, wl.H_I, wl.D_I), dtype=torch.bfloat16)
    w = torch.zeros((1, wl.H_I), dtype=torch.float32)
    for b in range(4):
        q[0, b, 32 * b], q[0, 4 + b, 32 * b] = 1.0, -1.0
        w[0, b], w[0, 4 + b] = 1.0, -1.0
    seq = hsa.PagedSeq(wl.seq_lens, wl.block_table, wl.page_size, wl.num_pages,
                       wl.q_seq[:1], wl.q_pos[:1], max_seq_len=int(wl.seq_lens.max()),
                       status=torch.zeros(1, dtype=torch.int32, device=DEV))
    sc = hsa.hsa_index_score(seq, q.to(DEV), w.to(DEV), k8, E.contiguous().to(DEV))
    check_status(seq)
    n = int(wl.q_pos[0]) + 1
    bt = wl.block_table[0].cpu().long()
    pos = torch.arange(n)
    slot = bt[pos // wl.page_size] * wl.page_size + pos % wl.page_size
    codes = code_of_slot[slot].numpy().astype(np.uint8)
    vals = oracle.e4m3_decode(codes)
    ref = sum(vals * np.exp2(E[slot, b].double().numpy() - 127) for b in range(4))
    assert len(set(codes.tolist())) == 254
    assert np.array_equal(sc[0, :n].cpu().numpy().astype(np.float64), ref)


@pytest.mark.parametrize("src_dtype", [torch.bfloat16, torch.float32])
def test_quantize_mx_bit_exact(src_dtype):
    """hsa_quantize_mx against the oracle's MX quantizer, scattered through a slot permutation:
    N(0,1) keys scaled per row by 2^-40..2^40, the hand-worked golden blocks, every E4M3
    midpoint at the top binade's scale, all-zero and sub-2^-119 blocks."""
    g = torch.Generator().manual_seed(21)
    x = torch.randn((4096, 128), generator=g) * torch.exp2(torch.randint(-40, 41, (4096, 1), generator=g).float())
    vals = oracle.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    mids = torch.from_numpy(((vals[:-1] + vals[1:]) / 2).astype(np.float32))
    mid_rows = torch.cat([mids, -mids, torch.zeros((-2 * mids.numel()) % 127)]).view(-1, 127)
    mid_rows = torch.cat([torch.full((mid_rows.shape[0], 1), 448.0), mid_rows], 1)   # E = 127
    edge = torch.zeros((3, 128))
    edge[1, :32] = 2.0 ** -130
    edge[1, 40] = -(2.0 ** -140)
    edge[2, 64:96] = torch.linspace(-1.0, 1.0, 32) * 3e38          # finite, near the float32 top
    x = torch.cat([x, mid_rows, edge]).to(src_dtype)
    assert torch.isfinite(x).all()
    n = x.shape[0]
    perm = torch.randperm(n, generator=g)
    codes, scales = hsa.hsa_quantize_mx(x.to(DEV), slot_mapping=perm.to(DEV), num_slots=n)
    rc, rs = oracle.mx_quantize_rows(x.float())
    assert np.array_equal(codes.cpu()[perm].numpy(), rc)
    assert np.array_equal(scales.cpu()[perm].numpy(), rs)
    # dequantized values are exact in fp32; in bf16 for every block with E >= 3
    ref = oracle.mx_dequantize_rows(rc, rs)
    d32 = hsa.hsa_dequantize_mx(torch.from_numpy(rc).to(DEV), torch.from_numpy(rs).to(DEV), torch.float32)
    assert np.array_equal(d32.cpu().numpy().astype(np.float64), ref)
    d16 = hsa.hsa_dequantize_mx(torch.from_numpy(rc).to(DEV), torch.from_numpy(rs).to(DEV))
    big = np.repeat(rs >= 3, 32, axis=1)
    assert np.array_equal(d16.float().cpu().numpy().astype(np.float64)[big], ref[big])


def test_index_score_paging_invariance_bitwise():
    wl = workloads.make("decode_bf16", DEV, B=4, L_min=300, L_max=1000)
    base = hsa.hsa_index_score(paged_seq(wl), wl.q_I, wl.w, wl.k_I)
    perm = torch.randperm(wl.num_pages, generator=torch.Generator().manual_seed(3)).to(DEV)
    moved = torch.empty_like(wl.k_I).view(wl.num_pages, wl.page_size, -1)
    moved[perm] = wl.k_I.view(wl.num_pages, wl.page_size, -1)
    wl2 = workloads.make("decode_bf16", DEV, B=4, L_min=300, L_max=1000)
    wl2.block_table = perm.to(torch.int32)[wl.block_table.long()]
    got = hsa.hsa_index_score(paged_seq(wl2), wl.q_I, wl.w, moved.view(-1, wl.D_I))
    for t in range(wl.T_q):
        n = int(wl.q_pos[t]) + 1
        assert torch.equal(got[t, :n], base[t, :n])


@pytest.mark.parametrize("ties", [False, True])
def test_topk_vs_oracle_bit_exact(ties):
    K = 64
    lens = [1, 63, 64, 65, 66, 200, 1000, 4097, 33, 64 * 1024 + 17, 70000, 2]
    T = len(lens)
    ld = max(lens)
    sc = workloads.random_scores(T, ld, seed=21, device=DEV, ties=ties)
    seq = hsa.PagedSeq(torch.tensor([ld], device=DEV), torch.zeros((1, ld), dtype=torch.int32, device=DEV),
                       1, ld, torch.zeros(T, dtype=torch.int32, device=DEV),
                       torch.tensor([n - 1 for n in lens], dtype=torch.int32, device=DEV), max_seq_len=ld)
    idx = hsa.hsa_topk(seq, sc, K)
    ref = oracle.topk(sc.cpu(), np.array(lens, dtype=np.int32), K)
    assert np.array_equal(idx.cpu().numpy(), ref)
    # short rows: staged in shared memory
    seq2 = hsa.PagedSeq(torch.tensor([3000], device=DEV), torch.zeros((1, 3000), dtype=torch.int32, device=DEV),
                        1, 3000, torch.zeros(5, dtype=torch.int32, device=DEV),
                        torch.tensor([2999, 100, 64, 63, 1500], dtype=torch.int32, device=DEV), max_seq_len=3000)
    sc2 = sc[:5, :3000].contiguous()
    idx2 = hsa.hsa_topk(seq2, sc2, K)
    ref2 = oracle.topk(sc2.cpu(), np.array([3000, 101, 65, 64, 1501], dtype=np.int32), K)
    assert np.array_equal(idx2.cpu().numpy(), ref2)


@pytest.mark.parametrize("T,ld,K", [
    (64, 9000, 2048),     # staged in shared memory, just long enough to sample
    (64, 20001, 2048),    # staged, odd row stride (unaligned row starts)
    (160, 40000, 2048),   # staged, the longest staged rows
    (12, 70001, 2048),    # read from L2, odd row stride
    (10, 131072, 2048),   # read from L2, the longest prefill context
    (80, 60003, 512),     # read from L2, small K
])
@pytest.mark.parametrize("dist", ["normal", "ties", "narrow", "constant", "clustered"])
def test_topk_launch_variants_bit_exact(T, ld, K, dist):
    """Every path of the Top-K kernel (rows staged in shared memory or read from L2, aligned or
    unaligned row starts, sampled candidates or the whole row) on score distributions that
    stress each step: spread values, heavy ties with +-0.0, values that all share their top 22
    key bits, constant rows whose candidates overflow shared memory, and the best keys packed
    into one window of 3 K positions (on rows read from L2 the candidates of the few warps
    that sweep the window overflow their stretches, so those rows are collected again by the
    count-then-collect sweeps)."""
    g = torch.Generator().manual_seed(T * 7 + ld)
    lens = torch.randint(1, ld + 1, (T,), generator=g)
    lens[0], lens[1], lens[2], lens[3] = ld, K, K + 1, min(ld, 3 * K + 5)
    sc = workloads.random_scores(T, ld, seed=ld % 97, device=DEV, ties=(dist == "ties"))
    if dist == "narrow":
        sc = 1.0 + sc.abs() * 1e-6
    elif dist == "constant":
        sc = torch.full_like(sc, 0.75)
        sc[1::2] = -0.0
    elif dist == "clustered":
        w0 = ld // 3
        sc[:, w0:w0 + 3 * K] += 1000.0
    seq = hsa.PagedSeq(torch.tensor([ld], device=DEV), torch.zeros((1, ld), dtype=torch.int32, device=DEV),
                       1, ld, torch.zeros(T, dtype=torch.int32, device=DEV),
                       (lens - 1).to(torch.int32).to(DEV), max_seq_len=ld,
                       status=torch.zeros(1, dtype=torch.int32, device=DEV))
    idx = hsa.hsa_topk(seq, sc, K)
    check_status(seq)
    ref = oracle.topk(sc.cpu(), lens.numpy().astype(np.int32), K)
    assert np.array_equal(idx.cpu().numpy(), ref)


def _attn_vs_oracle(wl, tol, idx=None, kv_group=None):
    gc = GpuCaches(wl, kv_group)
    seq = paged_seq(wl)
    if idx is None:
        idx = workloads.random_selection(wl.q_pos, wl.K, seed=wl.seed + 50)
    idx_d = idx.to(DEV)
    out, lse = hsa.hsa_sparse_mla_attn(seq, wl.q, gc.kv, idx_d, wl.D_v, wl.softmax_scale,
                                       kv_scale=gc.kv_scale, kv_rope=gc.kv_rope)
    check_status(seq)
    oc = OracleCaches(wl, kv_group=kv_group)
    ref, rlse = oracle.sparse_mla(oracle_paging(wl), wl.q.cpu(), oc.kv, idx, wl.D_v, wl.softmax_scale)
    ok, worst = attn_close(out.float().cpu().numpy(), ref, tol)
    assert ok, (wl.name, worst)
    l = lse.cpu().numpy()
    fin = np.isfinite(rlse)
    assert np.array_equal(np.isfinite(l), fin)
    np.testing.assert_allclose(l[fin], rlse[fin], rtol=1e-4, atol=1e-4)
    return out, lse


@pytest.mark.parametrize("name,kw,tol", [
    ("tiny_decode_fp32", {}, 1e-4),
    ("decode_bf16", dict(B=5, L_min=100, L_max=4000), 2e-2),
    ("decode_fp8", dict(B=3, L=3000), 6e-2),
    ("prefill_bf16", dict(T=2100), 2e-2),
])
def test_sparse_mla_vs_oracle(name, kw, tol):
    _attn_vs_oracle(workloads.make(name, DEV, **kw), tol)


@pytest.mark.parametrize("page_size", [16, 384])
def test_sparse_mla_page_sizes(page_size):
    """The gather's slot lookups with small pages and with a page size that is not a power of
    two, bf16 and FP8 caches."""
    _attn_vs_oracle(workloads.make("decode_bf16", DEV, B=3, L_min=2200, L_max=4000, page_size=page_size), 2e-2)
    _attn_vs_oracle(workloads.make("decode_fp8", DEV, B=2, L=2600, page_size=page_size), 6e-2)


@pytest.mark.parametrize("name,kw,block", [
    ("decode_bf16", dict(B=6, L_min=1500, L_max=9000), 64),
    ("prefill_bf16", dict(T=2400), 64),
    ("decode_bf16", dict(B=4, L_min=3000, L_max=5000), 16),
])
def test_topk_blocks_bit_exact_and_attention(name, kw, block):
    """Block-aligned selection on the GPU's own fp32 scores equals the oracle's rule bit for bit
    (rows shorter than K, partial last blocks, ties of block maxima included), keeps whole
    cache pages when block = page size, and the attention over it matches the oracle's."""
    wl = workloads.make(name, DEV, **kw)
    seq = paged_seq(wl)
    sc = hsa.hsa_index_score(seq, wl.q_I, wl.w, wl.k_I)
    sc_t = sc.clone()
    if wl.T_q > 3:                                  # ties between block maxima on row 2
        n2 = int(wl.q_pos[2]) + 1
        sc_t[2, :n2] = torch.floor(sc_t[2, :n2] * 2) / 2
    idx = hsa.hsa_topk_blocks(seq, sc_t, wl.K, block)
    check_status(seq)
    n_valid = (wl.q_pos + 1).cpu().numpy().astype(np.int32)
    ref = oracle.topk_blocks(sc_t.cpu(), n_valid, wl.K, block)
    assert np.array_equal(idx.cpu().numpy(), ref)
    if block == wl.page_size:                       # whole pages
        g = idx.cpu().numpy()
        for t in range(wl.T_q):
            sel = g[t][g[t] >= 0]
            if int(n_valid[t]) > wl.K:
                assert len(set((sel // block).tolist())) == wl.K // block
    _attn_vs_oracle(wl, 2e-2, idx.cpu())


@pytest.mark.parametrize("B", [3, 64])
def test_sparse_mla_short_rows_and_workspace(B):
    """Few rows (3) and the decode batch's 64, with a short row (11 of 32 tiles) and an empty row
    riding along, against the oracle; the workspace the library reports is not needed by the
    current kernel, so a call with none and a repeated call give the same bits."""
    wl = workloads.make("decode_bf16", DEV, B=B, L_min=2100, L_max=6000)
    idx = workloads.random_selection(wl.q_pos, wl.K, seed=11)
    idx[1, 700:] = -1                     # 11 of 32 tiles
    idx[2] = -1                           # nothing selected
    out, lse = _attn_vs_oracle(wl, 2e-2, idx)
    assert torch.all(out[2] == 0) and torch.all(torch.isneginf(lse[2]))
    seq = paged_seq(wl)
    need = hsa.hsa_sparse_mla_workspace_size(seq, wl.H, wl.D_qk, wl.D_v, wl.K)
    ws = torch.zeros(max(need, 1), dtype=torch.uint8, device=DEV)
    out_s, lse_s = hsa.hsa_sparse_mla_attn(seq, wl.q, wl.kv, idx.to(DEV), wl.D_v, wl.softmax_scale, ws=ws)
    out_2, lse_2 = hsa.hsa_sparse_mla_attn(seq, wl.q, wl.kv, idx.to(DEV), wl.D_v, wl.softmax_scale, ws=ws)
    check_status(seq)
    assert torch.equal(out_s, out) and torch.equal(lse_s, lse)
    assert torch.equal(out_2, out_s) and torch.equal(lse_2, lse_s)


@pytest.mark.parametrize("kv_group", [512, 128, 64])
@pytest.mark.parametrize("H", [128, 16])
def test_sparse_mla_fp8_scale_groups(kv_group, H):
    """FP8 latent cache with one scale per token (512), per the pages' 128-dim tile, and per 64
    dims, on the tensor-core kernel (128 heads) and the CUDA-core kernel (16 heads)."""
    wl = workloads.make("decode_fp8", DEV, B=3, L=2500, H=H)
    _attn_vs_oracle(wl, 6e-2, kv_group=kv_group)


@pytest.mark.parametrize("name,kw,tol", [
    ("decode_bf16", dict(B=4, L_min=100, L_max=3000), 2e-2),
    ("decode_fp8", dict(B=4, L=3000), 6e-2),
])
def test_sparse_mla_empty_rows_and_constant_values(name, kw, tol):
    wl = workloads.make(name, DEV, **kw)
    idx = workloads.random_selection(wl.q_pos, wl.K, seed=5)
    idx[1] = -1                       # a row that selects nothing
    idx[2, 1::2] = -1                 # holes inside a row
    out, lse = _attn_vs_oracle(wl, tol, idx)
    assert torch.all(out[1] == 0) and torch.all(torch.isneginf(lse[1]))
    wl.kv[:, :wl.D_v] = 1.0           # every value row is all ones -> output is ones
    gc = GpuCaches(wl)
    out2, _ = hsa.hsa_sparse_mla_attn(paged_seq(wl), wl.q, gc.kv, idx.to(DEV), wl.D_v, wl.softmax_scale,
                                      kv_scale=gc.kv_scale, kv_rope=gc.kv_rope)
    for t in (0, 2, 3):
        assert torch.allclose(out2[t].float(), torch.ones_like(out2[t].float()), atol=1e-2)


@pytest.mark.parametrize("group", [None, 32])
def test_quantize_index_bit_exact(group):
    wl = workloads.make("decode_fp8", DEV, B=2, L=2000)
    grp = wl.D_I if group is None else group
    n = wl.k_I.shape[0]
    perm = torch.randperm(n, generator=torch.Generator().manual_seed(1))
    slots = perm.to(DEV).to(torch.int64)
    codes, scales = hsa.hsa_quantize_index(wl.k_I, grp, slot_mapping=slots, num_slots=n)
    rc, rs = oracle.quantize_rows(wl.k_I.float().cpu(), grp)
    assert np.array_equal(codes.cpu()[perm].numpy(), rc)
    assert np.array_equal(scales.cpu()[perm].numpy(), rs)


def test_quantize_kv_bit_exact_and_rounding_ties():
    wl = workloads.make("decode_fp8", DEV, B=2, L=1024)
    codes, scales, rope = hsa.hsa_quantize_kv(wl.kv, wl.D_v, wl.D_v)
    rc, rs = oracle.quantize_rows(wl.kv[:, :wl.D_v].float().cpu(), wl.D_v)
    assert np.array_equal(codes.cpu().numpy(), rc) and np.array_equal(scales.cpu().numpy(), rs)
    assert torch.equal(rope, wl.kv[:, wl.D_v:])
    # rows whose max is 448 have scale 1 and are rounded as they are: every midpoint between
    # adjacent E4M3 values, and 4e6 random fp32 values, against the library's conversion
    vals = oracle.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    g = torch.Generator().manual_seed(9)
    rnd = (torch.randn(4_000_000, generator=g) * 60).clamp(-447, 447)
    x = torch.cat([torch.from_numpy(mids), -torch.from_numpy(mids), rnd])
    D = 126
    pad = (-x.numel()) % (D - 1)
    x = torch.cat([x, torch.zeros(pad)]).view(-1, D - 1)
    x = torch.cat([torch.full((x.shape[0], 1), 448.0), x], dim=1).contiguous()
    gcodes, gscales = hsa.hsa_quantize_index(x.to(DEV), D)
    assert torch.all(gscales == 1.0)
    ref = oracle.e4m3_encode(x.numpy().ravel()).reshape(x.shape)
    assert np.array_equal(gcodes.cpu().numpy(), ref)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_quantize_tiny_group_maxima_bit_exact(dtype):
    """Groups whose maximum is far below 448 / FLT_MAX (1e-37, 1e-40, 2^-64, 2^-65, 2^-140)
    and which hold zeros: codes and scales equal the oracle's bit for bit, and no NaN code
    appears.  The same rows through the KV quantizer (latent part) agree as well."""
    rng = np.random.default_rng(21)
    rows = []
    for amax in (1e-37, 1e-40, 2.0 ** -64, 2.0 ** -65, 2.0 ** -140, 1.0):
        base = rng.standard_normal(128)
        base[rng.random(128) < 0.25] = 0.0
        base = base / np.abs(base).max() * amax
        rows.append(base)
    x = torch.tensor(np.stack(rows), dtype=torch.float32).to(dtype)
    xf = x.float()
    for grp in (128, 32):
        codes, scales = hsa.hsa_quantize_index(x.to(DEV), grp)
        rc, rs = oracle.quantize_rows(xf, grp)
        assert np.array_equal(codes.cpu().numpy(), rc), grp
        assert np.array_equal(scales.cpu().numpy(), rs), grp
        assert not np.any((rc & 0x7F) == 0x7F)
    kv = torch.cat([x, torch.zeros((x.shape[0], 64), dtype=dtype)], dim=1).contiguous()
    kcodes, kscales, _ = hsa.hsa_quantize_kv(kv.to(DEV), 128, 128)
    rc, rs = oracle.quantize_rows(xf, 128)
    assert np.array_equal(kcodes.cpu().numpy(), rc) and np.array_equal(kscales.cpu().numpy(), rs)


def test_device_checks_flag_instead_of_faulting():
    wl = workloads.make("decode_bf16", DEV, B=3, L_min=200, L_max=600)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    bad = wl.block_table.clone()
    bad[1, 0] = wl.num_pages + 5      # page id out of range
    seq = hsa.PagedSeq(wl.seq_lens, bad, wl.page_size, wl.num_pages, wl.q_seq, wl.q_pos, q_run=1,
                       status=status)
    hsa.hsa_index_score(seq, wl.q_I, wl.w, wl.k_I)
    torch.cuda.synchronize()
    assert int(status.item()) & hsa.HSA_DEV_BAD_PAGE
    status.zero_()
    qpos = wl.q_pos.clone()
    qpos[0] = int(wl.seq_lens[0]) + 3  # position past the sequence end
    seq2 = hsa.PagedSeq(wl.seq_lens, wl.block_table, wl.page_size, wl.num_pages, wl.q_seq, qpos,
                        max_seq_len=int(wl.seq_lens.max()) + 8, status=status)
    hsa.hsa_topk(seq2, torch.zeros((3, int(wl.seq_lens.max()) + 8), device=DEV), 16)
    torch.cuda.synchronize()
    assert int(status.item()) & hsa.HSA_DEV_BAD_POS
    status.zero_()
    idx = workloads.random_selection(wl.q_pos, 64, seed=1).to(DEV)
    idx[0, 0] = int(wl.q_pos[0]) + 1   # selected position beyond the causal window
    hsa.hsa_sparse_mla_attn(paged_seq(wl, status), wl.q, wl.kv, idx, wl.D_v, wl.softmax_scale)
    torch.cuda.synchronize()
    assert int(status.item()) & hsa.HSA_DEV_BAD_POS


def test_sparse_mla_repeatable_and_clean():
    """Many launches of the same call give bitwise-identical results and never trip a device-side
    check: pipeline races between the two CTAs of a cluster would show up here first."""
    wl = workloads.make("decode_bf16", DEV, B=24, L_min=2100, L_max=6000)
    idx = workloads.random_selection(wl.q_pos, wl.K, seed=77).to(DEV)
    seq = paged_seq(wl)
    ref, ref_lse = hsa.hsa_sparse_mla_attn(seq, wl.q, wl.kv, idx, wl.D_v, wl.softmax_scale)
    for _ in range(30):
        out, lse = hsa.hsa_sparse_mla_attn(seq, wl.q, wl.kv, idx, wl.D_v, wl.softmax_scale)
        assert torch.equal(out, ref) and torch.equal(lse, ref_lse)
    check_status(seq)
