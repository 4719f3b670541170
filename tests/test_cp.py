"""Zigzag context-parallel prefill (host logic): the segment layout, the gathered block table,
and a two-rank gloo run on the CPU whose per-rank compute is the oracle, against the oracle's
one-process result for the whole sequence.  The library's kernels take the place of the oracle
on GPUs; that single-rank path is covered in test_gpu_prefill.py."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from sparse_index_attention_b200 import cp, workloads

TINY = dict(T=192, page_size=8, H_I=4, D_I=32, H=8, D_v=64, D_rope=16, K=16)


@pytest.mark.parametrize("world", [1, 2, 3, 4])
def test_segments_cover_every_position_once_with_equal_load(world):
    T = 2 * world * 40
    seen = torch.cat([cp.rank_positions(T, world, r) for r in range(world)])
    assert torch.equal(seen.sort().values, torch.arange(T, dtype=torch.int32))
    loads = cp.pair_loads(T, world)
    assert len(set(loads)) == 1 and sum(loads) == T * (T + 1) // 2
    with pytest.raises(ValueError):
        cp.segment_rows(T + 1, world)


@pytest.mark.parametrize("world,page", [(1, 4), (2, 8), (3, 4), (4, 2)])
def test_gathered_block_table_finds_every_position(world, page):
    """Build each rank's local cache of position ids, stack them as the all-gather does, and
    read every position back through the block table."""
    T = 2 * world * 3 * page
    local = [cp.rank_positions(T, world, r) for r in range(world)]
    gathered = torch.cat(local)
    bt = cp.gathered_block_table(T, world, page)
    assert sorted(bt.view(-1).tolist()) == list(range(T // page))
    for p in range(T):
        slot = int(bt[0, p // page]) * page + p % page
        assert int(gathered[slot]) == p


def _oracle_compute(seq_lens, block_table, page_size, num_pages, q_seq, q_pos, q_I, w, k, k_scale,
                    q, kv, kv_scale, kv_rope, K, D_v, softmax_scale, chunks):
    """Per-rank compute for the CPU runs: the oracle over the gathered paging and caches (FP8
    caches decoded by the oracle's own codec)."""
    if k_scale is not None:
        k = oracle.dequantize_rows(k, k_scale.numpy(), k.shape[1])
    if kv_scale is not None:
        lat = oracle.dequantize_rows(kv, kv_scale.numpy(), kv.shape[1])
        kv = np.concatenate([lat, kv_rope.float().numpy().astype(np.float64)], axis=1)
    pg = oracle.Paging(seq_lens, block_table, page_size, num_pages, q_seq, q_pos)
    _, idx, out, lse = oracle.sparse_index_attention(pg, q_I, w, k, q, kv, K, D_v, softmax_scale)
    return torch.from_numpy(out), torch.from_numpy(lse), torch.from_numpy(idx)


def _slots(wl, pos):
    pos = pos.long()
    return wl.block_table[0].long()[pos // wl.page_size] * wl.page_size + pos % wl.page_size


def _caches(wl, fp8):
    """The whole cache as the oracle reads it, in slot order: bf16 values, or FP8 codes with
    fp32 scales (per key; per token for the latent part) and bf16 rope."""
    if not fp8:
        return dict(k=wl.k_I, kv=wl.kv)
    kc, ks = oracle.quantize_rows(wl.k_I.float(), wl.D_I)
    vc, vs = oracle.quantize_rows(wl.kv[:, :wl.D_v].float(), wl.D_v)
    return dict(k=torch.from_numpy(kc), k_scale=torch.from_numpy(ks[:, 0].copy()),
                kv=torch.from_numpy(vc), kv_scale=torch.from_numpy(vs[:, 0].copy()),
                kv_rope=wl.kv[:, wl.D_v:].contiguous())


def _worker(rank, world, port, fp8, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        wl = workloads.make("prefill_bf16", **TINY)
        pos = cp.rank_positions(wl.T_q, world, rank)
        rows = pos.long()
        sl = _slots(wl, pos)
        c = {k: v[sl] for k, v in _caches(wl, fp8).items()}
        out, lse, idx = cp.prefill_zigzag_cp(
            wl.T_q, wl.page_size, wl.q_I[rows], wl.w[rows], wl.q[rows], c["k"], c["kv"], wl.K,
            wl.D_v, wl.softmax_scale, k_scale_local=c.get("k_scale"),
            kv_scale_local=c.get("kv_scale"), kv_rope_local=c.get("kv_rope"),
            gather_outputs=True, compute=_oracle_compute)
        q.put((rank, out.numpy(), lse.numpy(), idx.numpy(), pos.numpy()))
    finally:
        dist.destroy_process_group()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,fp8", [(2, False), (3, False), (2, True)])
def test_zigzag_cp_prefill_equals_one_process(world, fp8):
    """Every rank's rows, and the gathered outputs in position order, equal the one-process
    oracle over the whole sequence bit for bit; with FP8 caches the scales and the rope rows
    travel through the same all-gather as the codes."""
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, fp8, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted((q.get(timeout=120) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]

    wl = workloads.make("prefill_bf16", **TINY)
    c = _caches(wl, fp8)
    ref_out, ref_lse, ref_idx = _oracle_compute(
        wl.seq_lens, wl.block_table, wl.page_size, wl.num_pages, wl.q_seq, wl.q_pos, wl.q_I, wl.w,
        c["k"], c.get("k_scale"), wl.q, c["kv"], c.get("kv_scale"), c.get("kv_rope"), wl.K, wl.D_v,
        wl.softmax_scale, None)
    for rank, out, lse, idx, pos in got:
        assert np.array_equal(out, ref_out.numpy()) and np.array_equal(lse, ref_lse.numpy()), rank
        assert np.array_equal(idx, ref_idx.numpy()[pos]), rank


@pytest.mark.parametrize("world", [1, 2, 3])
def test_outputs_return_to_position_order(world):
    """Rows stacked in rank order (each rank: its two segments) come back in position order."""
    T = 2 * world * 5
    stacked = torch.cat([cp.rank_positions(T, world, r) for r in range(world)])
    assert torch.equal(cp._to_position_order(stacked, T, world), torch.arange(T, dtype=torch.int32))
