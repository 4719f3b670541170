"""Zigzag context parallelism for long causal prefill over several GPUs.

The sequence of T positions is cut into 2W equal segments for W ranks; rank r owns segments r
and 2W-1-r ("Efficient Inference Deployment and Optimization for Hybrid Attention LLMs", 5.2;
"Inference Adaptation and Performance Optimization for a Domestically Developed LLM's New
Architecture", 5.2).  Under a causal mask segment s carries work proportional to s + 1/2, so
every rank's pair carries the same total.  Each rank holds the index-key and latent cache pages
of its own two segments (it wrote them); one all-gather gives every rank the whole cache, and
its query rows then run the one-GPU path (``hsa_prefill_chunked``: index score, Top-K, sparse
MLA, one segment per stream) with no further exchange.  Optionally a second all-gather puts the
outputs of all ranks back in position order.

This module is host logic only: the arithmetic runs in the library's kernels and the exchange
is ``torch.distributed`` (NCCL on GPUs).  Multicast loads are not involved: the gathered pages
land in each rank's own memory before any kernel reads them.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist


def segment_rows(T: int, world: int, page_size: int = 1) -> int:
    """Positions per segment (T / 2W); it must be a whole number of cache pages."""
    n = 2 * world
    if T % n or (T // n) % page_size:
        raise ValueError(f"T = {T} must split into {n} segments of whole pages of {page_size}")
    return T // n


def rank_segments(T: int, world: int, rank: int) -> List[Tuple[int, int]]:
    """The two position ranges [p0, p1) rank `rank` owns: segments rank and 2W-1-rank."""
    S = segment_rows(T, world)
    return [(s * S, (s + 1) * S) for s in (rank, 2 * world - 1 - rank)]


def rank_positions(T: int, world: int, rank: int) -> torch.Tensor:
    """int32 positions of the rank's query rows: its first segment, then its second."""
    return torch.cat([torch.arange(p0, p1, dtype=torch.int32) for p0, p1 in rank_segments(T, world, rank)])


def gathered_block_table(T: int, world: int, page_size: int) -> torch.Tensor:
    """int32 [1, T / page_size] block table of the whole sequence over the gathered cache.

    Rank r's local cache holds its first segment's pages, then its second's; the all-gather
    stacks the ranks' local caches in rank order.  Logical page j of segment s therefore lives
    on rank src = s (s < W) or 2W-1-s (s >= W), local segment 0 or 1, and its physical page is
    src * 2P + local * P + (j - s * P) with P pages per segment."""
    P = segment_rows(T, world, page_size) // page_size
    table = torch.empty(2 * world * P, dtype=torch.int32)
    for s in range(2 * world):
        src, local = (s, 0) if s < world else (2 * world - 1 - s, 1)
        table[s * P:(s + 1) * P] = src * 2 * P + local * P + torch.arange(P, dtype=torch.int32)
    return table.view(1, -1)


def all_gather_rows(local: torch.Tensor, group=None) -> torch.Tensor:
    """Stack every rank's `local` [n, ...] along dim 0 in rank order (one collective)."""
    world = dist.get_world_size(group)
    local = local.contiguous()
    out = torch.empty((world * local.shape[0],) + tuple(local.shape[1:]), dtype=local.dtype,
                      device=local.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, local, group=group)
    else:
        dist.all_gather(list(out.chunk(world)), local, group=group)
    return out


def _library_compute(seq_lens, block_table, page_size, num_pages, q_seq, q_pos, q_I, w, k, k_scale,
                     q, kv, kv_scale, kv_rope, K, D_v, softmax_scale, chunks):
    import sparse_index_attention_b200 as hsa
    dev = q.device
    seq = hsa.PagedSeq(seq_lens.to(dev), block_table.to(dev), page_size, num_pages, q_seq.to(dev),
                       q_pos.to(dev), q_run=chunks[0][1] - chunks[0][0])
    return hsa.hsa_prefill_chunked(seq, q_I, w, k, k_scale, q, kv, kv_scale, kv_rope, K, D_v,
                                   softmax_scale, chunks)


def prefill_zigzag_cp(T: int, page_size: int, q_I, w, q, k_local, kv_local, K: int, D_v: int,
                      softmax_scale: float, k_scale_local=None, kv_scale_local=None,
                      kv_rope_local=None, group=None, gather_outputs: bool = False,
                      compute: Optional[Callable] = None):
    """Causal prefill of one sequence of T positions on W ranks in zigzag segments.

    Per rank: q_I [2S, H_I, D_I], w [2S, H_I], q [2S, H, D_qk] are the rows of its two segments
    (``rank_positions`` order); k_local [2S, D_I] and kv_local [2S, D_qk] (or the FP8 codes, with
    the matching ``*_scale_local`` / ``kv_rope_local`` rows) are the cache rows of the same
    positions, page by page.  Returns (out [2S, H, D_v], lse [2S, H], idx [2S, K]) for the rank's
    rows; with ``gather_outputs`` the outputs of all ranks in position order ([T, H, D_v],
    [T, H]) and the rank's idx.  ``compute`` defaults to the library's chunked prefill; it
    receives the gathered paging and caches and the rank's two segments as row chunks.
    """
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    S = segment_rows(T, world, page_size)
    if q.shape[0] != 2 * S or k_local.shape[0] != 2 * S or kv_local.shape[0] != 2 * S:
        raise ValueError("each rank passes the 2 * T / (2W) rows of its two segments")
    gather = lambda t: None if t is None else all_gather_rows(t, group)   # noqa: E731
    k, kv = gather(k_local), gather(kv_local)
    k_scale, kv_scale, kv_rope = gather(k_scale_local), gather(kv_scale_local), gather(kv_rope_local)
    bt = gathered_block_table(T, world, page_size)
    pos = rank_positions(T, world, rank)
    compute = compute or _library_compute
    out, lse, idx = compute(torch.tensor([T], dtype=torch.int32), bt, page_size,
                            bt.shape[1], torch.zeros(2 * S, dtype=torch.int32), pos, q_I, w, k,
                            k_scale, q, kv, kv_scale, kv_rope, K, D_v, softmax_scale,
                            [(0, S), (S, 2 * S)])
    if not gather_outputs:
        return out, lse, idx
    return _to_position_order(all_gather_rows(out, group), T, world), \
        _to_position_order(all_gather_rows(lse, group), T, world), idx


def _to_position_order(stacked: torch.Tensor, T: int, world: int) -> torch.Tensor:
    """Rows gathered in rank order (each rank: its two segments) back in position order."""
    S = T // (2 * world)
    full = torch.empty_like(stacked)
    for r in range(world):
        for j, (p0, p1) in enumerate(rank_segments(T, world, r)):
            full[p0:p1] = stacked[(2 * r + j) * S:(2 * r + j + 1) * S]
    return full


def pair_loads(T: int, world: int) -> Sequence[int]:
    """Causal (query, key) pairs each rank scores: sum over its positions p of p + 1."""
    return [sum(p1 * (p1 + 1) // 2 - p0 * (p0 + 1) // 2 for p0, p1 in rank_segments(T, world, r))
            for r in range(world)]
