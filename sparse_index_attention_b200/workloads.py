"""Seeded synthetic inputs for the sparse index attention path.

This module only draws random numbers and lays them out (sequence lengths, a random page
permutation for the block table, query rows and positions).  It holds none of the method's
arithmetic, so both the CUDA path and the CPU oracle can consume what it produces.

Every tensor X of a workload with seed ``c`` is drawn from its own ``torch.Generator`` seeded
with ``1000 * c + id(X)``; the ids are fixed below.  Floating point data is drawn as fp32
``randn``, scaled, then rounded to bf16 (round to nearest even) unless the workload is fp32.
FP8 workloads draw bf16 data here; each side quantizes it itself.

Named workloads (sizes as the pages' deployment scenarios use them: decode batches of long
contexts with Top-2048 selection over an MLA latent cache of 512 + 64 dims, 128 heads, and a
64-head x 128-dim indexer):

* ``tiny_decode_fp32``      B=1, L=256, 4 query rows at 252..255, 4x32 indexer, Top-32,
                            8 heads, latent 64 + rope 16, page 16, fp32.
* ``decode_bf16``           B=64, L ~ U[8192, 32768], one query row per sequence, bf16.
* ``prefill_bf16``          one sequence of 16384 tokens, every token a query, bf16.
* ``decode_fp8``            B=128, L=65536, FP8 index keys (one scale per key) and FP8 latent
                            KV (one scale per token) with a bf16 rope part.
* ``prefill_long_zigzag``   one sequence of 131072 tokens in 32 query chunks of 4096, issued
                            as pairs (i, 31-i); FP8 index keys, bf16 KV.
* ``decode_mxfp8``          ``decode_fp8``'s draws with the index queries and keys in MXFP8.
* ``decode_draft_bf16``     as ``decode_bf16`` but four query rows per sequence at its last
                            four positions (draft-verify decode).
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Tuple

import torch

# tensor ids used in the seed formula
ID_LENGTHS, ID_BLOCK_TABLE, ID_Q_I, ID_W, ID_K_I, ID_Q, ID_KV = 1, 2, 3, 4, 5, 6, 7

_CHUNK_ELEMS = 1 << 28  # draw big tensors in slices of 256 Mi elements


@dataclasses.dataclass
class Workload:
    name: str
    seed: int
    dtype: str                      # "f32" or "bf16": dtype of q_I, k_I, q, kv as drawn
    # paged sequences
    B: int
    seq_lens: torch.Tensor          # int32 [B]
    block_table: torch.Tensor       # int32 [B, max_pages]; entries past a sequence's pages are 0
    page_size: int
    num_pages: int
    # query rows
    T_q: int
    q_seq: torch.Tensor             # int32 [T_q]
    q_pos: torch.Tensor             # int32 [T_q]
    q_run: int                      # rows come in runs of this many rows of one sequence
    # indexer
    H_I: int
    D_I: int
    q_I: torch.Tensor               # [T_q, H_I, D_I]
    w: torch.Tensor                 # fp32 [T_q, H_I]
    k_I: torch.Tensor               # [num_pages * page_size, D_I] (bf16 source when index_fp8)
    index_fp8: bool
    # sparse MLA
    H: int
    D_qk: int
    D_v: int
    q: torch.Tensor                 # [T_q, H, D_qk]
    kv: torch.Tensor                # [num_pages * page_size, D_qk]: latent (D_v) ‖ rope
    kv_fp8: bool
    K: int
    softmax_scale: float
    chunks: Optional[List[Tuple[int, int]]] = None   # query-row ranges in issue order
    index_mx: bool = False          # index keys and queries in MXFP8 (E8M0 per 32 dims)

    @property
    def num_slots(self) -> int:
        return self.num_pages * self.page_size

    @property
    def D_rope(self) -> int:
        return self.D_qk - self.D_v


def _gen(device, seed: int, tid: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(1000 * seed + tid)
    return g


def _randn(shape, g, device, scale: float, dtype: torch.dtype) -> torch.Tensor:
    """fp32 randn * scale, rounded to `dtype`, drawn slice by slice along dim 0."""
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(shape[0], -1)
    per_row = flat.shape[1] if flat.dim() > 1 else 1
    rows = max(1, _CHUNK_ELEMS // max(per_row, 1))
    for r0 in range(0, shape[0], rows):
        r1 = min(shape[0], r0 + rows)
        x = torch.randn((r1 - r0,) + tuple(shape[1:]), generator=g, device=device,
                        dtype=torch.float32)
        if scale != 1.0:
            x.mul_(scale)
        out[r0:r1] = x.to(dtype)
    return out


def _paging(seq_lens: List[int], page_size: int, device, seed: int):
    pages = [math.ceil(L / page_size) for L in seq_lens]
    num_pages = sum(pages)
    perm = torch.randperm(num_pages, generator=_gen("cpu", seed, ID_BLOCK_TABLE))
    max_pages = max(pages)
    bt = torch.zeros((len(seq_lens), max_pages), dtype=torch.int32)
    off = 0
    for b, n in enumerate(pages):
        bt[b, :n] = perm[off:off + n].to(torch.int32)
        off += n
    return bt.to(device), num_pages


def _build(name, seed, device, dtype_s, seq_lens, page_size, q_seq, q_pos, q_run, H_I, D_I,
           w_scale, H, D_qk, D_v, qkv_scale, K, softmax_scale, index_fp8, kv_fp8, chunks=None,
           q_scale=None):
    dt = torch.float32 if dtype_s == "f32" else torch.bfloat16
    bt, num_pages = _paging(seq_lens, page_size, device, seed)
    slots = num_pages * page_size
    T_q = len(q_seq)
    q_I = _randn((T_q, H_I, D_I), _gen(device, seed, ID_Q_I), device, 1.0, dt)
    w = _randn((T_q, H_I), _gen(device, seed, ID_W), device, w_scale, torch.float32)
    k_I = _randn((slots, D_I), _gen(device, seed, ID_K_I), device, 1.0, dt)
    q = _randn((T_q, H, D_qk), _gen(device, seed, ID_Q), device,
               qkv_scale if q_scale is None else q_scale, dt)
    kv = _randn((slots, D_qk), _gen(device, seed, ID_KV), device, qkv_scale, dt)
    return Workload(
        name=name, seed=seed, dtype=dtype_s, B=len(seq_lens),
        seq_lens=torch.tensor(seq_lens, dtype=torch.int32, device=device), block_table=bt,
        page_size=page_size, num_pages=num_pages, T_q=T_q,
        q_seq=torch.tensor(q_seq, dtype=torch.int32, device=device),
        q_pos=torch.tensor(q_pos, dtype=torch.int32, device=device), q_run=q_run,
        H_I=H_I, D_I=D_I, q_I=q_I, w=w, k_I=k_I, index_fp8=index_fp8,
        H=H, D_qk=D_qk, D_v=D_v, q=q, kv=kv, kv_fp8=kv_fp8, K=K,
        softmax_scale=softmax_scale, chunks=chunks)


def _lengths(B, L_min, L_max, seed):
    if L_min == L_max:
        return [L_min] * B
    g = _gen("cpu", seed, ID_LENGTHS)
    return torch.randint(L_min, L_max + 1, (B,), generator=g).tolist()


# ------------------------------------------------------------------------------ recipes
def tiny_decode_fp32(device="cpu", seed=0, L=256, n_rows=4, page_size=16, H_I=4, D_I=32, H=8,
                     D_v=64, D_rope=16, K=32):
    q_pos = list(range(L - n_rows, L))
    D_qk = D_v + D_rope
    return _build("tiny_decode_fp32", seed, device, "f32", [L], page_size, [0] * n_rows, q_pos,
                  n_rows, H_I, D_I, 0.5, H, D_qk, D_v, 1.0, K, 1.0 / math.sqrt(D_qk),
                  False, False)


def decode_bf16(device="cpu", seed=1, B=64, L_min=8192, L_max=32768, page_size=64, H_I=64,
                D_I=128, H=128, D_v=512, D_rope=64, K=2048):
    lens = _lengths(B, L_min, L_max, seed)
    D_qk = D_v + D_rope
    return _build("decode_bf16", seed, device, "bf16", lens, page_size, list(range(B)),
                  [L - 1 for L in lens], 1, H_I, D_I, 1.0 / 8, H, D_qk, D_v, 0.5, K,
                  1.0 / math.sqrt(D_qk), False, False)


def prefill_bf16(device="cpu", seed=2, T=16384, page_size=64, H_I=64, D_I=128, H=128, D_v=512,
                 D_rope=64, K=2048):
    D_qk = D_v + D_rope
    return _build("prefill_bf16", seed, device, "bf16", [T], page_size, [0] * T, list(range(T)),
                  T, H_I, D_I, 1.0 / 8, H, D_qk, D_v, 0.5, K, 1.0 / math.sqrt(D_qk), False,
                  False)


def decode_fp8(device="cpu", seed=3, B=128, L=65536, page_size=64, H_I=64, D_I=128, H=128,
               D_v=512, D_rope=64, K=2048):
    D_qk = D_v + D_rope
    return _build("decode_fp8", seed, device, "bf16", [L] * B, page_size, list(range(B)),
                  [L - 1] * B, 1, H_I, D_I, 1.0 / 8, H, D_qk, D_v, 1.0, K,
                  1.0 / math.sqrt(D_qk), True, True)


def decode_mxfp8(device="cpu", seed=3, **kw):
    """decode_fp8 (same seed, so the same draws) with the index queries and keys in MXFP8: blocks
    of 32 dims sharing one power-of-two scale ("Inference Adaptation and Performance Optimization
    for a Domestically Developed LLM's New Architecture", section 4 table; "Day 0 Inference
    Adaptation and Optimization for Hybrid Attention Models", "Hierarchical Quantization").
    The latent cache stays FP8 with an fp32 scale per token."""
    wl = decode_fp8(device=device, seed=seed, **kw)
    return dataclasses.replace(wl, name="decode_mxfp8", index_mx=True)


def decode_draft_bf16(device="cpu", seed=5, B=64, n_draft=4, L_min=8192, L_max=32768,
                      page_size=64, H_I=64, D_I=128, H=128, D_v=512, D_rope=64, K=2048):
    """Draft-verify decode: each sequence checks n_draft drafted tokens in one step, so it has
    n_draft query rows at its last n_draft positions, each causal over its own prefix
    ("Day 0 Inference Adaptation and Optimization for Hybrid Attention Models", decoding
    acceleration reuse: the draft-verify paradigm; "Inference Adaptation and Performance
    Optimization for a Domestically Developed LLM's New Architecture", 6: speculative
    inference).  Same shapes and value recipe as decode_bf16 otherwise."""
    lens = _lengths(B, max(L_min, n_draft), max(L_max, n_draft), seed)
    D_qk = D_v + D_rope
    q_seq = [b for b in range(B) for _ in range(n_draft)]
    q_pos = [L - n_draft + i for L in lens for i in range(n_draft)]
    return _build("decode_draft_bf16", seed, device, "bf16", lens, page_size, q_seq, q_pos,
                  n_draft, H_I, D_I, 1.0 / 8, H, D_qk, D_v, 0.5, K, 1.0 / math.sqrt(D_qk),
                  False, False)


def zigzag_chunks(T: int, n_chunks: int) -> List[Tuple[int, int]]:
    """Query-row ranges issued as pairs (i, n_chunks-1-i) ("Efficient Inference Deployment and
    Optimization for Hybrid Attention LLMs", 5.2: segment i goes with segment 2N-1-i)."""
    if T % n_chunks or n_chunks % 2:
        raise ValueError("T must split into an even number of equal chunks")
    c = T // n_chunks
    order = []
    for i in range(n_chunks // 2):
        for j in (i, n_chunks - 1 - i):
            order.append((j * c, (j + 1) * c))
    return order


def prefill_long_zigzag(device="cpu", seed=4, T=131072, n_chunks=32, page_size=64, H_I=64,
                        D_I=128, H=128, D_v=512, D_rope=64, K=2048):
    D_qk = D_v + D_rope
    return _build("prefill_long_zigzag", seed, device, "bf16", [T], page_size, [0] * T,
                  list(range(T)), T // n_chunks, H_I, D_I, 1.0 / 8, H, D_qk, D_v, 0.5, K,
                  1.0 / math.sqrt(D_qk), True, False, chunks=zigzag_chunks(T, n_chunks))


RECIPES = {
    "tiny_decode_fp32": tiny_decode_fp32,
    "decode_bf16": decode_bf16,
    "prefill_bf16": prefill_bf16,
    "decode_fp8": decode_fp8,
    "decode_draft_bf16": decode_draft_bf16,
    "decode_mxfp8": decode_mxfp8,
    "prefill_long_zigzag": prefill_long_zigzag,
}


def make(name: str, device="cpu", **overrides) -> Workload:
    return RECIPES[name](device=device, **overrides)


def random_scores(T_q: int, ld: int, seed: int, device="cpu", ties: bool = False) -> torch.Tensor:
    """fp32 score rows for exercising Top-K on its own.  With ties=True values are drawn from a
    small integer set (with +-0.0 both present) so equal keys are common."""
    g = _gen(device, seed, 11)
    if ties:
        x = torch.randint(-3, 4, (T_q, ld), generator=g, device=device).to(torch.float32)
        neg0 = torch.randint(0, 2, (T_q, ld), generator=g, device=device).bool() & (x == 0)
        x[neg0] = -0.0
        return x
    return torch.randn((T_q, ld), generator=g, device=device, dtype=torch.float32)


def random_selection(pos: torch.Tensor, K: int, seed: int) -> torch.Tensor:
    """int32 [T_q, K]: for row t, min(pos_t+1, K) distinct positions in [0, pos_t], ascending,
    padded with -1 -- a valid Top-K output that does not depend on any scores."""
    g = _gen("cpu", seed, 12)
    pos = pos.to("cpu")
    out = torch.full((pos.shape[0], K), -1, dtype=torch.int32)
    for t, p in enumerate(pos.tolist()):
        n = p + 1
        if n <= K:
            out[t, :n] = torch.arange(n, dtype=torch.int32)
        else:
            sel = torch.randperm(n, generator=g)[:K].sort().values
            out[t] = sel.to(torch.int32)
    return out


def sample_rows(T_q: int, every: int, chunks: Optional[List[Tuple[int, int]]] = None,
                extra: Tuple[int, ...] = ()) -> List[int]:
    """Stratified query-row sample: every `every`-th row, the first and last row of each chunk,
    and the `extra` rows (e.g. the Top-K boundary 2046..2049)."""
    rows = set(range(0, T_q, every))
    rows.add(T_q - 1)
    for a, b in chunks or []:
        rows.update((a, b - 1))
    rows.update(r for r in extra if 0 <= r < T_q)
    return sorted(rows)
