"""The seeded input recipe (CPU): the seed formula, the layout invariants every kernel and the
oracle rely on (valid pages, positions inside their sequence, runs of rows of one sequence),
and determinism.  Sizes are reduced; the recipe is the same at full size."""
import math

import pytest
import torch

from sparse_index_attention_b200 import workloads

SMALL = {
    "tiny_decode_fp32": {},
    "decode_bf16": dict(B=5, L_min=100, L_max=700),
    "prefill_bf16": dict(T=300),
    "decode_fp8": dict(B=3, L=500),
    "prefill_long_zigzag": dict(T=512, n_chunks=4),
    "decode_mxfp8": dict(B=3, L=500),
    "decode_draft_bf16": dict(B=4, L_min=100, L_max=700),
}


def test_every_recipe_is_listed():
    assert set(SMALL) == set(workloads.RECIPES)


@pytest.mark.parametrize("name", sorted(SMALL))
def test_layout_invariants(name):
    wl = workloads.make(name, **SMALL[name])
    # every logical page of every sequence maps to a distinct physical page
    used = []
    for b in range(wl.B):
        n = math.ceil(int(wl.seq_lens[b]) / wl.page_size)
        used += wl.block_table[b, :n].tolist()
    assert sorted(used) == list(range(wl.num_pages))
    # query rows: inside their sequence, and runs of q_run rows share one sequence
    assert wl.q_seq.shape == wl.q_pos.shape == (wl.T_q,)
    assert bool(((wl.q_pos >= 0) & (wl.q_pos < wl.seq_lens[wl.q_seq.long()])).all())
    for r0 in range(0, wl.T_q, wl.q_run):
        assert len(set(wl.q_seq[r0:r0 + wl.q_run].tolist())) == 1
    # shapes and dtypes
    dt = torch.float32 if wl.dtype == "f32" else torch.bfloat16
    assert wl.q_I.shape == (wl.T_q, wl.H_I, wl.D_I) and wl.q_I.dtype == dt
    assert wl.w.shape == (wl.T_q, wl.H_I) and wl.w.dtype == torch.float32
    assert wl.k_I.shape == (wl.num_slots, wl.D_I) and wl.k_I.dtype == dt
    assert wl.q.shape == (wl.T_q, wl.H, wl.D_qk) and wl.kv.shape == (wl.num_slots, wl.D_qk)
    assert wl.D_qk == wl.D_v + wl.D_rope
    if wl.chunks is not None:
        assert sorted(wl.chunks) == [(i * (wl.T_q // len(wl.chunks)), (i + 1) * (wl.T_q // len(wl.chunks)))
                                     for i in range(len(wl.chunks))]


@pytest.mark.parametrize("name", sorted(SMALL))
def test_deterministic(name):
    a = workloads.make(name, **SMALL[name])
    b = workloads.make(name, **SMALL[name])
    for f in ("seq_lens", "block_table", "q_seq", "q_pos", "q_I", "w", "k_I", "q", "kv"):
        assert torch.equal(getattr(a, f), getattr(b, f)), f


def test_seed_formula():
    """Tensor X of a workload with seed c comes from torch.Generator(1000 c + id(X)): fp32 randn,
    scaled, rounded to bf16."""
    wl = workloads.make("decode_bf16", B=3, L_min=100, L_max=300)
    g = torch.Generator().manual_seed(1000 * wl.seed + workloads.ID_Q_I)
    want = torch.randn(wl.q_I.shape, generator=g).to(torch.bfloat16)
    assert torch.equal(wl.q_I, want)
    g = torch.Generator().manual_seed(1000 * wl.seed + workloads.ID_W)
    assert torch.equal(wl.w, torch.randn(wl.w.shape, generator=g) * (1.0 / 8))
    g = torch.Generator().manual_seed(1000 * wl.seed + workloads.ID_LENGTHS)
    assert wl.seq_lens.tolist() == torch.randint(100, 301, (3,), generator=g).tolist()


def test_variants_share_their_base_draws():
    fp8 = workloads.make("decode_fp8", B=2, L=300)
    mx = workloads.make("decode_mxfp8", B=2, L=300)
    assert mx.index_mx and not fp8.index_mx
    for f in ("q_I", "w", "k_I", "q", "kv", "block_table"):
        assert torch.equal(getattr(fp8, f), getattr(mx, f))
    d = workloads.make("decode_draft_bf16", B=3, n_draft=4, L_min=50, L_max=90)
    assert d.q_run == 4 and d.T_q == 12
    for b in range(3):
        L = int(d.seq_lens[b])
        assert d.q_pos[4 * b:4 * b + 4].tolist() == list(range(L - 4, L))
