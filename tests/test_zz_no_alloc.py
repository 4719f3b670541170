"""The no-allocation fused decode step (hsa_fused_decode_noalloc) against the allocating one
(hsa_fused_decode) on the same inputs, through the C ABI, two calls in a row on the library's
shared scratch.  Tolerances as in the other attention tests: 2e-2 (bf16 caches) and 6e-2 (FP8
caches), per element, relative to the magnitude; lse 1e-4.  This file is collected last and
also runs alone in a fresh process."""
import pytest
import torch

import sparse_index_attention_b200 as hsa
from sparse_index_attention_b200 import workloads

from helpers import GpuCaches, paged_seq

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _both(wl, gc, seq, q):
    out_ref, lse_ref, _, _ = hsa.hsa_fused_decode(seq, gc.q_I, wl.w, gc.k, gc.k_scale, q, gc.kv,
                                                  gc.kv_scale, gc.kv_rope, wl.K, wl.D_v,
                                                  wl.softmax_scale)
    out = torch.full_like(out_ref, float("nan"))
    lse = torch.full_like(lse_ref, float("nan"))
    hsa.hsa_fused_decode_noalloc(seq, gc.q_I, wl.w, gc.k, gc.k_scale, q, gc.kv, gc.kv_scale,
                                 gc.kv_rope, wl.K, wl.D_v, wl.softmax_scale, out, lse)
    torch.cuda.synchronize()
    return out, lse, out_ref, lse_ref


def _close(out, lse, out_ref, lse_ref, tol):
    assert torch.allclose(out.float(), out_ref.float(), atol=tol, rtol=tol)
    fin = torch.isfinite(lse_ref)
    assert torch.equal(fin, torch.isfinite(lse))
    assert torch.allclose(lse[fin], lse_ref[fin], atol=1e-4, rtol=1e-4)


@pytest.mark.parametrize("name,kw,tol", [
    ("decode_bf16", dict(B=8, L_min=1500, L_max=9000), 2e-2),
    ("decode_fp8", dict(B=6, L=5000), 6e-2),
])
def test_noalloc_matches_fused_decode_twice(name, kw, tol):
    wl = workloads.make(name, DEV, **kw)
    gc = GpuCaches(wl)
    seq = paged_seq(wl)
    # first call: the step's own inputs
    _close(*_both(wl, gc, seq, wl.q), tol)
    # second call in a row on the same scratch, with other query rows: the scratch still holds
    # the first call's scores and selections, which must not leak into this result
    g = torch.Generator(device=DEV).manual_seed(123)
    q2 = torch.randn(wl.q.shape, generator=g, device=DEV).to(wl.q.dtype)
    wl.q_I = torch.randn(wl.q_I.shape, generator=g, device=DEV).to(wl.q_I.dtype)
    gc2 = GpuCaches(wl)
    _close(*_both(wl, gc2, seq, q2), tol)
