"""Sparse index attention on B200: indexer score -> Top-K -> sparse MLA over a paged latent cache.

Thin Python binding of ``libhsa.so`` (C ABI in ``include/hsa.h``).  Every function here only
marshals torch tensors into pointers and sizes and calls the C entry point of the same name; all
computation happens in the library's CUDA kernels.  Output tensors that the caller does not pass
are allocated with torch on the input's device (PyTorch provides device memory and streams).

The library is loaded on first use; if ``libhsa.so`` has not been built the call raises
``RuntimeError`` -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhsa.so")

HSA_OK, HSA_ERR_INVALID_ARG, HSA_ERR_UNSUPPORTED, HSA_ERR_CUDA, HSA_ERR_WORKSPACE = 0, 1, 2, 3, 4
HSA_F32, HSA_BF16, HSA_E4M3, HSA_MXE4M3 = 0, 1, 2, 3
HSA_DEV_BAD_PAGE, HSA_DEV_BAD_POS, HSA_DEV_BAD_GROUP, HSA_DEV_TIMEOUT = 1, 2, 4, 8

_P = ctypes.c_void_p
_i32, _i64, _sz, _f32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float


class hsa_paged_seq_t(ctypes.Structure):
    _fields_ = [("B", _i32), ("seq_lens", _P), ("block_table", _P), ("bt_stride", _i64),
                ("page_size", _i32), ("num_pages", _i32), ("max_seq_len", _i32), ("T_q", _i32),
                ("q_seq", _P), ("q_pos", _P), ("q_run", _i32), ("status", _P)]


class hsa_index_args_t(ctypes.Structure):
    _fields_ = [("q_I", _P), ("q_dtype", ctypes.c_int), ("w", _P), ("H_I", _i32), ("D_I", _i32),
                ("k_cache", _P), ("k_dtype", ctypes.c_int), ("k_scale", _P), ("q_scale", _P)]


class hsa_attn_args_t(ctypes.Structure):
    _fields_ = [("q", _P), ("q_dtype", ctypes.c_int), ("H", _i32), ("D_qk", _i32), ("D_v", _i32),
                ("kv", _P), ("kv_dtype", ctypes.c_int), ("kv_scale", _P), ("kv_scale_group", _i32),
                ("kv_rope", _P),
                ("softmax_scale", _f32), ("out", _P), ("out_dtype", ctypes.c_int), ("lse", _P)]


class hsa_prolog_args_t(ctypes.Structure):
    _fields_ = [("n_new", _i64), ("slot_mapping", _P), ("num_slots", _i64),
                ("new_k", _P), ("new_k_dtype", ctypes.c_int), ("D_I", _i32),
                ("k_cache", _P), ("k_scale", _P), ("k_dtype", ctypes.c_int),
                ("new_kv", _P), ("new_kv_dtype", ctypes.c_int), ("D_v", _i32), ("D_rope", _i32),
                ("kv_group", _i32), ("kv_cache", _P), ("kv_scale", _P), ("kv_rope", _P),
                ("q_I", _P), ("q_I_dtype", ctypes.c_int), ("q_rows", _i64), ("q_I_out", _P),
                ("q_codes_out", _P), ("q_scale_out", _P)]


SYMBOLS = {
    "hsa_index_score": (ctypes.c_int, [_P, _P, ctypes.c_int, _P, _i32, _i32, _P, ctypes.c_int, _P,
                                       _P, _i64, _P]),
    "hsa_index_score_mx": (ctypes.c_int, [_P, _P, _P, _P, _i32, _i32, _P, _P, _P, _i64, _P]),
    "hsa_topk": (ctypes.c_int, [_P, _P, _i64, _i32, _P, _P]),
    "hsa_topk_blocks": (ctypes.c_int, [_P, _P, _i64, _i32, _i32, _P, _P]),
    "hsa_sparse_mla_workspace_size": (_sz, [_P, _i32, _i32, _i32, _i32]),
    "hsa_sparse_mla_attn": (ctypes.c_int, [_P, _P, ctypes.c_int, _i32, _i32, _i32, _P, ctypes.c_int,
                                           _P, _i32, _P, _P, _i32, _f32, _P, ctypes.c_int, _P, _P, _sz,
                                           _P]),
    "hsa_fused_decode_workspace_size": (_sz, [_P, _P, _i32]),
    "hsa_fused_decode": (ctypes.c_int, [_P, _P, _P, _i32, _P, _i64, _P, _P, _sz, _P, _P]),
    "hsa_fused_decode_noalloc": (ctypes.c_int, [_P, _P, _P, _i32, _P]),
    "hsa_prefill_chunked": (ctypes.c_int, [_P, _P, _P, _i32, _P, _i32, _P, _i32, _i64, _P, _P, _P, _P]),
    "hsa_quantize_index": (ctypes.c_int, [_P, ctypes.c_int, _i64, _i32, _i32, _P, _i64, _P, _P, _P]),
    "hsa_quantize_kv": (ctypes.c_int, [_P, ctypes.c_int, _i64, _i32, _i32, _i32, _P, _i64, _P, _P,
                                       _P, _P]),
    "hsa_quantize_mx": (ctypes.c_int, [_P, ctypes.c_int, _i64, _i32, _P, _i64, _P, _P, _P]),
    "hsa_dequantize_mx": (ctypes.c_int, [_P, _P, _i64, _i32, _P, ctypes.c_int, _P]),
    "hsa_mx_round": (ctypes.c_int, [_P, ctypes.c_int, _i64, _i32, _P, ctypes.c_int, _P]),
    "hsa_decode_prolog": (ctypes.c_int, [_P, _P, _P, _P, _P]),
    "hsa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "hsa_last_error_message": (ctypes.c_char_p, []),
    "hsa_version": (_i32, []),
    "hsa_launch_count": (ctypes.c_uint64, []),
}

_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """Load libhsa.so (raises RuntimeError if it was not built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with `python -m sparse_index_attention_b200.build`"
                    " (the CUDA library is required; there is no fallback)")
            L = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SYMBOLS.items():
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            _lib = L
    return _lib


class HsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        L = lib()
        msg = L.hsa_last_error_message().decode()
        super().__init__(f"{where}: {L.hsa_status_string(status).decode()}: {msg}")
        self.status = status


def _check(rc: int, where: str):
    if rc != HSA_OK:
        raise HsaError(rc, where)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return HSA_F32
    if t.dtype == torch.bfloat16:
        return HSA_BF16
    if t.dtype in (torch.uint8, getattr(torch, "float8_e4m3fn", torch.uint8)):
        return HSA_E4M3
    raise TypeError(f"unsupported dtype {t.dtype}")


def _key_dtype(k_cache: torch.Tensor, k_scale: Optional[torch.Tensor]) -> int:
    """Index keys: 8-bit codes with uint8 (E8M0) scales are MXFP8, with fp32 scales E4M3."""
    d = _dtype(k_cache)
    if d == HSA_E4M3 and k_scale is not None and k_scale.dtype == torch.uint8:
        return HSA_MXE4M3
    return d


def _stream(s) -> ctypes.c_void_p:
    if s is None:
        s = torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


class PagedSeq:
    """Paged sequences + query rows (hsa_paged_seq_t).  Keeps its tensors alive."""

    def __init__(self, seq_lens, block_table, page_size: int, num_pages: int, q_seq, q_pos,
                 max_seq_len: Optional[int] = None, q_run: int = 1, status=None):
        self.seq_lens = seq_lens.to(torch.int32).contiguous()
        self.block_table = block_table.to(torch.int32).contiguous()
        self.q_seq = q_seq.to(torch.int32).contiguous()
        self.q_pos = q_pos.to(torch.int32).contiguous()
        self.status = status
        self.page_size, self.num_pages, self.q_run = int(page_size), int(num_pages), int(q_run)
        self.max_seq_len = int(max_seq_len if max_seq_len is not None else self.seq_lens.max().item())
        self.T_q = int(self.q_seq.shape[0])
        self.B = int(self.seq_lens.shape[0])
        self.c = hsa_paged_seq_t(self.B, _ptr(self.seq_lens), _ptr(self.block_table),
                                 int(self.block_table.shape[1]), self.page_size, self.num_pages,
                                 self.max_seq_len, self.T_q, _ptr(self.q_seq), _ptr(self.q_pos),
                                 self.q_run, _ptr(status))

    def rows(self, r0: int, r1: int, q_run: Optional[int] = None) -> "PagedSeq":
        """Descriptor of query rows [r0, r1) (same sequences and caches)."""
        return PagedSeq(self.seq_lens, self.block_table, self.page_size, self.num_pages,
                        self.q_seq[r0:r1], self.q_pos[r0:r1], self.max_seq_len,
                        q_run if q_run is not None else self.q_run, self.status)

    @property
    def ref(self):
        return ctypes.byref(self.c)


# ------------------------------------------------------------------------------ entry points
def hsa_index_score(seq: PagedSeq, q_I, w, k_cache, k_scale=None, scores=None, ld: Optional[int] = None,
                    stream=None, q_scale=None):
    """Index scores [T_q, ld].  With q_scale (uint8 E8M0 [T_q, H_I, D_I / 32]) q_I holds MXFP8
    codes and the keys must be MXFP8 too: hsa_index_score_mx, the block-scaled path."""
    T_q, H_I, D_I = q_I.shape
    if scores is None:
        ld = ld or seq.max_seq_len
        scores = torch.empty((T_q, ld), dtype=torch.float32, device=q_I.device)
    ld = scores.shape[1]
    if q_scale is not None:
        _check(lib().hsa_index_score_mx(seq.ref, _ptr(q_I), _ptr(q_scale), _ptr(w), H_I, D_I,
                                        _ptr(k_cache), _ptr(k_scale), _ptr(scores), ld, _stream(stream)),
               "hsa_index_score_mx")
        return scores
    _check(lib().hsa_index_score(seq.ref, _ptr(q_I), _dtype(q_I), _ptr(w), H_I, D_I, _ptr(k_cache),
                                 _key_dtype(k_cache, k_scale), _ptr(k_scale), _ptr(scores), ld,
                                 _stream(stream)),
           "hsa_index_score")
    return scores


def hsa_topk(seq: PagedSeq, scores, K: int, idx=None, stream=None):
    if idx is None:
        idx = torch.empty((seq.T_q, K), dtype=torch.int32, device=scores.device)
    _check(lib().hsa_topk(seq.ref, _ptr(scores), scores.shape[1], K, _ptr(idx), _stream(stream)),
           "hsa_topk")
    return idx


def hsa_topk_blocks(seq: PagedSeq, scores, K: int, block: int, idx=None, stream=None):
    """Block-aligned selection: the K / block blocks of `block` positions with the highest block
    maximum, all their causal positions ascending, -1 padded (rows with n <= K select all)."""
    if idx is None:
        idx = torch.empty((seq.T_q, K), dtype=torch.int32, device=scores.device)
    _check(lib().hsa_topk_blocks(seq.ref, _ptr(scores), scores.shape[1], K, block, _ptr(idx),
                                 _stream(stream)),
           "hsa_topk_blocks")
    return idx


def hsa_sparse_mla_workspace_size(seq: PagedSeq, H: int, D_qk: int, D_v: int, K: int) -> int:
    return int(lib().hsa_sparse_mla_workspace_size(seq.ref, H, D_qk, D_v, K))


def _workspace(nbytes: int, device, ws):
    """Workspace of nbytes (at least one byte; the current attention kernels report 0 and use
    none), zero-filled, or the caller's own `ws`."""
    if ws is not None:
        return ws
    return torch.zeros(max(nbytes, 1), dtype=torch.uint8, device=device)


def _kv_group(kv, kv_scale, D_v: int) -> int:
    """Latent dims per KV scale: an FP8 cache's kv_scale holds D_v / group scales per slot."""
    if kv_scale is None or kv.dtype != torch.uint8:
        return D_v
    per_slot = kv_scale.numel() // kv.shape[0]
    if per_slot < 1 or kv_scale.numel() != per_slot * kv.shape[0] or D_v % per_slot:
        raise ValueError(f"kv_scale with {kv_scale.numel()} entries does not fit {kv.shape[0]} slots")
    return D_v // per_slot


def hsa_sparse_mla_attn(seq: PagedSeq, q, kv, idx, D_v: int, softmax_scale: float, kv_scale=None,
                        kv_rope=None, out=None, out_dtype=None, lse=True, ws=None, stream=None):
    """Returns (out [T_q, H, D_v], lse [T_q, H] or None).  kv is the packed [slots, D_qk] cache
    (fp32/bf16) or the uint8 latent codes [slots, D_v] with kv_scale ([slots] or
    [slots, D_v / group]: one scale per token or per group of latent dims) and kv_rope."""
    T_q, H, D_qk = q.shape
    K = idx.shape[1]
    if out is None:
        out = torch.empty((T_q, H, D_v), dtype=out_dtype or q.dtype, device=q.device)
    if lse is True:
        lse = torch.empty((T_q, H), dtype=torch.float32, device=q.device)
    elif lse is False:
        lse = None
    need = hsa_sparse_mla_workspace_size(seq, H, D_qk, D_v, K)
    ws = _workspace(need, q.device, ws)
    _check(lib().hsa_sparse_mla_attn(seq.ref, _ptr(q), _dtype(q), H, D_qk, D_v, _ptr(kv), _dtype(kv),
                                     _ptr(kv_scale), _kv_group(kv, kv_scale, D_v), _ptr(kv_rope),
                                     _ptr(idx), K,
                                     float(softmax_scale), _ptr(out), _dtype(out), _ptr(lse),
                                     _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "hsa_sparse_mla_attn")
    return out, lse


def _attn_struct(q, kv, D_v, softmax_scale, kv_scale, kv_rope, out, lse):
    T_q, H, D_qk = q.shape
    return hsa_attn_args_t(_ptr(q), _dtype(q), H, D_qk, D_v, _ptr(kv), _dtype(kv), _ptr(kv_scale),
                           _kv_group(kv, kv_scale, D_v), _ptr(kv_rope), float(softmax_scale), _ptr(out),
                           _dtype(out), _ptr(lse))


def hsa_fused_decode_workspace_size(seq: PagedSeq, q, kv, D_v: int, K: int) -> int:
    T_q, H, D_qk = q.shape
    at = hsa_attn_args_t(None, _dtype(q), H, D_qk, D_v, None, _dtype(kv), None, D_v, None, 1.0, None,
                         _dtype(q), None)
    return int(lib().hsa_fused_decode_workspace_size(seq.ref, ctypes.byref(at), K))


def hsa_fused_decode(seq: PagedSeq, q_I, w, k_cache, k_scale, q, kv, kv_scale, kv_rope, K: int,
                     D_v: int, softmax_scale: float, scores=None, idx=None, out=None, lse=True,
                     ws=None, stream=None, aux_stream=None, q_I_scale=None):
    """index score -> Top-K -> sparse MLA in one call.  Returns (out, lse, idx, scores).  With
    q_I_scale, q_I holds MXFP8 codes (keys MXFP8 too), as in hsa_index_score_mx."""
    T_q, H_I, D_I = q_I.shape
    _, H, D_qk = q.shape
    dev = q.device
    if scores is None:
        scores = torch.empty((T_q, seq.max_seq_len), dtype=torch.float32, device=dev)
    if idx is None:
        idx = torch.empty((T_q, K), dtype=torch.int32, device=dev)
    if out is None:
        out = torch.empty((T_q, H, D_v), dtype=q.dtype, device=dev)
    if lse is True:
        lse = torch.empty((T_q, H), dtype=torch.float32, device=dev)
    elif lse is False:
        lse = None
    ws = _workspace(hsa_fused_decode_workspace_size(seq, q, kv, D_v, K), dev, ws)
    ia = hsa_index_args_t(_ptr(q_I), HSA_MXE4M3 if q_I_scale is not None else _dtype(q_I), _ptr(w),
                          H_I, D_I, _ptr(k_cache), _key_dtype(k_cache, k_scale), _ptr(k_scale),
                          _ptr(q_I_scale))
    at = _attn_struct(q, kv, D_v, softmax_scale, kv_scale, kv_rope, out, lse)
    _check(lib().hsa_fused_decode(seq.ref, ctypes.byref(ia), ctypes.byref(at), K, _ptr(scores),
                                  scores.shape[1], _ptr(idx), _ptr(ws), ws.numel(), _stream(stream),
                                  None if aux_stream is None else ctypes.c_void_p(aux_stream.cuda_stream)),
           "hsa_fused_decode")
    return out, lse, idx, scores

def hsa_fused_decode_noalloc(seq: PagedSeq, q_I, w, k_cache, k_scale, q, kv, kv_scale, kv_rope, K: int,
                             D_v: int, softmax_scale: float, out, lse=None, stream=None, q_I_scale=None):
    """The fused decode step with its scores and selections in the library's own scratch
    (hsa_fused_decode_noalloc: for callers that may not allocate device memory).  ``out``
    [T_q, H, D_v] and ``lse`` [T_q, H] fp32 (or None) are the caller's; returns (out, lse)."""
    T_q, H_I, D_I = q_I.shape
    ia = hsa_index_args_t(_ptr(q_I), HSA_MXE4M3 if q_I_scale is not None else _dtype(q_I), _ptr(w),
                          H_I, D_I, _ptr(k_cache), _key_dtype(k_cache, k_scale), _ptr(k_scale),
                          _ptr(q_I_scale))
    at = _attn_struct(q, kv, D_v, softmax_scale, kv_scale, kv_rope, out, lse)
    _check(lib().hsa_fused_decode_noalloc(seq.ref, ctypes.byref(ia), ctypes.byref(at), K,
                                          _stream(stream)),
           "hsa_fused_decode_noalloc")
    return out, lse


class DecodeGraph:
    """One hsa_fused_decode step captured as a CUDA graph (the decode step in "graph mode"):
    replay() reruns the same kernels on the same buffers with a single graph launch and no
    per-step host work in the library.  The graph reads the tensors given here: write the next
    step's query rows into q_I, w and q (and the caches) before replay(); results land in
    .out, .lse, .idx and .scores.  With aux=True the step uses the two-stream form."""

    def __init__(self, seq: PagedSeq, q_I, w, k_cache, k_scale, q, kv, kv_scale, kv_rope, K: int,
                 D_v: int, softmax_scale: float, aux: bool = False):
        dev = q.device
        T_q, H, _ = q.shape
        self.scores = torch.empty((T_q, seq.max_seq_len), dtype=torch.float32, device=dev)
        self.idx = torch.empty((T_q, K), dtype=torch.int32, device=dev)
        self.out = torch.empty((T_q, H, D_v), dtype=q.dtype, device=dev)
        self.lse = torch.empty((T_q, H), dtype=torch.float32, device=dev)
        self.ws = _workspace(hsa_fused_decode_workspace_size(seq, q, kv, D_v, K), dev, None)
        self._aux = torch.cuda.Stream(device=dev) if aux else None
        args = (seq, q_I, w, k_cache, k_scale, q, kv, kv_scale, kv_rope, K, D_v, softmax_scale)
        cap = torch.cuda.Stream(device=dev)

        def step(stream):
            hsa_fused_decode(*args, scores=self.scores, idx=self.idx, out=self.out, lse=self.lse,
                             ws=self.ws, stream=stream, aux_stream=self._aux)
        cap.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(cap):
            step(cap)                       # first call outside the capture (kernel attributes)
        cap.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=cap, capture_error_mode="relaxed"):
            step(cap)
        self._args = args                   # keep every captured tensor alive

    def replay(self):
        self.graph.replay()
        return self.out, self.lse, self.idx, self.scores


def hsa_quantize_index(src, group: int, slot_mapping=None, num_slots: Optional[int] = None,
                       codes=None, scales=None, stream=None):
    """Rows [n, D] -> (codes uint8 [slots, D], scales fp32 [slots, D/group])."""
    n, D = src.shape
    num_slots = num_slots if num_slots is not None else n
    if codes is None:
        codes = torch.zeros((num_slots, D), dtype=torch.uint8, device=src.device)
    if scales is None:
        scales = torch.zeros((num_slots, D // group), dtype=torch.float32, device=src.device)
    _check(lib().hsa_quantize_index(_ptr(src), _dtype(src), n, D, group, _ptr(slot_mapping),
                                    num_slots, _ptr(codes), _ptr(scales), _stream(stream)),
           "hsa_quantize_index")
    return codes, scales


def hsa_quantize_kv(src, D_v: int, group: int, slot_mapping=None, num_slots: Optional[int] = None,
                    codes=None, scales=None, rope_cache=None, stream=None):
    """Rows [n, D_v + D_rope] (latent || rope) -> (codes [slots, D_v], scales [slots, D_v/group],
    rope bf16 [slots, D_rope])."""
    n, D = src.shape
    D_rope = D - D_v
    num_slots = num_slots if num_slots is not None else n
    dev = src.device
    if codes is None:
        codes = torch.zeros((num_slots, D_v), dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.zeros((num_slots, D_v // group), dtype=torch.float32, device=dev)
    if rope_cache is None:
        rope_cache = torch.zeros((num_slots, max(D_rope, 0)), dtype=torch.bfloat16, device=dev)
    _check(lib().hsa_quantize_kv(_ptr(src), _dtype(src), n, D_v, D_rope, group, _ptr(slot_mapping),
                                 num_slots, _ptr(codes), _ptr(scales), _ptr(rope_cache),
                                 _stream(stream)),
           "hsa_quantize_kv")
    return codes, scales, rope_cache


def hsa_quantize_mx(src, slot_mapping=None, num_slots: Optional[int] = None, codes=None,
                    scales=None, stream=None):
    """MXFP8: rows [n, D] (D a multiple of 32) -> (E4M3 codes uint8 [slots, D], E8M0 scale bytes
    uint8 [slots, D/32]).  With D = 128 the pair is an MXFP8 index key cache for
    ``hsa_index_score``."""
    n, D = src.shape
    num_slots = num_slots if num_slots is not None else n
    if codes is None:
        codes = torch.zeros((num_slots, D), dtype=torch.uint8, device=src.device)
    if scales is None:
        scales = torch.zeros((num_slots, D // 32), dtype=torch.uint8, device=src.device)
    _check(lib().hsa_quantize_mx(_ptr(src), _dtype(src), n, D, _ptr(slot_mapping), num_slots,
                                 _ptr(codes), _ptr(scales), _stream(stream)),
           "hsa_quantize_mx")
    return codes, scales


def hsa_dequantize_mx(codes, scales, dtype=torch.bfloat16, out=None, stream=None):
    """MXFP8 codes [n, D] + E8M0 bytes [n, D/32] -> values [n, D] (code * 2^(E - 127))."""
    n, D = codes.shape
    if out is None:
        out = torch.empty((n, D), dtype=dtype, device=codes.device)
    _check(lib().hsa_dequantize_mx(_ptr(codes), _ptr(scales), n, D, _ptr(out), _dtype(out),
                                   _stream(stream)),
           "hsa_dequantize_mx")
    return out


def mx_round(x, out=None, stream=None):
    """Index queries [..., D] rounded onto the MXFP8 grid and returned as bf16 (hsa_mx_round: the
    quantize-then-dequantize result of the MX rule in one kernel).  The bf16-query index kernels
    then score MXFP8 queries."""
    flat = x.reshape(-1, x.shape[-1])
    if out is None:
        out = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device)
    _check(lib().hsa_mx_round(_ptr(flat), _dtype(flat), flat.shape[0], flat.shape[1], _ptr(out),
                              _dtype(out), _stream(stream)),
           "hsa_mx_round")
    return out


def _cache_rows(t, name: str, width: int, dtype) -> int:
    """Slots of a flat paged cache tensor [slots, width] (a paged [P, page, width] view is
    accepted and flattened): a mismatch is an error, not a silently dropped row."""
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if width == 1 and t.dim() == 1:
        return t.numel()
    if t.dim() < 1 or t.shape[-1] != width or t.numel() % width:
        raise ValueError(f"{name}: shape {tuple(t.shape)} is not [slots, {width}]")
    return t.numel() // width


def hsa_decode_prolog(new_k, new_kv, slot_mapping, k_cache, k_scale, kv_cache, kv_scale, kv_rope,
                      q_I, q_I_out, D_v: int, kv_group: Optional[int] = None, streams=None,
                      stream=None, q_codes_out=None, q_scale_out=None):
    """The writes that precede a decode step, on three streams (hsa_decode_prolog): the new
    tokens' index keys into the index key cache, their latent rows into the FP8 latent cache,
    and the index queries rounded onto the MXFP8 grid into ``q_I_out`` ("Day 0 Inference
    Adaptation and Optimization for Hybrid Attention Models", "Sparse Attention Pipeline
    Optimization": independent prolog operators on concurrent streams; "Inference Adaptation and
    Performance Optimization for a Domestically Developed LLM's New Architecture", 3.3).
    ``stream`` (default: current) waits for all three, so a decode step issued on it next sees
    the new rows.

    new_k [n, D_I] and new_kv [n, D_v + D_rope] (F32/BF16) go to physical slots
    ``slot_mapping`` [n] (int64).  The index key cache is MXFP8 when ``k_scale`` is uint8
    (E8M0 bytes, [slots, D_I/32]) and E4M3 with one fp32 scale per key otherwise.  The latent
    cache is E4M3 with one fp32 scale per ``kv_group`` dims (default D_v) plus bf16 rope.
    With ``q_codes_out`` (uint8, q_I's size) and ``q_scale_out`` (uint8 [rows, D_I/32]) the
    queries are also quantized to MXFP8 codes and scales for the block-scaled index path.
    Results equal the same calls issued one after another on one stream."""
    n, D_I = new_k.shape
    D_rope = new_kv.shape[1] - D_v
    grp = kv_group or D_v
    mx = k_scale.dtype == torch.uint8
    slots = _cache_rows(k_cache, "k_cache", D_I, torch.uint8)
    if _cache_rows(k_scale, "k_scale", D_I // 32 if mx else 1, torch.uint8 if mx else torch.float32) != slots:
        raise ValueError("k_scale does not cover the key cache's slots")
    if _cache_rows(kv_cache, "kv_cache", D_v, torch.uint8) != slots or \
            _cache_rows(kv_scale, "kv_scale", D_v // grp, torch.float32) != slots or \
            _cache_rows(kv_rope, "kv_rope", D_rope, torch.bfloat16) != slots:
        raise ValueError("the latent cache tensors do not cover the key cache's slots")
    if slot_mapping.dtype != torch.int64 or slot_mapping.numel() != n:
        raise ValueError("slot_mapping must be int64 [n]")
    if q_I_out is not None and (q_I_out.dtype != torch.bfloat16 or q_I_out.numel() != q_I.numel()):
        raise ValueError("q_I_out must be bf16 with q_I's size")
    if q_codes_out is not None and (
            q_codes_out.dtype != torch.uint8 or q_codes_out.numel() != q_I.numel() or
            q_scale_out is None or q_scale_out.dtype != torch.uint8 or
            q_scale_out.numel() != q_I.numel() // 32):
        raise ValueError("q_codes_out / q_scale_out must be uint8 codes and E8M0 scales of q_I")
    if streams is None:
        streams = (torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream())
    flat_q = q_I.reshape(-1, D_I)
    a = hsa_prolog_args_t(n, _ptr(slot_mapping), slots, _ptr(new_k), _dtype(new_k), D_I,
                          _ptr(k_cache), _ptr(k_scale), HSA_MXE4M3 if mx else HSA_E4M3,
                          _ptr(new_kv), _dtype(new_kv), D_v, D_rope, grp, _ptr(kv_cache),
                          _ptr(kv_scale), _ptr(kv_rope), _ptr(flat_q), _dtype(flat_q),
                          flat_q.shape[0], _ptr(q_I_out), _ptr(q_codes_out), _ptr(q_scale_out))
    _check(lib().hsa_decode_prolog(ctypes.byref(a), _stream(stream), _stream(streams[0]),
                                   _stream(streams[1]), _stream(streams[2])),
           "hsa_decode_prolog")
    return q_I_out


def hsa_version() -> int:
    return int(lib().hsa_version())


def hsa_launch_count() -> int:
    """Kernels launched by the library from this host thread so far."""
    return int(lib().hsa_launch_count())


def prefill_score_buffers(seq: PagedSeq, chunks, device, n: int = 2):
    """Caller-owned fp32 score buffers for hsa_prefill_chunked: one [max chunk rows, max_seq_len]
    buffer per stream, allocated once and reused by every call."""
    rows_max = max(r1 - r0 for r0, r1 in chunks)
    return tuple(torch.empty((rows_max, seq.max_seq_len), dtype=torch.float32, device=device)
                 for _ in range(n))


def hsa_prefill_chunked(seq: PagedSeq, q_I, w, k_cache, k_scale, q, kv, kv_scale, kv_rope, K: int,
                        D_v: int, softmax_scale: float, chunks, out=None, lse=True, idx=None,
                        streams=None, score_bufs=None):
    """Causal prefill over query-row windows issued in the order of `chunks` [(r0, r1), ...].

    Consecutive chunks form pairs that run concurrently, one on each of two streams; with the
    zigzag order (chunk i paired with chunk 2N-1-i, "Efficient Inference Deployment and
    Optimization for Hybrid Attention LLMs", 5.2) every pair carries the same causal index work.
    Each chunk is hsa_index_score -> hsa_topk -> hsa_sparse_mla_attn on its rows, so its outputs
    land at the rows' own offsets and no restore step exists; the issue order cannot change any
    result.  This function marshals its arguments into one C-ABI call (hsa_prefill_chunked,
    which issues the chunks and orders the streams).  ``score_bufs`` (one per
    stream, from prefill_score_buffers) holds the chunks' scores; when it is not given, buffers
    are allocated for this call.  Returns (out, lse, idx).
    """
    T_q = q.shape[0]
    dev = q.device
    if out is None:
        out = torch.empty((T_q, q.shape[1], D_v), dtype=q.dtype, device=dev)
    if lse is True:
        lse = torch.empty((T_q, q.shape[1]), dtype=torch.float32, device=dev)
    elif lse is False:
        lse = None
    if idx is None:
        idx = torch.empty((T_q, K), dtype=torch.int32, device=dev)
    main = torch.cuda.current_stream()
    if streams is None:
        streams = (torch.cuda.Stream(), torch.cuda.Stream())
    own = score_bufs is None
    bufs = list(prefill_score_buffers(seq, chunks, dev, 2) if own else score_bufs)
    rows_max = max(r1 - r0 for r0, r1 in chunks)
    if len(bufs) < 2 or bufs[0].shape != bufs[1].shape or bufs[0].shape[0] < rows_max or \
            bufs[0].shape[1] < seq.max_seq_len or \
            not all(b.is_contiguous() and b.dtype == torch.float32 for b in bufs[:2]):
        raise ValueError("two contiguous fp32 score buffers of at least [max chunk rows, max_seq_len]")
    if len(streams) != 2:
        raise ValueError("streams must be a pair (the chunks alternate between them)")
    T_qI, H_I, D_I = q_I.shape
    ia = hsa_index_args_t(_ptr(q_I), _dtype(q_I), _ptr(w), H_I, D_I, _ptr(k_cache),
                          _key_dtype(k_cache, k_scale), _ptr(k_scale), None)
    at = _attn_struct(q, kv, D_v, softmax_scale, kv_scale, kv_rope, out, lse)
    flat = [x for rr in chunks for x in rr]
    arr = (ctypes.c_int32 * len(flat))(*flat)
    bp = (ctypes.c_void_p * 2)(bufs[0].data_ptr(), bufs[1].data_ptr())
    _check(lib().hsa_prefill_chunked(seq.ref, ctypes.byref(ia), ctypes.byref(at), K, arr, len(chunks),
                                     bp, bufs[0].shape[0], bufs[0].shape[1], _ptr(idx),
                                     _stream(main), _stream(streams[0]), _stream(streams[1])),
           "hsa_prefill_chunked")
    if own:
        for b, s in zip(bufs, streams):
            b.record_stream(s)
    return out, lse, idx
