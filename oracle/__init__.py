"""Float64 CPU oracle for the sparse index attention path.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()`` and by the
benchmark's CPU-baseline leg.  The product library (``sparse_index_attention_b200``) never
imports it, and it imports nothing from the product.  The arithmetic lives in ``oracle.c``
(plain C, float64, OpenMP over query rows); this module only marshals numpy arrays.

Inputs are widened exactly: bf16/fp32 tensors become float64 arrays, FP8 E4M3 codes are
decoded by the oracle's own codec (``e4m3_decode``) and multiplied by their fp32 scale, or, for
MXFP8 blocks, by 2^(E - 127) of their shared E8M0 scale byte (``mx_dequantize_rows``).

Page citations (title, section) are in ``oracle.c`` beside each function.  The end-to-end
composition ``sparse_index_attention`` follows the pipeline of "Day 0 Inference Adaptation and
Optimization for Hybrid Attention Models", "Sparse Attention Pipeline Optimization": score every
causal history position, keep the Top-K, attend over the selected latent rows only.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

OK, BAD_ARG, NOT_FINITE, SOFTMAX_SUM = 0, 1, 2, 3


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
               "-ffp-contract=off", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
            lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
            lib.oracle_e4m3_decode.restype = f64
            lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
            lib.oracle_e4m3_encode.restype = ctypes.c_uint8
            lib.oracle_quantize_rows.argtypes = [P, i64, i32, i32, P, P]
            lib.oracle_dequantize_rows.argtypes = [P, P, i64, i32, i32, P]
            lib.oracle_mx_quantize_rows.argtypes = [P, i64, i32, P, P]
            lib.oracle_mx_dequantize_rows.argtypes = [P, P, i64, i32, P]
            paging = [i32, P, P, i64, i32, i32, i32, P, P]
            lib.oracle_index_score.argtypes = paging + [i32, i32, P, P, P, P, i64]
            lib.oracle_topk.argtypes = [i32, P, P, i64, i32, P]
            lib.oracle_topk_blocks.argtypes = [i32, P, P, i64, i32, i32, P]
            lib.oracle_sparse_mla.argtypes = paging + [i32, i32, i32, P, P, P, i32, f64, P, P]
            lib.oracle_dense_attn.argtypes = paging + [i32, i32, i32, P, P, f64, P, P]
            for f in ("oracle_quantize_rows", "oracle_dequantize_rows", "oracle_mx_quantize_rows",
                      "oracle_mx_dequantize_rows", "oracle_index_score",
                      "oracle_topk", "oracle_topk_blocks", "oracle_sparse_mla", "oracle_dense_attn"):
                getattr(lib, f).restype = ctypes.c_int
            lib.oracle_num_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f64(x) -> np.ndarray:
    """Exact widening of a torch tensor (fp32 / bf16 / f16) or array to a contiguous float64."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu")
            if x.dtype in (torch.bfloat16, torch.float16):
                x = x.float()          # exact
            return np.ascontiguousarray(x.numpy().astype(np.float64))
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i32(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu").numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _check(rc: int, what: str):
    if rc != OK:
        raise OracleError(f"{what}: oracle status {rc}")


def num_threads() -> int:
    return int(_load().oracle_num_threads())


# ----------------------------------------------------------------------------- FP8 E4M3 codec
def e4m3_decode(codes) -> np.ndarray:
    lib = _load()
    c = np.asarray(codes, dtype=np.uint8)
    return np.vectorize(lambda v: lib.oracle_e4m3_decode(int(v)), otypes=[np.float64])(c)


def e4m3_encode(x) -> np.ndarray:
    lib = _load()
    a = np.asarray(x, dtype=np.float32)
    return np.vectorize(lambda v: lib.oracle_e4m3_encode(float(v)), otypes=[np.uint8])(a)


def quantize_rows(x, group: int):
    """Rows [n, D] (fp32-representable) -> (codes uint8 [n, D], scales fp32 [n, D/group])."""
    xf = np.ascontiguousarray(_f64(x).astype(np.float32))
    n, D = xf.shape
    codes = np.zeros((n, D), dtype=np.uint8)
    scales = np.zeros((n, D // group), dtype=np.float32)
    _check(_load().oracle_quantize_rows(_ptr(xf), n, D, group, _ptr(codes), _ptr(scales)),
           "quantize_rows")
    return codes, scales


def dequantize_rows(codes, scales, group: int) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(codes, dtype=np.uint8))
    s = np.ascontiguousarray(np.asarray(scales, dtype=np.float32))
    n, D = c.shape
    out = np.zeros((n, D), dtype=np.float64)
    _check(_load().oracle_dequantize_rows(_ptr(c), _ptr(s), n, D, group, _ptr(out)),
           "dequantize_rows")
    return out


def mx_quantize_rows(x):
    """MXFP8: rows [n, D] (fp32-representable, D a multiple of 32) -> (E4M3 codes uint8 [n, D],
    E8M0 scale bytes uint8 [n, D/32]); the rule is in ``oracle.c``."""
    xf = np.ascontiguousarray(_f64(x).astype(np.float32))
    n, D = xf.shape
    codes = np.zeros((n, D), dtype=np.uint8)
    scales = np.zeros((n, D // 32), dtype=np.uint8)
    _check(_load().oracle_mx_quantize_rows(_ptr(xf), n, D, _ptr(codes), _ptr(scales)),
           "mx_quantize_rows")
    return codes, scales


def mx_dequantize_rows(codes, scales) -> np.ndarray:
    """decode(code) * 2^(E - 127) per 32-element block, float64 (exact)."""
    c = np.ascontiguousarray(np.asarray(codes, dtype=np.uint8))
    s = np.ascontiguousarray(np.asarray(scales, dtype=np.uint8))
    n, D = c.shape
    out = np.zeros((n, D), dtype=np.float64)
    _check(_load().oracle_mx_dequantize_rows(_ptr(c), _ptr(s), n, D, _ptr(out)),
           "mx_dequantize_rows")
    return out


# ------------------------------------------------------------------------------ paged layout
class Paging:
    """Host copy of the paged-sequence description (see oracle.c, paged_slot)."""

    def __init__(self, seq_lens, block_table, page_size: int, num_pages: int, q_seq, q_pos):
        self.seq_lens = _i32(seq_lens)
        self.block_table = _i32(block_table)
        if self.block_table.ndim != 2:
            raise ValueError("block_table must be [B, max_pages]")
        self.B = int(self.seq_lens.shape[0])
        self.bt_stride = int(self.block_table.shape[1])
        self.page_size = int(page_size)
        self.num_pages = int(num_pages)
        self.q_seq = _i32(q_seq)
        self.q_pos = _i32(q_pos)
        self.T_q = int(self.q_seq.shape[0])

    def args(self):
        return [self.B, _ptr(self.seq_lens), _ptr(self.block_table), self.bt_stride,
                self.page_size, self.num_pages, self.T_q, _ptr(self.q_seq), _ptr(self.q_pos)]

    def subset(self, rows):
        rows = np.asarray(rows)
        return Paging(self.seq_lens, self.block_table, self.page_size, self.num_pages,
                      self.q_seq[rows], self.q_pos[rows])


# ------------------------------------------------------------------------------- the path
def index_score(pg: Paging, q_I, w, k, ld: int | None = None, fill: float = np.nan) -> np.ndarray:
    """I[t, s] for s <= q_pos[t]; other entries hold `fill`.  k: [slots, D_I] exact values."""
    qI, wt, kk = _f64(q_I), _f64(w), _f64(k)
    T_q, H_I, D_I = qI.shape
    if ld is None:
        ld = int(pg.q_pos.max()) + 1 if T_q else 1
    out = np.full((T_q, ld), fill, dtype=np.float64)
    _check(_load().oracle_index_score(*pg.args(), H_I, D_I, _ptr(qI), _ptr(wt), _ptr(kk),
                                      _ptr(out), ld), "index_score")
    return out


def topk(scores, n_valid, K: int) -> np.ndarray:
    """[T_q, K] int32: selected positions ascending, -1 padded (rows with n <= K select all)."""
    sc = _f64(scores)
    nv = _i32(n_valid)
    T_q, ld = sc.shape
    idx = np.zeros((T_q, K), dtype=np.int32)
    _check(_load().oracle_topk(T_q, _ptr(nv), _ptr(sc), ld, K, _ptr(idx)), "topk")
    return idx


def topk_blocks(scores, n_valid, K: int, block: int) -> np.ndarray:
    """[T_q, K] int32: block-aligned selection (the K / block blocks of `block` positions with the
    highest block maximum, ties to the lower block; all their causal positions), ascending, -1
    padded; rows with n <= K select all."""
    sc = _f64(scores)
    nv = _i32(n_valid)
    T_q, ld = sc.shape
    idx = np.zeros((T_q, K), dtype=np.int32)
    _check(_load().oracle_topk_blocks(T_q, _ptr(nv), _ptr(sc), ld, K, block, _ptr(idx)),
           "topk_blocks")
    return idx


def sparse_mla(pg: Paging, q, kv, idx, D_v: int, scale: float):
    """(out [T_q, H, D_v], lse [T_q, H]).  kv: [slots, D_qk] exact values (latent ‖ rope)."""
    qq, kk, ii = _f64(q), _f64(kv), _i32(idx)
    T_q, H, D_qk = qq.shape
    K = ii.shape[1]
    out = np.zeros((T_q, H, D_v), dtype=np.float64)
    lse = np.zeros((T_q, H), dtype=np.float64)
    _check(_load().oracle_sparse_mla(*pg.args(), H, D_qk, D_v, _ptr(qq), _ptr(kk), _ptr(ii), K,
                                     float(scale), _ptr(out), _ptr(lse)), "sparse_mla")
    return out, lse


def dense_attn(pg: Paging, q, kv, D_v: int, scale: float):
    qq, kk = _f64(q), _f64(kv)
    T_q, H, D_qk = qq.shape
    out = np.zeros((T_q, H, D_v), dtype=np.float64)
    lse = np.zeros((T_q, H), dtype=np.float64)
    _check(_load().oracle_dense_attn(*pg.args(), H, D_qk, D_v, _ptr(qq), _ptr(kk), float(scale),
                                     _ptr(out), _ptr(lse)), "dense_attn")
    return out, lse


def sparse_index_attention(pg: Paging, q_I, w, k, q, kv, K: int, D_v: int, scale: float):
    """The whole path: index scores -> Top-K -> sparse MLA.  Returns (scores, idx, out, lse)."""
    sc = index_score(pg, q_I, w, k)
    idx = topk(sc, pg.q_pos + 1, K)
    out, lse = sparse_mla(pg, q, kv, idx, D_v, scale)
    return sc, idx, out, lse
