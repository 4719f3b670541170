"""The C-ABI library loads and exports every entry point that include/hsa.h declares; argument
validation rejects bad calls before anything reaches a GPU (CPU only: no compute is launched)."""
import ctypes
import os
import re

import pytest

import sparse_index_attention_b200 as hsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "hsa.h")).read()
    return sorted(set(re.findall(r"HSA_API\s+[\w\s\*]+?\b(hsa_\w+)\s*\(", text)))


def test_header_declares_the_path():
    names = _declared()
    for n in ("hsa_index_score", "hsa_topk", "hsa_sparse_mla_attn", "hsa_fused_decode",
              "hsa_quantize_index", "hsa_quantize_kv", "hsa_quantize_mx", "hsa_dequantize_mx",
              "hsa_mx_round", "hsa_decode_prolog", "hsa_topk_blocks"):
        assert n in names


def test_library_exports_every_declared_symbol():
    L = hsa.lib()
    for name in _declared():
        assert hasattr(L, name), name
        assert name in hsa.SYMBOLS, f"binding lacks {name}"
    assert hsa.hsa_version() >= 100


def test_validation_without_gpu():
    L = hsa.lib()
    # NULL descriptor
    rc = L.hsa_topk(None, None, 0, 8, None, None)
    assert rc == hsa.HSA_ERR_INVALID_ARG
    assert b"seq" in L.hsa_last_error_message()
    # a descriptor with fake (never dereferenced) device pointers and bad sizes
    fake = ctypes.c_void_p(0x1000)
    seq = hsa.hsa_paged_seq_t(1, fake, fake, 4, 16, 4, 64, 2, fake, fake, 1, None)
    assert L.hsa_topk(ctypes.byref(seq), fake, 64, 0, fake, None) == hsa.HSA_ERR_INVALID_ARG
    assert L.hsa_topk(ctypes.byref(seq), fake, 32, 8, fake, None) == hsa.HSA_ERR_INVALID_ARG  # ld < max_seq_len
    bad = hsa.hsa_paged_seq_t(1, fake, fake, 2, 16, 4, 64, 2, fake, fake, 1, None)  # bt_stride too small
    assert L.hsa_topk(ctypes.byref(bad), fake, 64, 8, fake, None) == hsa.HSA_ERR_INVALID_ARG
    rc = L.hsa_index_score(ctypes.byref(seq), fake, hsa.HSA_E4M3, fake, 4, 32, fake, hsa.HSA_BF16,
                           None, fake, 64, None)
    assert rc == hsa.HSA_ERR_UNSUPPORTED                       # e4m3 queries are not a supported type
    rc = L.hsa_index_score(ctypes.byref(seq), fake, hsa.HSA_BF16, fake, 4, 32, fake, hsa.HSA_E4M3,
                           None, fake, 64, None)
    assert rc == hsa.HSA_ERR_INVALID_ARG                       # E4M3 keys without scales
    rc = L.hsa_index_score(ctypes.byref(seq), fake, hsa.HSA_MXE4M3, fake, 4, 32, fake, hsa.HSA_MXE4M3,
                           fake, fake, 64, None)
    assert rc == hsa.HSA_ERR_INVALID_ARG                       # MX queries without their scales
    rc = L.hsa_index_score_mx(ctypes.byref(seq), fake, None, fake, 4, 32, fake, fake, fake, 64, None)
    assert rc == hsa.HSA_ERR_INVALID_ARG                       # q_scale NULL
    rc = L.hsa_index_score_mx(ctypes.byref(seq), fake, ctypes.c_void_p(0x1004), fake, 4, 32, fake,
                              fake, fake, 64, None)
    assert rc == hsa.HSA_ERR_INVALID_ARG                       # q_scale not 16-byte aligned
    rc = L.hsa_index_score_mx(ctypes.byref(seq), fake, fake, fake, 4, 48, fake, fake, fake, 64, None)
    assert rc == hsa.HSA_ERR_INVALID_ARG                       # D_I not a multiple of 32
    # the no-allocation decode step rejects a step whose scores and selections exceed its
    # scratch before anything touches the device
    big = hsa.hsa_paged_seq_t(1, fake, fake, 2048, 64, 2048, 131072, 128, fake, fake, 1, None)
    ia = hsa.hsa_index_args_t(fake, hsa.HSA_BF16, fake, 64, 128, fake, hsa.HSA_BF16, None, None)
    at = hsa.hsa_attn_args_t(fake, hsa.HSA_BF16, 128, 576, 512, fake, hsa.HSA_BF16, None, 512, None,
                             0.04, fake, hsa.HSA_BF16, None)
    rc = L.hsa_fused_decode_noalloc(ctypes.byref(big), ctypes.byref(ia), ctypes.byref(at), 2048, None)
    assert rc == hsa.HSA_ERR_WORKSPACE and b"scratch" in L.hsa_last_error_message()
    # the chunked prefill checks its chunk list and score buffers before enqueuing anything
    pf = hsa.hsa_paged_seq_t(1, fake, fake, 64, 64, 64, 4096, 64, fake, fake, 1, None)
    bufs = (ctypes.c_void_p * 2)(0x1000, 0x2000)
    for chunks, rows in (([0, 100], 128), ([32, 32], 128), ([0, 64], 32)):
        arr = (ctypes.c_int32 * 2)(*chunks)
        rc = L.hsa_prefill_chunked(ctypes.byref(pf), ctypes.byref(ia), ctypes.byref(at), 2048, arr, 1,
                                   bufs, rows, 4096, fake, None, None, None)
        assert rc == hsa.HSA_ERR_INVALID_ARG and b"chunk" in L.hsa_last_error_message(), chunks
    rc = L.hsa_quantize_index(fake, hsa.HSA_BF16, 10, 128, 48, None, 10, fake, fake, None)
    assert rc == hsa.HSA_ERR_INVALID_ARG                       # group does not divide D
    # E4M3 latent cache: the scale group must be a multiple of 16 that divides D_v
    for group, want in ((24, hsa.HSA_ERR_INVALID_ARG), (48, hsa.HSA_ERR_INVALID_ARG)):
        rc = L.hsa_sparse_mla_attn(ctypes.byref(seq), fake, hsa.HSA_BF16, 8, 80, 64, fake, hsa.HSA_E4M3,
                                   fake, group, fake, fake, 32, 0.1, fake, hsa.HSA_BF16, None, None, 0,
                                   None)
        assert rc == want, group
        assert b"kv_scale_group" in L.hsa_last_error_message()
    # MXFP8 keys: scales required and 16-byte aligned, D_I a multiple of 32
    rc = L.hsa_index_score(ctypes.byref(seq), fake, hsa.HSA_BF16, fake, 4, 32, fake, hsa.HSA_MXE4M3,
                           None, fake, 64, None)
    assert rc == hsa.HSA_ERR_INVALID_ARG and b"k_scale" in L.hsa_last_error_message()
    rc = L.hsa_index_score(ctypes.byref(seq), fake, hsa.HSA_BF16, fake, 4, 48, fake, hsa.HSA_MXE4M3,
                           fake, fake, 64, None)
    assert rc == hsa.HSA_ERR_INVALID_ARG and b"multiple of 32" in L.hsa_last_error_message()
    rc = L.hsa_index_score(ctypes.byref(seq), fake, hsa.HSA_BF16, fake, 4, 32, fake, hsa.HSA_MXE4M3,
                           ctypes.c_void_p(0x1004), fake, 64, None)
    assert rc == hsa.HSA_ERR_INVALID_ARG and b"aligned" in L.hsa_last_error_message()
    # MXFP8 quantizer: blocks of 32, F32/BF16 sources
    assert L.hsa_quantize_mx(fake, hsa.HSA_BF16, 10, 48, None, 10, fake, fake, None) == hsa.HSA_ERR_INVALID_ARG
    assert L.hsa_quantize_mx(fake, hsa.HSA_E4M3, 10, 64, None, 10, fake, fake, None) == hsa.HSA_ERR_UNSUPPORTED
    assert L.hsa_quantize_mx(fake, hsa.HSA_BF16, 11, 64, None, 10, fake, fake, None) == hsa.HSA_ERR_INVALID_ARG
    assert L.hsa_dequantize_mx(fake, fake, 10, 40, fake, hsa.HSA_BF16, None) == hsa.HSA_ERR_INVALID_ARG
    assert L.hsa_dequantize_mx(fake, fake, 10, 64, fake, hsa.HSA_E4M3, None) == hsa.HSA_ERR_UNSUPPORTED
    assert L.hsa_quantize_mx(None, hsa.HSA_BF16, 0, 64, None, 0, None, None, None) == hsa.HSA_OK
    # cache-write quantizers: misaligned sources, scales, rope cache or slot mapping are refused
    odd = ctypes.c_void_p(0x1001)
    rc = L.hsa_quantize_index(odd, hsa.HSA_BF16, 10, 128, 128, None, 10, fake, fake, None)
    assert rc == hsa.HSA_ERR_INVALID_ARG and b"misaligned" in L.hsa_last_error_message()
    rc = L.hsa_quantize_index(fake, hsa.HSA_F32, 10, 128, 128, None, 10, fake, odd, None)
    assert rc == hsa.HSA_ERR_INVALID_ARG
    rc = L.hsa_quantize_kv(fake, hsa.HSA_BF16, 10, 512, 64, 512, odd, 10, fake, fake, fake, None)
    assert rc == hsa.HSA_ERR_INVALID_ARG
    rc = L.hsa_quantize_kv(fake, hsa.HSA_BF16, 10, 512, 64, 512, None, 10, fake, fake, odd, None)
    assert rc == hsa.HSA_ERR_INVALID_ARG
    rc = L.hsa_quantize_kv(odd, hsa.HSA_F32, 10, 512, 64, 512, None, 10, fake, fake, fake, None)
    assert rc == hsa.HSA_ERR_INVALID_ARG
    rc = L.hsa_quantize_mx(fake, hsa.HSA_BF16, 10, 64, odd, 10, fake, fake, None)
    assert rc == hsa.HSA_ERR_INVALID_ARG
    # MX rounding of queries: blocks of 32, partial overlap refused, in place allowed
    assert L.hsa_mx_round(fake, hsa.HSA_BF16, 4, 48, fake, hsa.HSA_BF16, None) == hsa.HSA_ERR_INVALID_ARG
    assert L.hsa_mx_round(fake, hsa.HSA_E4M3, 4, 64, fake, hsa.HSA_BF16, None) == hsa.HSA_ERR_UNSUPPORTED
    rc = L.hsa_mx_round(ctypes.c_void_p(0x1000), hsa.HSA_BF16, 4, 64, ctypes.c_void_p(0x1040),
                        hsa.HSA_BF16, None)
    assert rc == hsa.HSA_ERR_INVALID_ARG and b"overlap" in L.hsa_last_error_message()
    # decode prolog: every operator is checked before anything is enqueued
    pa = hsa.hsa_prolog_args_t(4, fake, 64, fake, hsa.HSA_BF16, 128, fake, fake, hsa.HSA_MXE4M3,
                               fake, hsa.HSA_BF16, 512, 64, 48, fake, fake, fake, fake, hsa.HSA_BF16,
                               8, fake)
    assert L.hsa_decode_prolog(ctypes.byref(pa), None, None, None, None) == hsa.HSA_ERR_INVALID_ARG
    pa.kv_group = 512
    pa.k_dtype = hsa.HSA_BF16
    assert L.hsa_decode_prolog(ctypes.byref(pa), None, None, None, None) == hsa.HSA_ERR_UNSUPPORTED
    pa.k_dtype = hsa.HSA_MXE4M3
    pa.slot_mapping = None
    assert L.hsa_decode_prolog(ctypes.byref(pa), None, None, None, None) == hsa.HSA_ERR_INVALID_ARG
    pa.slot_mapping = odd
    assert L.hsa_decode_prolog(ctypes.byref(pa), None, None, None, None) == hsa.HSA_ERR_INVALID_ARG
    assert L.hsa_decode_prolog(None, None, None, None, None) == hsa.HSA_ERR_INVALID_ARG
    # block-aligned selection: block >= 8 dividing K
    for blk in (4, 48, 0):
        rc = L.hsa_topk_blocks(ctypes.byref(seq), fake, 64, 64, blk, fake, None)
        assert rc == hsa.HSA_ERR_INVALID_ARG, blk
    assert L.hsa_topk_blocks(ctypes.byref(seq), fake, 32, 64, 16, fake, None) == hsa.HSA_ERR_INVALID_ARG
    # zero rows is a no-op, not an error
    empty = hsa.hsa_paged_seq_t(1, fake, fake, 4, 16, 4, 64, 0, None, None, 1, None)
    assert L.hsa_topk(ctypes.byref(empty), None, 64, 8, None, None) == hsa.HSA_OK


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(hsa, "_lib", None)
    monkeypatch.setattr(hsa, "LIB_PATH", "/nonexistent/libhsa.so")
    with pytest.raises(RuntimeError, match="no fallback"):
        hsa.lib()


def test_plain_c_program_links_and_validates(tmp_path):
    """The header compiles as C99 with warnings as errors, and a C program linked against
    libhsa.so gets the documented status codes from the host-side checks."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    assert gcc, "gcc is needed to build the C ABI check"
    hsa.lib()                                   # the library is built
    libdir = os.path.dirname(hsa.LIB_PATH)
    exe = str(tmp_path / "c_abi_check")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi_check.c"),
                    "-L", libdir, "-lhsa", "-Wl,-rpath," + libdir, "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "c abi ok"
