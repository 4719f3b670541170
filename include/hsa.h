/*
 * hsa.h -- C ABI of the sparse index attention library (libhsa.so) for NVIDIA B200 (sm_100a).
 *
 * The path, as the source pages state the problem ("Day 0 Inference Adaptation and
 * Optimization for Hybrid Attention Models", section "Sparse Attention Pipeline Optimization";
 * "Inference Adaptation and Performance Optimization for a Domestically Developed LLM's New
 * Architecture", section 3):
 *   1. a lightweight indexer scores every causal history position of every query row,
 *        I[t,s] = sum_j w[t,j] * ReLU( q_I[t,j,:] . k_I[s,:] ),   0 <= s <= p_t;
 *   2. a per-row Top-K keeps the K best positions (ties toward the lower position; rows with
 *      p_t + 1 <= K keep all of them);
 *   3. sparse MLA attention reads only the selected rows of the paged latent KV cache
 *      (latent c_kv || rope part per position, shared by every head) and attends over them.
 * FP8 storage of index keys and latent KV ("Hierarchical Quantization" on the first page;
 * the table of section 4 on the fifth) is written by hsa_quantize_index / hsa_quantize_kv
 * (E4M3 with fp32 scales) and hsa_quantize_mx (MXFP8: E8M0 scale per 32 elements).
 *
 * Conventions shared by every call
 *  - Memory: every tensor is caller-owned device memory, row-major and contiguous unless a
 *    stride is given.  The library never allocates device memory at run time.  Calls that need
 *    scratch take a workspace pointer and size; hsa_*_workspace_size() reports the bytes needed.
 *    The one exception is hsa_fused_decode_noalloc, whose scratch is a fixed array of the library
 *    itself (see there).
 *  - Streams: every call is asynchronous on the cudaStream_t passed in as `stream` (NULL = the
 *    legacy default stream).  Host-side argument checks happen before anything is enqueued.
 *  - Errors: every call returns an hsa_status_t.  HSA_ERR_INVALID_ARG: null pointer, size out of
 *    range, misaligned pointer; HSA_ERR_UNSUPPORTED: a dtype / shape combination no kernel
 *    implements; HSA_ERR_WORKSPACE: workspace too small; HSA_ERR_CUDA: a launch failed
 *    (hsa_last_error_message() names it).  Nothing is enqueued when a call returns an error.
 *  - Device-side checks: every kernel validates the page ids it reads from the block table, the
 *    positions it reads (q_pos < seq_len, selected index in [0, q_pos]) and the row grouping it
 *    relies on.  A failed check never faults: the access is skipped or redirected to page 0 and
 *    a bit is OR-ed into *seq->status (if non-null), so results are then undefined but the
 *    context stays usable.  Bits: HSA_DEV_BAD_PAGE, HSA_DEV_BAD_POS, HSA_DEV_BAD_GROUP,
 *    HSA_DEV_TIMEOUT (every wait inside a kernel is bounded; one that gives up makes the kernel
 *    leave early and sets this bit instead of hanging the GPU).
 *  - Threading: no mutable global state beyond a per-thread error message, a launch counter
 *    and hsa_fused_decode_noalloc's scratch (shared by its calls); calls on different streams
 *    may be issued from different host threads.
 */
#ifndef HSA_H_
#define HSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HSA_API __attribute__((visibility("default")))
#else
#define HSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum hsa_status {
    HSA_OK = 0,
    HSA_ERR_INVALID_ARG = 1,
    HSA_ERR_UNSUPPORTED = 2,
    HSA_ERR_CUDA = 3,
    HSA_ERR_WORKSPACE = 4
} hsa_status_t;

typedef enum hsa_dtype {
    HSA_F32 = 0,   /* IEEE binary32 */
    HSA_BF16 = 1,  /* bfloat16 */
    HSA_E4M3 = 2,  /* OCP FP8 E4M3 code, one byte; paired with fp32 scales */
    HSA_MXE4M3 = 3 /* MXFP8 (OCP Microscaling): E4M3 codes, and one E8M0 scale byte E, meaning
                      2^(E - 127), shared by each block of 32 consecutive elements */
} hsa_dtype_t;

/* device status bits (OR-ed into *hsa_paged_seq_t.status) */
#define HSA_DEV_BAD_PAGE 1u   /* block_table entry outside [0, num_pages) */
#define HSA_DEV_BAD_POS 2u    /* q_pos >= seq_len, or a selected index outside [0, q_pos] */
#define HSA_DEV_BAD_GROUP 4u  /* rows of one q_run disagree on their sequence */
#define HSA_DEV_TIMEOUT 8u    /* a pipeline wait inside a kernel gave up (the kernel returned early) */

/* Paged sequences and query rows.
 * Position s of sequence b lives in physical slot
 *     block_table[b * bt_stride + s / page_size] * page_size + s % page_size
 * of every paged cache (the indexer reads keys straight out of the paged cache: first page,
 * "Sparse Attention Pipeline Optimization"; gather through the page table, third page, 3.1).  Query row t belongs to
 * sequence q_seq[t] at absolute position q_pos[t] and sees positions 0..q_pos[t] (the causal
 * mask is generated from q_pos inside the kernels, with per-row offsets instead of a
 * per-sequence host loop, third page 3.1).  Top-K outputs are positions in this logical
 * numbering, the representation shared with the cache layer (third page, section 4). */
typedef struct hsa_paged_seq {
    int32_t B;                   /* number of sequences, >= 1 */
    const int32_t* seq_lens;     /* device [B]: context length of each sequence */
    const int32_t* block_table;  /* device [B, bt_stride]: physical page of each logical page */
    int64_t bt_stride;           /* elements between consecutive sequences' rows */
    int32_t page_size;           /* slots per page, >= 1 */
    int32_t num_pages;           /* physical pages in every paged cache */
    int32_t max_seq_len;         /* host-side upper bound of seq_lens[] (sizes launch grids) */
    int32_t T_q;                 /* number of query rows, >= 0 */
    const int32_t* q_seq;        /* device [T_q]: sequence of each query row */
    const int32_t* q_pos;        /* device [T_q]: absolute position of each query row */
    int32_t q_run;               /* rows come in runs of q_run consecutive rows of one sequence
                                    (the last run may be shorter); 1 = no promise */
    uint32_t* status;            /* device, nullable: device-side check bits are OR-ed here */
} hsa_paged_seq_t;

/* ---- 1. index score ---------------------------------------------------------------------
 * scores[t, s] = sum_{j<H_I} w[t,j] * max(0, sum_{d<D_I} q_I[t,j,d] * k(slot(t,s), d))
 * for 0 <= s <= q_pos[t]; entries s > q_pos[t] are not written.
 *   q_I      device [T_q, H_I, D_I], q_dtype F32 or BF16
 *   w        device fp32 [T_q, H_I] (head weights)
 *   k_cache  device [num_pages * page_size, D_I] of k_dtype F32, BF16, E4M3 or MXE4M3 (codes)
 *   k_scale  k_dtype E4M3: device fp32 [num_pages * page_size] (key = code * scale);
 *            k_dtype MXE4M3: device uint8 [num_pages * page_size, D_I / 32] E8M0 bytes, 16-byte
 *            aligned (key element d = code * 2^(E[d / 32] - 127), D_I a multiple of 32);
 *            else NULL
 *   scores   device fp32 [T_q, ld_scores], ld_scores >= max_seq_len
 * Pages: first page "Sparse Attention Pipeline Optimization" (per-head scores over the paged K
 * cache, summed with per-head weights); fifth page 3.1 (LI); BF16 and
 * quantized index paths, second page 3.1; MXFP8 index keys, fifth page 4 (table).  The
 * tensor-core kernel serves q BF16, k BF16/E4M3/MXE4M3, H_I = 64, D_I = 128, page_size a
 * multiple of 8; other shapes use a CUDA-core kernel.  With E4M3 keys a 16-byte-aligned k_scale
 * lets the codes go straight to 8-bit MMAs (each bf16 query split into two E4M3 parts); a
 * k_scale aligned to 4 bytes only is served by widening the codes, with the same contract. */
HSA_API hsa_status_t hsa_index_score(const hsa_paged_seq_t* seq, const void* q_I, hsa_dtype_t q_dtype,
                             const float* w, int32_t H_I, int32_t D_I, const void* k_cache,
                             hsa_dtype_t k_dtype, const void* k_scale, float* scores,
                             int64_t ld_scores, void* stream);

/* The index score with MXFP8 queries and keys: both operands are E4M3 codes with one E8M0 scale
 * byte per 32 dims, so the product runs as a block-scaled MMA on the codes themselves (first
 * page "Hierarchical Quantization": index Q and K in MXFP8; fifth page 4, table).
 *   scores[t, s] = sum_j w[t,j] * max(0, sum_d qv(t,j,d) * kv(slot(t,s), d)),
 *   qv(t,j,d) = q_codes[t,j,d] * 2^(q_scale[t,j,d/32] - 127)   (kv likewise from k_codes, k_scale)
 *   q_codes  device uint8 [T_q, H_I, D_I];  q_scale device uint8 [T_q, H_I, D_I / 32], 16-byte
 *            aligned (hsa_quantize_mx writes both from bf16 or fp32 queries)
 *   k_codes, k_scale, w, scores: as hsa_index_score with k_dtype MXE4M3.
 * D_I must be a multiple of 32.  The tensor-core kernel serves H_I = 64, D_I = 128, page_size a
 * multiple of 8; other shapes use a CUDA-core kernel.  Same errors as hsa_index_score. */
HSA_API hsa_status_t hsa_index_score_mx(const hsa_paged_seq_t* seq, const uint8_t* q_codes,
                                const uint8_t* q_scale, const float* w, int32_t H_I, int32_t D_I,
                                const uint8_t* k_codes, const uint8_t* k_scale, float* scores,
                                int64_t ld_scores, void* stream);

/* ---- 2. Top-K -----------------------------------------------------------------------------
 * For row t with n = q_pos[t] + 1 candidate positions:
 *   n <= K : idx[t] = 0, 1, ..., n-1, then -1 up to K;
 *   n >  K : the K positions first in the order (score descending, position ascending),
 *            written in ascending position order.  +0.0 and -0.0 are equal; NaN is outside the
 *            contract.
 *   scores  device fp32 [T_q, ld_scores] (entries past q_pos[t] are ignored)
 *   idx     device int32 [T_q, K], 1 <= K <= 65536
 * Pages: first page "Sparse Attention Pipeline Optimization" (Top-K of the weighted scores);
 * third page 3.1 (selection).  Needs no workspace. */
HSA_API hsa_status_t hsa_topk(const hsa_paged_seq_t* seq, const float* scores, int64_t ld_scores,
                      int32_t K, int32_t* idx, void* stream);

/* Block-aligned selection (third page, 3.1: the selection is aligned to cache blocks so that
 * the attention reads the cache in contiguous pieces).  For row t with n = q_pos[t] + 1:
 *   n <= K : as hsa_topk;
 *   n >  K : positions fall into blocks [b * block, (b + 1) * block) (the last one cut at n); a
 *            block scores the largest score of its positions; the K / block blocks first in the
 *            order (block score descending, block index ascending) are kept, and every position
 *            of a kept block is written, ascending, then -1 up to K (a kept partial last block
 *            leaves fewer than K).
 * block >= 8 and divides K; ceil(max_seq_len / block) may not exceed about 56000.  With block =
 * page_size each kept block is one whole cache page. */
HSA_API hsa_status_t hsa_topk_blocks(const hsa_paged_seq_t* seq, const float* scores,
                             int64_t ld_scores, int32_t K, int32_t block, int32_t* idx,
                             void* stream);

/* ---- 3. sparse MLA attention -----------------------------------------------------------
 * For row t, head h, over S_t = { idx[t,k] != -1 }:
 *   z_n = softmax_scale * sum_{d<D_qk} q[t,h,d] * key(n, d)
 *   out[t,h,:] = sum_n e^{z_n - m} * key(n, 0:D_v) / sum_n e^{z_n - m},  m = max_n z_n
 *   lse[t,h]   = m + log sum_n e^{z_n - m}        (empty S_t: out = 0, lse = -inf)
 * where key(n, :) is cache row slot(t, n): the latent part (D_v values, also the value) followed
 * by the rope part (D_qk - D_v values).
 *   q        device [T_q, H, D_qk], q_dtype F32 or BF16
 *   kv       kv_dtype F32 / BF16: device [slots, D_qk] packed latent || rope; kv_rope = NULL
 *            kv_dtype E4M3: device uint8 [slots, D_v] latent codes, kv_scale fp32
 *            [slots, D_v / kv_scale_group] (one scale per kv_scale_group consecutive latent dims
 *            of a token: D_v = one per token, 128 = the pages' tile; a multiple of 16 that
 *            divides D_v), kv_rope BF16 [slots, D_qk - D_v]; F32 / BF16 caches: kv_scale_group
 *            is ignored
 *   idx      device int32 [T_q, K]: positions in [0, q_pos[t]] or -1
 *   out      device [T_q, H, D_v] of out_dtype (F32 or BF16)
 *   lse      device fp32 [T_q, H] or NULL
 *   ws       workspace of at least hsa_sparse_mla_workspace_size() bytes, 256-byte aligned
 *            (the current kernels report 0 and need none; a call may pass NULL)
 * Pages: first page "Sparse Attention Pipeline Optimization" (indexed reads, block-wise fused
 * attention); third page 3.2 (partition by query, aggregate over the selected positions,
 * stage them in shared memory); fifth page 3 (SFA).  The tensor-core kernel serves q BF16,
 * kv BF16 or E4M3, H = 128, D_qk = 576, D_v = 512; other shapes use a CUDA-core kernel. */
HSA_API size_t hsa_sparse_mla_workspace_size(const hsa_paged_seq_t* seq, int32_t H, int32_t D_qk,
                                     int32_t D_v, int32_t K);
HSA_API hsa_status_t hsa_sparse_mla_attn(const hsa_paged_seq_t* seq, const void* q, hsa_dtype_t q_dtype,
                                 int32_t H, int32_t D_qk, int32_t D_v, const void* kv,
                                 hsa_dtype_t kv_dtype, const float* kv_scale, int32_t kv_scale_group,
                                 const void* kv_rope, const int32_t* idx, int32_t K,
                                 float softmax_scale, void* out,
                                 hsa_dtype_t out_dtype, float* lse, void* ws, size_t ws_bytes,
                                 void* stream);

/* ---- 4. fused decode step -----------------------------------------------------------------
 * hsa_index_score -> hsa_topk -> hsa_sparse_mla_attn on the same rows, results bitwise equal
 * to the three calls in sequence.  scores ([T_q, ld_scores] fp32) and idx ([T_q, K] int32) are
 * caller buffers that hold the intermediate results afterwards.  With stream_aux != NULL the
 * rows are split in two halves; the second half runs on stream_aux, overlapping the first
 * half's attention (event-ordered; stream_main waits for stream_aux before returning work to
 * the caller); the results are bitwise the same.  ws: as for hsa_sparse_mla_attn.  Pages: first page "Sparse Attention Pipeline Optimization" (fusing the decode
 * operators and running independent ones concurrently: indexer, then the sparse attention
 * kernel; several streams); fifth page 3.3 (operators on independent streams with event
 * synchronization).  The members of hsa_index_args_t and hsa_attn_args_t have the meaning of
 * the same-named arguments of hsa_index_score and hsa_sparse_mla_attn (k_scale: fp32 per key
 * for E4M3 keys, E8M0 bytes for MXE4M3 keys). */
typedef struct hsa_index_args {
    const void* q_I; hsa_dtype_t q_dtype; const float* w; int32_t H_I; int32_t D_I;
    const void* k_cache; hsa_dtype_t k_dtype; const void* k_scale;
    const void* q_scale;   /* q_dtype MXE4M3 (keys MXE4M3 too): the queries' E8M0 bytes, as in
                              hsa_index_score_mx; else ignored */
} hsa_index_args_t;

typedef struct hsa_attn_args {
    const void* q; hsa_dtype_t q_dtype; int32_t H; int32_t D_qk; int32_t D_v;
    const void* kv; hsa_dtype_t kv_dtype; const float* kv_scale; int32_t kv_scale_group;
    const void* kv_rope;
    float softmax_scale; void* out; hsa_dtype_t out_dtype; float* lse;
} hsa_attn_args_t;

HSA_API size_t hsa_fused_decode_workspace_size(const hsa_paged_seq_t* seq, const hsa_attn_args_t* attn,
                                       int32_t K);
HSA_API hsa_status_t hsa_fused_decode(const hsa_paged_seq_t* seq, const hsa_index_args_t* index,
                              const hsa_attn_args_t* attn, int32_t K, float* scores,
                              int64_t ld_scores, int32_t* idx, void* ws, size_t ws_bytes,
                              void* stream_main, void* stream_aux);

/* Causal prefill over query-row chunks (Python: hsa_prefill_chunked).  Chunk i covers rows
 * [chunks[2i], chunks[2i+1]) (host int32 array, non-empty, inside [0, T_q); with q_run > 1 its
 * bounds should be multiples of q_run) and runs hsa_index_score -> hsa_topk ->
 * hsa_sparse_mla_attn on those rows, on stream_a for even i and stream_b for odd i (NULL: the
 * calling stream), so consecutive chunks form pairs that run concurrently.  With the zigzag order
 * (chunk i of 2N paired with chunk 2N-1-i) every pair carries the same causal work ("Efficient
 * Inference Deployment and Optimization for Hybrid Attention LLMs", 5.2: zigzag load balancing;
 * its multi-GPU form is the same chunks on several ranks).  Outputs land at the rows' own
 * offsets of out / lse / idx ([T_q, ...]), so the order of the chunks changes no result.  Both
 * side streams first wait for the work already on `stream`, which then waits for both.
 *   score_bufs  host array of two device fp32 buffers [score_rows, ld_scores], one per side
 *               stream, reused chunk after chunk (score_rows >= the largest chunk's rows;
 *               ld_scores >= max_seq_len); they hold scores of the last chunks afterwards
 *   idx         device int32 [T_q, K]: every row's selection afterwards
 * index / attn as for hsa_fused_decode.  Needs no workspace. */
HSA_API hsa_status_t hsa_prefill_chunked(const hsa_paged_seq_t* seq, const hsa_index_args_t* index,
                                 const hsa_attn_args_t* attn, int32_t K, const int32_t* chunks,
                                 int32_t n_chunks, float* const* score_bufs, int32_t score_rows,
                                 int64_t ld_scores, int32_t* idx, void* stream, void* stream_a,
                                 void* stream_b);

/* The fused decode step for callers that may not allocate device memory: code that runs while
 * a CUDA graph is being captured (an allocation cannot be captured), and engines or plug-ins
 * whose device memory all belongs to a pool they do not manage.  hsa_fused_decode needs scores
 * and idx buffers from its caller; this variant keeps both in a scratch array that the library
 * itself declares, 40 MiB, held on every GPU where the library's kernels are loaded until the
 * process exits.  It calls no cudaMalloc or cudaFree and no allocating routine, runs on one
 * stream, and gives the same out and lse as hsa_fused_decode on that stream (the paper has no
 * counterpart: this is an interface for such callers, not a step of the method).
 *   The step's scores [T_q, ld] fp32, ld = max_seq_len rounded up to a multiple of 4, and its
 *   selections [T_q, K] int32, each rounded up to 256 bytes, must fit in the 40 MiB: a larger
 *   call returns HSA_ERR_WORKSPACE and enqueues nothing (the FP8 decode batch, 128 rows of 65536
 *   positions with K = 2048, needs 33 MiB).
 *   The first call on a device looks up the scratch's address there (with that device current);
 *   make that first call outside any stream capture.
 *   Every call on a device uses the same scratch, which keeps the last call's scores and
 *   selections (nothing in it needs to start at zero): calls that overlap on the GPU -- on
 *   different streams without ordering between them -- race on it and must not be made.
 * Arguments as for hsa_fused_decode; other errors as there. */
HSA_API hsa_status_t hsa_fused_decode_noalloc(const hsa_paged_seq_t* seq, const hsa_index_args_t* index,
                                      const hsa_attn_args_t* attn, int32_t K, void* stream);

/* ---- 5. FP8 quantizers (cache write) --------------------------------------------------------
 * Per row r and group g of `group` consecutive elements:
 *   amax = max |x|; scale = amax / 448 (fp32, round to nearest); inv = 448 / amax (fp32);
 *   code = E4M3(round-to-nearest-even, saturating, of x * inv);   amax == 0: scale 1, codes 0.
 *   A group with amax < 2^-64 is multiplied by 2^64 (exactly) before inv and the products are
 *   formed, so that inv cannot overflow float32; this changes no code where 448 / amax is
 *   finite.  scale is still amax / 448 (it may be subnormal, or 0 for an fp32 amax of a few
 *   times 2^-149).
 * Row r is written to physical slot slot_mapping[r] (slot_mapping NULL: slot r).
 * hsa_quantize_index: src [n_rows, D] F32/BF16 -> codes uint8 [slots, D], scales fp32
 *   [slots, D / group].  group = D gives one scale per key (the layout hsa_index_score reads);
 *   group = 32 is the pages' group size (MXFP8-style granularity with fp32 scales).
 * hsa_quantize_kv: src [n_rows, D_v + D_rope] F32/BF16 (latent || rope) -> latent codes uint8
 *   [slots, D_v], scales fp32 [slots, D_v / group], rope copied to rope_cache BF16
 *   [slots, D_rope].  group = D_v gives one scale per token (the layout hsa_sparse_mla_attn
 *   reads); group = 128 is the pages' tile size.
 * Pages: first page "Hierarchical Quantization"; second page 4.1 and 4.2; fifth page 4 (table:
 * index Q/K group 32, KV cache tile 128, dynamic scales). */
HSA_API hsa_status_t hsa_quantize_index(const void* src, hsa_dtype_t src_dtype, int64_t n_rows,
                                int32_t D, int32_t group, const int64_t* slot_mapping,
                                int64_t num_slots, uint8_t* codes, float* scales, void* stream);
HSA_API hsa_status_t hsa_quantize_kv(const void* src, hsa_dtype_t src_dtype, int64_t n_rows, int32_t D_v,
                             int32_t D_rope, int32_t group, const int64_t* slot_mapping,
                             int64_t num_slots, uint8_t* codes, float* scales, void* rope_cache,
                             void* stream);

/* ---- 6. MXFP8 block quantizer ------------------------------------------------------------
 * Per row r and block b of 32 consecutive elements (D a multiple of 32):
 *   amax = max |x|;  X = floor(log2(amax)) - 8, clamped to [-127, 127];  E = X + 127;
 *   code = E4M3(round-to-nearest-even, saturating, of x * 2^-X);   amax == 0: E = 0, codes 0.
 * (8 is the exponent of E4M3's top binade, 448 = 1.75 * 2^8, so the block maximum times 2^-X
 * lies in [256, 512); a value there above 448 saturates to 448, an error of up to 12.5 % that
 * the OCP Microscaling rule for the shared exponent accepts.)  From finite fp32 or bf16 data E
 * never exceeds 246.
 * hsa_quantize_mx: src [n_rows, D] F32/BF16 -> codes uint8 [slots, D], scales uint8
 *   [slots, D / 32]; row r goes to slot slot_mapping[r] (NULL: slot r).  With D = 128 this
 *   writes the MXE4M3 index key cache hsa_index_score reads; applied to q_I (slot_mapping
 *   NULL) it quantizes the index queries.
 * hsa_dequantize_mx: codes [n_rows, D] + scales [n_rows, D / 32] -> dst [n_rows, D] of
 *   dst_dtype F32 or BF16, value code * 2^(E - 127): exact in F32 for every E <= 246; exact in
 *   BF16 for E >= 3 (below that, values under the bf16 range round to nearest).  Writing MXFP8
 *   index queries back as bf16 lets the bf16-query index kernels consume them unchanged.
 * Pages: first page "Hierarchical Quantization" (index Q/K in MXFP8, group 32, shared
 * exponent); second page 4.1; fifth page 4 (table). */
HSA_API hsa_status_t hsa_quantize_mx(const void* src, hsa_dtype_t src_dtype, int64_t n_rows, int32_t D,
                             const int64_t* slot_mapping, int64_t num_slots, uint8_t* codes,
                             uint8_t* scales, void* stream);
HSA_API hsa_status_t hsa_dequantize_mx(const uint8_t* codes, const uint8_t* scales, int64_t n_rows,
                               int32_t D, void* dst, hsa_dtype_t dst_dtype, void* stream);

/* hsa_mx_round: src [n_rows, D] F32/BF16 -> dst [n_rows, D] F32/BF16 holding the MXFP8 values
 * (hsa_quantize_mx followed by hsa_dequantize_mx, bit for bit, in one kernel with no code or
 * scale bytes written to memory).  Index queries rounded this way let the bf16-query index
 * kernels score MXFP8 queries.  src and dst may not overlap partially (dst == src is allowed). */
HSA_API hsa_status_t hsa_mx_round(const void* src, hsa_dtype_t src_dtype, int64_t n_rows, int32_t D,
                          void* dst, hsa_dtype_t dst_dtype, void* stream);

/* ---- 7. decode prolog ---------------------------------------------------------------------
 * The writes that precede a decode step, as three independent operators on three streams:
 *   stream_k : the new tokens' index keys into the index key cache
 *              (k_dtype MXE4M3: hsa_quantize_mx, k_scale E8M0 bytes [num_slots, D_I / 32];
 *               k_dtype E4M3: hsa_quantize_index with one fp32 scale per key, k_scale
 *               [num_slots]);
 *   stream_kv: their latent rows into the FP8 latent cache (hsa_quantize_kv: codes
 *              [num_slots, D_v], fp32 scales [num_slots, D_v / kv_group], bf16 rope
 *              [num_slots, D_rope]);
 *   stream_q : the index queries q_I [q_rows, D_I] rounded onto the MXFP8 grid into q_I_out
 *              (bf16, hsa_mx_round; skipped when q_I_out is NULL), and / or quantized to MXFP8
 *              codes q_codes_out [q_rows, D_I] and E8M0 scales q_scale_out [q_rows, D_I / 32]
 *              for hsa_index_score_mx (hsa_quantize_mx; skipped when q_codes_out is NULL).
 * Each side stream first waits for the work already enqueued on `stream`, and `stream` then
 * waits for all three, so a decode step enqueued on `stream` next sees every write.  A NULL side
 * stream means `stream` itself.  Results equal the same calls issued one after another on one
 * stream.  new_k [n_new, D_I] and new_kv [n_new, D_v + D_rope] are F32 or BF16; token r goes to
 * physical slot slot_mapping[r] (int64, device).  Pages: first page "Sparse Attention Pipeline
 * Optimization" (the indexer's preparatory operators run on concurrent streams); fifth page
 * 3.2 and 3.3 (independent operators on separate streams, synchronized by events); the Q / K
 * projections and the K normalization themselves need model weights and are not part of this
 * library. */
typedef struct hsa_prolog_args {
    int64_t n_new;                /* new tokens, >= 0 */
    const int64_t* slot_mapping;  /* device [n_new] */
    int64_t num_slots;            /* slots of every paged cache */
    const void* new_k; hsa_dtype_t new_k_dtype; int32_t D_I;
    uint8_t* k_cache; void* k_scale; hsa_dtype_t k_dtype;
    const void* new_kv; hsa_dtype_t new_kv_dtype; int32_t D_v; int32_t D_rope; int32_t kv_group;
    uint8_t* kv_cache; float* kv_scale; void* kv_rope;
    const void* q_I; hsa_dtype_t q_I_dtype; int64_t q_rows;
    void* q_I_out;                /* bf16 [q_rows, D_I], or NULL */
    uint8_t* q_codes_out;         /* uint8 [q_rows, D_I], or NULL */
    uint8_t* q_scale_out;         /* uint8 [q_rows, D_I / 32] (with q_codes_out) */
} hsa_prolog_args_t;

HSA_API hsa_status_t hsa_decode_prolog(const hsa_prolog_args_t* args, void* stream, void* stream_k,
                               void* stream_kv, void* stream_q);

/* ---- diagnostics -------------------------------------------------------------------------- */
HSA_API const char* hsa_status_string(hsa_status_t s);
/* Text of the last error raised by a call on this host thread ("" if none). */
HSA_API const char* hsa_last_error_message(void);
/* Number of kernels this library has launched from the calling host thread since it was loaded
 * (a diagnostic for benchmarks: every kernel of the path is counted once per launch). */
HSA_API uint64_t hsa_launch_count(void);
/* Library version, major * 10000 + minor * 100 + patch. */
HSA_API int32_t hsa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* HSA_H_ */
