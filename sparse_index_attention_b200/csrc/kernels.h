// kernels.h -- internal launcher declarations (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace hsa {

// ---- index score ---------------------------------------------------------------------------
struct IndexScoreArgs {
    SeqView seq;
    int32_t max_seq_len;
    int32_t q_run;
    const void* q_I;
    hsa_dtype_t q_dtype;   // F32, BF16, or MXE4M3 (codes, with q_scale)
    const void* q_scale;   // MXE4M3 queries: E8M0 bytes, D_I / 32 per (row, head); else NULL
    const float* w;
    int32_t H_I, D_I;
    const void* k_cache;
    hsa_dtype_t k_dtype;
    const void* k_scale;   // E4M3: fp32 per key; MXE4M3: E8M0 bytes, D_I / 32 per key
    float* scores;
    int64_t ld;
};
cudaError_t launch_index_score_simt(const IndexScoreArgs& a, cudaStream_t st);
// Tensor-core path (tcgen05 + TMA).  Returns cudaErrorNotSupported when the shape is not served.
bool index_score_tc_supported(const IndexScoreArgs& a);
cudaError_t launch_index_score_tc(const IndexScoreArgs& a, cudaStream_t st);

// ---- top-k ---------------------------------------------------------------------------------
cudaError_t launch_topk(const SeqView& seq, int32_t max_seq_len, const float* scores, int64_t ld,
                        int32_t K, int32_t* idx, cudaStream_t st);

// Block-aligned selection: the K / block blocks of `block` positions with the highest block
// maximum, all their causal positions ascending (block >= 8, block | K).
cudaError_t launch_topk_blocks(const SeqView& seq, int32_t max_seq_len, const float* scores,
                               int64_t ld, int32_t K, int32_t block, int32_t* idx, cudaStream_t st);
size_t topk_blocks_smem(int32_t max_seq_len, int32_t K, int32_t block);

// ---- sparse MLA -------------------------------------------------------------------------------
struct SparseMlaArgs {
    SeqView seq;
    int32_t max_seq_len;
    const void* q;
    hsa_dtype_t q_dtype;
    int32_t H, D_qk, D_v;
    const void* kv;
    hsa_dtype_t kv_dtype;
    const float* kv_scale;
    int32_t kv_scale_group;   // E4M3: latent dims per scale (divides D_v); else D_v
    const void* kv_rope;
    const int32_t* idx;
    int32_t K;
    float softmax_scale;
    void* out;
    hsa_dtype_t out_dtype;
    float* lse;
    void* ws;
    size_t ws_bytes;
};
cudaError_t launch_sparse_mla_simt(const SparseMlaArgs& a, cudaStream_t st);
bool sparse_mla_tc_supported(const SparseMlaArgs& a);
size_t sparse_mla_tc_workspace(int32_t T_q, int32_t K);
cudaError_t launch_sparse_mla_tc(const SparseMlaArgs& a, cudaStream_t st);

// ---- quantizers ------------------------------------------------------------------------------
cudaError_t launch_quantize_rows(const void* src, hsa_dtype_t src_dtype, int64_t n_rows,
                                 int32_t src_stride, int32_t D, int32_t group,
                                 const int64_t* slot_mapping, int64_t num_slots, uint8_t* codes,
                                 float* scales, int32_t copy_cols, void* copy_dst,
                                 cudaStream_t st);
// MXFP8: 32-element blocks, E8M0 scale bytes, E4M3 codes (rule in hsa.h).
cudaError_t launch_quantize_mx(const void* src, hsa_dtype_t src_dtype, int64_t n_rows, int32_t D,
                               const int64_t* slot_mapping, int64_t num_slots, uint8_t* codes,
                               uint8_t* scales, cudaStream_t st);
// quantize_mx followed by dequantize_mx in one kernel (rows contiguous, no slot mapping).
cudaError_t launch_mx_round(const void* src, hsa_dtype_t src_dtype, int64_t n_rows, int32_t D,
                            void* dst, hsa_dtype_t dst_dtype, cudaStream_t st);
cudaError_t launch_dequantize_mx(const uint8_t* codes, const uint8_t* scales, int64_t n_rows,
                                 int32_t D, void* dst, hsa_dtype_t dst_dtype, cudaStream_t st);

}  // namespace hsa
