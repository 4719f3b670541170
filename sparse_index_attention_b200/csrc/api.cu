// api.cu -- the C ABI of libhsa (declared in include/hsa.h): argument validation, kernel
// dispatch and the two-stream fused decode step.  Every entry point validates its arguments on
// the host before enqueuing anything and reports failures as hsa_status_t.
#include <stdarg.h>
#include <stdio.h>

#include <mutex>
#include <string>

#include "kernels.h"

namespace {

thread_local std::string g_last_error;

hsa_status_t fail(hsa_status_t s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
hsa_status_t fail(hsa_status_t s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

hsa_status_t cuda_status(cudaError_t e, const char* what) {
    if (e == cudaSuccess) return HSA_OK;
    return fail(HSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define HSA_REQUIRE(cond, code, ...)                                  \
    do {                                                              \
        if (!(cond)) return fail((code), __VA_ARGS__);                \
    } while (0)

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t dtype_size(hsa_dtype_t d) { return d == HSA_F32 ? 4 : (d == HSA_BF16 ? 2 : 1); }

hsa_status_t check_seq(const hsa_paged_seq_t* s) {
    HSA_REQUIRE(s != nullptr, HSA_ERR_INVALID_ARG, "seq is NULL");
    HSA_REQUIRE(s->B >= 1, HSA_ERR_INVALID_ARG, "B = %d must be >= 1", s->B);
    HSA_REQUIRE(s->seq_lens && s->block_table, HSA_ERR_INVALID_ARG, "seq_lens / block_table NULL");
    HSA_REQUIRE(s->page_size >= 1 && s->num_pages >= 1, HSA_ERR_INVALID_ARG,
                "page_size = %d, num_pages = %d must be >= 1", s->page_size, s->num_pages);
    HSA_REQUIRE(s->max_seq_len >= 1, HSA_ERR_INVALID_ARG, "max_seq_len = %d must be >= 1",
                s->max_seq_len);
    HSA_REQUIRE(s->bt_stride >= hsa::ceil_div(s->max_seq_len, s->page_size), HSA_ERR_INVALID_ARG,
                "bt_stride = %lld cannot hold ceil(max_seq_len / page_size) pages",
                (long long)s->bt_stride);
    HSA_REQUIRE(s->T_q >= 0, HSA_ERR_INVALID_ARG, "T_q = %d < 0", s->T_q);
    HSA_REQUIRE(s->T_q == 0 || (s->q_seq && s->q_pos), HSA_ERR_INVALID_ARG, "q_seq / q_pos NULL");
    HSA_REQUIRE(s->q_run >= 1, HSA_ERR_INVALID_ARG, "q_run = %d must be >= 1", s->q_run);
    return HSA_OK;
}

hsa::SeqView view(const hsa_paged_seq_t* s) { return hsa::make_view(*s); }

// Row window [t0, t0 + n) of a descriptor (used by the fused call's two halves).
hsa_paged_seq_t sub_rows(const hsa_paged_seq_t& s, int32_t t0, int32_t n) {
    hsa_paged_seq_t r = s;
    r.T_q = n;
    r.q_seq = s.q_seq + t0;
    r.q_pos = s.q_pos + t0;
    return r;
}

hsa_status_t check_index(const hsa_paged_seq_t* seq, const void* q_I, hsa_dtype_t q_dtype,
                         const void* q_scale, const float* w, int32_t H_I, int32_t D_I,
                         const void* k_cache, hsa_dtype_t k_dtype, const void* k_scale,
                         const float* scores, int64_t ld) {
    hsa_status_t st = check_seq(seq);
    if (st != HSA_OK) return st;
    HSA_REQUIRE(H_I >= 1 && H_I <= 256 && D_I >= 1 && D_I <= 1024, HSA_ERR_INVALID_ARG,
                "H_I = %d, D_I = %d out of range", H_I, D_I);
    HSA_REQUIRE((size_t)H_I * D_I * 4 <= 160 * 1024, HSA_ERR_UNSUPPORTED,
                "H_I * D_I = %d too large", H_I * D_I);
    HSA_REQUIRE(q_dtype == HSA_F32 || q_dtype == HSA_BF16 || q_dtype == HSA_MXE4M3, HSA_ERR_UNSUPPORTED,
                "q_I dtype must be F32, BF16 or MXE4M3");
    HSA_REQUIRE(q_dtype != HSA_MXE4M3 || k_dtype == HSA_MXE4M3, HSA_ERR_UNSUPPORTED,
                "MXE4M3 queries need MXE4M3 keys");
    HSA_REQUIRE(k_dtype == HSA_F32 || k_dtype == HSA_BF16 || k_dtype == HSA_E4M3 ||
                    k_dtype == HSA_MXE4M3,
                HSA_ERR_UNSUPPORTED, "k dtype must be F32, BF16, E4M3 or MXE4M3");
    HSA_REQUIRE(k_dtype != HSA_MXE4M3 || D_I % 32 == 0, HSA_ERR_INVALID_ARG,
                "MXE4M3 keys need D_I a multiple of 32 (D_I = %d)", D_I);
    HSA_REQUIRE(ld >= seq->max_seq_len, HSA_ERR_INVALID_ARG, "ld_scores = %lld < max_seq_len",
                (long long)ld);
    if (seq->T_q > 0) {
        HSA_REQUIRE(q_I && w && k_cache && scores, HSA_ERR_INVALID_ARG, "NULL tensor pointer");
        HSA_REQUIRE((k_dtype != HSA_E4M3 && k_dtype != HSA_MXE4M3) || k_scale,
                    HSA_ERR_INVALID_ARG, "E4M3 and MXE4M3 keys need k_scale");
        HSA_REQUIRE(k_dtype != HSA_E4M3 || aligned(k_scale, 4), HSA_ERR_INVALID_ARG,
                    "misaligned k_scale");
        HSA_REQUIRE(k_dtype != HSA_MXE4M3 || aligned(k_scale, 16), HSA_ERR_INVALID_ARG,
                    "MXE4M3 k_scale must be 16-byte aligned");
        HSA_REQUIRE(q_dtype != HSA_MXE4M3 || (q_scale && aligned(q_scale, 16)), HSA_ERR_INVALID_ARG,
                    "MXE4M3 queries need q_scale, 16-byte aligned");
        HSA_REQUIRE(aligned(q_I, dtype_size(q_dtype)) && aligned(w, 4) && aligned(scores, 4) &&
                        aligned(k_cache, dtype_size(k_dtype)),
                    HSA_ERR_INVALID_ARG, "misaligned tensor pointer");
    }
    return HSA_OK;
}

hsa_status_t check_attn(const hsa_paged_seq_t* seq, const void* q, hsa_dtype_t q_dtype, int32_t H,
                        int32_t D_qk, int32_t D_v, const void* kv, hsa_dtype_t kv_dtype,
                        const float* kv_scale, int32_t kv_scale_group, const void* kv_rope,
                        const int32_t* idx, int32_t K, const void* out, hsa_dtype_t out_dtype) {
    hsa_status_t st = check_seq(seq);
    if (st != HSA_OK) return st;
    HSA_REQUIRE(H >= 1 && H <= 1024, HSA_ERR_INVALID_ARG, "H = %d out of range", H);
    HSA_REQUIRE(D_v >= 1 && D_v <= D_qk && D_qk <= 2048, HSA_ERR_INVALID_ARG,
                "D_qk = %d, D_v = %d out of range", D_qk, D_v);
    HSA_REQUIRE(K >= 1 && K <= 65536, HSA_ERR_INVALID_ARG, "K = %d out of range", K);
    HSA_REQUIRE(q_dtype == HSA_F32 || q_dtype == HSA_BF16, HSA_ERR_UNSUPPORTED,
                "q dtype must be F32 or BF16");
    HSA_REQUIRE(out_dtype == HSA_F32 || out_dtype == HSA_BF16, HSA_ERR_UNSUPPORTED,
                "out dtype must be F32 or BF16");
    HSA_REQUIRE(kv_dtype == HSA_F32 || kv_dtype == HSA_BF16 || kv_dtype == HSA_E4M3,
                HSA_ERR_UNSUPPORTED, "kv dtype must be F32, BF16 or E4M3");
    if (seq->T_q > 0) {
        HSA_REQUIRE(q && kv && idx && out, HSA_ERR_INVALID_ARG, "NULL tensor pointer");
        if (kv_dtype == HSA_E4M3) {
            HSA_REQUIRE(kv_scale && (kv_rope || D_qk == D_v), HSA_ERR_INVALID_ARG,
                        "E4M3 latent cache needs kv_scale and kv_rope");
            HSA_REQUIRE(kv_scale_group >= 16 && kv_scale_group % 16 == 0 && D_v % kv_scale_group == 0,
                        HSA_ERR_INVALID_ARG,
                        "kv_scale_group = %d must be a multiple of 16 that divides D_v = %d",
                        kv_scale_group, D_v);
        } else {
            HSA_REQUIRE(kv_rope == nullptr, HSA_ERR_INVALID_ARG,
                        "kv_rope must be NULL for a packed F32/BF16 cache");
        }
        HSA_REQUIRE(aligned(q, dtype_size(q_dtype)) && aligned(out, dtype_size(out_dtype)) &&
                        aligned(idx, 4) && aligned(kv, dtype_size(kv_dtype)),
                    HSA_ERR_INVALID_ARG, "misaligned tensor pointer");
    }
    return HSA_OK;
}

hsa::IndexScoreArgs index_args(const hsa_paged_seq_t* seq, const void* q_I, hsa_dtype_t q_dtype,
                               const void* q_scale, const float* w, int32_t H_I, int32_t D_I,
                               const void* k_cache, hsa_dtype_t k_dtype, const void* k_scale,
                               float* scores, int64_t ld) {
    hsa::IndexScoreArgs a;
    a.seq = view(seq);
    a.max_seq_len = seq->max_seq_len;
    a.q_run = seq->q_run;
    a.q_I = q_I;
    a.q_dtype = q_dtype;
    a.q_scale = q_dtype == HSA_MXE4M3 ? q_scale : nullptr;
    a.w = w;
    a.H_I = H_I;
    a.D_I = D_I;
    a.k_cache = k_cache;
    a.k_dtype = k_dtype;
    a.k_scale = k_scale;
    a.scores = scores;
    a.ld = ld;
    return a;
}

hsa_status_t run_index(const hsa::IndexScoreArgs& a, cudaStream_t st) {
    if (a.seq.T_q == 0) return HSA_OK;
    if (hsa::index_score_tc_supported(a))
        return cuda_status(hsa::launch_index_score_tc(a, st), "index_score (tensor core)");
    return cuda_status(hsa::launch_index_score_simt(a, st), "index_score");
}

hsa::SparseMlaArgs attn_args(const hsa_paged_seq_t* seq, const hsa_attn_args_t& at,
                             const int32_t* idx, int32_t K, void* ws, size_t ws_bytes) {
    hsa::SparseMlaArgs a;
    a.seq = view(seq);
    a.max_seq_len = seq->max_seq_len;
    a.q = at.q;
    a.q_dtype = at.q_dtype;
    a.H = at.H;
    a.D_qk = at.D_qk;
    a.D_v = at.D_v;
    a.kv = at.kv;
    a.kv_dtype = at.kv_dtype;
    a.kv_scale = at.kv_scale;
    a.kv_scale_group = at.kv_dtype == HSA_E4M3 ? at.kv_scale_group : at.D_v;
    a.kv_rope = at.kv_rope;
    a.idx = idx;
    a.K = K;
    a.softmax_scale = at.softmax_scale;
    a.out = at.out;
    a.out_dtype = at.out_dtype;
    a.lse = at.lse;
    a.ws = ws;
    a.ws_bytes = ws_bytes;
    return a;
}

size_t attn_ws_bytes(const hsa::SparseMlaArgs& a) {
    return hsa::sparse_mla_tc_supported(a) ? hsa::sparse_mla_tc_workspace(a.seq.T_q, a.K) : 0;
}

hsa_status_t run_attn(const hsa::SparseMlaArgs& a, cudaStream_t st) {
    if (a.seq.T_q == 0) return HSA_OK;
    if (hsa::sparse_mla_tc_supported(a)) {
        // the tensor-core kernel needs no workspace; one that is given must be 256-byte aligned
        HSA_REQUIRE(a.ws == nullptr || a.ws_bytes == 0 || aligned(a.ws, 256), HSA_ERR_WORKSPACE,
                    "workspace must be 256-byte aligned");
        return cuda_status(hsa::launch_sparse_mla_tc(a, st), "sparse_mla_attn (tensor core)");
    }
    return cuda_status(hsa::launch_sparse_mla_simt(a, st), "sparse_mla_attn");
}

hsa_attn_args_t make_attn(const void* q, hsa_dtype_t q_dtype, int32_t H, int32_t D_qk, int32_t D_v,
                          const void* kv, hsa_dtype_t kv_dtype, const float* kv_scale,
                          int32_t kv_scale_group, const void* kv_rope, float softmax_scale, void* out,
                          hsa_dtype_t out_dtype, float* lse) {
    hsa_attn_args_t a;
    a.q = q;
    a.q_dtype = q_dtype;
    a.H = H;
    a.D_qk = D_qk;
    a.D_v = D_v;
    a.kv = kv;
    a.kv_dtype = kv_dtype;
    a.kv_scale = kv_scale;
    a.kv_scale_group = kv_scale_group;
    a.kv_rope = kv_rope;
    a.softmax_scale = softmax_scale;
    a.out = out;
    a.out_dtype = out_dtype;
    a.lse = lse;
    return a;
}

// Host-side checks of the cache-write quantizers (shared by their entry points and the prolog,
// which checks every operator before it enqueues any).  D_rope = 0 and rope = NULL for index
// keys.
hsa_status_t check_quantize_rows(const void* src, hsa_dtype_t src_dtype, int64_t n_rows, int32_t D,
                                 int32_t D_rope, int32_t group, const int64_t* slot_mapping,
                                 int64_t num_slots, const uint8_t* codes, const float* scales,
                                 const void* rope) {
    HSA_REQUIRE(src_dtype == HSA_F32 || src_dtype == HSA_BF16, HSA_ERR_UNSUPPORTED,
                "source dtype must be F32 or BF16");
    HSA_REQUIRE(n_rows >= 0 && D >= 1 && D_rope >= 0 && group >= 1 && D % group == 0,
                HSA_ERR_INVALID_ARG, "need n_rows >= 0, D >= 1, D_rope >= 0, group | D "
                "(n_rows=%lld D=%d group=%d)", (long long)n_rows, D, group);
    HSA_REQUIRE(num_slots >= 0 && (slot_mapping || n_rows <= num_slots), HSA_ERR_INVALID_ARG,
                "identity slot mapping needs n_rows <= num_slots");
    if (n_rows == 0) return HSA_OK;
    HSA_REQUIRE(src && codes && scales && (D_rope == 0 || rope), HSA_ERR_INVALID_ARG,
                "NULL tensor pointer");
    HSA_REQUIRE(aligned(src, dtype_size(src_dtype)) && aligned(scales, 4) &&
                    (D_rope == 0 || aligned(rope, 2)) &&
                    (slot_mapping == nullptr || aligned(slot_mapping, 8)),
                HSA_ERR_INVALID_ARG, "misaligned source, scales, rope cache or slot mapping");
    return HSA_OK;
}

hsa_status_t check_quantize_mx(const void* src, hsa_dtype_t src_dtype, int64_t n_rows, int32_t D,
                               const int64_t* slot_mapping, int64_t num_slots, const uint8_t* codes,
                               const uint8_t* scales) {
    HSA_REQUIRE(src_dtype == HSA_F32 || src_dtype == HSA_BF16, HSA_ERR_UNSUPPORTED,
                "source dtype must be F32 or BF16");
    HSA_REQUIRE(n_rows >= 0 && D >= 32 && D % 32 == 0, HSA_ERR_INVALID_ARG,
                "need n_rows >= 0 and D a positive multiple of 32 (n_rows=%lld D=%d)",
                (long long)n_rows, D);
    HSA_REQUIRE(num_slots >= 0 && (slot_mapping || n_rows <= num_slots), HSA_ERR_INVALID_ARG,
                "identity slot mapping needs n_rows <= num_slots");
    if (n_rows == 0) return HSA_OK;
    HSA_REQUIRE(src && codes && scales, HSA_ERR_INVALID_ARG, "NULL tensor pointer");
    HSA_REQUIRE(aligned(src, dtype_size(src_dtype)) &&
                    (slot_mapping == nullptr || aligned(slot_mapping, 8)),
                HSA_ERR_INVALID_ARG, "misaligned source or slot mapping");
    return HSA_OK;
}

hsa_status_t check_mx_round(const void* src, hsa_dtype_t src_dtype, int64_t n_rows, int32_t D,
                            const void* dst, hsa_dtype_t dst_dtype) {
    HSA_REQUIRE((src_dtype == HSA_F32 || src_dtype == HSA_BF16) &&
                    (dst_dtype == HSA_F32 || dst_dtype == HSA_BF16),
                HSA_ERR_UNSUPPORTED, "source and destination dtypes must be F32 or BF16");
    HSA_REQUIRE(n_rows >= 0 && D >= 32 && D % 32 == 0, HSA_ERR_INVALID_ARG,
                "need n_rows >= 0 and D a positive multiple of 32 (n_rows=%lld D=%d)",
                (long long)n_rows, D);
    if (n_rows == 0) return HSA_OK;
    HSA_REQUIRE(src && dst, HSA_ERR_INVALID_ARG, "NULL tensor pointer");
    HSA_REQUIRE(aligned(src, dtype_size(src_dtype)) && aligned(dst, dtype_size(dst_dtype)),
                HSA_ERR_INVALID_ARG, "misaligned source or destination");
    const uintptr_t s0 = reinterpret_cast<uintptr_t>(src), d0 = reinterpret_cast<uintptr_t>(dst);
    const uintptr_t s1 = s0 + (uintptr_t)n_rows * D * dtype_size(src_dtype);
    const uintptr_t d1 = d0 + (uintptr_t)n_rows * D * dtype_size(dst_dtype);
    HSA_REQUIRE(s0 == d0 ? src_dtype == dst_dtype : (d1 <= s0 || s1 <= d0), HSA_ERR_INVALID_ARG,
                "source and destination overlap");
    return HSA_OK;
}

}  // namespace

uint64_t& hsa::launch_counter() {
    thread_local uint64_t n = 0;
    return n;
}

extern "C" {

uint64_t hsa_launch_count(void) { return hsa::launch_counter(); }

const char* hsa_status_string(hsa_status_t s) {
    switch (s) {
        case HSA_OK: return "HSA_OK";
        case HSA_ERR_INVALID_ARG: return "HSA_ERR_INVALID_ARG";
        case HSA_ERR_UNSUPPORTED: return "HSA_ERR_UNSUPPORTED";
        case HSA_ERR_CUDA: return "HSA_ERR_CUDA";
        case HSA_ERR_WORKSPACE: return "HSA_ERR_WORKSPACE";
    }
    return "HSA_ERR_UNKNOWN";
}

const char* hsa_last_error_message(void) { return g_last_error.c_str(); }

int32_t hsa_version(void) { return 400; }

hsa_status_t hsa_index_score(const hsa_paged_seq_t* seq, const void* q_I, hsa_dtype_t q_dtype,
                             const float* w, int32_t H_I, int32_t D_I, const void* k_cache,
                             hsa_dtype_t k_dtype, const void* k_scale, float* scores,
                             int64_t ld_scores, void* stream) {
    g_last_error.clear();
    hsa_status_t st = check_index(seq, q_I, q_dtype, nullptr, w, H_I, D_I, k_cache, k_dtype,
                                  k_scale, scores, ld_scores);
    if (st != HSA_OK) return st;
    return run_index(index_args(seq, q_I, q_dtype, nullptr, w, H_I, D_I, k_cache, k_dtype, k_scale,
                                scores, ld_scores),
                     (cudaStream_t)stream);
}

hsa_status_t hsa_index_score_mx(const hsa_paged_seq_t* seq, const uint8_t* q_codes,
                                const uint8_t* q_scale, const float* w, int32_t H_I, int32_t D_I,
                                const uint8_t* k_codes, const uint8_t* k_scale, float* scores,
                                int64_t ld_scores, void* stream) {
    g_last_error.clear();
    hsa_status_t st = check_index(seq, q_codes, HSA_MXE4M3, q_scale, w, H_I, D_I, k_codes,
                                  HSA_MXE4M3, k_scale, scores, ld_scores);
    if (st != HSA_OK) return st;
    return run_index(index_args(seq, q_codes, HSA_MXE4M3, q_scale, w, H_I, D_I, k_codes,
                                HSA_MXE4M3, k_scale, scores, ld_scores),
                     (cudaStream_t)stream);
}

hsa_status_t hsa_topk(const hsa_paged_seq_t* seq, const float* scores, int64_t ld_scores,
                      int32_t K, int32_t* idx, void* stream) {
    g_last_error.clear();
    hsa_status_t st = check_seq(seq);
    if (st != HSA_OK) return st;
    HSA_REQUIRE(K >= 1 && K <= 65536, HSA_ERR_INVALID_ARG, "K = %d out of range", K);
    HSA_REQUIRE(ld_scores >= seq->max_seq_len, HSA_ERR_INVALID_ARG, "ld_scores < max_seq_len");
    if (seq->T_q == 0) return HSA_OK;
    HSA_REQUIRE(scores && idx && aligned(scores, 4) && aligned(idx, 4), HSA_ERR_INVALID_ARG,
                "NULL or misaligned scores / idx");
    return cuda_status(hsa::launch_topk(view(seq), seq->max_seq_len, scores, ld_scores, K, idx,
                                        (cudaStream_t)stream),
                       "topk");
}

hsa_status_t hsa_topk_blocks(const hsa_paged_seq_t* seq, const float* scores, int64_t ld_scores,
                             int32_t K, int32_t block, int32_t* idx, void* stream) {
    g_last_error.clear();
    hsa_status_t st = check_seq(seq);
    if (st != HSA_OK) return st;
    HSA_REQUIRE(K >= 1 && K <= 65536, HSA_ERR_INVALID_ARG, "K = %d out of range", K);
    HSA_REQUIRE(block >= 8 && block <= K && K % block == 0, HSA_ERR_INVALID_ARG,
                "block = %d must be >= 8 and divide K = %d", block, K);
    HSA_REQUIRE(ld_scores >= seq->max_seq_len, HSA_ERR_INVALID_ARG, "ld_scores < max_seq_len");
    HSA_REQUIRE(hsa::topk_blocks_smem(seq->max_seq_len, K, block) <= 227 * 1024, HSA_ERR_UNSUPPORTED,
                "max_seq_len / block = %d blocks per row is too many", (int)hsa::ceil_div(seq->max_seq_len, block));
    if (seq->T_q == 0) return HSA_OK;
    HSA_REQUIRE(scores && idx && aligned(scores, 4) && aligned(idx, 4), HSA_ERR_INVALID_ARG,
                "NULL or misaligned scores / idx");
    return cuda_status(hsa::launch_topk_blocks(view(seq), seq->max_seq_len, scores, ld_scores, K,
                                               block, idx, (cudaStream_t)stream),
                       "topk_blocks");
}

size_t hsa_sparse_mla_workspace_size(const hsa_paged_seq_t* seq, int32_t H, int32_t D_qk,
                                     int32_t D_v, int32_t K) {
    if (seq == nullptr || seq->T_q <= 0) return 0;
    // the tensor-core kernel's need only depends on the shape, not on the pointers
    hsa_attn_args_t at = make_attn(nullptr, HSA_BF16, H, D_qk, D_v, nullptr, HSA_BF16, nullptr,
                                   D_v, nullptr, 1.f, nullptr, HSA_BF16, nullptr);
    return attn_ws_bytes(attn_args(seq, at, nullptr, K, nullptr, 0));
}

hsa_status_t hsa_sparse_mla_attn(const hsa_paged_seq_t* seq, const void* q, hsa_dtype_t q_dtype,
                                 int32_t H, int32_t D_qk, int32_t D_v, const void* kv,
                                 hsa_dtype_t kv_dtype, const float* kv_scale, int32_t kv_scale_group,
                                 const void* kv_rope, const int32_t* idx, int32_t K,
                                 float softmax_scale, void* out,
                                 hsa_dtype_t out_dtype, float* lse, void* ws, size_t ws_bytes,
                                 void* stream) {
    g_last_error.clear();
    hsa_status_t st = check_attn(seq, q, q_dtype, H, D_qk, D_v, kv, kv_dtype, kv_scale, kv_scale_group, kv_rope,
                                 idx, K, out, out_dtype);
    if (st != HSA_OK) return st;
    hsa_attn_args_t at = make_attn(q, q_dtype, H, D_qk, D_v, kv, kv_dtype, kv_scale, kv_scale_group, kv_rope,
                                   softmax_scale, out, out_dtype, lse);
    return run_attn(attn_args(seq, at, idx, K, ws, ws_bytes), (cudaStream_t)stream);
}

size_t hsa_fused_decode_workspace_size(const hsa_paged_seq_t* seq, const hsa_attn_args_t* attn,
                                       int32_t K) {
    if (seq == nullptr || attn == nullptr || seq->T_q <= 0) return 0;
    // each half of a two-stream call needs its own region; the sum of the halves' needs is
    // reported (the workspace need grows with the row count), rounded to 256 bytes each
    const int32_t t1 = seq->T_q / 2;
    hsa_paged_seq_t a = sub_rows(*seq, 0, t1), b = sub_rows(*seq, t1, seq->T_q - t1);
    size_t na = t1 > 0 ? attn_ws_bytes(attn_args(&a, *attn, nullptr, K, nullptr, 0)) : 0;
    size_t nb = attn_ws_bytes(attn_args(&b, *attn, nullptr, K, nullptr, 0));
    size_t nall = attn_ws_bytes(attn_args(seq, *attn, nullptr, K, nullptr, 0));
    na = (na + 255) / 256 * 256;
    nb = (nb + 255) / 256 * 256;
    return na + nb > nall ? na + nb : nall;
}

hsa_status_t hsa_fused_decode(const hsa_paged_seq_t* seq, const hsa_index_args_t* ix,
                              const hsa_attn_args_t* at, int32_t K, float* scores,
                              int64_t ld_scores, int32_t* idx, void* ws, size_t ws_bytes,
                              void* stream_main, void* stream_aux) {
    g_last_error.clear();
    HSA_REQUIRE(ix && at, HSA_ERR_INVALID_ARG, "index / attn args NULL");
    hsa_status_t st = check_index(seq, ix->q_I, ix->q_dtype, ix->q_scale, ix->w, ix->H_I, ix->D_I,
                                  ix->k_cache, ix->k_dtype, ix->k_scale, scores, ld_scores);
    if (st != HSA_OK) return st;
    st = check_attn(seq, at->q, at->q_dtype, at->H, at->D_qk, at->D_v, at->kv, at->kv_dtype,
                    at->kv_scale, at->kv_scale_group, at->kv_rope, idx, K, at->out, at->out_dtype);
    if (st != HSA_OK) return st;
    HSA_REQUIRE(K >= 1 && K <= 65536, HSA_ERR_INVALID_ARG, "K = %d out of range", K);
    if (seq->T_q == 0) return HSA_OK;
    HSA_REQUIRE(idx && aligned(idx, 4), HSA_ERR_INVALID_ARG, "idx NULL or misaligned");
    HSA_REQUIRE(ws == nullptr || ws_bytes == 0 || aligned(ws, 256), HSA_ERR_WORKSPACE,
                "workspace must be 256-byte aligned");

    cudaStream_t s0 = (cudaStream_t)stream_main, s1 = (cudaStream_t)stream_aux;
    // split point: half the rows, on a run boundary so no run is cut
    int32_t t1 = seq->T_q / 2;
    t1 -= t1 % seq->q_run;
    const bool two = s1 != nullptr && t1 > 0 && t1 < seq->T_q;

    auto one_part = [&](int32_t r0, int32_t n, void* pws, size_t pws_bytes, cudaStream_t s,
                        cudaEvent_t after_topk) -> hsa_status_t {
        hsa_paged_seq_t part = sub_rows(*seq, r0, n);
        const size_t qI = (size_t)r0 * ix->H_I * ix->D_I * dtype_size(ix->q_dtype);
        const void* qs = ix->q_dtype == HSA_MXE4M3
                             ? static_cast<const char*>(ix->q_scale) + (size_t)r0 * ix->H_I * (ix->D_I / 32)
                             : nullptr;
        hsa::IndexScoreArgs ia = index_args(
            &part, static_cast<const char*>(ix->q_I) + qI, ix->q_dtype, qs, ix->w + (size_t)r0 * ix->H_I,
            ix->H_I, ix->D_I, ix->k_cache, ix->k_dtype, ix->k_scale, scores + (size_t)r0 * ld_scores,
            ld_scores);
        hsa_status_t r = run_index(ia, s);
        if (r != HSA_OK) return r;
        r = cuda_status(hsa::launch_topk(view(&part), part.max_seq_len,
                                         scores + (size_t)r0 * ld_scores, ld_scores, K,
                                         idx + (size_t)r0 * K, s),
                        "topk");
        if (r != HSA_OK) return r;
        if (after_topk) {
            r = cuda_status(cudaEventRecord(after_topk, s), "cudaEventRecord");
            if (r != HSA_OK) return r;
        }
        hsa_attn_args_t pa = *at;
        pa.q = static_cast<const char*>(at->q) + (size_t)r0 * at->H * at->D_qk * dtype_size(at->q_dtype);
        pa.out = static_cast<char*>(at->out) + (size_t)r0 * at->H * at->D_v * dtype_size(at->out_dtype);
        pa.lse = at->lse ? at->lse + (size_t)r0 * at->H : nullptr;
        return run_attn(attn_args(&part, pa, idx + (size_t)r0 * K, K, pws, pws_bytes), s);
    };

    if (!two) return one_part(0, seq->T_q, ws, ws_bytes, s0, nullptr);

    // stream_main: rows [0, t1) index -> topk -> (event) -> attention
    // stream_aux : waits for that event, then rows [t1, T_q) index -> topk -> attention, so the
    //              second half's index stream overlaps the first half's attention
    cudaEvent_t ev_topk = nullptr, ev_done = nullptr;
    hsa_status_t r = cuda_status(cudaEventCreateWithFlags(&ev_topk, cudaEventDisableTiming), "event");
    if (r == HSA_OK) r = cuda_status(cudaEventCreateWithFlags(&ev_done, cudaEventDisableTiming), "event");
    hsa_paged_seq_t first = sub_rows(*seq, 0, t1);
    size_t ws0 = attn_ws_bytes(attn_args(&first, *at, nullptr, K, nullptr, 0));
    ws0 = (ws0 + 255) / 256 * 256;
    // each half takes its own region; a workspace too small for a half runs it with whole rows
    const bool ws_a = ws != nullptr && ws_bytes >= ws0;
    if (r == HSA_OK) r = one_part(0, t1, ws_a ? ws : nullptr, ws_a ? ws0 : 0, s0, ev_topk);
    if (r == HSA_OK) r = cuda_status(cudaStreamWaitEvent(s1, ev_topk, 0), "cudaStreamWaitEvent");
    if (r == HSA_OK)
        r = one_part(t1, seq->T_q - t1, ws_a ? static_cast<char*>(ws) + ws0 : nullptr,
                     ws_a ? ws_bytes - ws0 : 0, s1, nullptr);
    if (r == HSA_OK) r = cuda_status(cudaEventRecord(ev_done, s1), "cudaEventRecord");
    if (r == HSA_OK) r = cuda_status(cudaStreamWaitEvent(s0, ev_done, 0), "cudaStreamWaitEvent");
    if (ev_topk) cudaEventDestroy(ev_topk);
    if (ev_done) cudaEventDestroy(ev_done);
    return r;
}

hsa_status_t hsa_prefill_chunked(const hsa_paged_seq_t* seq, const hsa_index_args_t* ix,
                                 const hsa_attn_args_t* at, int32_t K, const int32_t* chunks,
                                 int32_t n_chunks, float* const* score_bufs, int32_t score_rows,
                                 int64_t ld_scores, int32_t* idx, void* stream, void* stream_a,
                                 void* stream_b) {
    g_last_error.clear();
    HSA_REQUIRE(ix && at, HSA_ERR_INVALID_ARG, "index / attn args NULL");
    HSA_REQUIRE(n_chunks >= 0 && (n_chunks == 0 || chunks), HSA_ERR_INVALID_ARG, "chunks NULL");
    HSA_REQUIRE(score_bufs && score_bufs[0] && score_bufs[1], HSA_ERR_INVALID_ARG,
                "two score buffers are needed");
    hsa_status_t st = check_index(seq, ix->q_I, ix->q_dtype, ix->q_scale, ix->w, ix->H_I, ix->D_I,
                                  ix->k_cache, ix->k_dtype, ix->k_scale, score_bufs[0], ld_scores);
    if (st != HSA_OK) return st;
    st = check_attn(seq, at->q, at->q_dtype, at->H, at->D_qk, at->D_v, at->kv, at->kv_dtype,
                    at->kv_scale, at->kv_scale_group, at->kv_rope, idx, K, at->out, at->out_dtype);
    if (st != HSA_OK) return st;
    HSA_REQUIRE(idx && aligned(idx, 4) && aligned(score_bufs[1], 4), HSA_ERR_INVALID_ARG,
                "idx NULL or a buffer misaligned");
    for (int32_t i = 0; i < n_chunks; ++i) {
        const int32_t r0 = chunks[2 * i], r1 = chunks[2 * i + 1];
        HSA_REQUIRE(0 <= r0 && r0 < r1 && r1 <= seq->T_q, HSA_ERR_INVALID_ARG,
                    "chunk %d = [%d, %d) outside [0, T_q = %d) or empty", i, r0, r1, seq->T_q);
        HSA_REQUIRE(r1 - r0 <= score_rows, HSA_ERR_INVALID_ARG,
                    "chunk %d has %d rows; the score buffers hold %d", i, r1 - r0, score_rows);
    }
    if (n_chunks == 0 || seq->T_q == 0) return HSA_OK;

    cudaStream_t s0 = (cudaStream_t)stream;
    const cudaStream_t side[2] = {stream_a ? (cudaStream_t)stream_a : s0,
                                  stream_b ? (cudaStream_t)stream_b : s0};
    cudaEvent_t ev[3] = {nullptr, nullptr, nullptr};
    hsa_status_t r = HSA_OK;
    for (int i = 0; i < 3 && r == HSA_OK; ++i)
        r = cuda_status(cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming), "cudaEventCreate");
    // fork: both side streams start after the work already on `stream`
    if (r == HSA_OK) r = cuda_status(cudaEventRecord(ev[0], s0), "cudaEventRecord");
    for (int i = 0; i < 2 && r == HSA_OK; ++i)
        if (side[i] != s0) r = cuda_status(cudaStreamWaitEvent(side[i], ev[0], 0), "cudaStreamWaitEvent");
    const size_t qsz = dtype_size(ix->q_dtype), asz = dtype_size(at->q_dtype), osz = dtype_size(at->out_dtype);
    for (int32_t i = 0; i < n_chunks && r == HSA_OK; ++i) {
        const int32_t r0 = chunks[2 * i], n = chunks[2 * i + 1] - r0;
        cudaStream_t s = side[i & 1];
        hsa_paged_seq_t part = sub_rows(*seq, r0, n);
        part.q_run = seq->q_run < n ? seq->q_run : n;
        float* sc = score_bufs[i & 1];
        const void* qs = ix->q_dtype == HSA_MXE4M3
                             ? static_cast<const char*>(ix->q_scale) + (size_t)r0 * ix->H_I * (ix->D_I / 32)
                             : nullptr;
        r = run_index(index_args(&part, static_cast<const char*>(ix->q_I) + (size_t)r0 * ix->H_I * ix->D_I * qsz,
                                 ix->q_dtype, qs, ix->w + (size_t)r0 * ix->H_I, ix->H_I, ix->D_I,
                                 ix->k_cache, ix->k_dtype, ix->k_scale, sc, ld_scores),
                      s);
        if (r != HSA_OK) break;
        r = cuda_status(hsa::launch_topk(view(&part), part.max_seq_len, sc, ld_scores, K,
                                         idx + (size_t)r0 * K, s),
                        "topk");
        if (r != HSA_OK) break;
        hsa_attn_args_t pa = *at;
        pa.q = static_cast<const char*>(at->q) + (size_t)r0 * at->H * at->D_qk * asz;
        pa.out = static_cast<char*>(at->out) + (size_t)r0 * at->H * at->D_v * osz;
        pa.lse = at->lse ? at->lse + (size_t)r0 * at->H : nullptr;
        r = run_attn(attn_args(&part, pa, idx + (size_t)r0 * K, K, nullptr, 0), s);
    }
    // join (also after a failed launch, so that nothing enqueued is left unordered)
    for (int i = 0; i < 2; ++i) {
        if (side[i] == s0 || ev[1 + i] == nullptr || ev[0] == nullptr) continue;
        hsa_status_t e = cuda_status(cudaEventRecord(ev[1 + i], side[i]), "cudaEventRecord");
        if (e == HSA_OK) e = cuda_status(cudaStreamWaitEvent(s0, ev[1 + i], 0), "cudaStreamWaitEvent");
        if (r == HSA_OK) r = e;
    }
    for (int i = 0; i < 3; ++i)
        if (ev[i]) cudaEventDestroy(ev[i]);
    return r;
}

hsa_status_t hsa_quantize_index(const void* src, hsa_dtype_t src_dtype, int64_t n_rows,
                                int32_t D, int32_t group, const int64_t* slot_mapping,
                                int64_t num_slots, uint8_t* codes, float* scales, void* stream) {
    g_last_error.clear();
    hsa_status_t st = check_quantize_rows(src, src_dtype, n_rows, D, 0, group, slot_mapping,
                                          num_slots, codes, scales, nullptr);
    if (st != HSA_OK || n_rows == 0) return st;
    return cuda_status(hsa::launch_quantize_rows(src, src_dtype, n_rows, D, D, group, slot_mapping,
                                                 num_slots, codes, scales, 0, nullptr,
                                                 (cudaStream_t)stream),
                       "quantize_index");
}

hsa_status_t hsa_quantize_kv(const void* src, hsa_dtype_t src_dtype, int64_t n_rows, int32_t D_v,
                             int32_t D_rope, int32_t group, const int64_t* slot_mapping,
                             int64_t num_slots, uint8_t* codes, float* scales, void* rope_cache,
                             void* stream) {
    g_last_error.clear();
    hsa_status_t st = check_quantize_rows(src, src_dtype, n_rows, D_v, D_rope, group, slot_mapping,
                                          num_slots, codes, scales, rope_cache);
    if (st != HSA_OK || n_rows == 0) return st;
    return cuda_status(hsa::launch_quantize_rows(src, src_dtype, n_rows, D_v + D_rope, D_v, group,
                                                 slot_mapping, num_slots, codes, scales, D_rope,
                                                 rope_cache, (cudaStream_t)stream),
                       "quantize_kv");
}

hsa_status_t hsa_quantize_mx(const void* src, hsa_dtype_t src_dtype, int64_t n_rows, int32_t D,
                             const int64_t* slot_mapping, int64_t num_slots, uint8_t* codes,
                             uint8_t* scales, void* stream) {
    g_last_error.clear();
    hsa_status_t st = check_quantize_mx(src, src_dtype, n_rows, D, slot_mapping, num_slots, codes,
                                        scales);
    if (st != HSA_OK || n_rows == 0) return st;
    return cuda_status(hsa::launch_quantize_mx(src, src_dtype, n_rows, D, slot_mapping, num_slots,
                                               codes, scales, (cudaStream_t)stream),
                       "quantize_mx");
}

hsa_status_t hsa_dequantize_mx(const uint8_t* codes, const uint8_t* scales, int64_t n_rows,
                               int32_t D, void* dst, hsa_dtype_t dst_dtype, void* stream) {
    g_last_error.clear();
    HSA_REQUIRE(dst_dtype == HSA_F32 || dst_dtype == HSA_BF16, HSA_ERR_UNSUPPORTED,
                "destination dtype must be F32 or BF16");
    HSA_REQUIRE(n_rows >= 0 && D >= 32 && D % 32 == 0, HSA_ERR_INVALID_ARG,
                "need n_rows >= 0 and D a positive multiple of 32 (n_rows=%lld D=%d)",
                (long long)n_rows, D);
    if (n_rows == 0) return HSA_OK;
    HSA_REQUIRE(codes && scales && dst, HSA_ERR_INVALID_ARG, "NULL tensor pointer");
    HSA_REQUIRE(aligned(dst, dtype_size(dst_dtype)), HSA_ERR_INVALID_ARG, "misaligned destination");
    return cuda_status(hsa::launch_dequantize_mx(codes, scales, n_rows, D, dst, dst_dtype,
                                                 (cudaStream_t)stream),
                       "dequantize_mx");
}

hsa_status_t hsa_mx_round(const void* src, hsa_dtype_t src_dtype, int64_t n_rows, int32_t D,
                          void* dst, hsa_dtype_t dst_dtype, void* stream) {
    g_last_error.clear();
    hsa_status_t st = check_mx_round(src, src_dtype, n_rows, D, dst, dst_dtype);
    if (st != HSA_OK || n_rows == 0) return st;
    return cuda_status(hsa::launch_mx_round(src, src_dtype, n_rows, D, dst, dst_dtype,
                                            (cudaStream_t)stream),
                       "mx_round");
}

hsa_status_t hsa_decode_prolog(const hsa_prolog_args_t* a, void* stream, void* stream_k,
                               void* stream_kv, void* stream_q) {
    g_last_error.clear();
    HSA_REQUIRE(a != nullptr, HSA_ERR_INVALID_ARG, "prolog args NULL");
    HSA_REQUIRE(a->n_new >= 0 && a->q_rows >= 0, HSA_ERR_INVALID_ARG, "need n_new >= 0, q_rows >= 0");
    HSA_REQUIRE(a->k_dtype == HSA_MXE4M3 || a->k_dtype == HSA_E4M3, HSA_ERR_UNSUPPORTED,
                "index key cache must be MXE4M3 or E4M3");
    HSA_REQUIRE(a->n_new == 0 || a->slot_mapping, HSA_ERR_INVALID_ARG, "slot_mapping NULL");
    // every operator's arguments are checked before anything is enqueued or any stream forked
    hsa_status_t st = HSA_OK;
    if (a->k_dtype == HSA_MXE4M3)
        st = check_quantize_mx(a->new_k, a->new_k_dtype, a->n_new, a->D_I, a->slot_mapping,
                               a->num_slots, a->k_cache, static_cast<uint8_t*>(a->k_scale));
    else
        st = check_quantize_rows(a->new_k, a->new_k_dtype, a->n_new, a->D_I, 0, a->D_I,
                                 a->slot_mapping, a->num_slots, a->k_cache,
                                 static_cast<float*>(a->k_scale), nullptr);
    if (st != HSA_OK) return st;
    st = check_quantize_rows(a->new_kv, a->new_kv_dtype, a->n_new, a->D_v, a->D_rope, a->kv_group,
                             a->slot_mapping, a->num_slots, a->kv_cache, a->kv_scale, a->kv_rope);
    if (st != HSA_OK) return st;
    const bool want_q = a->q_I_out != nullptr && a->q_rows > 0;
    if (want_q) {
        st = check_mx_round(a->q_I, a->q_I_dtype, a->q_rows, a->D_I, a->q_I_out, HSA_BF16);
        if (st != HSA_OK) return st;
    }
    const bool want_qc = a->q_codes_out != nullptr && a->q_rows > 0;
    if (want_qc) {
        st = check_quantize_mx(a->q_I, a->q_I_dtype, a->q_rows, a->D_I, nullptr, a->q_rows,
                               a->q_codes_out, a->q_scale_out);
        if (st != HSA_OK) return st;
    }
    cudaStream_t s0 = (cudaStream_t)stream;
    const cudaStream_t side[3] = {stream_k ? (cudaStream_t)stream_k : s0,
                                  stream_kv ? (cudaStream_t)stream_kv : s0,
                                  stream_q ? (cudaStream_t)stream_q : s0};
    cudaEvent_t ev[4] = {nullptr, nullptr, nullptr, nullptr};
    hsa_status_t r = HSA_OK;
    for (int i = 0; i < 4 && r == HSA_OK; ++i)
        r = cuda_status(cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming), "cudaEventCreate");
    // fork: each side stream starts after the work already on the main stream
    if (r == HSA_OK) r = cuda_status(cudaEventRecord(ev[0], s0), "cudaEventRecord");
    for (int i = 0; i < 3 && r == HSA_OK; ++i)
        if (side[i] != s0) r = cuda_status(cudaStreamWaitEvent(side[i], ev[0], 0), "cudaStreamWaitEvent");
    if (r == HSA_OK && a->n_new > 0) {
        if (a->k_dtype == HSA_MXE4M3)
            r = cuda_status(hsa::launch_quantize_mx(a->new_k, a->new_k_dtype, a->n_new, a->D_I,
                                                    a->slot_mapping, a->num_slots, a->k_cache,
                                                    static_cast<uint8_t*>(a->k_scale), side[0]),
                            "quantize_mx");
        else
            r = cuda_status(hsa::launch_quantize_rows(a->new_k, a->new_k_dtype, a->n_new, a->D_I,
                                                      a->D_I, a->D_I, a->slot_mapping, a->num_slots,
                                                      a->k_cache, static_cast<float*>(a->k_scale),
                                                      0, nullptr, side[0]),
                            "quantize_index");
        if (r == HSA_OK)
            r = cuda_status(hsa::launch_quantize_rows(a->new_kv, a->new_kv_dtype, a->n_new,
                                                      a->D_v + a->D_rope, a->D_v, a->kv_group,
                                                      a->slot_mapping, a->num_slots, a->kv_cache,
                                                      a->kv_scale, a->D_rope, a->kv_rope, side[1]),
                            "quantize_kv");
    }
    if (r == HSA_OK && want_q)
        r = cuda_status(hsa::launch_mx_round(a->q_I, a->q_I_dtype, a->q_rows, a->D_I, a->q_I_out,
                                             HSA_BF16, side[2]),
                        "mx_round");
    if (r == HSA_OK && want_qc)
        r = cuda_status(hsa::launch_quantize_mx(a->q_I, a->q_I_dtype, a->q_rows, a->D_I, nullptr,
                                                a->q_rows, a->q_codes_out, a->q_scale_out, side[2]),
                        "quantize_mx (queries)");
    // join (also after a failed launch, so that nothing enqueued is left unordered)
    for (int i = 0; i < 3; ++i) {
        if (side[i] == s0 || ev[1 + i] == nullptr || ev[0] == nullptr) continue;
        hsa_status_t e = cuda_status(cudaEventRecord(ev[1 + i], side[i]), "cudaEventRecord");
        if (e == HSA_OK) e = cuda_status(cudaStreamWaitEvent(s0, ev[1 + i], 0), "cudaStreamWaitEvent");
        if (r == HSA_OK) r = e;
    }
    for (int i = 0; i < 4; ++i)
        if (ev[i]) cudaEventDestroy(ev[i]);
    return r;
}

}  // extern "C"

// ---- the fused decode step without allocation -------------------------------------------------
// Scratch of hsa_fused_decode_noalloc: the step's scores, then its selections.  Every GPU on which
// the library's kernels are loaded holds these 40 MiB from then until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(40) << 20;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mutex;
uint8_t* g_noalloc_ptr[kNoAllocMaxDevices];   // the scratch's address on each device, once known

// The scratch's device address on the current device; the first call on a device looks it up
// (with that device current) and keeps it.
hsa_status_t noalloc_scratch(uint8_t** p) {
    int dev = -1;
    hsa_status_t r = cuda_status(cudaGetDevice(&dev), "cudaGetDevice");
    if (r != HSA_OK) return r;
    HSA_REQUIRE(dev >= 0 && dev < kNoAllocMaxDevices, HSA_ERR_UNSUPPORTED,
                "device %d: the no-allocation entry serves devices 0..%d", dev, kNoAllocMaxDevices - 1);
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* q = nullptr;
        r = cuda_status(cudaGetSymbolAddress(&q, g_noalloc_scratch), "cudaGetSymbolAddress (scratch)");
        if (r != HSA_OK) return r;
        g_noalloc_ptr[dev] = static_cast<uint8_t*>(q);
    }
    *p = g_noalloc_ptr[dev];
    return HSA_OK;
}

}  // namespace

extern "C" {

hsa_status_t hsa_fused_decode_noalloc(const hsa_paged_seq_t* seq, const hsa_index_args_t* ix,
                                      const hsa_attn_args_t* at, int32_t K, void* stream) {
    g_last_error.clear();
    HSA_REQUIRE(seq && ix && at, HSA_ERR_INVALID_ARG, "seq / index / attn args NULL");
    HSA_REQUIRE(seq->T_q >= 0 && seq->max_seq_len >= 1, HSA_ERR_INVALID_ARG,
                "T_q = %d, max_seq_len = %d", seq->T_q, seq->max_seq_len);
    HSA_REQUIRE(K >= 1 && K <= 65536, HSA_ERR_INVALID_ARG, "K = %d out of range", K);
    // scores [T_q, ld] fp32 (rows 16-byte aligned), then idx [T_q, K] int32
    const int64_t ld = ((int64_t)seq->max_seq_len + 3) / 4 * 4;
    const size_t score_bytes = ((size_t)seq->T_q * ld * 4 + 255) / 256 * 256;
    const size_t idx_bytes = ((size_t)seq->T_q * K * 4 + 255) / 256 * 256;
    HSA_REQUIRE(score_bytes + idx_bytes <= kNoAllocScratchBytes, HSA_ERR_WORKSPACE,
                "T_q = %d rows, max_seq_len = %d and K = %d need %zu bytes of scratch; the "
                "no-allocation entry holds %zu",
                seq->T_q, seq->max_seq_len, K, score_bytes + idx_bytes, kNoAllocScratchBytes);
    uint8_t* scratch = nullptr;
    hsa_status_t r = noalloc_scratch(&scratch);
    if (r != HSA_OK) return r;
    return hsa_fused_decode(seq, ix, at, K, reinterpret_cast<float*>(scratch), ld,
                            reinterpret_cast<int32_t*>(scratch + score_bytes), nullptr, 0, stream,
                            nullptr);
}

}  // extern "C"
