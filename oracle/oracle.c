/*
 * oracle.c -- plain, slow, float64 CPU reference of the sparse index attention path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes or calls this
 * file; only the tests, the package's smoke check and the benchmark's CPU-baseline leg load it.
 * It shares no header, helper, table or constant with the CUDA code.
 *
 * Every input is widened exactly to double (bf16 and fp32 are subsets of double; an e4m3 code
 * is decoded from the OCP 8-bit floating point definition and multiplied by its fp32 scale,
 * which is exact in double).  Loops are written in the order the definitions read; OpenMP only
 * spreads independent query rows over host threads.
 *
 * Sources (page title, section):
 *  [P1]  "Day 0 Inference Adaptation and Optimization for Hybrid Attention Models",
 *        "Sparse Attention Pipeline Optimization" (indexer scores every history position,
 *        per-head scores combined with per-head weights, Top-K, sparse attention reading only
 *        the selected KV rows) and
 *        "Hierarchical Quantization" (index path 8-bit, KV cache FP8 block quantization).
 *  [P2]  "Efficient Inference Deployment and Optimization for Hybrid Attention LLMs",
 *        sections 3.1 (indexer then sparse attention), 4.1/4.2 (quantization granularity),
 *        5.2 (Zigzag layout).
 *  [P3]  "Day-One Inference Adaptation for Very Large Hybrid-Attention Models",
 *        section 3.1 (selection operator: index computation + causal mask, paged gather) and
 *        3.2 (sparse attention over the selected positions).
 *  [P5]  "Inference Adaptation and Performance Optimization for a Domestically Developed
 *        LLM's New Architecture", section 3 (LI scoring/weighting/Top-K, SFA) and the
 *        tiered quantization table of section 4.
 *
 * The pages never write the indexer as a formula.  The oracle uses
 *     I[t,s] = sum_j w[t,j] * ReLU( sum_d q_I[t,j,d] * k_I[s,d] ),   s <= p_t,
 * which is the plainest reading of the pages' per-head scoring followed by a weighted sum over
 * heads ([P1], [P5] s3), with one key per position shared by all index heads.
 *
 * Parity pins: see tests/test_oracle_*.py (closed forms, invariants, brute force, library
 * routines).  No function here is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_NOT_FINITE 2
#define ORACLE_SOFTMAX_SUM 3

/* ------------------------------------------------------------------------------------------
 * OCP 8-bit floating point, E4M3 variant.
 * 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits.  Exponent field 0 encodes
 * subnormals 2^-6 * m/8.  There are no infinities; S.1111.111 is NaN, so the largest finite
 * magnitude is S.1111.110 = 2^8 * 1.75 = 448.  ([P1] "Hierarchical Quantization": the KV cache
 * and index keys are stored in FP8.)
 * ------------------------------------------------------------------------------------------ */
double oracle_e4m3_decode(uint8_t code) {
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double mag;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, -6);
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* Round an fp32 value to the nearest E4M3 value, ties to the even code, saturating finite
 * overflow to +-448 (the "satfinite" behaviour).  Written from the definition above: find the
 * spacing of representable values at |x|, round |x| to a multiple of it with
 * round-half-to-even, then re-encode. */
uint8_t oracle_e4m3_encode(float xf) {
    double x = (double)xf;
    uint8_t sign = (x < 0.0 || (x == 0.0 && signbit(x))) ? 0x80 : 0x00;
    double a = fabs(x);
    if (isnan(x)) return 0x7F | sign;
    if (a == 0.0) return sign;
    double spacing;
    if (a < ldexp(1.0, -6)) {
        spacing = ldexp(1.0, -9);                    /* subnormal grid */
    } else {
        int ex;
        frexp(a, &ex);                               /* a = f * 2^ex, f in [0.5, 1) */
        spacing = ldexp(1.0, (ex - 1) - 3);          /* 3 mantissa bits below the leading one */
    }
    double q = a / spacing;                          /* exact: spacing is a power of two */
    double r = nearbyint(q);                         /* default mode: round half to even */
    double v = r * spacing;
    if (v > 448.0) v = 448.0;
    /* re-encode v (now exactly representable) */
    uint8_t bits;
    if (v < ldexp(1.0, -6)) {
        bits = (uint8_t)(int)(v / ldexp(1.0, -9));   /* e = 0, m = v / 2^-9 */
    } else {
        int ex;
        double f = frexp(v, &ex);                    /* v = f * 2^ex, f in [0.5,1) */
        int e = (ex - 1) + 7;
        int m = (int)((f * 2.0 - 1.0) * 8.0);
        bits = (uint8_t)((e << 3) | m);
    }
    return (uint8_t)(bits | sign);
}

/* Dynamic per-group quantization of rows to E4M3 with one fp32 scale per group.
 * [P1] "Hierarchical Quantization", [P2] 4.1/4.2, [P5] s4 table: the scale is computed from the
 * data at write time ("dynamic").  The pages do not print the scale rule; the reading taken is
 * the max-abs rule: scale = amax / 448 (fp32, round to nearest), the values are multiplied by
 * inv = 448 / amax (fp32, round to nearest) and rounded to E4M3 (for amax < 2^-64 both amax and
 * the values are first lifted by 2^64, see below).  amax == 0 gives scale 1 and all-zero codes.  fp32 division and multiplication are reproduced exactly by doing them in
 * double and rounding once to float (double carries more than 2*24+2 bits).
 *   x: [n_rows, D] (fp32-representable values), codes: [n_rows, D], scales: [n_rows, D/group]. */
int oracle_quantize_rows(const float* x, int64_t n_rows, int32_t D, int32_t group,
                         uint8_t* codes, float* scales) {
    if (n_rows < 0 || D <= 0 || group <= 0 || D % group != 0) return ORACLE_BAD_ARG;
    int32_t ng = D / group;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_rows; ++r) {
        for (int32_t g = 0; g < ng; ++g) {
            const float* xs = x + r * D + (int64_t)g * group;
            double amax = 0.0;
            for (int32_t i = 0; i < group; ++i) {
                double a = fabs((double)xs[i]);
                if (a > amax) amax = a;
            }
            /* A group maximum below 2^-64 is multiplied by 2^64 (exact) before 448/amax is
             * formed, and so are the group's values before they are multiplied by it: 448/amax
             * itself would overflow float32 for amax < 448/FLT_MAX, and a zero of the group
             * would then become 0 * inf = NaN.  Where 448/amax is finite both the reciprocal
             * and the products only move by an exact power of two, so the codes are the same
             * as without the lift. */
            const double lift = amax < 0x1p-64 ? 0x1p64 : 1.0;
            float scale, inv;
            if (amax == 0.0) {
                scale = 1.0f;
                inv = 0.0f;
            } else {
                scale = (float)(amax / 448.0);
                inv = (float)(448.0 / (amax * lift));
            }
            scales[r * ng + g] = scale;
            for (int32_t i = 0; i < group; ++i) {
                float y = (float)((double)xs[i] * lift * (double)inv);
                codes[r * D + (int64_t)g * group + i] = amax == 0.0 ? 0 : oracle_e4m3_encode(y);
            }
        }
    }
    return ORACLE_OK;
}

/* value = decode(code) * scale, per group, into double. */
int oracle_dequantize_rows(const uint8_t* codes, const float* scales, int64_t n_rows, int32_t D,
                           int32_t group, double* out) {
    if (n_rows < 0 || D <= 0 || group <= 0 || D % group != 0) return ORACLE_BAD_ARG;
    int32_t ng = D / group;
    for (int64_t r = 0; r < n_rows; ++r)
        for (int32_t i = 0; i < D; ++i)
            out[r * D + i] = oracle_e4m3_decode(codes[r * D + i]) * (double)scales[r * ng + i / group];
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------------------------
 * MXFP8 (OCP Microscaling formats, FP8 E4M3 elements): every block of 32 consecutive elements
 * shares one E8M0 scale byte E meaning 2^(E - 127) (E = 255 is NaN and never produced).  The
 * pages store the index Q/K this way: dynamic per-group quantization, group size 32, a shared
 * exponent ([P1] "Hierarchical Quantization"; [P2] 4.1; [P5] section 4 table).  The pages do
 * not spell out how the shared exponent is chosen; the reading taken is the MX rule:
 *     X = floor(log2(amax)) - 8        (8 = exponent of the top E4M3 binade: 448 = 1.75 * 2^8)
 * clamped to [-127, 127], E = X + 127, and each element becomes the E4M3 code of x / 2^X
 * (round to nearest even, finite overflow saturating to +-448).  An all-zero block gets E = 0
 * and zero codes.  x / 2^X is a power-of-two rescaling, exact in double, and exact as a float
 * whenever it is at least 2^-126; below that every candidate rounds to code 0 either way.
 *   x: [n_rows, D] fp32-representable, D a multiple of 32; codes [n_rows, D]; scales
 *   [n_rows, D / 32] (one byte each).
 * ------------------------------------------------------------------------------------------ */
int oracle_mx_quantize_rows(const float* x, int64_t n_rows, int32_t D, uint8_t* codes,
                            uint8_t* scales) {
    if (n_rows < 0 || D <= 0 || D % 32 != 0) return ORACLE_BAD_ARG;
    const int32_t nb = D / 32;
    for (int64_t i = 0; i < n_rows * (int64_t)D; ++i)   /* the MX rule is defined on finite data */
        if (!isfinite(x[i])) return ORACLE_NOT_FINITE;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_rows; ++r) {
        for (int32_t b = 0; b < nb; ++b) {
            const float* xs = x + r * D + (int64_t)b * 32;
            uint8_t* cs = codes + r * D + (int64_t)b * 32;
            double amax = 0.0;
            for (int i = 0; i < 32; ++i) {
                double a = fabs((double)xs[i]);
                if (a > amax) amax = a;
            }
            if (amax == 0.0) {
                scales[r * nb + b] = 0;
                for (int i = 0; i < 32; ++i) cs[i] = 0;
                continue;
            }
            int e2;
            frexp(amax, &e2);               /* amax = m * 2^e2, m in [0.5, 1) */
            int X = (e2 - 1) - 8;           /* floor(log2(amax)) - 8 */
            if (X < -127) X = -127;
            if (X > 127) X = 127;
            scales[r * nb + b] = (uint8_t)(X + 127);
            for (int i = 0; i < 32; ++i)
                cs[i] = oracle_e4m3_encode((float)ldexp((double)xs[i], -X));
        }
    }
    return ORACLE_OK;
}

/* value = decode(code) * 2^(E - 127), into double (exact). */
int oracle_mx_dequantize_rows(const uint8_t* codes, const uint8_t* scales, int64_t n_rows,
                              int32_t D, double* out) {
    if (n_rows < 0 || D <= 0 || D % 32 != 0) return ORACLE_BAD_ARG;
    const int32_t nb = D / 32;
    for (int64_t r = 0; r < n_rows; ++r)
        for (int32_t i = 0; i < D; ++i) {
            const uint8_t E = scales[r * nb + i / 32];
            out[r * D + i] = E == 255 ? NAN : ldexp(oracle_e4m3_decode(codes[r * D + i]), (int)E - 127);
        }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------------------------
 * Paged cache addressing.  A sequence b stores position s in physical slot
 *     block_table[b][s / page_size] * page_size + s % page_size
 * ([P1]: the indexer reads keys straight out of the paged cache; [P3] 3.1 gather).  Returns -1 for an address outside
 * the cache, which the callers report as a bad argument.
 * ------------------------------------------------------------------------------------------ */
static int64_t paged_slot(const int32_t* block_table, int64_t bt_stride, int32_t page_size,
                          int32_t num_pages, int32_t b, int64_t s) {
    int32_t page = block_table[(int64_t)b * bt_stride + s / page_size];
    if (page < 0 || page >= num_pages) return -1;
    return (int64_t)page * page_size + s % page_size;
}

/* Index score, [P1] "Sparse Attention Pipeline Optimization", [P5] s3.1:
 *   for each query row t (sequence b = q_seq[t], position p = q_pos[t]) and each causal history
 *   position s in [0, p]:  I[t,s] = sum_j w[t,j] * max(0, sum_d q_I[t,j,d] * k[slot(b,s), d]).
 * Positions s > p are left untouched in `scores` (the caller's fill).
 *   q_I: [T_q, H_I, D_I], w: [T_q, H_I], k: [num_pages*page_size, D_I] (exact values),
 *   scores: [T_q, ld]. */
int oracle_index_score(int32_t B, const int32_t* seq_lens, const int32_t* block_table,
                       int64_t bt_stride, int32_t page_size, int32_t num_pages, int32_t T_q,
                       const int32_t* q_seq, const int32_t* q_pos, int32_t H_I, int32_t D_I,
                       const double* q_I, const double* w, const double* k, double* scores,
                       int64_t ld) {
    for (int32_t t = 0; t < T_q; ++t) {
        int32_t b = q_seq[t];
        if (b < 0 || b >= B || q_pos[t] < 0 || q_pos[t] >= seq_lens[b] || q_pos[t] >= ld)
            return ORACLE_BAD_ARG;
        for (int64_t s = 0; s <= q_pos[t]; ++s)
            if (paged_slot(block_table, bt_stride, page_size, num_pages, b, s) < 0)
                return ORACLE_BAD_ARG;
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int32_t t = 0; t < T_q; ++t) {
        int32_t b = q_seq[t];
        const double* qt = q_I + (int64_t)t * H_I * D_I;
        const double* wt = w + (int64_t)t * H_I;
        for (int64_t s = 0; s <= q_pos[t]; ++s) {
            const double* ks = k + paged_slot(block_table, bt_stride, page_size, num_pages, b, s) * D_I;
            double acc = 0.0;
            for (int32_t j = 0; j < H_I; ++j) {
                double dot = 0.0;
                for (int32_t d = 0; d < D_I; ++d) dot += qt[(int64_t)j * D_I + d] * ks[d];
                double relu = dot > 0.0 ? dot : 0.0;
                acc += wt[j] * relu;
            }
            scores[(int64_t)t * ld + s] = acc;
        }
    }
    return ORACLE_OK;
}

/* Top-K selection, [P1] "Sparse Attention Pipeline Optimization" ("selects the Top-K critical
 * positions"), [P3] 3.1.  Row t considers its causal positions s in [0, n_t) with n_t given.
 *  - n_t <= K: every position is selected; output 0..n_t-1 then -1 padding.
 *  - otherwise the K positions ranked first by (score descending, position ascending) are
 *    selected.
 * The output lists the selected positions in ascending order (the pages leave the order open;
 * ascending is the reading taken).  Algorithm: find the K-th largest score v by sorting a copy
 * of the row's scores; take every position with score > v, then positions with score == v in
 * increasing position until K are taken.  -0.0 and +0.0 compare equal (double comparison).
 * Returns ORACLE_NOT_FINITE if a considered score is not finite. */
static int cmp_desc(const void* a, const void* b) {
    double x = *(const double*)a, y = *(const double*)b;
    return (x < y) - (x > y);
}

int oracle_topk(int32_t T_q, const int32_t* n_valid, const double* scores, int64_t ld, int32_t K,
                int32_t* idx) {
    if (K <= 0) return ORACLE_BAD_ARG;
    for (int32_t t = 0; t < T_q; ++t) {
        if (n_valid[t] < 0 || n_valid[t] > ld) return ORACLE_BAD_ARG;
        for (int64_t s = 0; s < n_valid[t]; ++s)
            if (!isfinite(scores[(int64_t)t * ld + s])) return ORACLE_NOT_FINITE;
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int32_t t = 0; t < T_q; ++t) {
        const double* row = scores + (int64_t)t * ld;
        int32_t* out = idx + (int64_t)t * K;
        int64_t n = n_valid[t];
        if (n <= K) {
            for (int64_t i = 0; i < K; ++i) out[i] = i < n ? (int32_t)i : -1;
            continue;
        }
        double* tmp = (double*)malloc(sizeof(double) * (size_t)n);
        memcpy(tmp, row, sizeof(double) * (size_t)n);
        qsort(tmp, (size_t)n, sizeof(double), cmp_desc);
        double v = tmp[K - 1];
        free(tmp);
        int64_t greater = 0;
        for (int64_t s = 0; s < n; ++s) greater += row[s] > v;
        int64_t ties_wanted = K - greater, taken = 0;
        for (int64_t s = 0; s < n; ++s) {
            if (row[s] > v) {
                out[taken++] = (int32_t)s;
            } else if (row[s] == v && ties_wanted > 0) {
                out[taken++] = (int32_t)s;
                --ties_wanted;
            }
        }
    }
    return ORACLE_OK;
}

/* Block-aligned selection, [P3] 3.1 (the selection is aligned to cache blocks so that the sparse
 * attention that follows reads the cache in contiguous blocks).  The page does not spell out the
 * rule; the reading taken: row t's causal positions [0, n_t) fall into blocks of `block`
 * consecutive positions (the last one possibly partial); a block scores the maximum of its
 * positions' scores; rows with n_t <= K select every position as in oracle_topk; otherwise the
 * K / block blocks first in the order (block score descending, block index ascending) are
 * selected and every causal position of a selected block is kept.  Output: the kept positions
 * ascending, then -1 padding to K (a partial block can leave fewer than K).  block must divide K.
 * Algorithm: block maxima, then the same full-sort threshold rule as oracle_topk applied to the
 * blocks. */
int oracle_topk_blocks(int32_t T_q, const int32_t* n_valid, const double* scores, int64_t ld,
                       int32_t K, int32_t block, int32_t* idx) {
    if (K <= 0 || block <= 0 || K % block != 0) return ORACLE_BAD_ARG;
    for (int32_t t = 0; t < T_q; ++t) {
        if (n_valid[t] < 0 || n_valid[t] > ld) return ORACLE_BAD_ARG;
        for (int64_t s = 0; s < n_valid[t]; ++s)
            if (!isfinite(scores[(int64_t)t * ld + s])) return ORACLE_NOT_FINITE;
    }
    const int32_t kb = K / block;
#pragma omp parallel for schedule(dynamic, 1)
    for (int32_t t = 0; t < T_q; ++t) {
        const double* row = scores + (int64_t)t * ld;
        int32_t* out = idx + (int64_t)t * K;
        const int64_t n = n_valid[t];
        if (n <= K) {
            for (int64_t i = 0; i < K; ++i) out[i] = i < n ? (int32_t)i : -1;
            continue;
        }
        const int64_t nb = (n + block - 1) / block;
        double* bmax = (double*)malloc(sizeof(double) * (size_t)nb);
        double* tmp = (double*)malloc(sizeof(double) * (size_t)nb);
        char* keep = (char*)calloc((size_t)nb, 1);
        for (int64_t b = 0; b < nb; ++b) {
            double m = -INFINITY;
            for (int64_t s = b * block; s < (b + 1) * block && s < n; ++s)
                if (row[s] > m) m = row[s];
            bmax[b] = m;
        }
        memcpy(tmp, bmax, sizeof(double) * (size_t)nb);
        qsort(tmp, (size_t)nb, sizeof(double), cmp_desc);
        const double v = tmp[kb - 1];
        int64_t greater = 0;
        for (int64_t b = 0; b < nb; ++b) greater += bmax[b] > v;
        int64_t ties_wanted = kb - greater;
        for (int64_t b = 0; b < nb; ++b) {
            if (bmax[b] > v) {
                keep[b] = 1;
            } else if (bmax[b] == v && ties_wanted > 0) {
                keep[b] = 1;
                --ties_wanted;
            }
        }
        int64_t taken = 0;
        for (int64_t b = 0; b < nb; ++b)
            if (keep[b])
                for (int64_t s = b * block; s < (b + 1) * block && s < n; ++s) out[taken++] = (int32_t)s;
        for (; taken < K; ++taken) out[taken] = -1;
        free(bmax);
        free(tmp);
        free(keep);
    }
    return ORACLE_OK;
}

/* Sparse MLA attention over the selected latent rows, [P1] "Sparse Attention Pipeline
 * Optimization" ("reads only the selected entries ... block-wise fused attention"),
 * [P3] 3.2, [P5] s3 (SFA).  Each cache row holds the compressed latent c_kv (D_v values)
 * followed by the rope part (D_qk - D_v values); keys are the whole row, values are its first
 * D_v entries (the low-rank latent shared by all heads).
 *   S_t = { idx[t,k] : idx[t,k] != -1 }  (a multiset; duplicates are outside the contract)
 *   z_n   = scale * sum_{d < D_qk} q[t,h,d] * kv[slot(b,n), d]
 *   m     = max_n z_n
 *   out   = sum_n e^{z_n - m} kv[slot(b,n), 0:D_v] / sum_n e^{z_n - m}
 *   lse   = m + log sum_n e^{z_n - m}
 * An empty S_t gives out = 0 and lse = -inf.
 *   q: [T_q, H, D_qk], kv: [num_slots, D_qk] exact values, idx: [T_q, K],
 *   out: [T_q, H, D_v], lse: [T_q, H]. */
int oracle_sparse_mla(int32_t B, const int32_t* seq_lens, const int32_t* block_table,
                      int64_t bt_stride, int32_t page_size, int32_t num_pages, int32_t T_q,
                      const int32_t* q_seq, const int32_t* q_pos, int32_t H, int32_t D_qk,
                      int32_t D_v, const double* q, const double* kv, const int32_t* idx,
                      int32_t K, double scale, double* out, double* lse) {
    if (D_v <= 0 || D_v > D_qk || K <= 0) return ORACLE_BAD_ARG;
    for (int32_t t = 0; t < T_q; ++t) {
        int32_t b = q_seq[t];
        if (b < 0 || b >= B || q_pos[t] < 0 || q_pos[t] >= seq_lens[b]) return ORACLE_BAD_ARG;
        for (int32_t k = 0; k < K; ++k) {
            int32_t n = idx[(int64_t)t * K + k];
            if (n == -1) continue;
            if (n < 0 || n > q_pos[t]) return ORACLE_BAD_ARG;
            if (paged_slot(block_table, bt_stride, page_size, num_pages, b, n) < 0)
                return ORACLE_BAD_ARG;
        }
    }
    int status = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t th = 0; th < (int64_t)T_q * H; ++th) {
        int32_t t = (int32_t)(th / H), h = (int32_t)(th % H);
        int32_t b = q_seq[t];
        const double* qh = q + th * D_qk;
        const int32_t* sel = idx + (int64_t)t * K;
        double* o = out + th * D_v;
        double* z = (double*)malloc(sizeof(double) * (size_t)K);
        double m = -INFINITY;
        for (int32_t k = 0; k < K; ++k) {
            if (sel[k] == -1) continue;
            const double* row = kv + paged_slot(block_table, bt_stride, page_size, num_pages, b, sel[k]) * D_qk;
            double dot = 0.0;
            for (int32_t d = 0; d < D_qk; ++d) dot += qh[d] * row[d];
            z[k] = scale * dot;
            if (z[k] > m) m = z[k];
        }
        for (int32_t d = 0; d < D_v; ++d) o[d] = 0.0;
        double denom = 0.0;
        if (m != -INFINITY) {
            for (int32_t k = 0; k < K; ++k) {
                if (sel[k] == -1) continue;
                const double* row = kv + paged_slot(block_table, bt_stride, page_size, num_pages, b, sel[k]) * D_qk;
                double e = exp(z[k] - m);
                denom += e;
                for (int32_t d = 0; d < D_v; ++d) o[d] += e * row[d];
            }
            double psum = 0.0;
            for (int32_t k = 0; k < K; ++k)
                if (sel[k] != -1) psum += exp(z[k] - m) / denom;
            if (fabs(psum - 1.0) >= 1e-12) {
#pragma omp atomic write
                status = ORACLE_SOFTMAX_SUM;
            }
            for (int32_t d = 0; d < D_v; ++d) o[d] /= denom;
            lse[th] = m + log(denom);
        } else {
            lse[th] = -INFINITY;
        }
        free(z);
    }
    return status;
}

/* Dense causal attention over every history position s in [0, p_t] (textbook softmax
 * attention with the same key/value split as above).  Used to check that selecting K >= the
 * context length reproduces full attention. */
int oracle_dense_attn(int32_t B, const int32_t* seq_lens, const int32_t* block_table,
                      int64_t bt_stride, int32_t page_size, int32_t num_pages, int32_t T_q,
                      const int32_t* q_seq, const int32_t* q_pos, int32_t H, int32_t D_qk,
                      int32_t D_v, const double* q, const double* kv, double scale, double* out,
                      double* lse) {
    if (D_v <= 0 || D_v > D_qk) return ORACLE_BAD_ARG;
    for (int32_t t = 0; t < T_q; ++t) {
        int32_t b = q_seq[t];
        if (b < 0 || b >= B || q_pos[t] < 0 || q_pos[t] >= seq_lens[b]) return ORACLE_BAD_ARG;
        for (int64_t s = 0; s <= q_pos[t]; ++s)
            if (paged_slot(block_table, bt_stride, page_size, num_pages, b, s) < 0)
                return ORACLE_BAD_ARG;
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t th = 0; th < (int64_t)T_q * H; ++th) {
        int32_t t = (int32_t)(th / H);
        int32_t b = q_seq[t];
        int64_t n = (int64_t)q_pos[t] + 1;
        const double* qh = q + th * D_qk;
        double* o = out + th * D_v;
        double* z = (double*)malloc(sizeof(double) * (size_t)n);
        double m = -INFINITY;
        for (int64_t s = 0; s < n; ++s) {
            const double* row = kv + paged_slot(block_table, bt_stride, page_size, num_pages, b, s) * D_qk;
            double dot = 0.0;
            for (int32_t d = 0; d < D_qk; ++d) dot += qh[d] * row[d];
            z[s] = scale * dot;
            if (z[s] > m) m = z[s];
        }
        double denom = 0.0;
        for (int32_t d = 0; d < D_v; ++d) o[d] = 0.0;
        for (int64_t s = 0; s < n; ++s) {
            const double* row = kv + paged_slot(block_table, bt_stride, page_size, num_pages, b, s) * D_qk;
            double e = exp(z[s] - m);
            denom += e;
            for (int32_t d = 0; d < D_v; ++d) o[d] += e * row[d];
        }
        for (int32_t d = 0; d < D_v; ++d) o[d] /= denom;
        lse[th] = m + log(denom);
        free(z);
    }
    return ORACLE_OK;
}

/* Number of threads OpenMP would use (reported next to CPU timings). */
#ifdef _OPENMP
#include <omp.h>
#endif
int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
