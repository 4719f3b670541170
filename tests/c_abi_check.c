/*
 * c_abi_check.c -- a plain C99 consumer of include/hsa.h.  It links libhsa.so and exercises the
 * host-side argument checks, which answer before anything touches the device, so it runs on a
 * machine without a GPU.  The pointers below are placeholders that the library never
 * dereferences (every call here is rejected, or has no rows to process).
 */
#include <stdio.h>
#include <string.h>

#include "hsa.h"

#define CHECK(cond)                                                                         \
    do {                                                                                    \
        if (!(cond)) {                                                                      \
            fprintf(stderr, "line %d: %s failed (%s)\n", __LINE__, #cond,                   \
                    hsa_last_error_message());                                              \
            return 1;                                                                       \
        }                                                                                   \
    } while (0)

int main(void) {
    const void* fake = (const void*)0x1000;
    hsa_paged_seq_t seq;
    hsa_paged_seq_t empty;
    hsa_status_t st;

    CHECK(hsa_version() >= 300);
    CHECK(strlen(hsa_status_string(HSA_ERR_WORKSPACE)) > 0);

    /* a NULL descriptor is an argument error and says so */
    st = hsa_topk(NULL, NULL, 0, 8, NULL, NULL);
    CHECK(st == HSA_ERR_INVALID_ARG);
    CHECK(strstr(hsa_last_error_message(), "seq") != NULL);

    memset(&seq, 0, sizeof seq);
    seq.B = 1;
    seq.seq_lens = (const int32_t*)fake;
    seq.block_table = (const int32_t*)fake;
    seq.bt_stride = 4;
    seq.page_size = 16;
    seq.num_pages = 4;
    seq.max_seq_len = 64;
    seq.T_q = 2;
    seq.q_seq = (const int32_t*)fake;
    seq.q_pos = (const int32_t*)fake;
    seq.q_run = 1;

    /* K = 0 and ld < max_seq_len are rejected */
    CHECK(hsa_topk(&seq, (const float*)fake, 64, 0, (int32_t*)fake, NULL) == HSA_ERR_INVALID_ARG);
    CHECK(hsa_topk(&seq, (const float*)fake, 32, 8, (int32_t*)fake, NULL) == HSA_ERR_INVALID_ARG);

    /* MXFP8 keys need their E8M0 scale bytes, and D_I a multiple of 32 */
    st = hsa_index_score(&seq, fake, HSA_BF16, (const float*)fake, 4, 32, fake, HSA_MXE4M3, NULL,
                         (float*)fake, 64, NULL);
    CHECK(st == HSA_ERR_INVALID_ARG);
    st = hsa_index_score(&seq, fake, HSA_BF16, (const float*)fake, 4, 48, fake, HSA_MXE4M3, fake,
                         (float*)fake, 64, NULL);
    CHECK(st == HSA_ERR_INVALID_ARG);

    /* quantizers: group must divide D; MX blocks are 32 wide */
    CHECK(hsa_quantize_index(fake, HSA_BF16, 10, 128, 48, NULL, 10, (uint8_t*)fake, (float*)fake,
                             NULL) == HSA_ERR_INVALID_ARG);
    CHECK(hsa_quantize_mx(fake, HSA_BF16, 10, 48, NULL, 10, (uint8_t*)fake, (uint8_t*)fake, NULL) ==
          HSA_ERR_INVALID_ARG);
    CHECK(hsa_dequantize_mx((const uint8_t*)fake, (const uint8_t*)fake, 10, 64, (void*)fake,
                            HSA_E4M3, NULL) == HSA_ERR_UNSUPPORTED);

    /* MXFP8 queries: their scale bytes must be given, 16-byte aligned */
    st = hsa_index_score_mx(&seq, (const uint8_t*)fake, NULL, (const float*)fake, 4, 32,
                            (const uint8_t*)fake, (const uint8_t*)fake, (float*)fake, 64, NULL);
    CHECK(st == HSA_ERR_INVALID_ARG);

    /* the chunked prefill checks its chunk list: [0, 100) lies outside T_q = 2 */
    {
        hsa_index_args_t ia;
        hsa_attn_args_t at;
        int32_t chunks[2] = {0, 100};
        float* bufs[2] = {(float*)0x1000, (float*)0x2000};
        memset(&ia, 0, sizeof ia);
        memset(&at, 0, sizeof at);
        ia.q_I = fake; ia.q_dtype = HSA_BF16; ia.w = (const float*)fake; ia.H_I = 4; ia.D_I = 32;
        ia.k_cache = fake; ia.k_dtype = HSA_BF16;
        at.q = fake; at.q_dtype = HSA_BF16; at.H = 8; at.D_qk = 80; at.D_v = 64; at.kv = fake;
        at.kv_dtype = HSA_BF16; at.kv_scale_group = 64; at.softmax_scale = 0.1f;
        at.out = (void*)fake; at.out_dtype = HSA_BF16;
        st = hsa_prefill_chunked(&seq, &ia, &at, 32, chunks, 1, bufs, 128, 64, (int32_t*)fake, NULL,
                                 NULL, NULL);
        CHECK(st == HSA_ERR_INVALID_ARG);
        /* the no-allocation decode step rejects a step larger than its scratch before anything
           touches the device: 2 rows x 2^23 positions of fp32 scores */
        empty = seq;
        empty.max_seq_len = 1 << 23;
        st = hsa_fused_decode_noalloc(&empty, &ia, &at, 32, NULL);
        CHECK(st == HSA_ERR_WORKSPACE);
    }

    /* zero query rows is a no-op, not an error */
    empty = seq;
    empty.T_q = 0;
    empty.q_seq = NULL;
    empty.q_pos = NULL;
    CHECK(hsa_topk(&empty, NULL, 64, 8, NULL, NULL) == HSA_OK);
    CHECK(hsa_quantize_mx(NULL, HSA_BF16, 0, 64, NULL, 0, NULL, NULL, NULL) == HSA_OK);

    printf("c abi ok\n");
    return 0;
}
