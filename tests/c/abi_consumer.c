/* A plain C99 consumer of the C ABI: includes include/kq.h, links libkq.so and
 * calls the entry points whose answers need no GPU (block geometry, status
 * strings, and host-side argument checks, which return before any CUDA call).
 * Prints one "name value" line per check; the test compares them with the
 * values the header documents.  Pointer arguments are fake addresses that the
 * library never dereferences. */
#include <stdint.h>
#include <stdio.h>

#include "kq.h"

#define FAKE ((void*)(uintptr_t)0x10000)      /* 16-byte aligned, never touched */
#define MIS ((void*)(uintptr_t)0x10008)       /* 8 bytes off a 16-byte boundary */

int main(void) {
    static const int codecs[] = {KQ_Q4_0, KQ_Q8_0, KQ_Q4_K, KQ_Q5_K, KQ_Q6_K};
    unsigned i;
    for (i = 0; i < sizeof codecs / sizeof codecs[0]; ++i) {
        int vpb = 0, bpb = 0;
        const int rc = kq_block_info(codecs[i], &vpb, &bpb);
        printf("block_info_%d %d %d %d\n", codecs[i], rc, vpb, bpb);
    }
    printf("block_info_unknown %d\n", kq_block_info(3, NULL, NULL));
    for (i = 0; i <= 5; ++i) printf("status_string_%u %s\n", i, kq_status_string((int)i));

    const uint16_t* x = (const uint16_t*)FAKE;
    float* y = (float*)FAKE;
    printf("qmv_k_not_block_multiple %d\n", kq_qmv(KQ_Q4_K, FAKE, 16, 300, x, 1, y, NULL));
    printf("qmv_m_17 %d\n", kq_qmv(KQ_Q4_K, FAKE, 16, 256, x, 17, y, NULL));
    printf("qmv_unknown_codec %d\n", kq_qmv(3, FAKE, 16, 256, x, 1, y, NULL));
    printf("qmv_misaligned_w %d\n", kq_qmv(KQ_Q6_K, MIS, 16, 256, x, 1, y, NULL));
    printf("qmv_empty %d\n", kq_qmv(KQ_Q8_0, FAKE, 0, 32, x, 1, y, NULL));
    printf("qmm_null_x %d\n", kq_qmm(KQ_Q4_K, FAKE, 16, 256, NULL, 4, y, NULL));
    printf("dequantize_empty %d\n", kq_dequantize(KQ_Q6_K, FAKE, 0, 256, NULL, NULL));
    printf("gather_qmv_too_many_pairs %d\n",
           kq_gather_qmv(KQ_Q4_K, FAKE, 8, 64, 256, x, 0, (const int32_t*)FAKE, 4097, 2, y, NULL, NULL));
    printf("tile_map_small_cap %d\n",
           kq_expert_tile_map((const uint32_t*)FAKE, 1024, 8, (uint32_t*)FAKE, 23, (uint32_t*)FAKE, NULL, NULL));
    printf("glu_bad_act %d\n", kq_moe_glu_gather(KQ_Q4_K, FAKE, FAKE, 8, 64, 256, x, (const int32_t*)FAKE, 1, 2, 7,
                                                 0.0f, y, NULL, NULL));
    printf("mix_n_not_multiple_of_4 %d\n",
           kq_gather_mix(y, 8, 6, (const int32_t*)FAKE, y, 4, 2, y, NULL, NULL));
    return 0;
}
