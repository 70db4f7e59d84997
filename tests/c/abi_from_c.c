/* The C ABI used from plain C99: the header compiles as C, the library
 * links, and calls that fail host-side validation return their status and
 * name their clause without touching a device. */
#include <stdio.h>
#include <string.h>

#include "spa.h"

static int check(int got, int want, const char* clause) {
    if (got != want || strstr(spa_last_error_detail(), clause) == NULL) {
        printf("FAIL want %d got %d, detail '%s' lacks '%s'\n", want, got, spa_last_error_detail(), clause);
        return 1;
    }
    return 0;
}

int main(void) {
    int bad = 0;
    const uint16_t* q = (const uint16_t*)(uintptr_t)0x10000; /* never dereferenced */
    if (spa_abi_version() != SPA_ABI_VERSION) { printf("FAIL abi version\n"); bad++; }
    if (strcmp(spa_status_string(SPA_OK), "ok") != 0) { printf("FAIL status string\n"); bad++; }
    bad += check(spa_dequant_fp8_pages(NULL, NULL, -1, 64, 128, NULL, 1, 0, NULL, NULL, NULL),
                 SPA_ERR_INVALID_ARG, "num_pages < 0");
    bad += check(spa_paged_kv_write(NULL, NULL, -1, 128, NULL, NULL, NULL, 1, 1, 64, 1, NULL, NULL, NULL, NULL),
                 SPA_ERR_INVALID_ARG, "n_tokens < 0");
    bad += check(spa_unpack_d512_pages(NULL, 4, 0, NULL, 1, NULL, NULL, NULL), SPA_ERR_INVALID_ARG, "page_size < 1");
    bad += check(spa_sparse_sink_attn_fwd(q, 16384, 128, 4, 128, 96, NULL, NULL, 1, 64, NULL, 1, NULL, NULL, 0, 64,
                                          NULL, 0, NULL, 1, NULL, NULL, NULL, 0.088f, NULL, NULL, 1, NULL, 0, NULL,
                                          NULL),
                 SPA_ERR_UNSUPPORTED, "head_dim must be 64, 128 or 512");
    bad += check(spa_sparse_sink_attn_bwd(q, 16384, 128, 4, 128, 128, NULL, NULL, 1, 64, NULL, 1, NULL, NULL, 0, 64,
                                          NULL, 0, NULL, 1, NULL, NULL, NULL, 0.088f, NULL, NULL, NULL, NULL, NULL,
                                          NULL, NULL, NULL, NULL, 1, NULL, NULL),
                 SPA_ERR_INVALID_ARG, "k_raw, v_raw and pt_raw");
    if (spa_sparse_sink_attn_workspace_size(10, 128, 128, 1) != 0) { printf("FAIL workspace\n"); bad++; }
    printf(bad ? "FAILED %d\n" : "ok\n", bad);
    return bad != 0;
}
