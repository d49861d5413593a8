/* A plain C99 consumer of include/sekv.h: the header compiles as C, the library
 * links, and its host-only entry points behave as documented (no GPU needed:
 * every call below returns before touching the device). Exit code 0 = all
 * checks passed; otherwise the number of the first failed check. */
#include <stdio.h>
#include <string.h>

#include "sekv.h"

#define CHECK(n, cond)                                   \
    do {                                                 \
        if (!(cond)) {                                   \
            fprintf(stderr, "check %d failed: %s\n", n, #cond); \
            return n;                                    \
        }                                                \
    } while (0)

int main(void) {
    sekv_build_desc bd;
    sekv_decode_desc dd;
    sekv_fetch_desc fd;
    const char* s;
    /* the C compiler's view of the descriptors equals the library's */
    CHECK(1, sekv_desc_size(0) == sizeof(sekv_build_desc));
    CHECK(2, sekv_desc_size(1) == sizeof(sekv_decode_desc));
    CHECK(3, sekv_desc_size(2) == sizeof(sekv_fetch_desc));
    CHECK(4, sekv_desc_size(3) == 0);
    CHECK(5, sekv_version() == SEKV_VERSION);
    /* block = 2 len8 r8 + 2 r8 d: |S| = 13, rank 16 (r_S = 13 -> r8 = 16), d = 128 */
    CHECK(6, sekv_block_elems(13, 128, 16) == 2 * 16 * 16 + 2 * 16 * 128);
    CHECK(7, sekv_block_elems(0, 128, 16) == 0);
    CHECK(8, sekv_basis_region_bound(1024, 64, 2, 128, 16) % 64 == 0);
    s = sekv_status_str(SEKV_ERR_COLD_SPAN);
    CHECK(9, s != NULL && strlen(s) > 0);
    /* argument errors are reported before any launch */
    CHECK(10, sekv_build_spans(NULL, NULL) == SEKV_ERR_INVALID_ARG);
    CHECK(11, sekv_decode_attn(NULL, NULL) == SEKV_ERR_INVALID_ARG);
    memset(&bd, 0, sizeof bd);
    memset(&dd, 0, sizeof dd);
    memset(&fd, 0, sizeof fd);
    CHECK(12, sekv_build_spans(&bd, NULL) == SEKV_ERR_INVALID_ARG);
    CHECK(13, sekv_decode_attn(&dd, NULL) == SEKV_ERR_INVALID_ARG);
    CHECK(14, sekv_fetch_bases(&fd, NULL, NULL, NULL) == SEKV_ERR_INVALID_ARG);
    CHECK(15, sekv_merge_partials(NULL, NULL, 1, 1, 8, NULL, NULL, NULL) == SEKV_ERR_INVALID_ARG);
    s = sekv_last_error();
    CHECK(16, s != NULL && strlen(s) > 0);
    printf("ok\n");
    return 0;
}
