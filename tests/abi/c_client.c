/*
 * A plain C (C11) client of the library's C ABI, built and run by the CPU test
 * suite: it shows that include/sqa.h compiles as C, that every call it uses
 * links against the shared library, and that argument errors come back before
 * any launch (no GPU is needed for any call made here).  It prints one
 * "name value" line per check for the test to compare.
 */
#include <stdio.h>
#include <string.h>

#include "sqa.h"

int main(void) {
    const sqa_shape train = {32, 1024, 8, 4, 16};
    const sqa_shape decode = {32, 32768, 8, 4, 16};
    const sqa_shape bad_group = {2, 300, 6, 4, 16};
    const sqa_shape bad_dh = {2, 300, 8, 4, 48};
    char *p = (char *)0x100000; /* never dereferenced: every call below fails its checks first */
    float lse_dummy = 0.f;
    (void)lse_dummy;

    printf("version %d\n", sqa_version());
    printf("bwd_workspace %zu\n", sqa_bwd_workspace_bytes(train));
    printf("decode_workspace %zu\n", sqa_decode_workspace_bytes(decode));
    printf("decode_workspace_invalid %zu\n", sqa_decode_workspace_bytes(bad_group));
    printf("fwd_null %d\n", (int)sqa_fwd(NULL, p, p, p, (float *)p, train, 1, 0.f, NULL));
    printf("fwd_group %d\n", (int)sqa_fwd(p, p, p, p, (float *)p, bad_group, 1, 0.f, NULL));
    printf("fwd_dh %d\n", (int)sqa_fwd(p, p, p, p, (float *)p, bad_dh, 1, 0.f, NULL));
    printf("fwd_misaligned %d\n", (int)sqa_fwd(p + 2, p, p, p, (float *)p, train, 1, 0.f, NULL));
    printf("bwd_small_workspace %d\n",
           (int)sqa_bwd(p, p, p, p, p, (const float *)p, p, p, p, p, 16, train, 1, 0.f, NULL));
    printf("decode_null %d\n", (int)sqa_decode(p, NULL, p, NULL, p, (float *)p, p, 1 << 20, decode, 0.f, NULL));
    printf("timing_bad_kernel %d\n", (int)sqa_set_timing_events(7, NULL, NULL));
    printf("status_string_ok %d\n", sqa_status_string(SQA_OK) != NULL && strlen(sqa_status_string(SQA_OK)) > 0);
    /* the last error text names the failing argument */
    sqa_fwd(p, p, p, p, (float *)p, bad_dh, 1, 0.f, NULL);
    printf("last_error_nonempty %d\n", sqa_last_error() != NULL && strlen(sqa_last_error()) > 0);
    return 0;
}
