/* A plain C consumer of the q8 C ABI: compiles against include/q8.h as C11,
 * links libq8.so, and makes calls that return from host-side validation (no
 * device memory is touched).  Prints one line per check; exits non-zero on
 * the first unexpected status. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "q8.h"

static int expect(const char *what, q8_status got, q8_status want) {
    if (got != want) {
        printf("FAIL %s: %d (%s), want %d\n", what, (int)got, q8_status_string(got), (int)want);
        return 1;
    }
    printf("ok %s\n", what);
    return 0;
}

int main(void) {
    int bad = 0;
    if (q8_version() != Q8_VERSION) {
        printf("FAIL version %d != %d\n", q8_version(), Q8_VERSION);
        return 1;
    }
    printf("ok version %d\n", q8_version());
    if (strcmp(q8_status_string(Q8_OK), "ok") != 0) bad = 1;

    void *fake = (void *)(uintptr_t)0x10000;   /* never dereferenced */
    bad |= expect("quantize_weight null W",
                  q8_quantize_weight(NULL, Q8_BF16, 64, 128, 128, Q8_ASYM_INT8, Q8_U8, fake,
                                     (float *)fake, (float *)fake, NULL),
                  Q8_ERR_NULL);
    bad |= expect("quantize_act K % 32",
                  q8_quantize_act(fake, Q8_BF16, 16, 100, 100, Q8_SYM_INT8, 0.0f, fake,
                                  (float *)fake, (int32_t *)fake, NULL),
                  Q8_ERR_SHAPE);
    q8_weight_g4 g4 = {fake, (const float *)fake, 256, 512, 256, 96};
    bad |= expect("linear_w4a16 group 96",
                  q8_linear_w4a16(fake, Q8_BF16, 16, 512, 512, &g4, NULL, fake, 256, NULL),
                  Q8_ERR_SCHEME);
    q8_weight w = {fake, Q8_E4M3, (const float *)fake, NULL, 256, 128, 128};
    q8_act x = {fake, Q8_E4M3, (const float *)fake, NULL, 16, 128, 128};
    bad |= expect("linear_fp8_grouped 3 experts",
                  q8_linear_fp8_grouped(&x, &w, 3, (const int32_t *)fake, NULL, fake, 64, NULL),
                  Q8_ERR_SHAPE);
    bad |= expect("inject invalid code", q8_inject_failure((q8_status)42, 0), Q8_ERR_SCHEME);
    if (q8_workspace_size(Q8_OP_LINEAR_W8A8, 16, 64, 128) != 0 ||
        q8_workspace_size(Q8_OP_LINEAR_INT8_MIXED, 16, 64, 128) == 0) {
        printf("FAIL workspace sizes\n");
        bad = 1;
    } else {
        printf("ok workspace sizes\n");
    }
    return bad;
}
