/* A C99 caller of the library: include/moe.h compiles as C, the library links, and the calls
 * that need no device behave as the header states (sizes, argument errors before any launch, the
 * T == 0 no-op with null per-token pointers, status strings).  Exit code 0 on success. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "moe.h"

#define CHECK(cond, code)                                          \
    do {                                                           \
        if (!(cond)) {                                             \
            fprintf(stderr, "failed: %s (line %d)\n", #cond, __LINE__); \
            return code;                                           \
        }                                                          \
    } while (0)

int main(void) {
    moe_shape_t s;
    memset(&s, 0, sizeof s);
    s.T = 256; s.d = 7168; s.n_experts = 256; s.inter = 2048; s.top_k = 8;
    s.n_shared = 1; s.inter_shared = 2048; s.has_bias = 1;
    s.dtype = MOE_BF16; s.gate_mode = 0; s.routed_fmt = MOE_FMT_NATIVE;

    const size_t n = moe_workspace_bytes(&s);
    CHECK(n > 0, 1);
    CHECK(moe_layer_launches(&s) > 0, 2);

    /* an invalid shape: no workspace size, no launch count */
    moe_shape_t bad = s;
    bad.top_k = 300;
    CHECK(moe_workspace_bytes(&bad) == 0, 3);
    CHECK(moe_layer_launches(&bad) == -1, 4);

    /* argument errors return before any device work */
    void* fake = (void*)(uintptr_t)((uint64_t)1 << 40);          /* never dereferenced */
    CHECK(moe_route(&s, NULL, fake, NULL, fake, fake, fake, n, NULL) == MOE_ERR_INVALID_ARG, 5);
    CHECK(moe_route(&s, fake, fake, NULL, fake, fake, fake, n - 1, NULL) == MOE_ERR_WORKSPACE, 6);

    /* T == 0: a no-op, per-token pointers may be NULL */
    moe_shape_t e = s;
    e.T = 0;
    const size_t ne = moe_workspace_bytes(&e);
    CHECK(ne > 0, 7);
    CHECK(moe_route(&e, NULL, fake, NULL, NULL, NULL, fake, ne, NULL) == MOE_OK, 8);

    const char* v = moe_version();
    const char* m = moe_status_string(MOE_ERR_INVALID_ARG);
    CHECK(v && strlen(v) > 0 && m && strlen(m) > 0, 9);
    printf("%s\n%s\n", v, m);
    return 0;
}
