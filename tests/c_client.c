/* A plain C11 client of libjmoe.so: it includes the public header, links the library and makes the
 * calls whose result is decided on the host (sizes, argument validation, T = 0), so it runs without
 * a GPU.  Exit status 0 when every check holds; the first failed check is printed. */
#include <stdio.h>
#include <string.h>

#include "jmoe.h"

#define CHECK(cond)                                                    \
    do {                                                               \
        if (!(cond)) {                                                 \
            fprintf(stderr, "check failed, line %d: %s\n", __LINE__, #cond); \
            return 1;                                                  \
        }                                                              \
    } while (0)

int main(void) {
    /* a 256-byte aligned, never dereferenced stand-in for device pointers: every call below
     * returns from its host-side checks */
    void* const dev = (void*)(uintptr_t)0x100000;
    const uint16_t* x = (const uint16_t*)dev;
    const float* f = (const float*)dev;
    const int8_t* q = (const int8_t*)dev;
    uint16_t* y = (uint16_t*)dev;

    size_t ws = jamba_moe_workspace_size(32, 4096, 14336, 16, 2);
    CHECK(ws > (size_t)32 * 2 * 4096 * 4 && ws % 256 == 0);
    CHECK(jamba_moe_workspace_size(32, 4000, 14336, 16, 2) == 0);
    CHECK(jamba_moe_workspace_size(32, 4096, 14336, 8, 2) == 0);
    CHECK(jamba_mlp_workspace_size(32, 4096, 14336) > 0);
    CHECK(jamba_moe_workspace_size_fp8(32, 4096, 14336, 16, 2) > 0);

    CHECK(strcmp(jamba_moe_status_string(JMOE_OK), "ok") == 0);
    CHECK(strlen(jamba_moe_status_string(JMOE_ERR_SHAPE)) > 0);

    /* argument errors, found before anything is launched */
    CHECK(jamba_moe_forward(NULL, f, NULL, q, f, q, f, q, f, 8, 256, 512, 16, 2, y, NULL, NULL, dev, ws, NULL) ==
          JMOE_ERR_NULL);
    CHECK(jamba_moe_forward(x, f, NULL, q, f, q, f, q, f, 8, 256, 512, 8, 2, y, NULL, NULL, dev, ws, NULL) ==
          JMOE_ERR_SHAPE);
    CHECK(jamba_moe_forward(x, f, NULL, q, f, q, f, q, f, 8, 256, 500, 16, 2, y, NULL, NULL, dev, ws, NULL) ==
          JMOE_ERR_SHAPE);
    CHECK(jamba_moe_forward(x, f, NULL, q, f, q, f, q, f, 8, 256, 512, 16, 2, y, NULL, NULL, dev, 16, NULL) ==
          JMOE_ERR_WORKSPACE);
    CHECK(jamba_moe_forward((const uint16_t*)((const char*)dev + 2), f, NULL, q, f, q, f, q, f, 8, 256, 512, 16, 2,
                            y, NULL, NULL, dev, ws, NULL) == JMOE_ERR_ALIGN);
    CHECK(jamba_moe_quantize(x, 1, 4, 15, (int8_t*)dev, (float*)dev, NULL) == JMOE_ERR_SHAPE);
    CHECK(jamba_mlp_forward(x, q, f, q, f, q, NULL, 8, 256, 512, y, dev, ws, NULL) == JMOE_ERR_NULL);

    /* no token: nothing to do, pointers may be NULL */
    CHECK(jamba_moe_forward(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, 4096, 14336, 16, 2, NULL, NULL,
                            NULL, NULL, 0, NULL) == JMOE_OK);
    CHECK(jamba_mlp_forward(NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, 4096, 14336, NULL, NULL, 0, NULL) == JMOE_OK);

    printf("c client ok\n");
    return 0;
}
