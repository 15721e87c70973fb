/* The C ABI used from plain C (no CUDA headers, no GPU needed): the header compiles as C99,
 * the library links, and calls with bad arguments return their status without launching. */
#include <stdio.h>
#include <string.h>

#include "race_attn.h"

static int fails = 0;

static void expect(int cond, const char *what)
{
    if (!cond) {
        fprintf(stderr, "FAILED: %s\n", what);
        ++fails;
    }
}

int main(void)
{
    size_t fw = 0, bw = 0, cx = 0;
    expect(strcmp(race_status_string(RACE_OK), "RACE_OK") == 0, "status string");
    expect(race_attn_workspace_size(1, 1, 4096, 64, 16, 4, 1, 0, RACE_BF16, &fw) == RACE_OK && fw > 0,
           "forward workspace size");
    expect(race_attn_workspace_size(1, 1, 4096, 64, 16, 4, 1, 1, RACE_BF16, &bw) == RACE_OK && bw > fw,
           "backward workspace size");
    expect(race_attn_ctx_size(1, 1, 4096, 64, 16, 4, 1, &cx) == RACE_OK && cx == fw, "ctx size");
    expect(race_attn_workspace_size(1, 1, 4096, 60, 16, 4, 1, 0, RACE_BF16, &fw) == RACE_ERR_UNSUPPORTED,
           "d = 60 unsupported");
    /* NULL inputs: rejected before anything is launched */
    expect(race_attn_forward(NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, 1, 1, 4096, 64, 16, 4, 0.5f, 1,
                             RACE_BF16, NULL, 0, NULL) == RACE_ERR_INVALID_ARG,
           "forward with NULL pointers");
    expect(race_attn_backward(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL, NULL, NULL, 1, 1, 4096,
                              64, 16, 4, 0.5f, 1, RACE_BF16, NULL, 0, NULL) == RACE_ERR_INVALID_ARG,
           "backward with NULL pointers");
    expect(RACE_NOALLOC_SCRATCH_BYTES == (size_t)24 << 20, "scratch size constant");
    if (fails == 0) printf("abi_from_c ok\n");
    return fails != 0;
}
