/* A plain C99 client of include/mamba_scan.h: the header compiles as C with
 * every warning an error, the library links with nothing but the header, and
 * the calls that need no GPU (version, status strings, argument validation,
 * which runs before any device work) answer as documented. */
#include <stdint.h>
#include <stdio.h>

#include "mamba_scan.h"

static int fails = 0;
#define EXPECT(cond)                                                        \
    do {                                                                    \
        if (!(cond)) {                                                      \
            fprintf(stderr, "failed: %s (line %d)\n", #cond, __LINE__);     \
            ++fails;                                                        \
        }                                                                   \
    } while (0)

/* distinct fake device addresses: validation never dereferences them */
#define ADDR(x) ((void *)(uintptr_t)(x))

static int scan(void *u, void *out, int64_t batch, int64_t dstate, int dtype) {
    return mamba_scan_fwd(u, ADDR(0x200000), (const float *)ADDR(0x300000), ADDR(0x400000),
                          ADDR(0x500000), NULL, NULL, NULL, 1, out, NULL, batch, 4, 8, dstate,
                          dtype, (cudaStream_t)0);
}

int main(void) {
    int s;
    EXPECT((mamba_abi_version() >> 16) == 1);
    for (s = MAMBA_ERR_TIMEOUT; s <= MAMBA_OK; ++s)
        EXPECT(mamba_status_string(s) != NULL && mamba_status_string(s)[0] != '\0');

    EXPECT(scan(NULL, ADDR(0x600000), 2, 16, MAMBA_BF16) == MAMBA_ERR_NULL);
    EXPECT(scan(ADDR(0x100000), NULL, 2, 16, MAMBA_BF16) == MAMBA_ERR_NULL);
    EXPECT(scan(ADDR(0x100000), ADDR(0x600000), 0, 16, MAMBA_BF16) == MAMBA_ERR_SHAPE);
    EXPECT(scan(ADDR(0x100000), ADDR(0x600000), 2, 65, MAMBA_BF16) == MAMBA_ERR_UNSUPPORTED);
    EXPECT(scan(ADDR(0x100000), ADDR(0x600000), 2, 16, 7) == MAMBA_ERR_UNSUPPORTED);
    /* out two bytes into u (2 x 4 x 8 bf16 = 128 bytes): a partial overlap */
    EXPECT(scan(ADDR(0x100000), ADDR(0x100002), 2, 16, MAMBA_BF16) == MAMBA_ERR_OVERLAP);

    if (fails == 0) printf("ok\n");
    return fails == 0 ? 0 : 1;
}
