/*
 * A plain C client of the library's C ABI, compiled and run by the CPU test
 * suite (tests/test_abi.py).  It includes both public headers as C99 and calls
 * only the host-only entry points and host-side argument checks, so it needs no
 * GPU: every call here returns before any device is queried.
 */
#include <stdint.h>
#include <stdio.h>

#include "tg_attention.h"
#include "tg_gemm.h"

int main(void)
{
    int failures = 0;
#define EXPECT(cond)                                                   \
    do {                                                               \
        if (!(cond)) {                                                 \
            printf("FAIL line %d: %s\n", __LINE__, #cond);             \
            ++failures;                                                \
        }                                                              \
    } while (0)

    printf("version %d\n", tg_version());
    const int n = tg_num_configs();
    printf("configs %d\n", n);
    EXPECT(n > 0);
    for (int i = 0; i < n; ++i) {
        tg_config_t c;
        EXPECT(tg_config_info(i, &c) == TG_OK);
        EXPECT(c.id == i && c.block_m > 0 && c.block_n > 0 && c.block_k > 0);
    }
    tg_config_t pick;
    EXPECT(tg_gemm_select_config(8192, 8192, 8192, TG_EPILOGUE_BIAS_GELU, 148, &pick) == TG_OK);
    printf("8192 fused: config %d split %d\n", pick.id, pick.split);

    /* host-side rejections: nothing is launched */
    char *base = (char *)(uintptr_t)0x100000;
    EXPECT(tg_gemm(base, base + 0x100000, NULL, base + 0x200000, 64, 64, 64, 9, NULL) ==
           TG_ERR_INVALID_ARG);
    EXPECT(tg_gemm(base + 1, base + 0x100000, NULL, base + 0x200000, 64, 64, 64,
                   TG_EPILOGUE_NONE, NULL) == TG_ERR_MISALIGNED);
    EXPECT(tg_gemm(base, base + 0x100000, NULL, base + 0x200000, 0, 64, 64, TG_EPILOGUE_NONE,
                   NULL) == TG_OK);
    EXPECT(tg_attention_fwd(base, base + 0x100000, base + 0x200000, base + 0x300000, 1, 1, 8, 8,
                            96, 0, 0.0f, NULL) == TG_ERR_INVALID_ARG);

    int64_t units = -1, split = -1, grid = -1;
    EXPECT(tg_attention_plan(4, 16, 2048, 2048, 128, 0, TG_ATTN_SPLIT_AUTO, 148, &units, &split,
                             &grid) == TG_OK);
    printf("attention plan: units %lld split %lld grid %lld\n", (long long)units,
           (long long)split, (long long)grid);
    EXPECT(units == 512 && split == 68 && grid == 580);
    EXPECT(tg_attention_plan(1, 1, 8, 8, 64, 0, 7, 148, &units, &split, &grid) ==
           TG_ERR_INVALID_ARG);
    printf("status %s\n", tg_status_string(TG_ERR_TIMEOUT));
    printf("%s\n", failures ? "FAILED" : "OK");
    return failures ? 1 : 0;
}
