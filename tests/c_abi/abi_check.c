/* Plain C11 user of the library's headers: compiles against the public headers,
 * links libditattn.so and checks argument rejection without a GPU. */
#include <stdio.h>
#include <string.h>

#include "dit_attn.h"
#include "dit_cache.h"

static int fails = 0;
#define EXPECT(call, want)                                                          \
    do {                                                                            \
        dit_status got_ = (call);                                                   \
        if (got_ != (want)) {                                                       \
            printf("FAIL %s: %s (want %s)\n", #call, dit_status_string(got_),       \
                   dit_status_string(want));                                        \
            ++fails;                                                                \
        }                                                                           \
    } while (0)

int main(void) {
    char* q = (char*)0x10000000, *k = (char*)0x20000000, *v = (char*)0x30000000, *o = (char*)0x40000000;
    dit_cache_policy pol = {4, -1, 3, 0.24f};
    EXPECT(dit_attn_fwd(NULL, k, v, o, 1, 2, 256, 64, NULL, 0.f, NULL), DIT_ERR_INVALID_ARG);
    EXPECT(dit_attn_fwd(q, k, v, o, 1, 2, 256, 96, NULL, 0.f, NULL), DIT_ERR_UNSUPPORTED);
    EXPECT(dit_attn_fwd_ex(q, k, v, o, NULL, 1, 2, 0, 256, 64, NULL, NULL, 0.f, NULL), DIT_ERR_INVALID_ARG);
    EXPECT(fbc_rel_l1(q, k, 0, DIT_DTYPE_BF16, 0.1f, NULL, NULL, NULL, 0, NULL), DIT_ERR_INVALID_ARG);
    EXPECT(fbcache_step(q, k, 64, DIT_DTYPE_BF16, NULL, NULL, NULL, 0, 0, 0ull, NULL, 0, NULL), DIT_ERR_INVALID_ARG);
    EXPECT(fbcache_step(q, k, 64, DIT_DTYPE_BF16, &pol, (dit_cache_state*)o, NULL, 0, 0, 0ull, NULL, 0, NULL),
           DIT_ERR_WORKSPACE);
    EXPECT(dit_graph_launch(NULL, NULL), DIT_ERR_INVALID_ARG);
    if (dit_attn_q8_workspace_bytes(1, 24, 4608, 128, DIT_PV_FP8_E4M3) == 0) { puts("FAIL workspace size"); ++fails; }
    if (sizeof(dit_cache_state) != 40 || sizeof(dit_cache_trace) != 24) { puts("FAIL struct sizes"); ++fails; }
    if (strcmp(dit_status_string(DIT_ERR_TIMEOUT), "DIT_ERR_TIMEOUT") != 0) { puts("FAIL strings"); ++fails; }
    printf("%s\n", fails ? "abi check failed" : "abi check ok");
    return fails ? 1 : 0;
}
