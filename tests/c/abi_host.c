/* Host-only use of the C ABI from plain C: includes include/sinkattn.h, links
 * libsinkattn.so, and calls the entry points that answer on the host (version,
 * error strings, size queries, argument refusal).  No device is touched. */
#include <stdio.h>
#include <string.h>

#include "sinkattn.h"

int main(void) {
    static int32_t fake[64] __attribute__((aligned(16)));  /* never dereferenced */
    sinkattn_mask m;
    memset(&m, 0, sizeof m);
    m.causal = 1;
    m.cu_seqlens = fake;
    m.n_seq = 1;
    m.max_seqlen = 128;
    m.block_q = 64;
    m.block_k = 64;

    printf("version %d\n", sinkattn_version());
    printf("ok \"%s\"\n", sinkattn_error_string(SINKATTN_OK));
    printf("plan_bytes %zu\n", sinkattn_plan_bytes(128, 4, 2, &m));
    printf("plan_bytes_bad_heads %zu\n", sinkattn_plan_bytes(128, 3, 2, &m));
    printf("bwd_ws %zu\n", sinkattn_bwd_workspace_bytes(SINKATTN_BF16, 128, 4, 2, 64, &m));
    printf("decode_ws %zu\n", sinkattn_decode_workspace_bytes(32, 32, 128, 4));
    printf("imp_ws %zu\n", sinkattn_gate_importance_workspace_bytes(100, 32));
    printf("fwd_bad_d %d\n", sinkattn_fwd(SINKATTN_BF16, 128, 4, 2, 96, 0.125f, fake, fake, fake,
                                          NULL, &m, fake, 1 << 20, fake, (float *)fake, NULL,
                                          NULL));
    printf("gate_bad_t %d\n", sinkattn_gate_importance(0, 8, NULL, NULL, NULL, 0, NULL));
    return 0;
}
