/* The boundary's C ABI used from plain C: compiled against include/sp_region.h
 * and linked with the library, it calls the entry points that need no GPU
 * (plan counts, status strings, the activation-memory closed form, argument
 * validation) and prints what they return for the test to check. */
#include <stdio.h>
#include <string.h>

#include "sp_region.h"

int main(void)
{
    int32_t nf = 0, nb = 0;
    if (sp_plan_count(&nf, &nb) != SP_OK) return 1;
    printf("plans %d %d\n", nf, nb);

    double bytes = 0.0;
    /* A_TP+SP for s=2048 b=1 h=12288 a=96 t=8, 2 bytes per element */
    if (sp_activation_bytes(2048, 1, 12288, 96, 8, 2, 2.0, &bytes) != SP_OK) return 2;
    printf("activation %.1f\n", bytes);
    printf("bad_mode %d\n", sp_activation_bytes(2048, 1, 12288, 96, 8, 7, 2.0, &bytes));

    printf("status %s\n", sp_status_string(SP_ERR_INVALID_ARG));

    /* s not divisible by t: rejected before any device work */
    sp_cfg cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.s = 6; cfg.b = 1; cfg.h = 64; cfg.t = 4;
    cfg.dtype = SP_BF16; cfg.norm = SP_LAYERNORM; cfg.eps = 1e-5f;
    size_t ws = 0;
    printf("bad_cfg %d\n", sp_bwd_workspace_bytes(&cfg, 0, &ws));

    /* ring attention's workspace query: shapes it does not take, and a NULL
     * result pointer, are answered before any device query */
    memset(&cfg, 0, sizeof(cfg));
    cfg.s = 384; cfg.b = 1; cfg.h = 128; cfg.t = 2;   /* s / t = 192 */
    cfg.dtype = SP_BF16; cfg.norm = SP_LAYERNORM; cfg.eps = 1e-5f;
    printf("attn_ragged %d\n", sp_ring_attention_workspace_bytes(&cfg, 1, 0, &ws));
    cfg.s = 256; cfg.t = 1; cfg.h = 64;                /* head dimension 64 */
    printf("attn_head64 %d\n", sp_ring_attention_workspace_bytes(&cfg, 1, 0, &ws));
    cfg.h = 128;
    printf("attn_null %d\n", sp_ring_attention_workspace_bytes(&cfg, 1, 0, NULL));
    return 0;
}
