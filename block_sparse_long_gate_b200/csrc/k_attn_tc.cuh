// k_attn_tc.cuh - block-sparse attention on the sm_100a tensor cores (tcgen05).
#pragma once
#include "k_attn_common.cuh"

static int run_attention_tc(const AttnParams& a, cudaStream_t st) {
    (void)a;
    (void)st;
    return MOBA_ERR_UNSUPPORTED;
}
