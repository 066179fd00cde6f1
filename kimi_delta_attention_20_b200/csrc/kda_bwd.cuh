// Launch parameters of the backward of the chunk forward (kda_bwd.cu).
#pragma once

#include <stdint.h>

namespace kda {

// Launch parameters of the backward (device pointers).
struct BwdParams {
    const void *q, *k, *v, *g, *beta, *dout;
    const float *S0, *dSf;
    void *dq, *dk, *dv, *dg, *dbeta;
    float *dS0;
    const int32_t *cu_seqlens;  // may be null: sequence n = tokens [n*T, (n+1)*T)
    int T, N, H;
    float scale;
    int use_l2, has_lb;
    float lb;
    int beta_prob;
    float *ckpt;                // state checkpoints
    float *scratch;             // per CTA of the reverse sweep: the decayed states of one stretch
    int *ckpt_off;              // varlen: [N+1] first checkpoint of each sequence (device-computed)
};

}  // namespace kda
